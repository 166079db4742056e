// The 64 x 64 logit tile engine used by compress and head_match: each of 4 warps holds 16 query
// rows of Q in registers (bf16 mma fragments); 64 keys are staged in shared memory with a 16-byte
// XOR swizzle (conflict-free ldmatrix); S = Q K^T accumulates in fp32.
#pragma once

#include "common.cuh"

namespace iamap {

constexpr int kTile = 64;        // block size B (rows and columns of a tile)
constexpr int kTileThreads = 128;

// Q fragments of one warp: rows r0 (= lane/4) and r0 + 8 of the warp's 16 rows, all d dims.
// Rows at or beyond `rows_valid` read as zero.
template <int D>
__device__ __forceinline__ void load_q_frags(uint32_t (&qf)[D / 16][4],
                                             const __nv_bfloat16* __restrict__ qb, int64_t rs,
                                             int iA, int iB, int rows_valid, int lane) {
  const int t4 = lane & 3;
  const bool vA = iA < rows_valid, vB = iB < rows_valid;
  const uint32_t* pA = reinterpret_cast<const uint32_t*>(qb + (int64_t)(vA ? iA : 0) * rs);
  const uint32_t* pB = reinterpret_cast<const uint32_t*>(qb + (int64_t)(vB ? iB : 0) * rs);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const int w = kk * 8 + t4;  // 32-bit word index of dims (kk*16 + 2*t4, +1)
    qf[kk][0] = vA ? __ldg(pA + w) : 0u;
    qf[kk][1] = vB ? __ldg(pB + w) : 0u;
    qf[kk][2] = vA ? __ldg(pA + w + 4) : 0u;
    qf[kk][3] = vB ? __ldg(pB + w + 4) : 0u;
  }
}

// Async copy of keys [key0, key0 + 64) (rows beyond `keys_valid` zero-filled) into a swizzled
// [64][D] bf16 tile: 16-byte chunk c of row r is stored at chunk c ^ (r & 7).
template <int D>
__device__ __forceinline__ void load_k_tile(uint32_t sK, const __nv_bfloat16* __restrict__ kb,
                                            int64_t rs, int key0, int keys_valid, int tid) {
  constexpr int CH = D / 8;
#pragma unroll
  for (int c = tid; c < kTile * CH; c += kTileThreads) {
    const int r = c / CH, ch = c % CH;
    const int key = key0 + r;
    const bool valid = key < keys_valid;
    const __nv_bfloat16* src = kb + (int64_t)(valid ? key : 0) * rs + ch * 8;
    const uint32_t dst = sK + (uint32_t)((r * D + ((ch ^ (r & 7)) << 3)) * 2);
    cp_async16(dst, src, valid);
  }
}

// acc[nt][e]: rows (lane/4) [e<2] and (lane/4 + 8) [e>=2] of the warp's 16 rows, keys
// nt*8 + 2*(lane%4) + (e&1).
template <int D>
__device__ __forceinline__ void qk_tile(const uint32_t (&qf)[D / 16][4], uint32_t sK,
                                        float (&acc)[8][4], int lane) {
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
  const int m = lane >> 3, rr = lane & 7;
#pragma unroll
  for (int nt2 = 0; nt2 < 4; ++nt2) {
    const int key = nt2 * 16 + (m >> 1) * 8 + rr;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int ch = kk * 2 + (m & 1);
      const uint32_t addr = sK + (uint32_t)((key * D + ((ch ^ (key & 7)) << 3)) * 2);
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(addr, b0, b1, b2, b3);
      mma_bf16_16816(acc[2 * nt2], qf[kk], b0, b1);
      mma_bf16_16816(acc[2 * nt2 + 1], qf[kk], b2, b3);
    }
  }
}

// Scales the raw dot products into the log2 domain, adds the local bias and applies the causal
// mask (key > row -> -inf). Rows and keys are sequence-local indices.
__device__ __forceinline__ void scale_mask_tile(float (&acc)[8][4], int iA, int iB, int j0,
                                                float scale_log2, int bias_window,
                                                float bias_log2, int lane) {
  const int t4 = lane & 3;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = e < 2 ? iA : iB;
      const int j = j0 + nt * 8 + 2 * t4 + (e & 1);
      float v = acc[nt][e] * scale_log2;
      if (bias_window > 0 && i - j >= 0 && i - j < bias_window) v += bias_log2;
      acc[nt][e] = j > i ? -INFINITY : v;
    }
}

__device__ __forceinline__ float quad_max(float x) {
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
  return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
}
__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  return x + __shfl_xor_sync(0xffffffffu, x, 2);
}

}  // namespace iamap
