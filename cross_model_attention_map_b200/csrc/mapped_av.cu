// mapped_av: for every stored block of the block-sparse sender map, mix the sender heads by W on
// chip, multiply by the receiver's V and accumulate the output; no dense receiver map is formed.
// (MapFlow news page, storage-and-execution part, third component; head mapping as a learned
// linear combination of sender heads: its layer/head-mapping paragraph.)
//
// One CTA per (row block, group of 4 receiver heads), 16 warps. For each stored column block J of
// the row block:
//   1. the present sender tiles stream through shared memory in chunks of 4 (cp.async, double
//      buffered) and every thread accumulates P_r = sum_s W[r, s] * Pt_s for 8 positions and the
//      4 receiver heads of the CTA (fp32), absent heads contributing nothing;
//   2. P_r is rounded to bf16 into a swizzled [64][64] tile per receiver head;
//   3. warp w computes O_r[16 rows] += P_r . V_r[J] with mma.sync (bf16 in, fp32 accumulate)
//      for receiver head r = w / 4 of the group, V_r[J] staged in shared memory.
// The output rows are written once, after the last column block.
// This form serves receiver layers wider than the tensor-core kernel's cluster (H_r > 32) and
// narrow ones whose cluster would have one CTA, or two with at most 16 sender heads (there it is
// the faster of the two; see use_tensor_core_path below); the tensor-core, cluster-cooperative
// kernel (mapped_av_tc.cu) handles the rest of H_r <= 32.
#include "internal.h"

namespace iamap {

constexpr int kAvThreads = 512;
constexpr int kAvGroup = 4;       // receiver heads per CTA
constexpr int kAvChunk = 4;       // sender tiles per shared-memory buffer
constexpr int kT = 64;            // block size
constexpr int kTileElems = kT * kT;

struct AvParams {
  const int32_t* cu;
  SeqTables tab;
  int H_s;
  int H_r;
  int H_kv;     // value heads (H_r / H_kv consecutive receiver heads share one)
  int groups;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const unsigned long long* headmask;
  const int64_t* val_off;
  const __nv_bfloat16* vals;
  int64_t capacity;
  const float* W;
  int seqs_per_w;   // sequences per mixing matrix (several layers per launch; 0 = one W)
  const __nv_bfloat16* v;
  float* out;
  unsigned int* status;
};

template <int DV>
static constexpr size_t av_smem_bytes() {
  return (size_t)2 * kAvChunk * kTileElems * 2      // sender tiles, 2 buffers
         + (size_t)kAvGroup * kTileElems * 2         // mixed P_r tiles
         + (size_t)kAvGroup * kT * DV * 2            // V_r[J] tiles
         + sizeof(float) * kAvGroup * 64             // W rows of the group
         + sizeof(float) * kAvGroup * 64;            // W columns of the present heads
}

template <int DV>
__global__ void __launch_bounds__(kAvThreads, 1) mapped_av_kernel(AvParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  __nv_bfloat16* sT = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sP = sT + 2 * kAvChunk * kTileElems;
  __nv_bfloat16* sV = sP + kAvGroup * kTileElems;
  float* sW = reinterpret_cast<float*>(sV + kAvGroup * kT * DV);
  float* sWp = sW + kAvGroup * 64;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int item = blockIdx.x / p.groups;
  const int grp = blockIdx.x - item * p.groups;
  const int2 it = p.tab.items[item];
  const int s = it.x, I = it.y;
  const int seq0 = p.cu[s];                 // V token of key 0
  const int orow0 = p.tab.qoff[s];          // output row of the sequence-local row 0
  const int L = p.cu[s + 1] - seq0;
  const int rb = tab_rb(p.tab, s, I);
  const int r0 = grp * kAvGroup;
  const int G = min(kAvGroup, p.H_r - r0);
  const int64_t vrs = (int64_t)p.H_kv * DV;  // V row stride (elements)
  const int kv_grp = p.H_r / p.H_kv;
  const float* Wl = p.W + (p.seqs_per_w ? (int64_t)(s / p.seqs_per_w) * p.H_r * p.H_s : 0);

  for (int e = tid; e < kAvGroup * 64; e += kAvThreads) {
    const int r = e / 64, hs = e % 64;
    sW[e] = (r < G && hs < p.H_s) ? Wl[(int64_t)(r0 + r) * p.H_s + hs] : 0.f;
  }

  // PV role of this warp: 16 rows, one receiver head of the group.
  const int pv_rows = 16 * (warp & 3);
  const int pv_head = warp >> 2;
  float o[DV / 8][4];
#pragma unroll
  for (int nt = 0; nt < DV / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;

  // Mixing role of this thread: 8 consecutive positions of one row.
  const int mix_row = tid >> 3, mix_col = (tid & 7) * 8;

  const int u0 = p.row_ptr[rb], u1 = p.row_ptr[rb + 1];
  bool bad_index = false;
  for (int u = u0; u < u1; ++u) {
    const int J = p.col_idx[u];
    const unsigned long long m = p.headmask[u];
    const int64_t base = p.val_off[u];
    const int k = __popcll(m);
    __syncthreads();  // previous block's readers of sWp / sP / sV are done
    if (tid < 64 && ((m >> tid) & 1ull)) {
      const int rank = __popcll(m & ((1ull << tid) - 1ull));
#pragma unroll
      for (int r = 0; r < kAvGroup; ++r) sWp[r * 64 + rank] = sW[r * 64 + tid];
    }
    // V_r[J] for the group's receiver heads (rows past the sequence end read as zero).
    {
      constexpr int CH = DV / 8;
      for (int c = tid; c < kAvGroup * kT * CH; c += kAvThreads) {
        const int r = c / (kT * CH), rem = c % (kT * CH);
        const int j = rem / CH, ch = rem % CH;
        const int tok = J * kT + j;
        const bool valid = r < G && tok < L;
        const __nv_bfloat16* src =
            p.v + (valid ? ((int64_t)(seq0 + tok) * vrs + (int64_t)((r0 + r) / kv_grp) * DV + ch * 8)
                         : 0);
        const uint32_t dst = smem_u32(sV + r * kT * DV + j * DV + ((ch ^ (j & 7)) << 3));
        cp_async16(dst, src, valid);
      }
      cp_async_commit();
    }
    auto load_chunk = [&](int c, int buf) {
      for (int e = tid; e < kAvChunk * kTileElems / 8; e += kAvThreads) {
        const int t = e / (kTileElems / 8), off = e % (kTileElems / 8);
        const int hr = c * kAvChunk + t;
        const bool valid = hr < k && base >= 0 && base + k <= p.capacity;
        if (hr < k && !valid) bad_index = true;
        // row i of head rank hr: (i * k + hr) * 64 elements into the block
        const int i = off >> 3, ch = off & 7;
        const __nv_bfloat16* src =
            p.vals + (valid ? base * kTileElems + ((int64_t)i * k + hr) * kT + ch * 8 : 0);
        cp_async16(smem_u32(sT + (buf * kAvChunk + t) * kTileElems + off * 8), src, valid);
      }
    };
    const int nchunks = (k + kAvChunk - 1) / kAvChunk;
    float acc[8][kAvGroup];
#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
      for (int r = 0; r < kAvGroup; ++r) acc[e][r] = 0.f;
    load_chunk(0, 0);
    cp_async_commit();
    for (int c = 0; c < nchunks; ++c) {
      if (c + 1 < nchunks) load_chunk(c + 1, (c + 1) & 1);
      cp_async_commit();
      cp_async_wait<1>();
      __syncthreads();
      const int tmax = min(kAvChunk, k - c * kAvChunk);
      for (int t = 0; t < tmax; ++t) {
        const uint4 raw = *reinterpret_cast<const uint4*>(
            sT + ((c & 1) * kAvChunk + t) * kTileElems + mix_row * kT + mix_col);
        const __nv_bfloat162* pv = reinterpret_cast<const __nv_bfloat162*>(&raw);
        float pf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(pv[e]);
          pf[2 * e] = f.x;
          pf[2 * e + 1] = f.y;
        }
        const int hr = c * kAvChunk + t;
#pragma unroll
        for (int r = 0; r < kAvGroup; ++r) {
          const float w = sWp[r * 64 + hr];
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e][r] = fmaf(w, pf[e], acc[e][r]);
        }
      }
      __syncthreads();
    }
    cp_async_wait<0>();
    // Mixed maps to bf16, swizzled [64][64] per receiver head.
#pragma unroll
    for (int r = 0; r < kAvGroup; ++r) {
      uint4 packed;
      packed.x = pack_bf16(acc[0][r], acc[1][r]);
      packed.y = pack_bf16(acc[2][r], acc[3][r]);
      packed.z = pack_bf16(acc[4][r], acc[5][r]);
      packed.w = pack_bf16(acc[6][r], acc[7][r]);
      const int ch = mix_col >> 3;
      *reinterpret_cast<uint4*>(sP + r * kTileElems + mix_row * kT + ((ch ^ (mix_row & 7)) << 3)) =
          packed;
    }
    __syncthreads();
    if (pv_head < G) {
      const __nv_bfloat16* P = sP + pv_head * kTileElems;
      const __nv_bfloat16* V = sV + pv_head * kT * DV;
      const int mq = lane >> 3, rr = lane & 7;
#pragma unroll
      for (int kk = 0; kk < kT / 16; ++kk) {
        uint32_t a[4];
        {
          const int row = pv_rows + (mq & 1) * 8 + rr;
          const int ch = kk * 2 + (mq >> 1);
          ldmatrix_x4(smem_u32(P + row * kT + ((ch ^ (row & 7)) << 3)), a[0], a[1], a[2], a[3]);
        }
#pragma unroll
        for (int nt2 = 0; nt2 < DV / 16; ++nt2) {
          const int j = kk * 16 + (mq & 1) * 8 + rr;
          const int ch = nt2 * 2 + (mq >> 1);
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4_trans(smem_u32(V + j * DV + ((ch ^ (j & 7)) << 3)), b0, b1, b2, b3);
          mma_bf16_16816(o[2 * nt2], a, b0, b1);
          mma_bf16_16816(o[2 * nt2 + 1], a, b2, b3);
        }
      }
    }
  }
  if (bad_index) raise_status(p.status, IAMAP_DEV_BAD_INDEX);
  // Output rows of this row block (rows past the sequence end are not written).
  if (pv_head < G) {
    const int g = lane >> 2, t4 = lane & 3;
    const int r = r0 + pv_head;
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int i = I * kT + pv_rows + g + 8 * hr;
      if (i < L) {
        float* dst = p.out + ((int64_t)(orow0 + i) * p.H_r + r) * DV;
#pragma unroll
        for (int nt = 0; nt < DV / 8; ++nt)
          *reinterpret_cast<float2*>(dst + nt * 8 + 2 * t4) =
              make_float2(o[nt][2 * hr], o[nt][2 * hr + 1]);
      }
    }
  }
}

template <int DV>
static int launch_av(const AvParams& p, int64_t num_items, cudaStream_t stream) {
  const size_t smem = av_smem_bytes<DV>();
  IAMAP_CUDA_CHECK(cudaFuncSetAttribute(mapped_av_kernel<DV>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  const int64_t grid = num_items * p.groups;
  if (grid > 0) {
    mapped_av_kernel<DV><<<(unsigned)grid, kAvThreads, smem, stream>>>(p);
    IAMAP_LAUNCH_CHECK("mapped_av_kernel");
  }
  return IAMAP_OK;
}

// The tensor-core kernel spreads the receiver heads of a row block over a cluster of
// C = ceil(H_r / 4) CTAs. With one CTA per cluster, or two and at most 16 sender heads, the few
// CTAs each mix and read out most of the block alone, and this kernel (one CTA per row block and
// group of 4 receiver heads, no cluster exchange) is the faster one: measured on a B200, 4x at
// H_r = 4, 1.1x to 2x at H_r = 8 with H_s <= 16, even at H_r = 8 with H_s = 32, and the cluster
// kernel ahead from H_r = 12 on (1.2x to 3.5x).
static bool use_tensor_core_path(const MappedAvArgs& a) {
  if (!mapped_av_tc_supported(a.H_s, a.H_r, a.d_v)) return false;
  const int C = (a.H_r + kAvGroup - 1) / kAvGroup;
  return C > 2 || (C == 2 && a.H_s > 16);
}

int mapped_av_impl(const MappedAvArgs& a, cudaStream_t stream) {
  if (use_tensor_core_path(a)) return mapped_av_tc_impl(a, stream);
  AvParams p{};
  p.cu = a.cu_seqlens;
  p.tab = a.tab;
  p.H_s = a.H_s;
  p.H_r = a.H_r;
  p.H_kv = a.H_kv > 0 ? a.H_kv : a.H_r;
  p.groups = (a.H_r + kAvGroup - 1) / kAvGroup;
  p.row_ptr = a.row_ptr;
  p.col_idx = a.col_idx;
  p.headmask = reinterpret_cast<const unsigned long long*>(a.headmask);
  p.val_off = a.val_off;
  p.vals = static_cast<const __nv_bfloat16*>(a.vals);
  p.capacity = a.capacity;
  p.W = a.W;
  p.seqs_per_w = a.seqs_per_w;
  p.v = static_cast<const __nv_bfloat16*>(a.v);
  p.out = a.out;
  p.status = a.status;
  return a.d_v == 64 ? launch_av<64>(p, a.plan.num_rowblocks, stream)
                     : launch_av<128>(p, a.plan.num_rowblocks, stream);
}

}  // namespace iamap
