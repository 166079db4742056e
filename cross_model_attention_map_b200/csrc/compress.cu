// map_compress: a sender's causal softmax attention per head -> block-sparse (BSR) map.
//
// Follows the two stages of the MapFlow news page ("PKU MapFlow: cross-model attention map reuse",
// storage-and-execution part, first component): block-level statistics first, then extraction of
// the blocks kept by cumulative attention probability, without a dense n x n matrix.
//
// Stage 1 (compress_kernel<D, false>), one CTA per (row block, sender head): one sweep over the
// causal key tiles with an online softmax. For every (row, column block) it keeps the log2-sum of
// that block's exponentials in shared memory, so that once the row's log-sum-exp is known the
// block mass sum_i exp(c_iJ - lse_i) follows without a second sweep. The CTA then sorts the masses
// of its row block, takes the cumulative-mass prefix and ORs its head bit into the dense head
// mask of every kept causal block.
// Union index (row_count / row_scan / row_fill): the union of the heads' kept blocks per row
// block, with head masks and tile offsets.
// Stage 2 (compress_kernel<D, true>): recomputes each kept tile with the same arithmetic as
// stage 1 and writes exp(s - lse) as bf16 at its BSR position. The k present heads of a stored
// block are interleaved by row: row i of head rank t is at (i * k + t) * 64 within the block, so
// one tile row of all present heads is a contiguous run (what mapped_av loads).
#include "qk_tile.cuh"
#include "internal.h"

namespace iamap {

struct CompressParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const int32_t* cu;
  SeqTables tab;
  int64_t n;
  int64_t ncb;
  int H_s;
  int max_nb;
  float scale_log2;
  int bias_window;
  float bias_log2;
  float tau;
  float* lse;
  float* mass;
  unsigned long long* headmask_dense;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const unsigned long long* headmask;
  const int64_t* val_off;
  __nv_bfloat16* vals;
  int64_t capacity;
  unsigned int* status;
};

static size_t stats_smem_bytes(int D, int max_nb) {
  const size_t cstride = (size_t)max_nb + 1;
  return (size_t)2 * kTile * D * 2                       // key tiles (2 stages)
         + sizeof(float) * (kTile * cstride + kTile)      // cbuf + lse_s
         + sizeof(float) * 2 * (size_t)max_nb             // mass_s + sorted_s
         + sizeof(int) * (size_t)max_nb                   // rank_s
         + sizeof(float) * kTileThreads;                  // scan partials
}
static size_t extract_smem_bytes(int D, int max_nb) {
  return (size_t)2 * kTile * D * 2                       // key tiles (2 stages)
         + (size_t)kTile * kTile * 2                      // bf16 staging tile
         + sizeof(int64_t) * (size_t)max_nb               // own block base tiles
         + sizeof(int) * 2 * (size_t)max_nb               // own column blocks, (rank, k)
         + 16;                                            // own count
}

// Block-wide exclusive scan of x[0..n) (n <= 4 * kTileThreads) in place.
__device__ void block_exclusive_scan(float* x, int n, float* part, int tid) {
  const int per = (n + kTileThreads - 1) / kTileThreads;
  float loc[4];
  float tot = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    loc[e] = 0.f;
    if (e < per) {
      const int idx = tid * per + e;
      const float v = idx < n ? x[idx] : 0.f;
      loc[e] = tot;
      tot += v;
    }
  }
  const int lane = tid & 31, warp = tid >> 5;
  float inc = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) part[warp] = inc;
  __syncthreads();
  float woff = 0.f;
  for (int w = 0; w < warp; ++w) woff += part[w];
  const float base = woff + inc - tot;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    if (e < per) {
      const int idx = tid * per + e;
      if (idx < n) x[idx] = base + loc[e];
    }
  }
  __syncthreads();
}

template <int D, bool EXTRACT>
__global__ void __launch_bounds__(kTileThreads) compress_kernel(CompressParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
  const int item = blockIdx.x / p.H_s;
  const int h = blockIdx.x - item * p.H_s;
  const int2 it = p.tab.items[item];
  const int s = it.x, I = it.y;
  const int seq0 = p.cu[s];
  const int L = p.cu[s + 1] - seq0;
  const int row0 = I * kTile;
  const int R = min(kTile, L - row0);
  const int64_t rs = (int64_t)p.H_s * D;
  const __nv_bfloat16* qb = p.q + (int64_t)seq0 * rs + (int64_t)h * D;
  const __nv_bfloat16* kb = p.k + (int64_t)seq0 * rs + (int64_t)h * D;
  const int rb = tab_rb(p.tab, s, I);
  const int64_t cb0 = tab_cb(p.tab, s, I);

  const uint32_t sK0 = smem_u32(smem);
  constexpr uint32_t kStage = kTile * D * 2;
  unsigned char* rest = smem + 2 * kStage;

  uint32_t qf[D / 16][4];
  const int iA = row0 + 16 * warp + g, iB = iA + 8;  // sequence-local rows of this thread
  load_q_frags<D>(qf, qb, rs, iA, iB, L, lane);
  const bool vA = iA < L, vB = iB < L;
  float* lse_row = p.lse + (int64_t)h * p.n + seq0;  // lse of sequence-local row i: lse_row[i]

  if constexpr (!EXTRACT) {
    const int cstride = p.max_nb + 1;
    float* cbuf = reinterpret_cast<float*>(rest);       // [64][cstride]
    float* lse_s = cbuf + kTile * cstride;               // [64] (log2 domain)
    float* mass_s = lse_s + kTile;                        // [max_nb]
    float* sorted_s = mass_s + p.max_nb;                  // [max_nb]
    int* rank_s = reinterpret_cast<int*>(sorted_s + p.max_nb);
    float* part_s = reinterpret_cast<float*>(rank_s + p.max_nb);

    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    load_k_tile<D>(sK0, kb, rs, 0, L, tid);
    cp_async_commit();
    for (int J = 0; J <= I; ++J) {
      if (J < I) load_k_tile<D>(sK0 + ((J + 1) & 1) * kStage, kb, rs, (J + 1) * kTile, L, tid);
      cp_async_commit();
      cp_async_wait<1>();
      __syncthreads();
      float acc[8][4];
      qk_tile<D>(qf, sK0 + (J & 1) * kStage, acc, lane);
      scale_mask_tile(acc, iA, iB, J * kTile, p.scale_log2, p.bias_window, p.bias_log2, lane);
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        float mx = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
          mx = fmaxf(mx, fmaxf(acc[nt][2 * hr], acc[nt][2 * hr + 1]));
        mx = quad_max(mx);
        const float mnew = fmaxf(m_run[hr], mx);
        const float ref = mnew == -INFINITY ? 0.f : mnew;
        float sum = 0.f;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
          sum += ex2(acc[nt][2 * hr] - ref) + ex2(acc[nt][2 * hr + 1] - ref);
        sum = quad_sum(sum);
        l_run[hr] = l_run[hr] * ex2(m_run[hr] - ref) + sum;
        m_run[hr] = mnew;
        if (t4 == 0) cbuf[(16 * warp + g + 8 * hr) * cstride + J] = ref + lg2(sum);
      }
      __syncthreads();
    }
    // Row log-sum-exp: log2 domain in shared memory, natural log in the output.
    if (t4 == 0) {
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int r = 16 * warp + g + 8 * hr;
        const float l2 = m_run[hr] + lg2(l_run[hr]);
        lse_s[r] = l2;
        if (hr ? vB : vA) lse_row[row0 + r] = l2 * kLn2;
      }
    }
    __syncthreads();
    // Block masses over the valid rows.
    const int nJ = I + 1;
    float* mass_out = p.mass + (int64_t)h * p.ncb + cb0;
    for (int J = tid; J < nJ; J += kTileThreads) {
      float acc = 0.f;
      for (int r = 0; r < R; ++r) acc += ex2(cbuf[r * cstride + J] - lse_s[r]);
      mass_s[J] = acc;
      mass_out[J] = acc;
    }
    __syncthreads();
    // Cumulative-mass choice: order by decreasing mass (ties: lower J first); keep a block while
    // the mass before it is below tau * R.
    unsigned long long* hm_out = p.headmask_dense + cb0;
    const unsigned long long bit = 1ull << h;
    if (p.tau >= 1.f) {
      for (int J = tid; J < nJ; J += kTileThreads) atomicOr(hm_out + J, bit);
      return;
    }
    for (int J = tid; J < nJ; J += kTileThreads) {
      const float mJ = mass_s[J];
      int rank = 0;
      for (int J2 = 0; J2 < nJ; ++J2) {
        const float m2 = mass_s[J2];
        rank += (m2 > mJ) || (m2 == mJ && J2 < J);
      }
      rank_s[J] = rank;
      sorted_s[rank] = mJ;
    }
    __syncthreads();
    block_exclusive_scan(sorted_s, nJ, part_s, tid);
    const float thr = p.tau * (float)R;
    for (int J = tid; J < nJ; J += kTileThreads)
      if (sorted_s[rank_s[J]] < thr) atomicOr(hm_out + J, bit);
  } else {
    __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(rest);          // [64][64] swizzled
    int64_t* own_base = reinterpret_cast<int64_t*>(rest + kTile * kTile * 2);  // [max_nb]
    int* own_J = reinterpret_cast<int*>(own_base + p.max_nb);                // [max_nb]
    int* own_rk = own_J + p.max_nb;                                           // rank | k << 8
    int* own_cnt = own_rk + p.max_nb;
    // The column blocks this head keeps in this row block, with their tile indices.
    if (warp == 0) {
      const int u0 = p.row_ptr[rb], u1 = p.row_ptr[rb + 1];
      int cnt = 0;
      const unsigned long long below = (1ull << h) - 1ull;
      for (int base = u0; base < u1; base += 32) {
        const int u = base + lane;
        unsigned long long m = 0;
        bool own = false;
        if (u < u1) {
          m = p.headmask[u];
          own = (m >> h) & 1ull;
        }
        const unsigned b = __ballot_sync(0xffffffffu, own);
        if (own) {
          const int pos = cnt + __popc(b & ((1u << lane) - 1u));
          own_J[pos] = p.col_idx[u];
          own_base[pos] = p.val_off[u];
          own_rk[pos] = __popcll(m & below) | (__popcll(m) << 8);
        }
        cnt += __popc(b);
      }
      if (lane == 0) *own_cnt = cnt;
    }
    // Row log-sum-exp of this thread's two rows, log2 domain.
    const float lA = vA ? lse_row[iA] * kLog2e : 0.f;
    const float lB = vB ? lse_row[iB] * kLog2e : 0.f;
    __syncthreads();
    const int cnt = *own_cnt;
    if (cnt > 0) {
      load_k_tile<D>(sK0, kb, rs, own_J[0] * kTile, L, tid);
      cp_async_commit();
    }
    bool cap_flag = false;
    for (int t = 0; t < cnt; ++t) {
      if (t + 1 < cnt)
        load_k_tile<D>(sK0 + ((t + 1) & 1) * kStage, kb, rs, own_J[t + 1] * kTile, L, tid);
      cp_async_commit();
      cp_async_wait<1>();
      __syncthreads();
      const int J = own_J[t];
      float acc[8][4];
      qk_tile<D>(qf, sK0 + (t & 1) * kStage, acc, lane);
      scale_mask_tile(acc, iA, iB, J * kTile, p.scale_log2, p.bias_window, p.bias_log2, lane);
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float p0 = vA ? ex2(acc[nt][0] - lA) : 0.f;
        const float p1 = vA ? ex2(acc[nt][1] - lA) : 0.f;
        const float p2 = vB ? ex2(acc[nt][2] - lB) : 0.f;
        const float p3 = vB ? ex2(acc[nt][3] - lB) : 0.f;
        const int rA = 16 * warp + g, rB = rA + 8;
        *reinterpret_cast<uint32_t*>(stage + rA * kTile + ((nt ^ (rA & 7)) << 3) + 2 * t4) =
            pack_bf16(p0, p1);
        *reinterpret_cast<uint32_t*>(stage + rB * kTile + ((nt ^ (rB & 7)) << 3) + 2 * t4) =
            pack_bf16(p2, p3);
      }
      __syncthreads();
      const int64_t base = own_base[t];
      const int rank = own_rk[t] & 255, kk = own_rk[t] >> 8;
      if (base >= 0 && base + kk <= p.capacity) {
        __nv_bfloat16* blk = p.vals + base * (kTile * kTile) + (int64_t)rank * kTile;
#pragma unroll
        for (int c = tid; c < kTile * 8; c += kTileThreads) {
          const int r = c >> 3, ch = c & 7;
          *reinterpret_cast<uint4*>(blk + (int64_t)r * kk * kTile + ch * 8) =
              *reinterpret_cast<const uint4*>(stage + r * kTile + ((ch ^ (r & 7)) << 3));
        }
      } else {
        cap_flag = true;
      }
    }
    if (cap_flag && tid == 0) raise_status(p.status, IAMAP_DEV_CAPACITY);
  }
}

// ------------------------------------------------------------------------------------------------
// Union BSR index
// ------------------------------------------------------------------------------------------------

// One warp per row block: number of stored column blocks (row_ptr[rb], scanned later) and tiles.
__global__ void row_count_kernel(const unsigned long long* __restrict__ hm_dense, SeqTables tab,
                                 int64_t num_rowblocks, int32_t* __restrict__ row_ptr) {
  const int64_t item = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (item >= num_rowblocks) return;
  const int2 it = tab.items[item];
  const int rb = tab_rb(tab, it.x, it.y);
  const int64_t cb0 = tab_cb(tab, it.x, it.y);
  int cnt = 0;
  long long tiles = 0;
  for (int J = lane; J <= it.y; J += 32) {
    const unsigned long long m = hm_dense[cb0 + J];
    cnt += m != 0ull;
    tiles += __popcll(m);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    tiles += __shfl_xor_sync(0xffffffffu, tiles, o);
  }
  if (lane == 0) {
    row_ptr[rb] = cnt;
    tab.row_tiles[rb] = tiles;
  }
}

// One CTA of 1024 threads: exclusive scans of the per-row counts (in place) and tiles.
__global__ void __launch_bounds__(1024) row_scan_kernel(int32_t* __restrict__ row_ptr,
                                                        int64_t* __restrict__ row_tiles,
                                                        int64_t nrb, int64_t* __restrict__ counts) {
  __shared__ long long part_c[32], part_t[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t per = (nrb + 1023) / 1024;
  const int64_t b0 = tid * per, b1 = min(nrb, b0 + per);
  long long c = 0, t = 0;
  for (int64_t i = b0; i < b1; ++i) {
    c += row_ptr[i];
    t += row_tiles[i];
  }
  long long ic = c, itl = t;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long yc = __shfl_up_sync(0xffffffffu, ic, o);
    const long long yt = __shfl_up_sync(0xffffffffu, itl, o);
    if (lane >= o) {
      ic += yc;
      itl += yt;
    }
  }
  if (lane == 31) {
    part_c[warp] = ic;
    part_t[warp] = itl;
  }
  __syncthreads();
  long long oc = 0, ot = 0;
  for (int w = 0; w < warp; ++w) {
    oc += part_c[w];
    ot += part_t[w];
  }
  long long rc = oc + ic - c, rt = ot + itl - t;
  for (int64_t i = b0; i < b1; ++i) {
    const long long xc = row_ptr[i], xt = row_tiles[i];
    row_ptr[i] = (int32_t)rc;
    row_tiles[i] = rt;
    rc += xc;
    rt += xt;
  }
  if (tid == 1023) {
    row_ptr[nrb] = (int32_t)rc;
    counts[0] = rc;
    counts[1] = rt;
  }
}

// One warp per row block: writes col_idx / headmask / val_off of its stored column blocks.
__global__ void row_fill_kernel(const unsigned long long* __restrict__ hm_dense, SeqTables tab,
                                int64_t num_rowblocks, const int32_t* __restrict__ row_ptr,
                                int32_t* __restrict__ col_idx,
                                unsigned long long* __restrict__ headmask,
                                int64_t* __restrict__ val_off) {
  const int64_t item = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (item >= num_rowblocks) return;
  const int2 it = tab.items[item];
  const int rb = tab_rb(tab, it.x, it.y);
  const int64_t cb0 = tab_cb(tab, it.x, it.y);
  int u = row_ptr[rb];
  long long toff = tab.row_tiles[rb];
  for (int base = 0; base <= it.y; base += 32) {
    const int J = base + lane;
    const unsigned long long m = J <= it.y ? hm_dense[cb0 + J] : 0ull;
    const unsigned b = __ballot_sync(0xffffffffu, m != 0ull);
    const int pc = __popcll(m);
    int incl = pc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (m != 0ull) {
      const int pos = u + __popc(b & ((1u << lane) - 1u));
      col_idx[pos] = J;
      headmask[pos] = m;
      val_off[pos] = toff + (incl - pc);
    }
    u += __popc(b);
    toff += __shfl_sync(0xffffffffu, incl, 31);
  }
}

// Zero-fills up to 64 tiles after the last written tile (within capacity): consumers may read
// a fixed number of tiles past a block's last present head.
__global__ void zero_tail_kernel(__nv_bfloat16* __restrict__ vals,
                                 const int64_t* __restrict__ counts, int64_t capacity) {
  const int64_t tile = counts[1] + blockIdx.x;
  if (tile >= capacity) return;
  uint4* dst = reinterpret_cast<uint4*>(vals + tile * (kTile * kTile));
  for (int c = threadIdx.x; c < kTile * kTile / 8; c += blockDim.x) dst[c] = make_uint4(0, 0, 0, 0);
}

// ------------------------------------------------------------------------------------------------
// Host launchers
// ------------------------------------------------------------------------------------------------

template <int D, bool EXTRACT>
static int launch_compress_kernel(const CompressParams& p, int64_t num_rowblocks, size_t smem,
                                  cudaStream_t stream) {
  auto kern = compress_kernel<D, EXTRACT>;
  IAMAP_CUDA_CHECK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)smem));
  const int64_t grid = num_rowblocks * p.H_s;
  if (grid > 0) {
    kern<<<(unsigned)grid, kTileThreads, smem, stream>>>(p);
    IAMAP_LAUNCH_CHECK(EXTRACT ? "compress extract" : "compress stats");
  }
  return IAMAP_OK;
}

int compress_stats_impl(const CompressArgs& a, cudaStream_t stream) {
  CompressParams p{};
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k = static_cast<const __nv_bfloat16*>(a.k);
  p.cu = a.cu_seqlens;
  p.tab = a.tab;
  p.n = a.n;
  p.ncb = a.plan.num_causal_blocks;
  p.H_s = a.H_s;
  p.max_nb = a.plan.max_nb;
  p.scale_log2 = kLog2e / sqrtf((float)a.d);
  p.bias_window = a.bias_window;
  p.bias_log2 = a.bias_value * kLog2e;
  p.tau = a.tau;
  p.lse = a.lse;
  p.mass = a.mass;
  p.headmask_dense = reinterpret_cast<unsigned long long*>(a.headmask_dense);
  p.status = a.status;
  IAMAP_CUDA_CHECK(cudaMemsetAsync(a.headmask_dense, 0,
                                   sizeof(uint64_t) * (size_t)a.plan.num_causal_blocks, stream));
  const size_t smem = stats_smem_bytes(a.d, a.plan.max_nb);
  int rc = compress_tc_supported(a.d, a.plan.max_nb) ? compress_stats_tc_launch(a, stream)
           : a.d == 64 ? launch_compress_kernel<64, false>(p, a.plan.num_rowblocks, smem, stream)
                       : launch_compress_kernel<128, false>(p, a.plan.num_rowblocks, smem, stream);
  if (rc) return rc;
  const int64_t nrb = a.plan.num_rowblocks;
  const unsigned wgrid = (unsigned)((nrb * 32 + 255) / 256);
  if (wgrid > 0) {
    row_count_kernel<<<wgrid, 256, 0, stream>>>(p.headmask_dense, a.tab, nrb, a.row_ptr);
    IAMAP_LAUNCH_CHECK("row_count_kernel");
  }
  // (with no row blocks this writes row_ptr[0] = 0 and zero counts)
  row_scan_kernel<<<1, 1024, 0, stream>>>(a.row_ptr, a.tab.row_tiles, nrb, a.counts);
  IAMAP_LAUNCH_CHECK("row_scan_kernel");
  if (wgrid > 0) {
    row_fill_kernel<<<wgrid, 256, 0, stream>>>(p.headmask_dense, a.tab, nrb, a.row_ptr, a.col_idx,
                                               reinterpret_cast<unsigned long long*>(a.headmask),
                                               a.val_off);
    IAMAP_LAUNCH_CHECK("row_fill_kernel");
  }
  return IAMAP_OK;
}

int compress_extract_impl(const CompressArgs& a, cudaStream_t stream) {
  CompressParams p{};
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k = static_cast<const __nv_bfloat16*>(a.k);
  p.cu = a.cu_seqlens;
  p.tab = a.tab;
  p.n = a.n;
  p.ncb = a.plan.num_causal_blocks;
  p.H_s = a.H_s;
  p.max_nb = a.plan.max_nb;
  p.scale_log2 = kLog2e / sqrtf((float)a.d);
  p.bias_window = a.bias_window;
  p.bias_log2 = a.bias_value * kLog2e;
  p.lse = const_cast<float*>(a.lse_in);
  p.row_ptr = a.row_ptr_in;
  p.col_idx = a.col_idx_in;
  p.headmask = reinterpret_cast<const unsigned long long*>(a.headmask_in);
  p.val_off = a.val_off_in;
  p.vals = static_cast<__nv_bfloat16*>(a.vals);
  p.capacity = a.capacity;
  p.status = a.status;
  const size_t smem = extract_smem_bytes(a.d, a.plan.max_nb);
  int rc = compress_tc_supported(a.d, a.plan.max_nb) ? compress_extract_tc_launch(a, stream)
           : a.d == 64 ? launch_compress_kernel<64, true>(p, a.plan.num_rowblocks, smem, stream)
                       : launch_compress_kernel<128, true>(p, a.plan.num_rowblocks, smem, stream);
  if (rc) return rc;
  if (a.capacity > 0) {
    zero_tail_kernel<<<64, 256, 0, stream>>>(p.vals, a.counts_in, a.capacity);
    IAMAP_LAUNCH_CHECK("zero_tail_kernel");
  }
  return IAMAP_OK;
}

size_t compress_stats_smem(int d, int max_nb) { return stats_smem_bytes(d, max_nb); }
size_t compress_extract_smem(int d, int max_nb) { return extract_smem_bytes(d, max_nb); }

}  // namespace iamap
