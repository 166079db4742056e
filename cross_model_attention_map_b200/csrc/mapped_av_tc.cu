// mapped_av on the 5th-generation tensor cores, one thread-block cluster per row block.
//
// What it computes is the fused mapping + value aggregation of the MapFlow news page ("PKU
// MapFlow: cross-model attention map reuse", storage-and-execution part, third component): for
// every stored block (I, J) of the block-sparse sender map, P_r = sum_s W[r, s] Pt_s is formed on
// chip and O_r[rows of I] += P_r . V_r[rows of J]; no dense receiver map exists anywhere.
//
// Work split. A CTA can keep O accumulators of 4 receiver heads x 64 rows x d_v in TMEM, so a row
// block needs C = ceil(H_r / 4) CTAs; they form one cluster and split the sender tiles instead of
// each reading all of them:
//   * CTA c TMA-loads rows [2*c0, 2*c1) of every present sender tile of the block. The values of
//     a stored block are interleaved by row (row i of head rank t at line i*k + t), so one tile
//     row of all k present heads is one contiguous run of k lines of 128 B: one box per row,
//     whose lines are the K-stack of an MN-major, 128-byte-swizzled operand. It mixes them for ALL receiver
//     heads: D[128 positions][N = H_r] = P[128][K = heads] . W'[N][K] with tcgen05.mma, where W'
//     holds the W columns of the present heads (zero past them).
//   * The mixed rows are rounded to bf16, transposed (stmatrix) through a 2 KB per-warp scratch into 16-byte
//     runs of 8 positions of one receiver head, and stored with st.async straight into the receive
//     buffer of the CTA owning that head, at their place in its K-major, 128-byte-swizzled tile;
//     the bytes count on that CTA's mbarrier.
//   * Each CTA accumulates O_r^T[d_v][64 rows] += V_r[J]^T . P_r^T for its 4 heads: V_r[J] is the
//     MN-major A operand (TMA), the received P_r the K-major B operand; accumulators stay in TMEM
//     across the whole row and are written once.
// No TMA multicast is used: every CTA loads its own tiles.
//
// Roles: warps 0, 8, 9, 10 load the sender slices, warp 7 builds W', warps 6, 11, 17, 18 load
// the V tiles (one receiver head each), one thread of warp 1 issues the mixing MMAs and one
// thread of warp 12 the P.V MMAs (two issuers: MMA and commit issue costs add up on one thread).
// Two groups of four warps (2-5 and 13-16) take the even and the odd chunk pairs of every stored
// block: they read the mixing results out of TMEM, transpose and send them; the first group also
// writes the output. Every wait is bounded (2 s, then IAMAP_DEV_TIMEOUT).
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "internal.h"
#include "tc_utils.cuh"

namespace iamap {

// ------------------------------------------------------------------------------------------------
// Tensor-map encoding through the runtime's driver entry point
// ------------------------------------------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
static std::once_flag g_encode_once;

int encode_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                        uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer) {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) return set_error(IAMAP_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return set_error(IAMAP_ERR_INVALID_ARG, "tensor map encoding failed (%d)", (int)r);
  return IAMAP_OK;
}

int encode_tmap_3d_bf16(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                        uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1,
                        uint32_t b2) {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) return set_error(IAMAP_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return set_error(IAMAP_ERR_INVALID_ARG, "3-D tensor map encoding failed (%d)", (int)r);
  return IAMAP_OK;
}

namespace tcav {

constexpr int kG = 4;            // receiver heads per CTA (O in TMEM: 4 x 64 columns)
constexpr int kMaxNP = 12;       // sender-slice ring: as many slots as shared memory allows
// A thread that issues TMA loads waits ~5 ns per 128-byte line of the box (measured on a B200:
// 0.31 us for a 16 KB contiguous box, 0.49 us for a V tile spread over 64 tokens, i.e. 33-52 GB/s
// per issuing thread, against ~130 GB/s per SM from L2 with four issuers), so the loads are
// spread over several producer warps: four for the sender slices and one per receiver head for
// the V tiles (each a single 3-D box of both 64-dim halves). Ring slot s is always loaded by
// producer warp s mod 4, so the uses of a slot are issued in order by one thread: a wait for the
// release of use u - 1 never runs while use u - 2 is still pending (an mbarrier parity wait two
// phases ahead would pass at once and let a load overwrite a slot still in use).
constexpr int kPWarps = 4, kVWarps = 4;
constexpr int kND = 8;           // mixing-result TMEM slots (chunks)
constexpr int kNG = kND / 2;     // ... committed and released in pairs of chunks (one commit costs
                                 // ~90 ns of issue time on a B200, an MMA ~25 ns)
constexpr int kNGh = kNG / 2;    // pair slots of each readout group: even pairs of a block use
                                 // slots 0-1, odd pairs slots 2-3, so that every slot has one
                                 // consumer that takes its phases in order
constexpr int kNV = 4;           // V tiles: one slot per receiver head of the CTA
constexpr int kRecv = 2;         // exchange rounds in flight: receive buffers of 4 heads x 8 KB
constexpr int kThreads = 608;    // 19 warps
constexpr int kEpiWarps = 8;     // two readout groups of four warps
constexpr int kMixCol = 256;     // first TMEM column of the mixing slots
constexpr uint32_t kTmemCols = 512;

// barrier indices
enum {
  P_FULL = 0, P_EMPTY = P_FULL + kMaxNP, W_FULL = P_EMPTY + kMaxNP, W_EMPTY = W_FULL + 2,
  D_FULL = W_EMPTY + 2, D_EMPTY = D_FULL + kNG, RECV_FULL = D_EMPTY + kNG, BUF_FREE = RECV_FULL + kRecv,
  V_FULL = BUF_FREE + kRecv, O_FULL = V_FULL + kNV, MIX_DONE = O_FULL + 1,
  NUM_BARS = MIX_DONE + 1
};

struct __align__(64) Params {
  CUtensorMap p_maps[8];   // BSR values viewed [capacity * 64 lines][64]; box {64, 8 * (i + 1)}
  CUtensorMap v_map;       // V viewed [head-halves][n][64]; box {64, 64, d_v / 64}
  const int32_t* cu;
  SeqTables tab;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const unsigned long long* headmask;
  const int64_t* val_off;
  const float* W;
  float* out;
  unsigned int* status;
  int H_s, H_r, d_v, C, NR, KH, RB, NP;
  int grp;                 // receiver heads per value head (grouped values; 1 = one each)
  int seqs_per_w;          // sequences per mixing matrix (several layers per launch; 0 = one W)
  uint32_t off_p, off_w, off_scr, off_recv, off_v, off_wf, off_bar;
};

__device__ __forceinline__ uint32_t bar_addr(uint32_t base, int i) { return base + 8u * (uint32_t)i; }

__global__ void __launch_bounds__(kThreads, 1) mapped_av_tc_kernel(const __grid_constant__ Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + p.off_bar;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + p.off_bar + 8 * NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int C = p.C;
  const int NP = p.NP;
  const uint32_t crank = tc::cluster_rank();
  const int item = blockIdx.x / C;
  const int2 it = p.tab.items[item];
  const int s = it.x, I = it.y;
  const int seq0 = p.cu[s];                 // V token of key 0
  const int orow0 = p.tab.qoff[s];          // output row of the sequence-local row 0
  const int L = p.cu[s + 1] - seq0;
  const int rb = tab_rb(p.tab, s, I);
  const int u0 = p.row_ptr[rb];
  const int T = p.row_ptr[rb + 1] - u0;
  const int r0 = (int)crank * kG;
  const int G = max(0, min(kG, p.H_r - r0));
  const int c0 = (32 * (int)crank) / C, c1 = (32 * ((int)crank + 1)) / C;
  const uint32_t p_box = (uint32_t)p.RB * 128u;   // one box: RB lines of 128 B
  const uint32_t p_stage = 2u * p_box;
  const uint32_t w_stage = (uint32_t)p.NR * 128u;
  const uint32_t v_stage = (uint32_t)p.d_v * 128u;

  // ---- set-up: barriers, zeroed sender ring and its 1 KB tail (lines the MMA reads past a box
  // must be finite: their weights are zero), W, TMEM ----
  if (tid == 0) {
    for (int i = 0; i < NUM_BARS; ++i) {
      uint32_t cnt = 1;
      if (i >= D_EMPTY && i < D_EMPTY + kNG) cnt = 4;
      if (i >= BUF_FREE && i < BUF_FREE + kRecv) cnt = (uint32_t)C;
      tc::mbar_init(bar_addr(bars, i), cnt);
    }
    misc[1] = 0;
    tc::fence_barrier_init();
  }
  {
    uint4* z = reinterpret_cast<uint4*>(smem + p.off_p);
    const int nz = (int)((NP * p_stage + 1024u) / 16);
    for (int i = tid; i < nz; i += kThreads) z[i] = make_uint4(0, 0, 0, 0);
    float* wf = reinterpret_cast<float*>(smem + p.off_wf);   // W transposed: [H_s][H_r]
    const float* Wl = p.W + (p.seqs_per_w ? (int64_t)(s / p.seqs_per_w) * p.H_r * p.H_s : 0);
    for (int i = tid; i < p.H_r * p.H_s; i += kThreads) {
      const int r = i / p.H_s, h = i - r * p.H_s;
      wf[h * p.H_r + r] = Wl[i];
    }
    tc::fence_proxy_async_smem();
  }
  if (warp == 1) tc::tmem_alloc(smem_u32(misc), kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  tc::cluster_sync();  // every CTA's barriers exist before any remote copy or arrival
  const uint32_t tmem = misc[0];

  if (warp == 0 || (warp >= 8 && warp < 8 + kPWarps - 1)) {
    // ------------------------------ sender slices (chunks round-robin over 4 warps) ------------
    const int pw = warp == 0 ? 0 : warp - 7;
    const int nch = c1 - c0;
    int q = 0;
    if (lane == 0) {
      const uint64_t pol = tc::policy_evict_first();   // each stored tile is read once
      if (pw == 0)
        for (int i = 0; i < 8; ++i) tc::prefetch_tmap(&p.p_maps[i]);
      unsigned long long m_next = T > 0 ? p.headmask[u0] : 0ull;
      int64_t off_next = T > 0 ? p.val_off[u0] : 0;
      for (int t = 0; t < T; ++t) {
        const unsigned long long m = m_next;
        const int64_t off = off_next;
        if (t + 1 < T) {
          m_next = p.headmask[u0 + t + 1];
          off_next = p.val_off[u0 + t + 1];
        }
        const int k = __popcll(m);
        const int k8 = (k + 7) >> 3;
        const int y0 = (int)(off * 64);   // first line of the block
        for (int c = 0; c < nch; ++c, ++q) {
          if ((q % NP) % kPWarps != pw) continue;   // slot q % NP is always loaded by one warp
          const int ps = q % NP;
          if (q >= NP) tc::wait_bar(bar_addr(bars, P_EMPTY + ps), ((q / NP) - 1) & 1, abort_flag, p.status);
          tc::mbar_expect_tx(bar_addr(bars, P_FULL + ps), 2u * (uint32_t)k8 * 8u * 128u);
          const uint32_t dst = sbase + p.off_p + ps * p_stage;
          tc::tma_load_2d_hint(dst, &p.p_maps[k8 - 1], 0, y0 + (2 * (c0 + c)) * k,
                               bar_addr(bars, P_FULL + ps), pol);
          tc::tma_load_2d_hint(dst + p_box, &p.p_maps[k8 - 1], 0, y0 + (2 * (c0 + c) + 1) * k,
                               bar_addr(bars, P_FULL + ps), pol);
        }
      }
      // drain: the final load of every slot, where this warp issued it, has landed (earlier uses
      // of a slot are two phases back and must not be waited on)
      for (int qq = max(0, q - NP); qq < q; ++qq)
        if ((qq % NP) % kPWarps == pw) tc::drain_bar(bar_addr(bars, P_FULL + qq % NP), (qq / NP) & 1);
    }
  } else if (warp == 7) {
    // ------------------------------ W' of each stored block ------------------------------
    // row r = receiver head r; column t = W[r][t-th present sender head]; zero past k and for
    // padding rows. The present-head list comes from two ballots.
    const float* wf = reinterpret_cast<const float*>(smem + p.off_wf);
    unsigned char* hl = smem + p.off_bar + 8 * NUM_BARS + 16;   // 64-byte head list
    unsigned long long m_next = T > 0 ? p.headmask[u0] : 0ull;
    for (int t = 0; t < T; ++t) {
      const unsigned long long m = m_next;
      if (t + 1 < T) m_next = p.headmask[u0 + t + 1];
      const int k = __popcll(m);
      const int ws = t & 1;
      if (t >= 2) tc::wait_bar(bar_addr(bars, W_EMPTY + ws), ((t - 2) >> 1) & 1, abort_flag, p.status);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int h = 32 * half + lane;
        const bool present = (m >> h) & 1ull;
        const unsigned b = __ballot_sync(0xffffffffu, present);
        const int base = half ? __popcll(m & 0xffffffffull) : 0;
        if (present) hl[base + __popc(b & ((1u << lane) - 1u))] = (unsigned char)h;
      }
      __syncwarp();
      if (lane < p.NR) {
        const int r = lane;
        unsigned char* row = smem + p.off_w + ws * w_stage + r * 128;
        const bool real = r < p.H_r;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int tt = 8 * c + e;
            f[e] = (real && tt < k) ? wf[hl[tt] * p.H_r + r] : 0.f;
          }
          uint4 pk;
          pk.x = pack_bf16(f[0], f[1]);
          pk.y = pack_bf16(f[2], f[3]);
          pk.z = pack_bf16(f[4], f[5]);
          pk.w = pack_bf16(f[6], f[7]);
          *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) = pk;
        }
      }
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar_addr(bars, W_FULL + ws));
      __syncwarp();
    }
  } else if (warp == 6 || warp == 11 || warp == 17 || warp == 18) {
    // ------------------------------ V tiles (one warp per receiver head) ----------------------
    // slot rl holds V_rl[J] of the current block; it is refilled once the P.V of the previous
    // block has completed in every CTA of the cluster (the receive-buffer release of that round,
    // which includes this CTA's own), so each slot is used once per block. That barrier cannot
    // run two phases ahead of this wait: its next phase needs this CTA's P.V of block t, which
    // needs the V tiles loaded after it.
    const int vw = warp == 6 ? 0 : warp == 11 ? 1 : warp == 17 ? 2 : 3;
    const int halves = p.d_v / 64;
    if (lane == 0) {
      const uint64_t pol = tc::policy_evict_last();    // V_r[J] is read again by later row blocks
      if (vw == 0) tc::prefetch_tmap(&p.v_map);
      int J_next = T > 0 ? p.col_idx[u0] : 0;
      for (int t = 0; t < T; ++t) {
        const int J = J_next;
        if (t + 1 < T) J_next = p.col_idx[u0 + t + 1];
        if (t >= 1) tc::wait_bar(bar_addr(bars, BUF_FREE + (t - 1) % kRecv), ((t - 1) / kRecv) & 1, abort_flag, p.status);
        for (int rl = vw; rl < G; rl += kVWarps) {
          tc::mbar_expect_tx(bar_addr(bars, V_FULL + rl), v_stage);
          tc::tma_load_3d_hint(sbase + p.off_v + rl * v_stage, &p.v_map, 0, seq0 + J * 64,
                               ((r0 + rl) / p.grp) * halves, bar_addr(bars, V_FULL + rl), pol);
        }
      }
      if (T > 0)
        for (int rl = vw; rl < G; rl += kVWarps) tc::drain_bar(bar_addr(bars, V_FULL + rl), (T - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------ mixing MMAs ------------------------------
    if (lane == 0) {
      const uint32_t id_mix = tc::idesc_bf16(128, p.NR, 1, 0);
      const int nch = c1 - c0;
      const int npair = (nch + 1) >> 1;
      int q = 0;
      int k_next = T > 0 ? __popcll(p.headmask[u0]) : 0;
      for (int t = 0; t < T; ++t) {
        const int ksteps = (k_next + 15) >> 4;
        if (t + 1 < T) k_next = __popcll(p.headmask[u0 + t + 1]);
        const int ws = t & 1;
        tc::wait_bar(bar_addr(bars, W_FULL + ws), (t >> 1) & 1, abort_flag, p.status);
        const uint32_t wb = sbase + p.off_w + ws * w_stage;
        for (int c = 0; c < nch; c += 2) {
          // pair lp of the block goes to readout group lp & 1, which takes its pairs in order
          const int lp = c >> 1, g = lp & 1;
          const int gp = t * ((npair + 1 - g) >> 1) + (lp >> 1);
          const int gs = g * kNGh + gp % kNGh;
          if (gp >= kNGh) tc::wait_bar(bar_addr(bars, D_EMPTY + gs), ((gp / kNGh) - 1) & 1, abort_flag, p.status);
          const int nj = min(2, nch - c);
          for (int j = 0; j < nj; ++j) {
            const int qq = q + c + j, ps = qq % NP;
            tc::wait_bar(bar_addr(bars, P_FULL + ps), (qq / NP) & 1, abort_flag, p.status);
            tc::tc_fence_after();
            const uint32_t pa = sbase + p.off_p + ps * p_stage;
            const uint32_t d = tmem + (uint32_t)kMixCol + (uint32_t)(2 * gs + j) * (uint32_t)p.NR;
            for (int kk = 0; kk < ksteps; ++kk) {
              const uint64_t a = tc::sdesc_sw128(pa + kk * 2048u, p_box, 1024u);
              const uint64_t b = tc::sdesc_sw128(wb + kk * 32u, 16u, 1024u);
              tc::mma_bf16(d, a, b, id_mix, kk > 0 ? 1u : 0u);
            }
          }
          tc::mma_commit(bar_addr(bars, D_FULL + gs));
        }
        q += nch;   // W' of this block is released by the readout of its last pair
      }
      tc::mma_commit(bar_addr(bars, MIX_DONE));
      tc::drain_bar(bar_addr(bars, MIX_DONE), 0);   // every mixing MMA completed before TMEM is freed
    }
  } else if (warp == 12) {
    // ------------------------------ P.V MMAs ------------------------------
    if (lane == 0) {
      const uint32_t id_pv = tc::idesc_bf16(128, 64, 1, 0);
      const uint32_t v_lbo = p.d_v == 128 ? 8192u : 0u;
      const uint16_t all_ctas = (uint16_t)((1u << C) - 1u);
      for (int t = 0; t < T; ++t) {
        const int rs = t % kRecv;
        tc::mbar_expect_tx(bar_addr(bars, RECV_FULL + rs), (uint32_t)G * 8192u);
        tc::wait_bar(bar_addr(bars, RECV_FULL + rs), (t / kRecv) & 1, abort_flag, p.status);
        tc::tc_fence_after();
        tc::fence_proxy_async_smem();  // peers' st.async data, read next by the tensor cores
        for (int rl = 0; rl < G; ++rl) {
          tc::wait_bar(bar_addr(bars, V_FULL + rl), t & 1, abort_flag, p.status);
          tc::tc_fence_after();
          const uint32_t va = sbase + p.off_v + rl * v_stage;
          const uint32_t pb = sbase + p.off_recv + (uint32_t)rs * (kG * 8192u) + (uint32_t)rl * 8192u;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t a = tc::sdesc_sw128(va + kk * 2048u, v_lbo, 1024u);
            const uint64_t b = tc::sdesc_sw128(pb + kk * 32u, 16u, 1024u);
            tc::mma_bf16(tmem + (uint32_t)rl * 64u, a, b, id_pv, (t > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc::mma_commit_to_cluster(bar_addr(bars, BUF_FREE + rs), all_ctas);
      }
      tc::mma_commit(bar_addr(bars, O_FULL));
      tc::drain_bar(bar_addr(bars, O_FULL), 0);   // every P.V MMA completed before TMEM is freed
    }
  } else {
    // ------------------------------ readout, exchange, output (warps 2-5, 13-16) ----------------
    // group eg takes the pairs lp = eg, eg + 2, ... of every block
    const int eg = warp >= 13 ? 1 : 0;
    const int e = warp & 3;               // TMEM lane quarter of this warp
    const uint32_t lane_base = (uint32_t)(32 * e) << 16;
    const int ew = eg * 4 + (warp - (eg ? 13 : 2));   // 0..7
    unsigned char* scr = smem + p.off_scr + ew * 2048;   // [32 heads][32 positions] bf16
    const uint32_t scr_u32 = smem_u32(scr);
    const int o = lane & 3;               // this lane's 16-byte run: positions 8*o .. 8*o+7
    const int rq = lane >> 2;             // this lane's heads: 8*v + rq
    const int nch = c1 - c0;
    const int npair = (nch + 1) >> 1;
    const bool releaser = (warp == 2 || warp == 13) && lane == 0;
    const int npg = (npair + 1 - eg) >> 1;   // pairs of this group per block
    for (int t = 0; t < T; ++t) {
      const int ss = t % kRecv;
      const int q = t * nch;          // this block's first chunk (global order)
      int gp = t * npg;               // its first pair within this group
      // the receive buffers of round t - kRecv are free once every peer's P.V of that round completed
      if (t >= kRecv) tc::wait_bar(bar_addr(bars, BUF_FREE + ss), ((t - kRecv) / kRecv) & 1, abort_flag, p.status);
      const uint32_t recv_local = sbase + p.off_recv + (uint32_t)ss * (kG * 8192u);
      const uint32_t rbar_local = bar_addr(bars, RECV_FULL + ss);
      for (int cc = 2 * eg; cc < nch; cc += 4) {
        // one pair of chunks (cc, cc + 1): both TMEM loads before one wait
        const int gs = eg * kNGh + gp % kNGh;
        const int nj = min(2, nch - cc);
        tc::wait_bar(bar_addr(bars, D_FULL + gs), (gp / kNGh) & 1, abort_flag, p.status);
        // the pair's mixing MMAs completed: their sender slots can be refilled, and after the
        // block's last pair (its commit covers every earlier MMA) the block's W' as well
        if (releaser) {
          for (int jj = 0; jj < nj; ++jj) tc::mbar_arrive(bar_addr(bars, P_EMPTY + (q + cc + jj) % NP));
          if (cc + 2 >= nch) tc::mbar_arrive(bar_addr(bars, W_EMPTY + (t & 1)));
        }
        tc::tc_fence_after();
        // chunk j in the fragment shape: v[j][16 hh + 4 m + k] = position 16 hh + 8 (k >= 2) + lane / 4
        // of this warp's 32, receiver head 8 m + 2 (lane % 4) + (k & 1)
        uint32_t v[2][32];
        const uint32_t ta = tmem + lane_base + (uint32_t)kMixCol + (uint32_t)(2 * gs) * (uint32_t)p.NR;
        if (p.NR == 32) {
          IAMAP_TMEM_LD_FRAG16(ta, v[0]);
          IAMAP_TMEM_LD_FRAG16(ta + (16u << 16), v[0] + 16);
          if (nj == 2) {
            IAMAP_TMEM_LD_FRAG16(ta + 32u, v[1]);
            IAMAP_TMEM_LD_FRAG16(ta + 32u + (16u << 16), v[1] + 16);
          }
        } else {
          IAMAP_TMEM_LD_FRAG8(ta, v[0]);
          IAMAP_TMEM_LD_FRAG8(ta + (16u << 16), v[0] + 16);
          if (nj == 2) {
            IAMAP_TMEM_LD_FRAG8(ta + 16u, v[1]);
            IAMAP_TMEM_LD_FRAG8(ta + 16u + (16u << 16), v[1] + 16);
          }
        }
        tc::tmem_ld_wait();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar_addr(bars, D_EMPTY + gs));
        ++gp;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          if (j >= nj) break;
          const int ch = c0 + cc + j;
          // transpose into [head][32 positions] rows: each 8 positions x 8 heads tile is stored
          // transposed by stmatrix, so that a row holds 16-byte runs of one head; the run of
          // position octet po of head r sits at 16 * (po ^ ((r >> 1) & 3)), which keeps both
          // the stores and the reads below free of bank conflicts
#pragma unroll
          for (int po = 0; po < 4; ++po) {
            const int b = 16 * (po >> 1) + 2 * (po & 1);
            const uint32_t a = scr_u32 + (uint32_t)lane * 64u + ((uint32_t)(po ^ ((lane >> 1) & 3)) << 4);
            const uint32_t q0 = pack_bf16(__uint_as_float(v[j][b]), __uint_as_float(v[j][b + 1]));
            const uint32_t q1 = pack_bf16(__uint_as_float(v[j][b + 4]), __uint_as_float(v[j][b + 5]));
            if (p.NR == 32) {
              const uint32_t q2 = pack_bf16(__uint_as_float(v[j][b + 8]), __uint_as_float(v[j][b + 9]));
              const uint32_t q3 = pack_bf16(__uint_as_float(v[j][b + 12]), __uint_as_float(v[j][b + 13]));
              tc::stmatrix_x4_trans(a, q0, q1, q2, q3);
            } else {
              tc::stmatrix_x4_trans(a, q0, q1, 0u, 0u);   // heads 16-31 do not exist
            }
          }
          __syncwarp();
          const int pos0 = 32 * e;                          // this warp's first position in the chunk
          const int arow = 2 * ch + (pos0 >> 6);            // tile row
          const int jc = ((pos0 & 63) >> 3) + o;            // 16-byte chunk of the row
          const uint32_t row_off = (uint32_t)arow * 128u + ((uint32_t)(jc ^ (arow & 7)) << 4);
#pragma unroll
          for (int vv = 0; vv < 4; ++vv) {
            const int r = 8 * vv + rq;
            if (r < p.H_r) {
              const uint4 val = *reinterpret_cast<const uint4*>(scr + r * 64 + ((o ^ ((r >> 1) & 3)) << 4));
              const uint32_t c2 = (uint32_t)(r >> 2);
              const uint32_t dst = tc::map_to_cta(recv_local + (uint32_t)(r & 3) * 8192u + row_off, c2);
              tc::st_async_v4(dst, val, tc::map_to_cta(rbar_local, c2));
            }
          }
          __syncwarp();
        }
      }
    }
    // output rows (first group): TMEM lane = d_v index, column = rl * 64 + row of the block
    const int dv = 32 * e + lane;
    if (eg == 0) {
      tc::wait_bar(bar_addr(bars, O_FULL), 0, abort_flag, p.status);
      tc::tc_fence_after();
    }
    if (eg == 0 && 32 * e < p.d_v) {
      for (int rl = 0; rl < G; ++rl) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t v[32];
          IAMAP_TMEM_LD32(tmem + lane_base + (uint32_t)(rl * 64 + half * 32), v);
          tc::tmem_ld_wait();
          float* o = p.out + ((int64_t)(orow0 + I * 64 + half * 32) * p.H_r + r0 + rl) * p.d_v + dv;
#pragma unroll
          for (int ii = 0; ii < 32; ++ii)
            if (I * 64 + half * 32 + ii < L)
              o[(int64_t)ii * p.H_r * p.d_v] = T > 0 ? __uint_as_float(v[ii]) : 0.f;
        }
      }
    }
    // the last kRecv exchange rounds: every peer's P.V commit has arrived here and every peer's copy
    // into this CTA has landed, so nothing remote targets this CTA's shared memory once it exits.
    // These waits ignore the abort flag (bounded at 200 ms each): after a timeout elsewhere the
    // other threads skip their waits, and a remote arrival must still not outlive the CTA.
    if (eg == 0)
      for (int t = max(0, T - kRecv); t < T; ++t) {
        tc::drain_bar(bar_addr(bars, BUF_FREE + t % kRecv), (t / kRecv) & 1);
        tc::drain_bar(bar_addr(bars, RECV_FULL + t % kRecv), (t / kRecv) & 1);
      }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
  tc::cluster_sync();
}

}  // namespace tcav

static size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool mapped_av_tc_supported(int H_s, int H_r, int d_v) {
  return H_s >= 1 && H_s <= 64 && H_r >= 1 && H_r <= 32 && (d_v == 64 || d_v == 128);
}

int mapped_av_tc_impl(const MappedAvArgs& a, cudaStream_t stream) {
  using namespace tcav;
  Params p{};
  const int C = (a.H_r + kG - 1) / kG;
  p.C = C;
  p.H_s = a.H_s;
  p.H_r = a.H_r;
  p.d_v = a.d_v;
  p.NR = a.H_r <= 16 ? 16 : 32;
  p.KH = (a.H_s + 15) / 16 * 16;
  p.RB = (a.H_s + 7) / 8 * 8;
  // everything but the sender ring, then as many ring slots as fit (at most kMaxNP)
  const size_t fixed = (size_t)2 * p.NR * 128 + 1024 + (size_t)kRecv * kG * 8192 + (size_t)kNV * a.d_v * 128 +
                       (size_t)kEpiWarps * 2048 + sizeof(float) * (size_t)a.H_r * a.H_s + 8 * NUM_BARS + 96 + 4096;
  const size_t p_stage_b = (size_t)2 * p.RB * 128;
  const size_t budget = 232448 - 1024;
  p.NP = (int)std::min<size_t>(kMaxNP, (budget - fixed - 1024) / p_stage_b);
  if (p.NP < 2) return set_error(IAMAP_ERR_UNSUPPORTED, "mapped_av: sender ring does not fit");
  size_t off = 0;
  p.off_p = (uint32_t)off;
  off += (size_t)p.NP * p_stage_b + 1024;   // ring + tail read past the last box
  off = round_up(off, 1024);
  p.off_w = (uint32_t)off;
  off += (size_t)2 * p.NR * 128;
  off = round_up(off, 1024);
  p.off_recv = (uint32_t)off;
  off += (size_t)kRecv * kG * 8192;
  p.off_v = (uint32_t)off;
  off += (size_t)kNV * a.d_v * 128;
  p.off_scr = (uint32_t)off;
  off += (size_t)kEpiWarps * 2048;
  p.off_wf = (uint32_t)off;
  off += sizeof(float) * (size_t)a.H_r * a.H_s;
  off = round_up(off, 8);
  p.off_bar = (uint32_t)off;
  off += 8 * NUM_BARS + 16 + 64;   // barriers, TMEM address + abort flag, head list
  const size_t smem = off + 1024;  // alignment slack
  if (smem > 232448)
    return set_error(IAMAP_ERR_UNSUPPORTED, "mapped_av needs %zu bytes of shared memory", smem);

  const uint64_t cap = (uint64_t)std::max<int64_t>(a.capacity, 1);
  for (int i = 0; i < 8; ++i) {
    int rc = encode_tmap_2d_bf16(&p.p_maps[i], a.vals, 64, cap * 64, 128, 64, (uint32_t)(8 * (i + 1)));
    if (rc) return rc;
  }
  const int H_kv = a.H_kv > 0 ? a.H_kv : a.H_r;
  p.grp = a.H_r / H_kv;
  const int64_t n_v = a.n_k > 0 ? a.n_k : a.n;
  int rc = encode_tmap_3d_bf16(&p.v_map, a.v, 64, (uint64_t)n_v, (uint64_t)H_kv * (a.d_v / 64),
                               (uint64_t)H_kv * a.d_v * 2, 128, 64, 64, (uint32_t)(a.d_v / 64));
  if (rc) return rc;
  p.cu = a.cu_seqlens;
  p.tab = a.tab;
  p.row_ptr = a.row_ptr;
  p.col_idx = a.col_idx;
  p.headmask = reinterpret_cast<const unsigned long long*>(a.headmask);
  p.val_off = a.val_off;
  p.W = a.W;
  p.seqs_per_w = a.seqs_per_w;
  p.out = a.out;
  p.status = a.status;

  IAMAP_CUDA_CHECK(cudaFuncSetAttribute(mapped_av_tc_kernel,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  if (a.plan.num_rowblocks == 0) return IAMAP_OK;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.plan.num_rowblocks * C), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  IAMAP_CUDA_CHECK(cudaOccupancyMaxActiveClusters(&clusters, mapped_av_tc_kernel, &cfg));
  if (clusters < 1)
    return set_error(IAMAP_ERR_UNSUPPORTED, "a cluster of %d CTAs with %zu bytes each cannot be "
                     "scheduled", C, smem);
  IAMAP_CUDA_CHECK(cudaLaunchKernelEx(&cfg, mapped_av_tc_kernel, p));
  return IAMAP_OK;
}

}  // namespace iamap
