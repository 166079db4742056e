// head_match: IAM's calibration step ("IAM: Efficient Inference through Attention Mapping between
// Different-scale LLMs" notes, Method section 1 -- cosine similarity of flattened attention
// matrices -- and section 4 -- for each head of each mapped large layer, the most similar
// small-model head; prompts longer than tau_t are truncated).
//
// 1. maps_kernel<D>: one CTA per (head, row block) computes the causal softmax map rows of the
//    first n_used tokens (two sweeps over the key tiles: row log-sum-exp, then probabilities) as
//    bf16 64 x 64 tiles in causal-block order, zeros above the diagonal and past n_used. The
//    flattened map of a head is its tiles' rows in order: 64-element chunks c = tile * 64 + row.
//    The maps of all heads are stored chunk-major (chunk c of head hh is the 128-byte line
//    c * heads + hh), so that the Gram reads each chunk of 128 heads as one contiguous 16 KB run.
//    The squared norm and the sum of the bf16 map are accumulated alongside. (Prompts of 1024+
//    tokens take the tcgen05 compress kernels instead, which write the same layout.)
// 2. gram_tc_kernel: C_raw = A_large . A_small^T over the flattened maps on the tcgen05 tensor
//    cores (split-K; operands by TMA with 128-byte swizzle from the chunk-major maps viewed
//    {64, heads, chunks}, fp32 accumulator in TMEM, atomic fp32 reduction of the K splits).
// 3. finalize_kernel: the similarity of every (large, small) pair from C_raw and each map's sum and
//    squared norm, and the argmax per large head (lowest small-head index on ties). The method
//    section of the IAM notes compares cosine similarity, Minkowski distance and the Pearson
//    correlation of the flattened maps: cosine = C / (|a| |b|); Pearson = the cosine of the
//    maps less their means over the n_used x n_used entries; Minkowski with p = 2 (Euclidean):
//    |a - b|^2 = |a|^2 + |b|^2 - 2 C, reported negated so that larger is more similar.
// 4. consistency_kernel: how many large heads two mappings (e.g. prefill and a later prefix)
//    send to the same small head (IAM notes, method section 3).
#include <algorithm>
#include <vector>

#include "qk_tile.cuh"
#include "tc_utils.cuh"
#include "internal.h"

namespace iamap {

struct MapsParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  int n, n_used, H, L_layers;
  int nb;            // row blocks of the n_used prefix
  int64_t tiles;     // causal tiles per head
  float scale_log2;
  __nv_bfloat16* maps;   // [heads][tiles][64][64]
  float* norm2;          // [heads] squared norm of the rounded map
  float* sum1;           // [heads] sum of the rounded map
};

template <int D>
__global__ void __launch_bounds__(kTileThreads) maps_kernel(MapsParams p) {
  __shared__ __align__(128) __nv_bfloat16 sK[2 * kTile * D];
  __shared__ __align__(128) __nv_bfloat16 stage[kTile * kTile];
  __shared__ float red[kTileThreads / 32], red1[kTileThreads / 32];
  const int heads = p.H * p.L_layers;
  const int I = p.nb - 1 - (int)(blockIdx.x / heads);
  const int head = blockIdx.x % heads;
  const int layer = head / p.H, hh = head % p.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
  const int64_t rs = (int64_t)p.H * D;
  const __nv_bfloat16* qb = p.q + ((int64_t)layer * p.n * p.H + hh) * D;
  const __nv_bfloat16* kb = p.k + ((int64_t)layer * p.n * p.H + hh) * D;
  const int L = p.n_used;
  const int row0 = I * kTile;
  const uint32_t sK0 = smem_u32(sK);
  constexpr uint32_t kStage = kTile * D * 2;

  uint32_t qf[D / 16][4];
  const int iA = row0 + 16 * warp + g, iB = iA + 8;
  load_q_frags<D>(qf, qb, rs, iA, iB, L, lane);
  const bool vA = iA < L, vB = iB < L;

  // Sweep 1: row max and sum (online), log2 domain.
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
    scale_mask_tile(acc, iA, iB, J * kTile, p.scale_log2, 0, 0.f, lane);
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) mx = fmaxf(mx, fmaxf(acc[nt][2 * hr], acc[nt][2 * hr + 1]));
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
    }
    __syncthreads();
  }
  const float lA = m_run[0] + lg2(l_run[0]);
  const float lB = m_run[1] + lg2(l_run[1]);

  // Sweep 2: probabilities as bf16 tiles; squared norm of the rounded values.
  // chunk-major: row r of tile t of this head is line (t * 64 + r) * heads + head
  __nv_bfloat16* out = p.maps + ((int64_t)I * (I + 1) / 2 * kTile * heads + head) * kTile;
  float nrm = 0.f, tot = 0.f;
  load_k_tile<D>(sK0, kb, rs, 0, L, tid);
  cp_async_commit();
  for (int J = 0; J <= I; ++J) {
    if (J < I) load_k_tile<D>(sK0 + ((J + 1) & 1) * kStage, kb, rs, (J + 1) * kTile, L, tid);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    float acc[8][4];
    qk_tile<D>(qf, sK0 + (J & 1) * kStage, acc, lane);
    scale_mask_tile(acc, iA, iB, J * kTile, p.scale_log2, 0, 0.f, lane);
    const int rA = 16 * warp + g, rB = rA + 8;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const uint32_t wa = pack_bf16(vA ? ex2(acc[nt][0] - lA) : 0.f, vA ? ex2(acc[nt][1] - lA) : 0.f);
      const uint32_t wb = pack_bf16(vB ? ex2(acc[nt][2] - lB) : 0.f, vB ? ex2(acc[nt][3] - lB) : 0.f);
      const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wa));
      const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wb));
      nrm += fa.x * fa.x + fa.y * fa.y + fb.x * fb.x + fb.y * fb.y;
      tot += (fa.x + fa.y) + (fb.x + fb.y);
      *reinterpret_cast<uint32_t*>(stage + rA * kTile + ((nt ^ (rA & 7)) << 3) + 2 * t4) = wa;
      *reinterpret_cast<uint32_t*>(stage + rB * kTile + ((nt ^ (rB & 7)) << 3) + 2 * t4) = wb;
    }
    __syncthreads();
    __nv_bfloat16* dst = out + (int64_t)J * kTile * heads * kTile;
    for (int c = tid; c < kTile * 8; c += kTileThreads) {
      const int r = c >> 3, ch = c & 7;
      *reinterpret_cast<uint4*>(dst + (int64_t)r * heads * kTile + ch * 8) =
          *reinterpret_cast<const uint4*>(stage + r * kTile + ((ch ^ (r & 7)) << 3));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    nrm += __shfl_xor_sync(0xffffffffu, nrm, o);
    tot += __shfl_xor_sync(0xffffffffu, tot, o);
  }
  if (lane == 0) {
    red[warp] = nrm;
    red1[warp] = tot;
  }
  __syncthreads();
  if (tid == 0) {
    atomicAdd(p.norm2 + head, red[0] + red[1] + red[2] + red[3]);
    atomicAdd(p.sum1 + head, red1[0] + red1[1] + red1[2] + red1[3]);
  }
}

// ------------------------------------------------------------------------------------------------
// Gram on tcgen05: CTA (M tile of 128 large heads, N tile of BN small heads, K split). Warp 0
// loads A, warp 1 loads B (one 64-element K step per stage, 5 stages), lane 0 of warp 2 issues
// 4 MMAs (128 x BN x 16) per stage and frees the stage with a commit; warps 2-5 then read the
// accumulator (TMEM lane = large head, column = small head) and add it into C.
// ------------------------------------------------------------------------------------------------
constexpr int kGtStages = 5, kGtThreads = 192;

struct GramTcParams {
  CUtensorMap a_map;   // maps_large viewed {64, M heads, K / 64 chunks} bf16, box {64, 128, 1}
  CUtensorMap b_map;   // maps_small viewed {64, N heads, K / 64 chunks} bf16, box {64, BN, 1}
  int M, N, BN;
  int64_t K, k_per_split;
  float* C;
  unsigned int* status;
};

__global__ void __launch_bounds__(kGtThreads, 1) gram_tc_kernel(const __grid_constant__ GramTcParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t a_stage = 128u * 128u, b_stage = (uint32_t)p.BN * 128u;
  const uint32_t stage = a_stage + b_stage;
  uint64_t* bar_mem = reinterpret_cast<uint64_t*>(smem + kGtStages * stage);
  uint32_t* misc = reinterpret_cast<uint32_t*>(bar_mem + 2 * kGtStages + 1);   // [0] tmem [1] abort
  const uint32_t bars = smem_u32(bar_mem);
  auto FULL = [&](int i) { return bars + 8u * (uint32_t)i; };
  auto EMPTY = [&](int i) { return bars + 8u * (uint32_t)(kGtStages + i); };
  const uint32_t DONE = bars + 8u * (uint32_t)(2 * kGtStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * 128, n0 = blockIdx.y * p.BN;
  const int64_t k0 = (int64_t)blockIdx.z * p.k_per_split;
  const int64_t k1 = min(p.K, k0 + p.k_per_split);
  const int nsteps = (int)((k1 - k0) / 64);   // K and the split are multiples of 64

  if (tid == 0) {
    for (int i = 0; i < kGtStages; ++i) {
      tc::mbar_init(FULL(i), 2);    // one expect_tx arrival from each producer
      tc::mbar_init(EMPTY(i), 1);
    }
    tc::mbar_init(DONE, 1);
    misc[1] = 0;
    tc::fence_barrier_init();
  }
  if (warp == 2) tc::tmem_alloc(smem_u32(misc), 256);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp < 2) {
    if (lane == 0) {
      const CUtensorMap* map = warp == 0 ? &p.a_map : &p.b_map;
      const uint32_t off = warp == 0 ? 0u : a_stage;
      const uint32_t bytes = warp == 0 ? a_stage : b_stage;
      const int y = warp == 0 ? m0 : n0;
      tc::prefetch_tmap(map);
      for (int st = 0; st < nsteps; ++st) {
        const int b = st % kGtStages;
        if (st >= kGtStages)
          tc::wait_bar(EMPTY(b), ((st / kGtStages) - 1) & 1, abort_flag, p.status);
        tc::mbar_expect_tx(FULL(b), bytes);
        tc::tma_load_3d(sbase + b * stage + off, map, 0, y, (int)(k0 / 64 + st), FULL(b));
      }
      for (int st = max(0, nsteps - kGtStages); st < nsteps; ++st)
        tc::drain_bar(FULL(st % kGtStages), (st / kGtStages) & 1);
    }
  } else {
    if (warp == 2 && lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(128, p.BN, 0, 0);
      for (int st = 0; st < nsteps; ++st) {
        const int b = st % kGtStages;
        tc::wait_bar(FULL(b), (st / kGtStages) & 1, abort_flag, p.status);
        tc::tc_fence_after();
        const uint32_t sa = sbase + b * stage, sb = sa + a_stage;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc::mma_bf16(tmem, tc::sdesc_sw128(sa + kk * 32u, 16u, 1024u),
                       tc::sdesc_sw128(sb + kk * 32u, 16u, 1024u), idesc,
                       (st > 0 || kk > 0) ? 1u : 0u);
        tc::mma_commit(EMPTY(b));
      }
      tc::mma_commit(DONE);
    }
    __syncwarp();
    // accumulator readout: warp w reads TMEM lane quarter w % 4
    tc::wait_bar(DONE, 0, abort_flag, p.status);
    tc::tc_fence_after();
    const int q = warp & 3;
    const int m = m0 + 32 * q + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(32 * q) << 16);
    for (int c0 = 0; c0 < p.BN; c0 += 16) {
      uint32_t v[16];
      IAMAP_TMEM_LD16(t_lane + (uint32_t)c0, v);
      tc::tmem_ld_wait();
      if (nsteps > 0 && m < p.M)
#pragma unroll
        for (int e = 0; e < 16; ++e)
          if (n0 + c0 + e < p.N) atomicAdd(p.C + (int64_t)m * p.N + n0 + c0 + e, __uint_as_float(v[e]));
    }
    if (warp == 2 && lane == 0) tc::drain_bar(DONE, 0);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 256);
  }
}

// One warp per large head: similarity row and argmax (ties: lowest index).
__global__ void finalize_kernel(const float* __restrict__ craw, const float* __restrict__ n2_large,
                                const float* __restrict__ n2_small, const float* __restrict__ s1_large,
                                const float* __restrict__ s1_small, int M, int N, int metric,
                                float n_elems, float* __restrict__ sim, int32_t* __restrict__ argmax) {
  const int m = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (m >= M) return;
  const float nl2 = n2_large[m], sl = s1_large[m];
  const float inv_n = 1.f / n_elems;
  const float var_l = fmaxf(nl2 - sl * sl * inv_n, 0.f);
  float best = -INFINITY;
  int bi = 0x7fffffff;
  for (int s = lane; s < N; s += 32) {
    const float cr = craw[(int64_t)m * N + s];
    float c;
    if (metric == IAMAP_SIM_PEARSON) {
      const float ss = s1_small[s];
      const float var_s = fmaxf(n2_small[s] - ss * ss * inv_n, 0.f);
      c = (cr - sl * ss * inv_n) / sqrtf(var_l * var_s);
    } else if (metric == IAMAP_SIM_EUCLIDEAN) {
      c = -sqrtf(fmaxf(nl2 + n2_small[s] - 2.f * cr, 0.f));
    } else {
      c = cr / (sqrtf(nl2) * sqrtf(n2_small[s]));
    }
    if (sim) sim[(int64_t)m * N + s] = c;
    if (c > best) {
      best = c;
      bi = s;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ob > best || (ob == best && oi < bi)) {
      best = ob;
      bi = oi;
    }
  }
  if (lane == 0) argmax[m] = bi;
}

// agree = number of i < n with a[i] == b[i] (one CTA).
__global__ void __launch_bounds__(1024) consistency_kernel(const int32_t* __restrict__ a,
                                                           const int32_t* __restrict__ b, int n,
                                                           int32_t* __restrict__ agree) {
  __shared__ int part[32];
  int c = 0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) c += a[i] == b[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += part[w];
    *agree = t;
  }
}

int consistency_impl(const int32_t* a, const int32_t* b, int n, int32_t* agree,
                     cudaStream_t stream) {
  consistency_kernel<<<1, 1024, 0, stream>>>(a, b, n, agree);
  IAMAP_LAUNCH_CHECK("consistency_kernel");
  return IAMAP_OK;
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct HmLayout {
  int nb;
  int64_t tiles;
  size_t maps_small, maps_large, norms, craw, total;
  // tensor-core maps: per model, row log-sum-exp, scheduling tables, cu and token offsets
  size_t lse_small, lse_large, tab_small, tab_large, seq_small, seq_large;
};

static HmLayout hm_layout(int L_s, int H_small, int L_l, int H_large, int n_used) {
  HmLayout l;
  l.nb = (n_used + kTile - 1) / kTile;
  l.tiles = (int64_t)l.nb * (l.nb + 1) / 2;
  const size_t per_head = (size_t)l.tiles * kTile * kTile * 2;
  const size_t NS = (size_t)L_s * H_small, NL = (size_t)L_l * H_large;
  l.maps_small = align256(per_head * NS);
  l.maps_large = align256(per_head * NL);
  l.norms = align256(sizeof(float) * 2 * (NS + NL));   // squared norms, then sums
  l.craw = align256(sizeof(float) * NS * NL);
  l.lse_small = align256(sizeof(float) * NS * (size_t)n_used);
  l.lse_large = align256(sizeof(float) * NL * (size_t)n_used);
  l.tab_small = align256(seq_tables_bytes(L_s, (int64_t)L_s * l.nb));
  l.tab_large = align256(seq_tables_bytes(L_l, (int64_t)L_l * l.nb));
  l.seq_small = align256(sizeof(int32_t) * 2 * (size_t)(L_s + 1));
  l.seq_large = align256(sizeof(int32_t) * 2 * (size_t)(L_l + 1));
  l.total = l.maps_small + l.maps_large + l.norms + l.craw + l.lse_small + l.lse_large +
            l.tab_small + l.tab_large + l.seq_small + l.seq_large;
  return l;
}

size_t head_match_ws_bytes(int L_s, int H_small, int L_l, int H_large, int n_used) {
  return hm_layout(L_s, H_small, L_l, H_large, n_used).total;
}

template <int D>
static int launch_maps(const MapsParams& p, cudaStream_t stream) {
  const int64_t grid = (int64_t)p.nb * p.H * p.L_layers;
  if (grid > 0) {
    maps_kernel<D><<<(unsigned)grid, kTileThreads, 0, stream>>>(p);
    IAMAP_LAUNCH_CHECK("maps_kernel");
  }
  return IAMAP_OK;
}

// cu[s] = s * n_used (s <= L), tok0[s] = s * n (s < L): the layers of a [L, n, H, d] tensor as
// sequences of n_used tokens.
__global__ void hm_seq_kernel(int L, int n, int n_used, int32_t* cu, int32_t* tok0) {
  for (int s = threadIdx.x; s <= L; s += blockDim.x) {
    cu[s] = s * n_used;
    tok0[s] = s * n;
  }
}

// Maps of one model on the tensor cores: row statistics (compress stage 1 without masses), then
// every causal tile of every head written head-major with the maps' sums and squared norms.
static int maps_tc(const void* q, const void* k, int L, int H, int d, int n, int n_used,
                   int nb, int64_t tiles, float* lse, char* tab_ws, size_t tab_bytes,
                   int32_t* seq, __nv_bfloat16* maps, float* norm2, float* sum1,
                   unsigned int* status, cudaStream_t stream) {
  std::vector<int32_t> cu_host(L + 1);
  for (int s = 0; s <= L; ++s) cu_host[s] = s * n_used;
  CompressArgs c;
  int rc = make_plan(cu_host.data(), L, kTile, (int64_t)L * n_used, &c.plan);
  if (rc) return rc;
  int32_t* cu = seq;
  int32_t* tok0 = seq + (L + 1);
  hm_seq_kernel<<<1, 256, 0, stream>>>(L, n, n_used, cu, tok0);
  IAMAP_LAUNCH_CHECK("hm_seq_kernel");
  if (seq_tables_bytes(L, c.plan.num_rowblocks) > tab_bytes)
    return set_error(IAMAP_ERR_WORKSPACE, "head_match: scheduling tables do not fit");
  c.tab = carve_seq_tables(tab_ws, L, c.plan.num_rowblocks);
  rc = launch_build_tables(cu, L, kTile, c.plan.max_nb, c.tab, stream);
  if (rc) return rc;
  c.q = q;
  c.k = k;
  c.cu_seqlens = cu;
  c.num_seqs = L;
  c.n = (int64_t)L * n_used;
  c.n_tok = (int64_t)L * n;
  c.tok0 = tok0;
  c.H_s = H;
  c.d = d;
  c.tau = 1.f;
  c.lse = lse;
  c.mass = nullptr;
  c.status = status;
  rc = compress_stats_tc_launch(c, stream);
  if (rc) return rc;
  c.lse_in = lse;
  c.dense = 1;
  c.dense_tiles = tiles;
  c.vals = maps;
  c.capacity = (int64_t)L * H * tiles;
  c.norm2 = norm2;
  c.sum1 = sum1;
  (void)nb;
  return compress_extract_tc_launch(c, stream);
}

int head_match_impl(const HeadMatchArgs& a, cudaStream_t stream) {
  const HmLayout l = hm_layout(a.L_s, a.H_small, a.L_l, a.H_large, a.n_used);
  char* ws = static_cast<char*>(a.ws);
  __nv_bfloat16* maps_small = reinterpret_cast<__nv_bfloat16*>(ws);
  __nv_bfloat16* maps_large = reinterpret_cast<__nv_bfloat16*>(ws + l.maps_small);
  float* norms = reinterpret_cast<float*>(ws + l.maps_small + l.maps_large);
  float* craw = reinterpret_cast<float*>(ws + l.maps_small + l.maps_large + l.norms);
  const int NS = a.L_s * a.H_small, NL = a.L_l * a.H_large;
  IAMAP_CUDA_CHECK(cudaMemsetAsync(norms, 0, l.norms + l.craw, stream));

  // Maps on the tensor cores (the tcgen05 compress kernels) for prompts of 1024+ tokens: at
  // n_used = 1024 a calibration took 0.975 ms this way and 1.037 ms with the mma.sync kernel on
  // a B200. Shorter prompts keep the mma.sync kernel, whose CTAs need no TMEM set-up.
  const bool tc_maps = a.n_used >= 1024 && compress_tc_supported(a.d_small, l.nb) &&
                       compress_tc_supported(a.d_large, l.nb);
  if (tc_maps) {
    char* p = ws + l.maps_small + l.maps_large + l.norms + l.craw;
    float* lse_s = reinterpret_cast<float*>(p);
    float* lse_l = reinterpret_cast<float*>(p + l.lse_small);
    char* tab_s = p + l.lse_small + l.lse_large;
    char* tab_l = tab_s + l.tab_small;
    int32_t* seq_s = reinterpret_cast<int32_t*>(tab_l + l.tab_large);
    int32_t* seq_l = reinterpret_cast<int32_t*>(tab_l + l.tab_large + l.seq_small);
    int rc = maps_tc(a.q_small, a.k_small, a.L_s, a.H_small, a.d_small, a.n, a.n_used, l.nb,
                     l.tiles, lse_s, tab_s, l.tab_small, seq_s, maps_small, norms,
                     norms + NS + NL, a.status, stream);
    if (!rc)
      rc = maps_tc(a.q_large, a.k_large, a.L_l, a.H_large, a.d_large, a.n, a.n_used, l.nb,
                   l.tiles, lse_l, tab_l, l.tab_large, seq_l, maps_large, norms + NS,
                   norms + NS + NL + NS, a.status, stream);
    if (rc) return rc;
  } else {
  MapsParams ps{};
  ps.q = static_cast<const __nv_bfloat16*>(a.q_small);
  ps.k = static_cast<const __nv_bfloat16*>(a.k_small);
  ps.n = a.n;
  ps.n_used = a.n_used;
  ps.H = a.H_small;
  ps.L_layers = a.L_s;
  ps.nb = l.nb;
  ps.tiles = l.tiles;
  ps.scale_log2 = kLog2e / sqrtf((float)a.d_small);
  ps.maps = maps_small;
  ps.norm2 = norms;
  ps.sum1 = norms + NS + NL;
  int rc = a.d_small == 64 ? launch_maps<64>(ps, stream) : launch_maps<128>(ps, stream);
  if (rc) return rc;
  MapsParams pl = ps;
  pl.q = static_cast<const __nv_bfloat16*>(a.q_large);
  pl.k = static_cast<const __nv_bfloat16*>(a.k_large);
  pl.H = a.H_large;
  pl.L_layers = a.L_l;
  pl.scale_log2 = kLog2e / sqrtf((float)a.d_large);
  pl.maps = maps_large;
  pl.norm2 = norms + NS;
  pl.sum1 = norms + NS + NL + NS;
  rc = a.d_large == 64 ? launch_maps<64>(pl, stream) : launch_maps<128>(pl, stream);
  if (rc) return rc;
  }

  {
    GramTcParams gp{};
    const int64_t K = l.tiles * kTile * kTile;
    const int ntn = (NS + 255) / 256;                       // N tiles of at most 256 small heads
    gp.BN = ((NS + ntn - 1) / ntn + 15) / 16 * 16;
    gp.M = NL;
    gp.N = NS;
    gp.K = K;
    gp.C = craw;
    gp.status = a.status;
    // chunk-major maps: {64 elements, heads, K / 64 chunks}; heads past N read as zeros
    int rc2 = encode_tmap_3d_bf16(&gp.a_map, maps_large, 64, (uint64_t)NL, (uint64_t)(K / 64),
                                  128, (uint64_t)NL * 128, 64, 128, 1);
    if (!rc2) rc2 = encode_tmap_3d_bf16(&gp.b_map, maps_small, 64, (uint64_t)NS, (uint64_t)(K / 64),
                                        128, (uint64_t)NS * 128, 64, (uint32_t)gp.BN, 1);
    if (rc2) return rc2;
    const int tm = (NL + 127) / 128, tn = (NS + gp.BN - 1) / gp.BN;
    DeviceContext* ctx = device_context();
    const int sms = ctx ? ctx->num_sms : 148;
    int splits = std::max(1, sms / (tm * tn));
    int64_t kps = (K + splits - 1) / splits;
    kps = (kps + 63) / 64 * 64;
    splits = (int)((K + kps - 1) / kps);
    gp.k_per_split = kps;
    const size_t gsmem = 1024 + (size_t)kGtStages * (128 * 128 + (size_t)gp.BN * 128) +
                         8 * (2 * kGtStages + 1) + 16;
    IAMAP_CUDA_CHECK(cudaFuncSetAttribute(gram_tc_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gsmem));
    gram_tc_kernel<<<dim3(tm, tn, splits), kGtThreads, gsmem, stream>>>(gp);
    IAMAP_LAUNCH_CHECK("gram_tc_kernel");
  }
  finalize_kernel<<<(NL * 32 + 255) / 256, 256, 0, stream>>>(
      craw, norms + NS, norms, norms + NS + NL + NS, norms + NS + NL, NL, NS, a.metric,
      (float)a.n_used * (float)a.n_used, a.sim, a.argmax);
  IAMAP_LAUNCH_CHECK("finalize_kernel");
  return IAMAP_OK;
}

}  // namespace iamap
