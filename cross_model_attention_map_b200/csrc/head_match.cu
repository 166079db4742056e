// head_match: IAM's calibration step ("IAM: Efficient Inference through Attention Mapping between
// Different-scale LLMs" notes, Method section 1 -- cosine similarity of flattened attention
// matrices -- and section 4 -- for each head of each mapped large layer, the most similar
// small-model head; prompts longer than tau_t are truncated).
//
// 1. maps_kernel<D>: one CTA per (head, row block) computes the causal softmax map rows of the
//    first n_used tokens (two sweeps over the key tiles: row log-sum-exp, then probabilities) and
//    writes them as bf16 64 x 64 tiles in causal-block order, zeros above the diagonal and past
//    n_used. The flattened map of a head is its run of tiles. The squared norm of the bf16 map is
//    accumulated alongside.
// 2. gram_kernel: C_raw = A_large . A_small^T over the flattened maps (split-K, mma.sync,
//    fp32 accumulate, atomic fp32 reduction of the K splits).
// 3. finalize_kernel: the similarity of every (large, small) pair from C_raw and each map's sum and
//    squared norm, and the argmax per large head (lowest small-head index on ties). The method
//    section of the IAM notes compares cosine similarity, Minkowski distance and the Pearson
//    correlation of the flattened maps: cosine = C / (|a| |b|); Pearson = the cosine of the
//    maps less their means over the n_used x n_used entries; Minkowski with p = 2 (Euclidean):
//    |a - b|^2 = |a|^2 + |b|^2 - 2 C, reported negated so that larger is more similar.
// 4. consistency_kernel: how many large heads two mappings (e.g. prefill and a later prefix)
//    send to the same small head (IAM notes, method section 3).
#include "qk_tile.cuh"
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
  __nv_bfloat16* out = p.maps + ((int64_t)head * p.tiles + (int64_t)I * (I + 1) / 2) * kTile * kTile;
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
    uint4* dst = reinterpret_cast<uint4*>(out + (int64_t)J * kTile * kTile);
    for (int c = tid; c < kTile * 8; c += kTileThreads) {
      const int r = c >> 3, ch = c & 7;
      dst[c] = *reinterpret_cast<const uint4*>(stage + r * kTile + ((ch ^ (r & 7)) << 3));
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

// C_raw[M x N] += A[M x K] . B[N x K]^T over one K split. 128 x 128 output tile, 8 warps of
// 64 x 32, K staged 64 at a time through a 3-stage cp.async ring with a 16-byte XOR swizzle.
constexpr int kGBM = 128, kGBN = 128, kGBK = 64, kGStages = 3, kGThreads = 256;

struct GramParams {
  const __nv_bfloat16* A;
  const __nv_bfloat16* B;
  int M, N;
  int64_t K;
  int64_t k_per_split;
  float* C;
};

__global__ void __launch_bounds__(kGThreads) gram_kernel(GramParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  __nv_bfloat16* sA = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sB = sA + kGStages * kGBM * kGBK;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * kGBM, n0 = blockIdx.y * kGBN;
  const int64_t k0 = (int64_t)blockIdx.z * p.k_per_split;
  const int64_t k1 = min(p.K, k0 + p.k_per_split);
  const int nsteps = (int)((k1 - k0 + kGBK - 1) / kGBK);
  const int wm = (warp >> 2) * 64, wn = (warp & 3) * 32;

  auto load_stage = [&](int step, int buf) {
    const int64_t kk = k0 + (int64_t)step * kGBK;
    for (int c = tid; c < kGBM * 8; c += kGThreads) {
      const int r = c >> 3, ch = c & 7;
      const bool va = (m0 + r) < p.M && kk + ch * 8 < k1;
      const __nv_bfloat16* src = p.A + (va ? ((int64_t)(m0 + r) * p.K + kk + ch * 8) : 0);
      cp_async16(smem_u32(sA + (buf * kGBM + r) * kGBK + ((ch ^ (r & 7)) << 3)), src, va);
      const bool vb = (n0 + r) < p.N && kk + ch * 8 < k1;
      const __nv_bfloat16* srb = p.B + (vb ? ((int64_t)(n0 + r) * p.K + kk + ch * 8) : 0);
      cp_async16(smem_u32(sB + (buf * kGBN + r) * kGBK + ((ch ^ (r & 7)) << 3)), srb, vb);
    }
  };

  float acc[4][4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[a][b][e] = 0.f;

  for (int s = 0; s < kGStages - 1; ++s) {
    if (s < nsteps) load_stage(s, s);
    cp_async_commit();
  }
  const int mq = lane >> 3, rr = lane & 7;
  for (int step = 0; step < nsteps; ++step) {
    cp_async_wait<kGStages - 2>();
    __syncthreads();
    const int nxt = step + kGStages - 1;
    if (nxt < nsteps) load_stage(nxt, nxt % kGStages);
    cp_async_commit();
    const int buf = step % kGStages;
    const __nv_bfloat16* A = sA + buf * kGBM * kGBK;
    const __nv_bfloat16* B = sB + buf * kGBN * kGBK;
#pragma unroll
    for (int ks = 0; ks < kGBK / 16; ++ks) {
      uint32_t af[4][4];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        const int row = wm + mt * 16 + (mq & 1) * 8 + rr;
        const int ch = ks * 2 + (mq >> 1);
        ldmatrix_x4(smem_u32(A + row * kGBK + ((ch ^ (row & 7)) << 3)), af[mt][0], af[mt][1],
                    af[mt][2], af[mt][3]);
      }
#pragma unroll
      for (int nt2 = 0; nt2 < 2; ++nt2) {
        const int row = wn + nt2 * 16 + (mq >> 1) * 8 + rr;
        const int ch = ks * 2 + (mq & 1);
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4(smem_u32(B + row * kGBK + ((ch ^ (row & 7)) << 3)), b0, b1, b2, b3);
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          mma_bf16_16816(acc[mt][2 * nt2], af[mt], b0, b1);
          mma_bf16_16816(acc[mt][2 * nt2 + 1], af[mt], b2, b3);
        }
      }
    }
  }
  cp_async_wait<0>();
  const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int m = m0 + wm + mt * 16 + g + (e >= 2 ? 8 : 0);
        const int nn = n0 + wn + nt * 8 + 2 * t4 + (e & 1);
        if (m < p.M && nn < p.N) atomicAdd(p.C + (int64_t)m * p.N + nn, acc[mt][nt][e]);
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
  l.total = l.maps_small + l.maps_large + l.norms + l.craw;
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

int head_match_impl(const HeadMatchArgs& a, cudaStream_t stream) {
  const HmLayout l = hm_layout(a.L_s, a.H_small, a.L_l, a.H_large, a.n_used);
  char* ws = static_cast<char*>(a.ws);
  __nv_bfloat16* maps_small = reinterpret_cast<__nv_bfloat16*>(ws);
  __nv_bfloat16* maps_large = reinterpret_cast<__nv_bfloat16*>(ws + l.maps_small);
  float* norms = reinterpret_cast<float*>(ws + l.maps_small + l.maps_large);
  float* craw = reinterpret_cast<float*>(ws + l.maps_small + l.maps_large + l.norms);
  const int NS = a.L_s * a.H_small, NL = a.L_l * a.H_large;
  IAMAP_CUDA_CHECK(cudaMemsetAsync(norms, 0, l.norms + l.craw, stream));

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

  GramParams gp{};
  gp.A = maps_large;
  gp.B = maps_small;
  gp.M = NL;
  gp.N = NS;
  gp.K = l.tiles * kTile * kTile;
  const int tm = (NL + kGBM - 1) / kGBM, tn = (NS + kGBN - 1) / kGBN;
  DeviceContext* ctx = device_context();
  const int sms = ctx ? ctx->num_sms : 148;
  int splits = (2 * sms + tm * tn - 1) / (tm * tn);
  int64_t kps = (gp.K + splits - 1) / splits;
  kps = (kps + kGBK - 1) / kGBK * kGBK;
  splits = (int)((gp.K + kps - 1) / kps);
  gp.k_per_split = kps;
  gp.C = craw;
  const size_t gsmem = (size_t)kGStages * (kGBM + kGBN) * kGBK * 2;
  IAMAP_CUDA_CHECK(cudaFuncSetAttribute(gram_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)gsmem));
  gram_kernel<<<dim3(tm, tn, splits), kGThreads, gsmem, stream>>>(gp);
  IAMAP_LAUNCH_CHECK("gram_kernel");
  finalize_kernel<<<(NL * 32 + 255) / 256, 256, 0, stream>>>(
      craw, norms + NS, norms, norms + NS + NL + NS, norms + NS + NL, NL, NS, a.metric,
      (float)a.n_used * (float)a.n_used, a.sim, a.argmax);
  IAMAP_LAUNCH_CHECK("finalize_kernel");
  return IAMAP_OK;
}

}  // namespace iamap
