// map_compress on the 5th-generation tensor cores (tcgen05, TMEM accumulators, TMA operand loads).
//
// Same two stages as compress.cu (MapFlow news page, "PKU MapFlow: cross-model attention map
// reuse", storage-and-execution part, first component: block statistics first, then extraction
// of the blocks kept by cumulative attention probability), with the work of one CTA widened to a
// pair of row blocks (I0 = 2P, I1 = 2P + 1: 128 query rows, one per TMEM lane) of one sender head.
//
// Stage 1 (stats_tc_kernel): S = Q K^T for 128 keys at a time (column blocks 2T, 2T + 1) lands in
// one of two 128-column TMEM buffers (tile T in buffer T % 2). Sixteen softmax warps, four per SM
// sub-partition, read it back, one thread per (row, column block): the warps of even tiles and
// those of odd tiles run side by side, so that the exponentials of one set overlap the waits of
// the other. The block's log2-sum c_iJ = log2 sum_j 2^(s_ij log2(e)/sqrt(d)) is kept in TMEM
// column 256 + J. Afterwards the same threads form lse_i from the c values, the block masses
// sum_i 2^(c_iJ - lse_i) (a 32 x 32 butterfly per warp sums over rows), and the cumulative-mass
// choice of each row block. Rows with more than 256 column blocks (sequences longer than 16384
// tokens) take the mma.sync kernel instead.
//
// Stage 2 (extract_tc_kernel): for every column block J that this head keeps in I0 or I1,
// S = Q K_J^T (128 x 64) is recomputed into TMEM; two groups of four warps take alternate blocks
// and write exp(s - lse) as bf16 rows of the stored tiles, through a per-warp staging buffer so
// that each 128-byte tile row leaves as one coalesced run (rows of the k present heads of a
// stored block are interleaved: row i of head rank t is line i * k + t of the block).
//
// Roles: stats (576 threads) warps 0-15 softmax, warp 16 TMA producer (lanes 0 and 1: the two
// 64-dim panels of each key tile), warp 17 MMA issuer and TMEM owner; extract (320 threads)
// warps 0-7 writers, warp 8 TMA producer, warp 9 MMA issuer and TMEM owner. Every wait is bounded
// (2 s; then IAMAP_DEV_TIMEOUT and an orderly exit).
#include <algorithm>

#include "tc_utils.cuh"
#include "exp2_fma.cuh"
#include "internal.h"

namespace iamap {
namespace tccomp {

constexpr int kRows = 128;         // query rows per CTA (row blocks 2P, 2P + 1)
constexpr int kThreads = 320;      // extract: warps 0-7 writers, 8 TMA, 9 MMA
constexpr int kSThreads = 576;     // stats: warps 0-15 softmax, 16 TMA, 17 MMA
constexpr int kSMmaWarp = 17;
constexpr int kSoft = 512;         // stats: softmax threads
constexpr int kSStages = 4;        // stats: key-tile ring (128 keys per tile)
constexpr int kXStages = 2;        // extract: key-tile ring (64 keys per tile)
constexpr int kCCol = 256;         // stats: TMEM column of c_i0
constexpr int kMaxNb = 256;        // stats: column blocks per row kept in TMEM
constexpr uint32_t kPanel128 = 128u * 128u;   // 128 rows x 64 bf16 (one 128-byte swizzle span)
constexpr uint32_t kPanel64 = 64u * 128u;

enum { Q_FULL = 0, K_FULL = 1, K_EMPTY = K_FULL + kSStages, S_FULL = K_EMPTY + kSStages,
       S_EMPTY = S_FULL + 2, NUM_BARS = S_EMPTY + 2 };
constexpr int kXBufs = 4;          // extract: S buffers of 64 TMEM columns (two per writer group)
enum { XQ_FULL = 0, XK_FULL = 1, XK_EMPTY = XK_FULL + kXStages, XS_FULL = XK_EMPTY + kXStages,
       XS_EMPTY = XS_FULL + kXBufs, X_NUM_BARS = XS_EMPTY + kXBufs };
// extract with the sender's own output (O_s = P V_s accumulated in TMEM): a ring of value tiles,
// two staging buffers per writer group that hold the bf16 P tile the P.V MMA reads, and the
// completion of the last P.V MMA
constexpr int kVStages = 3;
constexpr int kOLag = 2;           // P.V of block t is issued after the QK^T of block t + kOLag
enum { XV_FULL = X_NUM_BARS, XV_EMPTY = XV_FULL + kVStages, XP_READY = XV_EMPTY + kVStages,
       XP_FREE = XP_READY + 4, XO_FULL = XP_FREE + 4, XO_NUM_BARS = XO_FULL + 1 };

struct StatsParams {
  CUtensorMap q_map;   // {64, n, H_s * D / 64} bf16, box {64, 128, 1}
  CUtensorMap k_map;   // same geometry
  const int32_t* cu;
  const int32_t* tok0;   // first q/k token of each sequence; null: cu (packed sequences)
  SeqTables tab;
  int64_t n, ncb;
  int H_s;
  float scale_log2;
  int bias_window;
  float bias_log2;
  float tau;
  float* lse;
  float* mass;           // null: row statistics only (no masses, no choice)
  int head_group;        // heads per group of the grid order
  unsigned long long* headmask_dense;
  unsigned int* status;
};

struct ExtractParams {
  CUtensorMap q_map;   // box {64, 128, 1}
  CUtensorMap k_map;   // box {64, 64, 1}
  const int32_t* cu;
  const int32_t* tok0;   // as in StatsParams
  SeqTables tab;
  int64_t n;
  int H_s;
  float scale_log2;
  int bias_window;
  float bias_log2;
  int head_group;        // heads per group of the grid order
  const float* lse;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const unsigned long long* headmask;
  const int64_t* val_off;
  __nv_bfloat16* vals;
  int64_t capacity;
  unsigned int* status;
  // dense mode (head_match maps): every causal tile of every head, chunk-major: row r of tile
  // t = I(I+1)/2 + J of head hh = s * H_s + h is the 128-byte line (t * 64 + r) * dense_heads + hh,
  // so that one 64-element chunk of the flattened maps of all heads is contiguous; with the
  // sum and the squared norm of each head's rounded map added into sum1 / norm2
  int dense;
  int64_t dense_tiles;
  int dense_heads;
  CUtensorMap dense_map;   // dense mode: vals viewed {64, dense_heads, dense_tiles * 64}, box {64, 1, 32}
  float* norm2;
  float* sum1;
  // sender output (extract_tc_kernel<D, true>): V_s bf16 viewed {64, n_k, H_s * d_vs / 64}, box
  // {64, 64, d_vs / 64}; o_s fp32 [n, H_s, d_vs]
  CUtensorMap vs_map;
  float* o_s;
  int d_vs;
};

__device__ __forceinline__ uint32_t bar_addr(uint32_t bars, int i) { return bars + 8u * (uint32_t)i; }

__device__ __forceinline__ void tmem_st1(uint32_t taddr, float x) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(__float_as_uint(x))
               : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// x[e] = this lane's value of column e; returns the sum over the warp's 32 lanes of column
// `lane` (31 shuffles: each step halves the columns a lane holds).
__device__ __forceinline__ float transpose_sum32(float (&x)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool upper = (lane & w) != 0;
#pragma unroll
    for (int e = 0; e < w; ++e) {
      const float send = upper ? x[e] : x[e + w];
      const float keep = upper ? x[e + w] : x[e];
      x[e] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  return x[0];
}

// Exclusive prefix sums of x[0..n) (n <= 256) in place, by one warp.
__device__ __forceinline__ void warp_exclusive_scan256(float* x, int n, int lane) {
  float loc[8];
  float tot = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int idx = lane * 8 + e;
    const float v = idx < n ? x[idx] : 0.f;
    loc[e] = tot;
    tot += v;
  }
  float inc = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  const float base = inc - tot;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int idx = lane * 8 + e;
    if (idx < n) x[idx] = base + loc[e];
  }
}

__device__ __forceinline__ unsigned char* align1024(unsigned char* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

// One thread's 64 logits of column block J (keys j0 .. j0 + 63) of row i: x_j = s_j * sc
// (+ bias_log2 where 0 <= i - j < bias_window), x_j = -inf above the diagonal. The block's
// log2-sum c = log2 sum_j 2^(x_j) = m + log2 sum_j 2^(x_j - m) with m = max_j x_j is taken in two
// passes, the max and then the exponentials, so that other work can sit between them.

// A block with every key present and no bias: max of the raw scores (3-input max).
__device__ __forceinline__ float raw_max64(const uint32_t (&v)[64]) {
  float m[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) m[k] = fmaxf(__uint_as_float(v[k]), __uint_as_float(v[k + 4]));
#pragma unroll
  for (int e = 8; e < 64; e += 8) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a = __uint_as_float(v[e + k]), b = __uint_as_float(v[e + 4 + k]);
      asm("max.f32 %0, %0, %1, %2;" : "+f"(m[k]) : "f"(a), "f"(b));
    }
  }
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(m[0]), "f"(m[1]), "f"(fmaxf(m[2], m[3])));
  return r;
}

// Any other block: the x_j replace v (scaled, biased, masked); returns their max.
__device__ __forceinline__ float masked_max64(uint32_t (&v)[64], int i, int j0, float sc,
                                              int bias_window, float bias_log2) {
  float m8[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) m8[k] = -INFINITY;
#pragma unroll
  for (int e = 0; e < 64; ++e) {
    const int j = j0 + e;
    float y = __uint_as_float(v[e]) * sc;
    if (bias_window > 0 && i - j >= 0 && i - j < bias_window) y += bias_log2;
    y = j > i ? -INFINITY : y;
    v[e] = __float_as_uint(y);
    m8[e & 7] = fmaxf(m8[e & 7], y);
  }
  return fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
               fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
}

// Number of the 32 column pairs of a plain block whose exponentials run on the FMA pipe
// (exp2_fma.cuh); the rest use ex2 on the MUFU unit. 0 by default: on a B200, prefill8k stats
// took 0.44 ms with 0 pairs, 0.45 with 8, 0.46 with 12 and 0.50 with 16 (at 1965 MHz), since the
// MUFU unit is not this loop's only limit and the polynomial costs more issue slots than it frees.
#ifndef IAMAP_STATS_FMA_PAIRS
#define IAMAP_STATS_FMA_PAIRS 0
#endif
constexpr int kFmaPairs = IAMAP_STATS_FMA_PAIRS;

__device__ __forceinline__ constexpr bool fma_pair(int q) {
  return (q * kFmaPairs) % 32 < kFmaPairs;   // spread evenly over the block
}

// sum_j 2^(s_j * sc + nm) over a plain block (nm = -max_j s_j * sc), packed pairs.
__device__ __forceinline__ float plain_exp2_sum64(const uint32_t (&v)[64], float sc, float nm) {
  const uint64_t sc2 = f2_splat(sc), nm2 = f2_splat(nm);
  uint64_t acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = f2_splat(0.f);
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const uint64_t x = f2_fma(f2_pack(__uint_as_float(v[2 * q]), __uint_as_float(v[2 * q + 1])),
                              sc2, nm2);
    uint64_t e;
    if (fma_pair(q)) {
      e = exp2_fma_x2(x);
    } else {
      float x0, x1;
      f2_unpack(x, x0, x1);
      e = f2_pack(ex2(x0), ex2(x1));
    }
    acc[q & 3] = f2_add(acc[q & 3], e);
  }
  const uint64_t t = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
  float a, b;
  f2_unpack(t, a, b);
  return a + b;
}

// sum_j 2^(x_j - m) over a block whose x_j are in v (masked_max64), m > -inf.
__device__ __forceinline__ float masked_exp2_sum64(const uint32_t (&v)[64], float m) {
  float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int e = 0; e < 64; ++e) s4[e & 3] += ex2(__uint_as_float(v[e]) - m);
  return (s4[0] + s4[1]) + (s4[2] + s4[3]);
}

// ------------------------------------------------------------------------------------------------
// Stage 1: block statistics, masses and the per-head choice
// ------------------------------------------------------------------------------------------------

template <int D>
__global__ void __launch_bounds__(kSThreads, 1) stats_tc_kernel(const __grid_constant__ StatsParams p) {
  constexpr int NPAN = D / 64;
  constexpr uint32_t kQBytes = NPAN * kPanel128;
  constexpr uint32_t kKStage = NPAN * kPanel128;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = align1024(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase, sK = sbase + kQBytes;
  float* aux = reinterpret_cast<float*>(smem + kQBytes + kSStages * kKStage);
  float* ml_m = aux;                  // [4][128] max (log2) of each softmax group's c values
  float* ml_l = ml_m + 4 * kRows;     // [4][128] their sums of exponentials
  float* lse_s = ml_l + 4 * kRows;    // [128] row lse (log2)
  float* part = lse_s + kRows;        // [4][256] per-quarter column sums
  float* mass_s = part + 4 * kMaxNb;  // [2][256]
  float* sorted_s = mass_s + 2 * kMaxNb;
  int* rank_s = reinterpret_cast<int*>(sorted_s + 2 * kMaxNb);
  uint64_t* bar_mem = reinterpret_cast<uint64_t*>(rank_s + 2 * kMaxNb);
  uint32_t* misc = reinterpret_cast<uint32_t*>(bar_mem + NUM_BARS);   // [0] tmem, [1] abort
  const uint32_t bars = smem_u32(bar_mem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // grid order (head group, pair, head in group): the CTAs resident at one time read the keys
  // of one group of head_group heads, which fit in L2 together, while neighbouring CTAs still
  // read neighbouring heads of one key tile (contiguous in the token-major K)
  const int num_pairs = (int)(gridDim.x / (unsigned)p.H_s);
  const int hgs = p.head_group;
  const int g0 = (int)(blockIdx.x / (unsigned)(num_pairs * hgs)) * hgs;   // first head of the group
  const int gsz = min(hgs, p.H_s - g0);
  const int rem = blockIdx.x - g0 * num_pairs;
  const int pair = rem / gsz;
  const int h = g0 + (rem - pair * gsz);
  const int2 it = p.tab.pairs[pair];
  const int s = it.x, I0 = it.y, P = I0 >> 1;
  const int row0 = p.tab.qoff[s];           // packed lse row of the sequence-local row 0
  const int ktok0 = p.tok0 ? p.tok0[s] : p.cu[s];   // k token of key 0
  const int qtok0 = p.tok0 ? p.tok0[s] : row0;      // q token of row 0
  const int L = p.cu[s + 1] - p.cu[s];
  const int nb = p.tab.nb[s];
  const int Ifirst = p.tab.I0[s];           // first row block of the chunk (0: whole sequence)
  const int nT = P + 1;                     // key tiles of 128

  if (tid == 0) {
    for (int i = 0; i < NUM_BARS; ++i)
      tc::mbar_init(bar_addr(bars, i), (i >= S_EMPTY && i < S_EMPTY + 2) ? 8u
                                       : (i >= K_FULL && i < K_FULL + kSStages) ? (uint32_t)NPAN
                                                                                : 1u);
    misc[1] = 0;
    tc::fence_barrier_init();
  }
  if (warp == kSMmaWarp) tc::tmem_alloc(smem_u32(misc), 512);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == kSMmaWarp - 1) {
    // ------------------------------ TMA: Q once, then the key tiles ------------------------------
    // One thread issues a 16 KB box only every ~0.3 us, so the two 64-dim panels of each key tile
    // come from two lanes (lane 0: panel 0 and Q, lane 1: panel 1), each arriving on K_FULL.
    const int pan = lane;
    if (pan < NPAN) {
      if (pan == 0) {
        tc::prefetch_tmap(&p.q_map);
        tc::mbar_expect_tx(bar_addr(bars, Q_FULL), kQBytes);
#pragma unroll
        for (int qp = 0; qp < NPAN; ++qp)
          tc::tma_load_3d_hint(sQ + qp * kPanel128, &p.q_map, 0, qtok0 + kRows * P, h * NPAN + qp,
                               bar_addr(bars, Q_FULL), tc::policy_evict_first());
      }
      tc::prefetch_tmap(&p.k_map);
      for (int T = 0; T < nT; ++T) {
        const int st = T % kSStages;
        if (T >= kSStages)
          tc::wait_bar(bar_addr(bars, K_EMPTY + st), ((T / kSStages) - 1) & 1, abort_flag, p.status);
        tc::mbar_expect_tx(bar_addr(bars, K_FULL + st), kPanel128);
        // keys are read again by the other row-block pairs of this head group (kept in L2);
        // the CTA's Q rows are read once
        tc::tma_load_3d_hint(sK + st * kKStage + pan * kPanel128, &p.k_map, 0, ktok0 + 128 * T,
                             h * NPAN + pan, bar_addr(bars, K_FULL + st), tc::policy_evict_last());
      }
      for (int T = max(0, nT - kSStages); T < nT; ++T)
        tc::drain_bar(bar_addr(bars, K_FULL + T % kSStages), (T / kSStages) & 1);
      if (pan == 0) tc::drain_bar(bar_addr(bars, Q_FULL), 0);
    }
  } else if (warp == kSMmaWarp) {
    // ------------------------------ MMA: S_b = Q K_T^T (128 x 128, fp32 in TMEM) ----------------
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(128, 128, 0, 0);
      tc::wait_bar(bar_addr(bars, Q_FULL), 0, abort_flag, p.status);
      for (int T = 0; T < nT; ++T) {
        const int st = T % kSStages, b = T & 1;
        tc::wait_bar(bar_addr(bars, K_FULL + st), (T / kSStages) & 1, abort_flag, p.status);
        if (T >= 2) tc::wait_bar(bar_addr(bars, S_EMPTY + b), ((T - 2) >> 1) & 1, abort_flag, p.status);
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * kPanel128 + (uint32_t)(kk & 3) * 32u;
          const uint64_t a = tc::sdesc_sw128(sQ + off, 16u, 1024u);
          const uint64_t bd = tc::sdesc_sw128(sK + st * kKStage + off, 16u, 1024u);
          tc::mma_bf16(tmem + (uint32_t)b * 128u, a, bd, idesc, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(bar_addr(bars, K_EMPTY + st));
        tc::mma_commit(bar_addr(bars, S_FULL + b));
      }
      if (nT > 0) tc::drain_bar(bar_addr(bars, S_FULL + ((nT - 1) & 1)), ((nT - 1) >> 1) & 1);
    }
  } else {
    // ------------------------------ softmax: one thread per (row, column block) -----------------
    // 16 warps, four per SM sub-partition: the warp's lane quarter qd gives its 32 rows, g the
    // column block 2T + g of a tile and tp the tiles it takes (T % 2 == tp, TMEM buffer tp). The
    // two tile parities run side by side, so one warp's waits (TMEM load, barriers, dependent
    // arithmetic) overlap the other warps' exponentials.
    const int qd = warp & 3, grp = warp >> 2, g = grp & 1, tp = grp >> 1;
    const int r = 32 * qd + lane;                 // TMEM lane = pair-local row
    const int Ir = I0 + (r >> 6);                 // row block (uniform over the warp)
    const int i = kRows * P + r;                  // sequence-local row
    const bool valid = i < L && Ir >= Ifirst;
    const uint32_t t_lane = (uint32_t)(32 * qd) << 16;
    const float sc = p.scale_log2;
    uint32_t v[64];
    for (int T = tp; T < nT; T += 2) {
      const int J = 2 * T + g;
      const bool has = J <= Ir;
      tc::wait_bar(bar_addr(bars, S_FULL + tp), (T >> 1) & 1, abort_flag, p.status);
      tc::tc_fence_after();
      if (has) {
        const uint32_t col = (uint32_t)(tp * 128 + g * 64);
        IAMAP_TMEM_LD32(tmem + t_lane + col, v);
        IAMAP_TMEM_LD32(tmem + t_lane + col + 32u, (v + 32));
        tc::tmem_ld_wait();
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar_addr(bars, S_EMPTY + tp));
      if (has) {
        float c;
        if (J < Ir && !(p.bias_window > 0 && i - 64 * J - 63 < p.bias_window)) {
          const float m = raw_max64(v) * sc;
          c = m + lg2(plain_exp2_sum64(v, sc, -m));
        } else {
          const float m = masked_max64(v, i, 64 * J, sc, p.bias_window, p.bias_log2);
          c = m == -INFINITY ? -INFINITY : m + lg2(masked_exp2_sum64(v, m));
        }
        tmem_st1(tmem + t_lane + (uint32_t)(kCCol + J), c);
      }
    }
    tmem_st_wait();
    tc::tc_fence_before();
    tc::named_bar(1, kSoft);
    tc::tc_fence_after();

    // ---- row log-sum-exp from the row's c values: group grp takes the 32-column chunks
    // ch = grp mod 4, then the four partial (max, sum) pairs are combined ----
    const int nJ = min(2 * P + 2, nb);
    {
      float m_acc = -INFINITY, l_acc = 0.f;
      for (int ch = grp; ch * 32 < nJ; ch += 4) {
        uint32_t cv[32];
        IAMAP_TMEM_LD32(tmem + t_lane + (uint32_t)(kCCol + 32 * ch), cv);
        tc::tmem_ld_wait();
        float cm = -INFINITY;
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (32 * ch + e <= Ir) cm = fmaxf(cm, __uint_as_float(cv[e]));
        if (cm > -INFINITY) {
          float cs = 0.f;
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (32 * ch + e <= Ir) cs += ex2(__uint_as_float(cv[e]) - cm);
          if (cm > m_acc) {
            l_acc = l_acc * ex2(m_acc - cm) + cs;
            m_acc = cm;
          } else {
            l_acc += cs * ex2(cm - m_acc);
          }
        }
      }
      ml_m[grp * kRows + r] = m_acc;
      ml_l[grp * kRows + r] = l_acc;
    }
    tc::named_bar(1, kSoft);
    if (grp == 0) {
      float m = ml_m[r];
#pragma unroll
      for (int k = 1; k < 4; ++k) m = fmaxf(m, ml_m[k * kRows + r]);
      float lse2 = -INFINITY;
      if (m > -INFINITY) {
        float l = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) l += ml_l[k * kRows + r] * ex2(ml_m[k * kRows + r] - m);
        lse2 = m + lg2(l);
      }
      lse_s[r] = lse2;
      if (valid) p.lse[(int64_t)h * p.n + row0 + i] = lse2 * kLn2;
    }
    tc::named_bar(1, kSoft);
    if (p.mass != nullptr) {

    // ---- block masses: sum over the valid rows of 2^(c_iJ - lse_i) ----
    const float lr = lse_s[r];
    for (int ch = grp; ch * 32 < nJ; ch += 4) {
      uint32_t cv[32];
      IAMAP_TMEM_LD32(tmem + t_lane + (uint32_t)(kCCol + 32 * ch), cv);
      tc::tmem_ld_wait();
      float x[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int J = 32 * ch + e;
        x[e] = (valid && J <= Ir) ? ex2(__uint_as_float(cv[e]) - lr) : 0.f;
      }
      part[qd * kMaxNb + 32 * ch + lane] = transpose_sum32(x, lane);
    }
    tc::named_bar(1, kSoft);
    for (int idx = tid; idx < 2 * kMaxNb; idx += kSoft) {
      const int k = idx / kMaxNb, J = idx - k * kMaxNb;
      const int I = I0 + k;
      if (I < nb && I >= Ifirst && J <= I) {
        const float m = part[(2 * k) * kMaxNb + J] + part[(2 * k + 1) * kMaxNb + J];
        mass_s[k * kMaxNb + J] = m;
        p.mass[(int64_t)h * p.ncb + tab_cb(p.tab, s, I) + J] = m;
      }
    }
    tc::named_bar(1, kSoft);

    // ---- cumulative-mass choice per row block: decreasing mass (ties: lower J first); a block
    // is kept while the mass before it is below tau * R ----
    const unsigned long long bit = 1ull << h;
    if (p.tau >= 1.f) {
      for (int idx = tid; idx < 2 * kMaxNb; idx += kSoft) {
        const int k = idx / kMaxNb, J = idx - k * kMaxNb, I = I0 + k;
        if (I < nb && I >= Ifirst && J <= I)
          atomicOr(p.headmask_dense + tab_cb(p.tab, s, I) + J, bit);
      }
    } else {
      for (int idx = tid; idx < 2 * kMaxNb; idx += kSoft) {
        const int k = idx / kMaxNb, J = idx - k * kMaxNb, I = I0 + k;
        if (I < nb && I >= Ifirst && J <= I) {
          const float* ms = mass_s + k * kMaxNb;
          const float mJ = ms[J];
          int rank = 0;
          for (int J2 = 0; J2 <= I; ++J2) {
            const float m2 = ms[J2];
            rank += (m2 > mJ) || (m2 == mJ && J2 < J);
          }
          rank_s[k * kMaxNb + J] = rank;
          sorted_s[k * kMaxNb + rank] = mJ;
        }
      }
      tc::named_bar(1, kSoft);
      if (warp < 2 && I0 + warp < nb && I0 + warp >= Ifirst)
        warp_exclusive_scan256(sorted_s + warp * kMaxNb, I0 + warp + 1, lane);
      tc::named_bar(1, kSoft);
      for (int idx = tid; idx < 2 * kMaxNb; idx += kSoft) {
        const int k = idx / kMaxNb, J = idx - k * kMaxNb, I = I0 + k;
        if (I < nb && I >= Ifirst && J <= I) {
          const float R = (float)min(64, L - 64 * I);
          if (sorted_s[k * kMaxNb + rank_s[k * kMaxNb + J]] < p.tau * R)
            atomicOr(p.headmask_dense + tab_cb(p.tab, s, I) + J, bit);
        }
      }
    }
    }   // masses
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == kSMmaWarp) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------------------------
// Stage 2: extraction of the kept tiles
// ------------------------------------------------------------------------------------------------

// OUT: also the sender's own attention output O_s = P V_s (MapFlow news page, the paragraphs on
// the attention map as the shared state: the sender runs its own attention, the receiver reuses
// its probabilities). Then every causal column block is visited, not only the kept ones; the
// bf16 P tile a writer group stages for the stores is also the A operand of a
// 128 x d_vs x 64 MMA into TMEM columns 256 .. 256 + d_vs, with the value tile as B. The row's
// final lse is known here, so P is normalised as computed and O_s needs no rescaling.
template <int D, bool OUT>
__global__ void __launch_bounds__(kThreads, OUT ? 1 : 2) extract_tc_kernel(const __grid_constant__ ExtractParams p) {
  constexpr int NPAN = D / 64;
  constexpr uint32_t kQBytes = NPAN * kPanel128;
  constexpr uint32_t kKStage = NPAN * kPanel64;
  constexpr uint32_t kVStage = 2 * kPanel64;               // room for d_vs up to 128
  constexpr int kBars = OUT ? XO_NUM_BARS : X_NUM_BARS;
  constexpr uint32_t kTmemCols = OUT ? 512u : 256u;
  constexpr int kStageBufs = OUT ? 2 : 1;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = align1024(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase, sK = sbase + kQBytes;
  const uint32_t sV = sK + kXStages * kKStage;             // OUT: value-tile ring
  unsigned char* stage_all = smem + kQBytes + kXStages * kKStage + (OUT ? kVStages * kVStage : 0);
  // 8 warps x 4 KB per staging buffer
  int64_t* base_s = reinterpret_cast<int64_t*>(stage_all + kStageBufs * 8 * 4096);   // [2][256]
  int* rk_s = reinterpret_cast<int*>(base_s + 2 * kMaxNb);               // [2][256] rank | k << 16
  int* ulist = rk_s + 2 * kMaxNb;                                        // [256] union of J
  uint64_t* bar_mem = reinterpret_cast<uint64_t*>(ulist + kMaxNb);
  uint32_t* misc = reinterpret_cast<uint32_t*>(bar_mem + kBars);         // [0] tmem [1] abort [2] count
  const uint32_t bars = smem_u32(bar_mem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // grid order (head group, pair, head in group): the CTAs resident at one time read the keys
  // of one group of head_group heads, which fit in L2 together, while neighbouring CTAs still
  // read neighbouring heads of one key tile (contiguous in the token-major K)
  const int num_pairs = (int)(gridDim.x / (unsigned)p.H_s);
  const int hgs = p.head_group;
  const int g0 = (int)(blockIdx.x / (unsigned)(num_pairs * hgs)) * hgs;   // first head of the group
  const int gsz = min(hgs, p.H_s - g0);
  const int rem = blockIdx.x - g0 * num_pairs;
  const int pair = rem / gsz;
  const int h = g0 + (rem - pair * gsz);
  const int2 it = p.tab.pairs[pair];
  const int s = it.x, I0 = it.y, P = I0 >> 1;
  const int row0 = p.tab.qoff[s];           // packed lse row of the sequence-local row 0
  const int ktok0 = p.tok0 ? p.tok0[s] : p.cu[s];
  const int qtok0 = p.tok0 ? p.tok0[s] : row0;
  const int L = p.cu[s + 1] - p.cu[s];
  const int nb = p.tab.nb[s];
  const int Ifirst = p.tab.I0[s];
  const int nJ = min(2 * P + 2, nb);

  if (tid == 0) {
    for (int i = 0; i < kBars; ++i) {
      uint32_t cnt = 1;
      if (i >= XS_EMPTY && i < XS_EMPTY + kXBufs) cnt = 4;
      if (OUT && i >= XP_READY && i < XP_READY + 4) cnt = 4;
      tc::mbar_init(bar_addr(bars, i), cnt);
    }
    misc[1] = 0;
    tc::fence_barrier_init();
  }
  for (int idx = tid; idx < 2 * kMaxNb; idx += kThreads) base_s[idx] = -1;
  if (warp == 9) tc::tmem_alloc(smem_u32(misc), kTmemCols);
  __syncthreads();
  // this head's stored blocks in row blocks I0 and I1, by column block
  if (p.dense) {
    for (int idx = tid; idx < 2 * kMaxNb; idx += kThreads) {
      const int k = idx / kMaxNb, J = idx - k * kMaxNb, I = I0 + k;
      if (I < nb && J <= I) {
        // the tile's rows are lines of a "block" of dense_heads interleaved heads (rank hh)
        base_s[idx] = ((int64_t)I * (I + 1) / 2 + J) * p.dense_heads;
        rk_s[idx] = (s * p.H_s + h) | (p.dense_heads << 16);
      }
    }
  } else if (warp < 2 && I0 + warp < nb && I0 + warp >= Ifirst) {
    const int rb = tab_rb(p.tab, s, I0 + warp);
    const int u0 = p.row_ptr[rb], u1 = p.row_ptr[rb + 1];
    const unsigned long long below = (1ull << h) - 1ull;
    for (int u = u0 + lane; u < u1; u += 32) {
      const unsigned long long m = p.headmask[u];
      if ((m >> h) & 1ull) {
        const int J = p.col_idx[u];
        base_s[warp * kMaxNb + J] = p.val_off[u];
        rk_s[warp * kMaxNb + J] = __popcll(m & below) | (__popcll(m) << 16);
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    // the column blocks to visit: the union of the kept ones, or (OUT) all causal ones
    int cnt = 0;
    for (int J0 = 0; J0 < nJ; J0 += 32) {
      const int J = J0 + lane;
      const bool any = J < nJ && (OUT || base_s[J] >= 0 || base_s[kMaxNb + J] >= 0);
      const unsigned bal = __ballot_sync(0xffffffffu, any);
      if (any) ulist[cnt + __popc(bal & ((1u << lane) - 1u))] = J;
      cnt += __popc(bal);
    }
    if (lane == 0) misc[2] = (uint32_t)cnt;
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = misc[0];
  const int nU = (int)misc[2];

  if (warp == 8) {
    if (lane == 0) {
      tc::prefetch_tmap(&p.q_map);
      tc::prefetch_tmap(&p.k_map);
      if (OUT) tc::prefetch_tmap(&p.vs_map);
      const uint32_t vbytes = OUT ? (uint32_t)p.d_vs * 128u : 0u;
      tc::mbar_expect_tx(bar_addr(bars, XQ_FULL), kQBytes);
#pragma unroll
      for (int pan = 0; pan < NPAN; ++pan)
        tc::tma_load_3d_hint(sQ + pan * kPanel128, &p.q_map, 0, qtok0 + kRows * P, h * NPAN + pan,
                             bar_addr(bars, XQ_FULL), tc::policy_evict_first());
      for (int t = 0; t < nU; ++t) {
        const int st = t % kXStages;
        if (t >= kXStages)
          tc::wait_bar(bar_addr(bars, XK_EMPTY + st), ((t / kXStages) - 1) & 1, abort_flag, p.status);
        tc::mbar_expect_tx(bar_addr(bars, XK_FULL + st), kKStage);
        const int J = ulist[t];
#pragma unroll
        for (int pan = 0; pan < NPAN; ++pan)
          tc::tma_load_3d_hint(sK + st * kKStage + pan * kPanel64, &p.k_map, 0, ktok0 + 64 * J,
                               h * NPAN + pan, bar_addr(bars, XK_FULL + st), tc::policy_evict_last());
        if (OUT) {
          // value tile of block t (both 64-dim halves in one box); its slot is free once the
          // P.V MMA of block t - kVStages completed
          const int vs = t % kVStages;
          if (t >= kVStages)
            tc::wait_bar(bar_addr(bars, XV_EMPTY + vs), ((t / kVStages) - 1) & 1, abort_flag, p.status);
          tc::mbar_expect_tx(bar_addr(bars, XV_FULL + vs), vbytes);
          tc::tma_load_3d(sV + vs * kVStage, &p.vs_map, 0, ktok0 + 64 * J, h * (p.d_vs / 64),
                          bar_addr(bars, XV_FULL + vs));
        }
      }
      for (int t = max(0, nU - kXStages); t < nU; ++t)
        tc::drain_bar(bar_addr(bars, XK_FULL + t % kXStages), (t / kXStages) & 1);
      if (OUT)
        for (int t = max(0, nU - kVStages); t < nU; ++t)
          tc::drain_bar(bar_addr(bars, XV_FULL + t % kVStages), (t / kVStages) & 1);
      tc::drain_bar(bar_addr(bars, XQ_FULL), 0);
    }
  } else if (warp == 9) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(128, 64, 0, 0);
      // O_s += P_t . V_s[J_t]: P from the staging buffer of block t's writer group (K-major,
      // 128 rows x 64 keys), V MN-major (d_vs columns per key; the second 64-dim half 8 KB on)
      auto issue_pv = [&](int t) {
        const int G = t & 1, c = t >> 1, sb = c & 1, u = c >> 1, vs = t % kVStages;
        tc::wait_bar(bar_addr(bars, XP_READY + 2 * G + sb), u & 1, abort_flag, p.status);
        tc::wait_bar(bar_addr(bars, XV_FULL + vs), (t / kVStages) & 1, abort_flag, p.status);
        tc::tc_fence_after();
        const uint32_t pa = smem_u32(stage_all) + (uint32_t)(sb * 8 + 4 * G) * 4096u;
        const uint32_t va = sV + (uint32_t)vs * kVStage;
        const uint32_t id_pv = tc::idesc_bf16(128, p.d_vs, 0, 1);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t a = tc::sdesc_sw128(pa + kk * 32u, 16u, 1024u);
          const uint64_t b = tc::sdesc_sw128(va + kk * 2048u, 8192u, 1024u);
          tc::mma_bf16(tmem + 256u, a, b, id_pv, (t > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(bar_addr(bars, XP_FREE + 2 * G + sb));
        tc::mma_commit(bar_addr(bars, XV_EMPTY + vs));
      };
      tc::wait_bar(bar_addr(bars, XQ_FULL), 0, abort_flag, p.status);
      for (int t = 0; t < nU; ++t) {
        const int st = t % kXStages, b = t & (kXBufs - 1);
        tc::wait_bar(bar_addr(bars, XK_FULL + st), (t / kXStages) & 1, abort_flag, p.status);
        if (t >= kXBufs) tc::wait_bar(bar_addr(bars, XS_EMPTY + b), ((t - kXBufs) >> 2) & 1, abort_flag, p.status);
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (uint32_t)(kk & 3) * 32u;
          const uint64_t a = tc::sdesc_sw128(sQ + (uint32_t)(kk >> 2) * kPanel128 + ko, 16u, 1024u);
          const uint64_t bd = tc::sdesc_sw128(sK + st * kKStage + (uint32_t)(kk >> 2) * kPanel64 + ko, 16u, 1024u);
          tc::mma_bf16(tmem + (uint32_t)b * 64u, a, bd, idesc, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(bar_addr(bars, XK_EMPTY + st));
        tc::mma_commit(bar_addr(bars, XS_FULL + b));
        if (OUT && t >= kOLag) issue_pv(t - kOLag);
      }
      if (OUT) {
        for (int t = max(0, nU - kOLag); t < nU; ++t) issue_pv(t);
        tc::mma_commit(bar_addr(bars, XO_FULL));
        tc::drain_bar(bar_addr(bars, XO_FULL), 0);
      } else if (nU > 0) {
        tc::drain_bar(bar_addr(bars, XS_FULL + ((nU - 1) & (kXBufs - 1))), ((nU - 1) >> 2) & 1);
      }
    }
  } else {
    // ------------------------------ writers: group G takes the blocks t = G, G + 2, ... --------
    const int qd = warp & 3, G = warp >> 2;
    const int r = 32 * qd + lane;
    const int kb = r >> 6;                        // 0: row block I0, 1: I1 (uniform over the warp)
    const int Ir = I0 + kb;
    const int i = kRows * P + r;
    const bool valid = i < L && Ir >= Ifirst;
    const int il = r & 63;                        // row within the tile
    const uint32_t t_lane = (uint32_t)(32 * qd) << 16;
    const float sc = p.scale_log2;
    const float lse2 = valid ? p.lse[(int64_t)h * p.n + row0 + i] * kLog2e : 0.f;
    bool cap_flag = false;
    float acc1 = 0.f, acc2 = 0.f;   // dense mode: sum and squared norm of this row's rounded values
    for (int t = G; t < nU; t += 2) {
      const int b = t & (kXBufs - 1);
      const int c = t >> 1, sb = OUT ? (c & 1) : 0;
      unsigned char* stg = stage_all + (sb * 8 + warp) * 4096;
      tc::wait_bar(bar_addr(bars, XS_FULL + b), (t >> 2) & 1, abort_flag, p.status);
      tc::tc_fence_after();
      const int J = ulist[t];
      const int64_t base = base_s[kb * kMaxNb + J];
      const int rk = rk_s[kb * kMaxNb + J];
      const int rank = rk & 0xffff, k = rk >> 16;
      // OUT: every block feeds the P.V MMA, so every block's P is staged
      const bool stage = OUT || base >= 0;
      if (stage) {
        // exp(s - lse) of this row, 32 columns at a time, staged as bf16 (16-byte chunk c of
        // the row at c ^ (row & 7))
        const int j0 = 64 * J;
        const bool fast = J < Ir && !(p.bias_window > 0 && i - j0 - 63 < p.bias_window);
        uint32_t v[64];
        IAMAP_TMEM_LD32(tmem + t_lane + (uint32_t)(b * 64), v);
        IAMAP_TMEM_LD32(tmem + t_lane + (uint32_t)(b * 64 + 32), (v + 32));
        tc::tmem_ld_wait();
        if (OUT && c >= 2)   // the P.V MMA of this buffer's previous block has read it
          tc::wait_bar(bar_addr(bars, XP_FREE + 2 * G + sb), ((c >> 1) - 1) & 1, abort_flag, p.status);
        if (!OUT && p.dense) {   // the tensor store of this warp's previous tile has read it
          if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
          __syncwarp();
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[16];
          if (fast) {
            const float nl = -lse2;
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float a0 = valid ? ex2(fmaf(__uint_as_float(v[32 * half + e]), sc, nl)) : 0.f;
              const float a1 = valid ? ex2(fmaf(__uint_as_float(v[32 * half + e + 1]), sc, nl)) : 0.f;
              pk[e >> 1] = pack_bf16(a0, a1);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float a[2];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int j = j0 + 32 * half + e + u;
                float x = __uint_as_float(v[32 * half + e + u]) * sc;
                if (p.bias_window > 0 && i - j >= 0 && i - j < p.bias_window) x += p.bias_log2;
                a[u] = (valid && j <= i) ? ex2(x - lse2) : 0.f;
              }
              pk[e >> 1] = pack_bf16(a[0], a[1]);
            }
          }
          if (p.norm2) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pk[e]));
              acc1 += f.x + f.y;
              acc2 = fmaf(f.x, f.x, fmaf(f.y, f.y, acc2));
            }
          }
#pragma unroll
          for (int cq = 0; cq < 4; ++cq) {
            const int cc = 4 * half + cq;
            *reinterpret_cast<uint4*>(stg + lane * 128 + ((cc ^ (lane & 7)) << 4)) =
                make_uint4(pk[4 * cq], pk[4 * cq + 1], pk[4 * cq + 2], pk[4 * cq + 3]);
          }
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar_addr(bars, XS_EMPTY + b));
      if (OUT) {
        // the staged tile goes to the tensor cores (async proxy) as well as to the stores below
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar_addr(bars, XP_READY + 2 * G + sb));
      }
      if (base < 0) continue;
      if (!OUT && p.dense) {
        // dense mode: the staged 32 rows are one box of the chunk-major maps (32 chunks of head
        // rank, staged with the same 128-byte swizzle); one tensor store, read asynchronously
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int chunk0 = (int)(base / k) * 64 + (il - lane);
          asm volatile(
              "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];\n\t"
              "cp.async.bulk.commit_group;" ::"l"(&p.dense_map),
              "r"(0), "r"(rank), "r"(chunk0), "r"(smem_u32(stg))
              : "memory");
        }
        continue;
      }
      // write 4 tile rows of 128 B per step
      __syncwarp();
      if (base + k <= p.capacity) {
        __nv_bfloat16* blk = p.vals + base * (64 * 64) + (int64_t)rank * 64;
        const int cl = lane & 7;
#pragma unroll
        for (int step = 0; step < 8; ++step) {
          const int row = 4 * step + (lane >> 3);          // warp-local row
          const uint4 val = *reinterpret_cast<const uint4*>(stg + row * 128 + ((cl ^ (row & 7)) << 4));
          const int tr = (il - lane) + row;                 // tile row of that warp-local row
          // streaming store: each tile is read once, by mapped_av, long after this kernel; it
          // should not displace the keys the grid order keeps in L2
          __stcs(reinterpret_cast<uint4*>(blk + (int64_t)tr * k * 64 + cl * 8), val);
        }
      } else {
        cap_flag = true;
      }
      __syncwarp();
    }
    if (!OUT && p.dense && lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    if (cap_flag && lane == 0) raise_status(p.status, IAMAP_DEV_CAPACITY);
    if (p.norm2) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        acc1 += __shfl_xor_sync(0xffffffffu, acc1, o);
        acc2 += __shfl_xor_sync(0xffffffffu, acc2, o);
      }
      if (lane == 0) {
        atomicAdd(p.sum1 + (int64_t)s * p.H_s + h, acc1);
        atomicAdd(p.norm2 + (int64_t)s * p.H_s + h, acc2);
      }
    }
    if (OUT) {
      // O_s rows out of TMEM: group G takes columns [G * d_vs / 2, (G + 1) * d_vs / 2), 32 at a
      // time, transposed through this warp's staging slice so that each row leaves as 128-byte
      // runs (4 rows per store instruction)
      tc::wait_bar(bar_addr(bars, XO_FULL), 0, abort_flag, p.status);
      tc::tc_fence_after();
      const int half_cols = p.d_vs / 2;
      float* scr = reinterpret_cast<float*>(stage_all + warp * 4096);   // [32 rows][32 floats]
      for (int c0 = G * half_cols; c0 < (G + 1) * half_cols; c0 += 32) {
        uint32_t v[32];
        IAMAP_TMEM_LD32(tmem + t_lane + 256u + (uint32_t)c0, v);
        tc::tmem_ld_wait();
#pragma unroll
        for (int cq = 0; cq < 8; ++cq)
          *reinterpret_cast<uint4*>(scr + lane * 32 + ((cq ^ (lane & 7)) << 2)) =
              make_uint4(v[4 * cq], v[4 * cq + 1], v[4 * cq + 2], v[4 * cq + 3]);
        __syncwarp();
        const int cl = lane & 7;
#pragma unroll
        for (int step = 0; step < 8; ++step) {
          const int row = 4 * step + (lane >> 3);           // warp-local row
          const int ir = kRows * P + 32 * qd + row;         // its sequence-local row
          const int Irr = I0 + ((32 * qd + row) >> 6);
          if (ir < L && Irr >= Ifirst) {
            const uint4 val = *reinterpret_cast<const uint4*>(scr + row * 32 + ((cl ^ (row & 7)) << 2));
            *reinterpret_cast<uint4*>(p.o_s + ((int64_t)(row0 + ir) * p.H_s + h) * p.d_vs + c0 + 4 * cl) = val;
          }
        }
        __syncwarp();
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
static size_t stats_smem() {
  return 1024 + (size_t)(D / 64) * kPanel128 * (1 + kSStages) +
         sizeof(float) * (4 * kRows + 4 * kRows + kRows + 4 * kMaxNb + 2 * kMaxNb + 2 * kMaxNb) +
         sizeof(int) * 2 * kMaxNb + 8 * NUM_BARS + 16;
}
template <int D, bool OUT>
static size_t extract_smem() {
  return 1024 + (size_t)(D / 64) * (kPanel128 + kXStages * kPanel64) +
         (OUT ? (size_t)kVStages * 2 * kPanel64 + 2 * 8 * 4096 : 8 * 4096) +
         sizeof(int64_t) * 2 * kMaxNb + sizeof(int) * 3 * kMaxNb +
         8 * (OUT ? (int)XO_NUM_BARS : (int)X_NUM_BARS) + 16;
}

}  // namespace tccomp

bool compress_tc_supported(int d, int max_nb) {
  return (d == 64 || d == 128) && max_nb <= tccomp::kMaxNb;
}

static int encode_qk_map(CUtensorMap* map, const void* base, int64_t n, int H_s, int d, int box_rows) {
  return encode_tmap_3d_bf16(map, base, 64, (uint64_t)n, (uint64_t)H_s * (d / 64),
                             (uint64_t)H_s * d * 2, 128, 64, (uint32_t)box_rows, 1);
}

// Heads per group of the grid order: as many as have their keys (n_key x d bf16 each) fit in
// kHeadGroupBytes, so that one group's keys stay in L2 (126 MB) while its CTAs run (varlen40k:
// 9 of 40 heads per group, extract 6.0 -> 5.3 ms; prefill8k: all 32 heads, the plain pair order).
#ifndef IAMAP_HEAD_GROUP_MB
#define IAMAP_HEAD_GROUP_MB 96
#endif
constexpr int64_t kHeadGroupBytes = (int64_t)IAMAP_HEAD_GROUP_MB << 20;
static int head_group_for(int64_t n_key, int d, int H_s) {
  const int64_t per_head = std::max<int64_t>(1, n_key * d * 2);
  return (int)std::max<int64_t>(1, std::min<int64_t>(H_s, kHeadGroupBytes / per_head));
}

int compress_stats_tc_launch(const CompressArgs& a, cudaStream_t stream) {
  using namespace tccomp;
  StatsParams p{};
  const int64_t n_tok = a.n_tok > 0 ? a.n_tok : a.n;
  const int64_t n_key = a.n_k > 0 ? a.n_k : n_tok;
  int rc = encode_qk_map(&p.q_map, a.q, n_tok, a.H_s, a.d, 128);
  if (!rc) rc = encode_qk_map(&p.k_map, a.k, n_key, a.H_s, a.d, 128);
  if (rc) return rc;
  p.cu = a.cu_seqlens;
  p.tok0 = a.tok0;
  p.tab = a.tab;
  p.n = a.n;
  p.ncb = a.plan.num_causal_blocks;
  p.H_s = a.H_s;
  p.head_group = head_group_for(n_key, a.d, a.H_s);
  p.scale_log2 = kLog2e / sqrtf((float)a.d);
  p.bias_window = a.bias_window;
  p.bias_log2 = a.bias_value * kLog2e;
  p.tau = a.tau;
  p.lse = a.lse;
  p.mass = a.mass;
  p.headmask_dense = reinterpret_cast<unsigned long long*>(a.headmask_dense);
  p.status = a.status;
  // one CTA per SM: it holds all 512 TMEM columns
  const size_t smem = std::max<size_t>(a.d == 64 ? stats_smem<64>() : stats_smem<128>(), 120 * 1024);
  auto kern = a.d == 64 ? stats_tc_kernel<64> : stats_tc_kernel<128>;
  IAMAP_CUDA_CHECK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  const int64_t grid = a.plan.num_pairs * a.H_s;
  if (grid > 0) {
    kern<<<(unsigned)grid, kSThreads, smem, stream>>>(p);
    IAMAP_LAUNCH_CHECK("compress stats (tcgen05)");
  }
  return IAMAP_OK;
}

int compress_extract_tc_launch(const CompressArgs& a, cudaStream_t stream) {
  using namespace tccomp;
  ExtractParams p{};
  const int64_t n_tok = a.n_tok > 0 ? a.n_tok : a.n;
  const int64_t n_key = a.n_k > 0 ? a.n_k : n_tok;
  int rc = encode_qk_map(&p.q_map, a.q, n_tok, a.H_s, a.d, 128);
  if (!rc) rc = encode_qk_map(&p.k_map, a.k, n_key, a.H_s, a.d, 64);
  if (rc) return rc;
  p.cu = a.cu_seqlens;
  p.tok0 = a.tok0;
  p.dense = a.dense;
  p.dense_tiles = a.dense_tiles;
  p.dense_heads = a.dense && a.dense_tiles > 0 ? (int)(a.capacity / a.dense_tiles) : 0;
  if (a.dense) {
    // one warp's 32 rows of a tile: 32 chunks of one head, 128 B each, dense_heads lines apart
    rc = encode_tmap_3d_bf16(&p.dense_map, a.vals, 64, (uint64_t)p.dense_heads,
                             (uint64_t)a.dense_tiles * 64, 128, (uint64_t)p.dense_heads * 128, 64,
                             1, 32);
    if (rc) return rc;
  }
  p.norm2 = a.norm2;
  p.sum1 = a.sum1;
  p.tab = a.tab;
  p.n = a.n;
  p.H_s = a.H_s;
  p.head_group = head_group_for(n_key, a.d, a.H_s);
  p.scale_log2 = kLog2e / sqrtf((float)a.d);
  p.bias_window = a.bias_window;
  p.bias_log2 = a.bias_value * kLog2e;
  p.lse = a.lse_in;
  p.row_ptr = a.row_ptr_in;
  p.col_idx = a.col_idx_in;
  p.headmask = reinterpret_cast<const unsigned long long*>(a.headmask_in);
  p.val_off = a.val_off_in;
  p.vals = static_cast<__nv_bfloat16*>(a.vals);
  p.capacity = a.capacity;
  p.status = a.status;
  const bool out = a.o_s != nullptr;
  if (out) {
    if (a.dense || !a.v_s || (a.d_vs != 64 && a.d_vs != 128))
      return set_error(IAMAP_ERR_INVALID_ARG, "sender output needs v_s and d_vs of 64 or 128");
    rc = encode_tmap_3d_bf16(&p.vs_map, a.v_s, 64, (uint64_t)n_key, (uint64_t)a.H_s * (a.d_vs / 64),
                             (uint64_t)a.H_s * a.d_vs * 2, 128, 64, 64, (uint32_t)(a.d_vs / 64));
    if (rc) return rc;
    p.o_s = a.o_s;
    p.d_vs = a.d_vs;
  }
  const size_t smem = out ? (a.d == 64 ? extract_smem<64, true>() : extract_smem<128, true>())
                          : (a.d == 64 ? extract_smem<64, false>() : extract_smem<128, false>());
  auto kern = out ? (a.d == 64 ? extract_tc_kernel<64, true> : extract_tc_kernel<128, true>)
                  : (a.d == 64 ? extract_tc_kernel<64, false> : extract_tc_kernel<128, false>);
  IAMAP_CUDA_CHECK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  const int64_t grid = a.plan.num_pairs * a.H_s;
  if (grid > 0) {
    kern<<<(unsigned)grid, kThreads, smem, stream>>>(p);
    IAMAP_LAUNCH_CHECK("compress extract (tcgen05)");
  }
  return IAMAP_OK;
}

}  // namespace iamap
