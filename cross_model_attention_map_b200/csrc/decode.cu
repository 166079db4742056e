// mapped_av_paged: the decode step of a mapped layer. The large model's mapped layer reuses the
// small model's attention row directly (no Q/K projection, no QK^T, no K cache) and only streams
// its own V cache ("IAM: Efficient Inference through Attention Mapping between Different-scale
// LLMs" notes, Method section 4, decode bullet); with a general W the row is the linear
// combination of sender heads used by mapped_av.
//
//   out[b, r, :] = sum_{j < ctx[b]} (sum_s W[r, s] p[b, s, j]) V[page(b, j), j % page, r, :]
//
// The V cache stream dominates (bytes read once), so the kernel is a coalesced GEMV on CUDA
// cores: CTA (chunk of pages, sequence b, slice of 8192 output elements) walks its pages; each
// thread owns four 16-byte chunks of the [H_r * d_v] token row and accumulates fp32, with the
// loads of four tokens in flight. The mixed weights of up to 128 tokens are formed in shared
// memory at a time. Partial sums per page chunk go to the workspace and a second kernel adds them
// in a fixed order (deterministic).
#include <algorithm>

#include "internal.h"

namespace iamap {

constexpr int kDecThreads = 256;
constexpr int kDecCPT = 4;                                  // 16-byte chunks per thread
constexpr int kDecSlice = kDecThreads * kDecCPT * 8;        // output elements per CTA slice
constexpr int kDecMaxPage = 32;                             // largest page size supported
constexpr int kDecMaxH = 128;                               // largest H_s / H_r supported

struct DecParams {
  const float* p_rows;
  int ctx_stride;
  const float* W;
  const __nv_bfloat16* v;
  int64_t num_pages;
  const int32_t* page_table;
  int max_pages;
  int page_size;
  const int32_t* ctx_lens;
  int H_s, H_r, d_v;
  int kv_grp;   // receiver heads per value head
  int chunks, ppc;
  float* partial;
  unsigned int* status;
};

// Mixed weights of kDecGroupTok tokens are formed at a time in shared memory:
// s_w[t][r] = sum_s W[r, s] p[b, s, j0 + t] (W read through L1).
constexpr int kDecGroupTok = 128;
constexpr int kDecUnroll = 3;                               // tokens whose loads are in flight

__global__ void __launch_bounds__(kDecThreads, 2) paged_gemv_kernel(DecParams p) {
  extern __shared__ float s_w[];                   // [kDecGroupTok][H_r]
  const int chunk = blockIdx.x, b = blockIdx.y, slice = blockIdx.z;
  const int tid = threadIdx.x;
  const int E = p.H_r * p.d_v;                    // output elements per sequence
  const int Ev = (p.H_r / p.kv_grp) * p.d_v;      // value elements per token
  const int ctx = p.ctx_lens[b];
  const int npages = (ctx + p.page_size - 1) / p.page_size;
  const int pg0 = chunk * p.ppc, pg1 = min(npages, pg0 + p.ppc);
  const int e0 = slice * kDecSlice;
  const int gpages = max(1, kDecGroupTok / p.page_size);    // pages per weight group

  float acc[kDecCPT][8];
#pragma unroll
  for (int c = 0; c < kDecCPT; ++c)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[c][e] = 0.f;
  int head_of[kDecCPT];
  int voff[kDecCPT];   // element offset of this chunk in a token's value row
  bool live[kDecCPT];
#pragma unroll
  for (int c = 0; c < kDecCPT; ++c) {
    const int e = e0 + (c * kDecThreads + tid) * 8;
    live[c] = e < E;
    head_of[c] = live[c] ? e / p.d_v : 0;
    voff[c] = live[c] ? (head_of[c] / p.kv_grp) * p.d_v + (e - head_of[c] * p.d_v) : 0;
  }
  const float* prow = p.p_rows + (int64_t)b * p.H_s * p.ctx_stride;
  bool bad = false;
  for (int gp0 = pg0; gp0 < pg1; gp0 += gpages) {
    const int gp1 = min(pg1, gp0 + gpages);
    const int j0 = gp0 * p.page_size;
    const int ntok = min(ctx, gp1 * p.page_size) - j0;
    __syncthreads();   // the previous group's weights are no longer read
    for (int e = tid; e < ntok * p.H_r; e += kDecThreads) {
      const int r = e / ntok, t = e - r * ntok;       // consecutive threads: consecutive tokens
      float w = 0.f;
      for (int sh = 0; sh < p.H_s; ++sh)
        w = fmaf(__ldg(p.W + r * p.H_s + sh), __ldg(prow + (int64_t)sh * p.ctx_stride + j0 + t), w);
      s_w[t * p.H_r + r] = w;
    }
    __syncthreads();
    for (int pi = gp0; pi < gp1; ++pi) {
      const int pg = p.page_table[(int64_t)b * p.max_pages + pi];
      if (pg < 0 || pg >= p.num_pages) {
        bad = true;
        continue;
      }
      const int tb = (pi - gp0) * p.page_size;          // first token of the page in the group
      const int nslot = min(p.page_size, ctx - pi * p.page_size);
      const __nv_bfloat16* vpage = p.v + (int64_t)pg * p.page_size * Ev;
      for (int t0 = 0; t0 < nslot; t0 += kDecUnroll) {
        uint4 raw[kDecUnroll][kDecCPT];
#pragma unroll
        for (int u = 0; u < kDecUnroll; ++u)
#pragma unroll
          for (int c = 0; c < kDecCPT; ++c)
            if (live[c] && t0 + u < nslot)
              // streaming loads: the V cache is read once per step (0.140 -> 0.136 ms on the
              // decode configuration)
              raw[u][c] = __ldcs(reinterpret_cast<const uint4*>(vpage + (int64_t)(t0 + u) * Ev + voff[c]));
#pragma unroll
        for (int u = 0; u < kDecUnroll; ++u) {
          if (t0 + u >= nslot) break;
#pragma unroll
          for (int c = 0; c < kDecCPT; ++c) {
            if (!live[c]) continue;
            const float w = s_w[(tb + t0 + u) * p.H_r + head_of[c]];
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[u][c]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(h2[e]);
              acc[c][2 * e] = fmaf(w, f.x, acc[c][2 * e]);
              acc[c][2 * e + 1] = fmaf(w, f.y, acc[c][2 * e + 1]);
            }
          }
        }
      }
    }
  }
  if (bad) raise_status(p.status, IAMAP_DEV_BAD_INDEX);
  float* dst = p.partial + ((int64_t)b * p.chunks + chunk) * E + e0;
#pragma unroll
  for (int c = 0; c < kDecCPT; ++c) {
    if (!live[c]) continue;
    float4* d4 = reinterpret_cast<float4*>(dst + (c * kDecThreads + tid) * 8);
    d4[0] = make_float4(acc[c][0], acc[c][1], acc[c][2], acc[c][3]);
    d4[1] = make_float4(acc[c][4], acc[c][5], acc[c][6], acc[c][7]);
  }
}

__global__ void paged_reduce_kernel(const float* __restrict__ partial, int chunks, int E,
                                    float* __restrict__ out) {
  const int b = blockIdx.y;
  const int e = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (e >= E) return;
  const float* src = partial + (int64_t)b * chunks * E + e;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c = 0; c < chunks; ++c) {
    const float4 x = *reinterpret_cast<const float4*>(src + (int64_t)c * E);
    acc.x += x.x;
    acc.y += x.y;
    acc.z += x.z;
    acc.w += x.w;
  }
  *reinterpret_cast<float4*>(out + (int64_t)b * E + e) = acc;
}

void paged_split(int batch, int max_ctx, int page_size, int num_sms, int* chunks,
                 int* pages_per_chunk) {
  const int npages = (max_ctx + page_size - 1) / page_size;
  int want = (2 * num_sms + batch - 1) / batch;
  if (want < 1) want = 1;
  int ppc = (npages + want - 1) / want;
  if (ppc < 1) ppc = 1;
  int ch = (npages + ppc - 1) / ppc;
  if (ch < 1) ch = 1;
  *chunks = ch;
  *pages_per_chunk = ppc;
}

int mapped_av_paged_impl(const PagedArgs& a, cudaStream_t stream) {
  if (a.page_size > kDecMaxPage || a.H_s > kDecMaxH || a.H_r > kDecMaxH)
    return set_error(IAMAP_ERR_UNSUPPORTED, "page_size <= %d and H_s, H_r <= %d required",
                     kDecMaxPage, kDecMaxH);
  DecParams p{};
  p.p_rows = a.p_rows;
  p.ctx_stride = a.ctx_stride;
  p.W = a.W;
  p.v = static_cast<const __nv_bfloat16*>(a.v_pages);
  p.num_pages = a.num_pages;
  p.page_table = a.page_table;
  p.max_pages = a.max_pages;
  p.page_size = a.page_size;
  p.ctx_lens = a.ctx_lens;
  p.H_s = a.H_s;
  p.H_r = a.H_r;
  p.d_v = a.d_v;
  p.kv_grp = a.H_r / (a.H_kv > 0 ? a.H_kv : a.H_r);
  p.chunks = a.chunks;
  p.ppc = a.pages_per_chunk;
  p.partial = a.partial;
  p.status = a.status;
  const int E = a.H_r * a.d_v;
  dim3 grid(a.chunks, a.batch, (E + kDecSlice - 1) / kDecSlice);
  const int gtok = std::max(1, kDecGroupTok / a.page_size) * a.page_size;
  const size_t smem = sizeof(float) * (size_t)gtok * a.H_r;
  IAMAP_CUDA_CHECK(cudaFuncSetAttribute(paged_gemv_kernel,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  paged_gemv_kernel<<<grid, kDecThreads, smem, stream>>>(p);
  IAMAP_LAUNCH_CHECK("paged_gemv_kernel");
  dim3 rgrid((E / 4 + 255) / 256, a.batch);
  paged_reduce_kernel<<<rgrid, 256, 0, stream>>>(a.partial, a.chunks, E, a.out);
  IAMAP_LAUNCH_CHECK("paged_reduce_kernel");
  return IAMAP_OK;
}

}  // namespace iamap
