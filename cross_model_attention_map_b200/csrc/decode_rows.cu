// iamap_sender_rows: the small model's attention row of one decode step, the row a mapped layer
// of the large model reuses ("IAM: Efficient Inference through Attention Mapping between
// Different-scale LLMs" notes, Method section 4, decode bullet: the mapped layer takes the small
// model's attention directly).
//
//   p[b, h, j] = exp(q[b, h] . k[b, j, h] / sqrt(d) - lse[b, h]),  j < ctx[b]
//
// with the keys in a paged cache. Two kernels: scores of a chunk of keys per CTA (one key per
// thread, its d bf16 values read as 16-byte vectors) written in the log2 domain, with the chunk's
// (max, sum of exponentials); then every chunk combines the partials of its row into the row's
// log-sum-exp and normalises its keys in place. Entries j >= ctx[b] up to ctx_stride are zeroed.
#include <algorithm>
#include <cfloat>

#include "internal.h"

namespace iamap {
namespace {

constexpr int kRowThreads = 256;
constexpr int kRowChunk = 512;      // keys per CTA
constexpr int kRowMaxD = 128;

struct RowParams {
  const __nv_bfloat16* q;       // [batch, H_s, d]
  const __nv_bfloat16* k;       // [num_pages, page_size, H_s, d]
  int64_t num_pages;
  const int32_t* page_table;    // [batch, max_pages]
  int max_pages, page_size;
  const int32_t* ctx_lens;
  int H_s, d;
  float scale_log2;
  float* p;                     // [batch, H_s, ctx_stride]
  int ctx_stride;
  float2* part;                 // [batch * H_s][nchunk]: (max, sum of 2^(x - max)) in log2
  int nchunk;
  unsigned int* status;
};

__device__ __forceinline__ float2 combine(float2 a, float2 b) {
  const float m = fmaxf(a.x, b.x);
  if (m == -INFINITY) return make_float2(-INFINITY, 0.f);
  return make_float2(m, a.y * ex2(a.x - m) + b.y * ex2(b.x - m));
}

__global__ void __launch_bounds__(kRowThreads) sender_scores_kernel(RowParams p) {
  __shared__ float q_s[kRowMaxD];
  __shared__ float2 red[kRowThreads / 32];
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ctx = p.ctx_lens[b];
  for (int e = tid; e < p.d; e += kRowThreads)
    q_s[e] = __bfloat162float(p.q[((int64_t)b * p.H_s + h) * p.d + e]);
  __syncthreads();
  float* row = p.p + ((int64_t)b * p.H_s + h) * p.ctx_stride;
  float2 acc = make_float2(-INFINITY, 0.f);
  bool bad = false;
  for (int j = c * kRowChunk + tid; j < min(ctx, (c + 1) * kRowChunk); j += kRowThreads) {
    const int page = p.page_table[(int64_t)b * p.max_pages + j / p.page_size];
    float x = -INFINITY;
    if (page >= 0 && page < p.num_pages) {
      const uint4* kv = reinterpret_cast<const uint4*>(
          p.k + (((int64_t)page * p.page_size + j % p.page_size) * p.H_s + h) * p.d);
      float dot = 0.f;
      for (int v = 0; v < p.d / 8; ++v) {
        const uint4 u = kv[v];
        const __nv_bfloat162* e2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float2 f = __bfloat1622float2(e2[t]);
          dot = fmaf(f.x, q_s[8 * v + 2 * t], dot);
          dot = fmaf(f.y, q_s[8 * v + 2 * t + 1], dot);
        }
      }
      x = dot * p.scale_log2;
    } else {
      bad = true;
    }
    row[j] = x;
    acc = combine(acc, make_float2(x, 1.f));
  }
  if (bad) raise_status(p.status, IAMAP_DEV_BAD_INDEX);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float2 other = make_float2(__shfl_xor_sync(0xffffffffu, acc.x, o),
                                     __shfl_xor_sync(0xffffffffu, acc.y, o));
    acc = combine(acc, other);
  }
  if (lane == 0) red[warp] = acc;
  __syncthreads();
  if (tid == 0) {
    float2 r = red[0];
    for (int w = 1; w < kRowThreads / 32; ++w) r = combine(r, red[w]);
    p.part[((int64_t)b * p.H_s + h) * p.nchunk + c] = r;
  }
}

__global__ void __launch_bounds__(kRowThreads) sender_norm_kernel(RowParams p) {
  __shared__ float lse_s;
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const int ctx = p.ctx_lens[b];
  if (tid == 0) {
    const float2* part = p.part + ((int64_t)b * p.H_s + h) * p.nchunk;
    float2 r = make_float2(-INFINITY, 0.f);
    const int used = (ctx + kRowChunk - 1) / kRowChunk;
    for (int i = 0; i < used; ++i) r = combine(r, part[i]);   // same order in every CTA
    lse_s = r.x == -INFINITY ? INFINITY : r.x + lg2(r.y);
  }
  __syncthreads();
  const float lse = lse_s;
  float* row = p.p + ((int64_t)b * p.H_s + h) * p.ctx_stride;
  for (int j = c * kRowChunk + tid; j < min(p.ctx_stride, (c + 1) * kRowChunk); j += kRowThreads)
    row[j] = j < ctx ? ex2(row[j] - lse) : 0.f;
}

}  // namespace
}  // namespace iamap

using namespace iamap;

extern "C" size_t iamap_sender_rows_workspace_bytes(int batch, int H_s, int ctx_stride) {
  if (batch < 1 || H_s < 1 || ctx_stride < 1) return 0;
  const int nchunk = (ctx_stride + kRowChunk - 1) / kRowChunk;
  return sizeof(float2) * (size_t)batch * H_s * nchunk;
}

extern "C" int iamap_sender_rows(const void* q, const void* k_pages, int64_t num_pages,
                                 const int32_t* page_table, int max_pages, int page_size,
                                 const int32_t* ctx_lens, const int32_t* ctx_lens_host, int batch,
                                 int H_s, int d, float* p_rows, int ctx_stride, void* ws,
                                 size_t ws_bytes, void* stream) {
  clear_error();
  if (!q || !k_pages || !page_table || !ctx_lens || !ctx_lens_host || !p_rows)
    return set_error(IAMAP_ERR_INVALID_ARG, "null pointer");
  if (batch < 1 || H_s < 1 || page_size < 1 || max_pages < 0 || num_pages < 0 || ctx_stride < 1)
    return set_error(IAMAP_ERR_INVALID_ARG, "bad sizes");
  if (d < 8 || d > kRowMaxD || d % 8 != 0)
    return set_error(IAMAP_ERR_UNSUPPORTED, "head dim must be a multiple of 8 up to %d", kRowMaxD);
  if ((reinterpret_cast<uintptr_t>(k_pages) & 15u) != 0)
    return set_error(IAMAP_ERR_INVALID_ARG, "k_pages must be 16-byte aligned");
  for (int b = 0; b < batch; ++b) {
    const int c = ctx_lens_host[b];
    if (c < 0 || c > ctx_stride || (int64_t)c > (int64_t)max_pages * page_size)
      return set_error(IAMAP_ERR_INVALID_ARG, "ctx_lens[%d]=%d exceeds the row or page table", b, c);
  }
  const int nchunk = (ctx_stride + kRowChunk - 1) / kRowChunk;
  const size_t need = sizeof(float2) * (size_t)batch * H_s * nchunk;
  if (!ws || ws_bytes < need)
    return set_error(IAMAP_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                     ws_bytes);
  DeviceContext* ctx = device_context();
  if (!ctx) return IAMAP_ERR_CUDA;
  RowParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k_pages);
  p.num_pages = num_pages;
  p.page_table = page_table;
  p.max_pages = max_pages;
  p.page_size = page_size;
  p.ctx_lens = ctx_lens;
  p.H_s = H_s;
  p.d = d;
  p.scale_log2 = kLog2e / sqrtf((float)d);
  p.p = p_rows;
  p.ctx_stride = ctx_stride;
  p.part = static_cast<float2*>(ws);
  p.nchunk = nchunk;
  p.status = ctx->status;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const dim3 grid(nchunk, H_s, batch);
  sender_scores_kernel<<<grid, kRowThreads, 0, st>>>(p);
  IAMAP_LAUNCH_CHECK("sender_scores_kernel");
  sender_norm_kernel<<<grid, kRowThreads, 0, st>>>(p);
  IAMAP_LAUNCH_CHECK("sender_norm_kernel");
  return IAMAP_OK;
}
