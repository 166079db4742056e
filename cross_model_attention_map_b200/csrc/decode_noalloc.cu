// iamap_mapped_av_paged_noalloc: the paged decode step for callers that cannot allocate device
// memory when they call us.
//
// Some callers must not allocate at call time: a serving engine that reserved nearly all of the
// GPU's memory for its paged KV cache when it started (a cudaMalloc here could fail, or steal
// memory the engine has budgeted), or a runtime that forbids cudaMalloc on its decode loop because
// cudaMalloc synchronises the device and stalls every stream. Such callers can still hand us their
// inputs and outputs, but not a workspace. This entry point therefore keeps the split partial
// sums of the decode kernel in a fixed array that is part of the library's device image, and
// neither it nor anything it calls allocates: no cudaMalloc, no cudaFree, no torch allocation, not
// even the status word the other entry points create on first use.
//
// Limits and behaviour:
//   * The scratch array holds kNoAllocScratchFloats floats (16 MiB). It belongs to this file's
//     device module. With CUDA's lazy module loading (the default) the module, and with it the
//     16 MiB of device memory, is loaded by the first call on each device (the address look-up
//     below), not when the library is loaded; the decode kernels' own module likewise loads on
//     its first launch. So the FIRST call on a device does take device memory, and may
//     synchronise. Make that first call at start-up, before reserving the rest of the GPU's memory
//     and before any stream capture; from then on the device holds the array until the process
//     exits, and calls allocate nothing.
//   * A call whose split partial sums (batch x chunks x H_r x d_v floats, chunks chosen as in
//     iamap_mapped_av_paged) do not fit returns IAMAP_ERR_CAPACITY without launching anything.
//   * The device address of the array is looked up with cudaGetSymbolAddress, with the device
//     current, and cached per (device, current context). A call from another context on the same
//     device (a driver-API context, or the primary context re-created after cudaDeviceReset)
//     looks it up again, so a stale address is never used.
//   * All calls on a device share the one array, and it keeps the previous call's contents. The
//     kernel writes every partial sum it later reads, so nothing needs clearing between calls, but
//     two calls whose work overlaps on the GPU (different streams, no ordering between them) race
//     on the array and corrupt each other's results. Order such calls on one stream.
//   * Page-table entries outside [0, num_pages) are skipped (they contribute nothing) and, since
//     this entry point has no status word, they are not reported.
#include <mutex>

#include "internal.h"

namespace iamap {

constexpr size_t kNoAllocScratchFloats = (size_t)4 << 20;  // 16 MiB of fp32 partial sums
constexpr int kNoAllocMaxDevices = 64;

// File-scope device array. In host code `g_noalloc_scratch` is only a host-side stand-in for the
// symbol: its device address must come from cudaGetSymbolAddress, never from taking &g_... here.
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

static std::mutex g_noalloc_mutex;
struct NoAllocSlot {
  void* ctx = nullptr;    // the context the address was looked up in
  float* ptr = nullptr;
};
static NoAllocSlot g_noalloc_slot[kNoAllocMaxDevices];

// The current context of the calling thread (cuCtxGetCurrent through the runtime's driver entry
// point, so the library needs no libcuda link).
static int current_context(void** ctx) {
  using GetCurrent = int (*)(void**);
  static GetCurrent fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<GetCurrent>(f);
  });
  if (!fn) return set_error(IAMAP_ERR_CUDA, "cuCtxGetCurrent is unavailable");
  if (fn(ctx) != 0) return set_error(IAMAP_ERR_CUDA, "cuCtxGetCurrent failed");
  return IAMAP_OK;
}

// Device address of the scratch array in the current context of the current device (looked up
// once per device and context).
static int noalloc_scratch(float** out) {
  int dev = -1;
  IAMAP_CUDA_CHECK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kNoAllocMaxDevices)
    return set_error(IAMAP_ERR_UNSUPPORTED, "device ordinal %d beyond %d", dev, kNoAllocMaxDevices);
  void* ctx = nullptr;
  int rc = current_context(&ctx);
  if (rc) return rc;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  NoAllocSlot& slot = g_noalloc_slot[dev];
  if (ctx == nullptr || slot.ptr == nullptr || slot.ctx != ctx) {
    // (a thread with no current context gets the device's primary context from the look-up)
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return set_error(IAMAP_ERR_CUDA, "cudaGetSymbolAddress of the decode scratch failed: %s",
                       cudaGetErrorString(e));
    rc = current_context(&ctx);
    if (rc) return rc;
    slot.ctx = ctx;
    slot.ptr = static_cast<float*>(p);
  }
  *out = slot.ptr;
  return IAMAP_OK;
}

}  // namespace iamap

using namespace iamap;

extern "C" int iamap_mapped_av_paged_noalloc(const float* p_rows, int ctx_stride, const float* W,
                                             const void* v_pages, int64_t num_pages,
                                             const int32_t* page_table, int max_pages,
                                             int page_size, const int32_t* ctx_lens,
                                             const int32_t* ctx_lens_host, int batch, int H_s,
                                             int H_r, int d_v, float* out, void* stream) {
  clear_error();
  if (!p_rows || !W || !v_pages || !page_table || !ctx_lens || !ctx_lens_host || !out)
    return set_error(IAMAP_ERR_INVALID_ARG, "null pointer");
  if (batch < 1 || H_s < 1 || H_r < 1 || page_size < 1 || max_pages < 0 || num_pages < 0)
    return set_error(IAMAP_ERR_INVALID_ARG, "bad sizes");
  if (d_v % 8 != 0) return set_error(IAMAP_ERR_UNSUPPORTED, "d_v must be a multiple of 8");
  if ((reinterpret_cast<uintptr_t>(v_pages) & 15u) || (reinterpret_cast<uintptr_t>(out) & 15u))
    return set_error(IAMAP_ERR_INVALID_ARG, "v_pages and out must be 16-byte aligned");
  int max_ctx = 0;
  for (int b = 0; b < batch; ++b) {
    const int c = ctx_lens_host[b];
    if (c < 0 || c > ctx_stride || (int64_t)c > (int64_t)max_pages * page_size)
      return set_error(IAMAP_ERR_INVALID_ARG, "ctx_lens[%d]=%d exceeds the row or page table", b, c);
    if (c > max_ctx) max_ctx = c;
  }
  int dev = -1, sms = 0;
  IAMAP_CUDA_CHECK(cudaGetDevice(&dev));
  IAMAP_CUDA_CHECK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  PagedArgs a;
  paged_split(batch, max_ctx, page_size, sms, &a.chunks, &a.pages_per_chunk);
  const size_t need = (size_t)batch * a.chunks * H_r * d_v;
  if (need > kNoAllocScratchFloats)
    return set_error(IAMAP_ERR_CAPACITY,
                     "partial sums need %zu bytes; the fixed scratch of this entry point holds "
                     "%zu bytes (use iamap_mapped_av_paged with a workspace)",
                     need * sizeof(float), kNoAllocScratchFloats * sizeof(float));
  float* scratch = nullptr;
  int rc = noalloc_scratch(&scratch);
  if (rc) return rc;
  a.p_rows = p_rows;
  a.ctx_stride = ctx_stride;
  a.W = W;
  a.v_pages = v_pages;
  a.num_pages = num_pages;
  a.page_table = page_table;
  a.max_pages = max_pages;
  a.page_size = page_size;
  a.ctx_lens = ctx_lens;
  a.max_ctx = max_ctx;
  a.batch = batch;
  a.H_s = H_s;
  a.H_r = H_r;
  a.d_v = d_v;
  a.out = out;
  a.partial = scratch;
  a.status = nullptr;
  return mapped_av_paged_impl(a, static_cast<cudaStream_t>(stream));
}
