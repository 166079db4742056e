// iamap_prefill_steps_host: prefill steps of one mapped layer pair on host-resident inputs, with
// the host <-> device copies inside the library.
//
// Every step uploads its own q, k, v, W from (pinned) host memory, runs compress and mapped_av,
// and reads its output back to host memory. Two device sets of inputs and outputs (the `io`
// buffer) let the upload of step i + 1 and the read-back of step i - 1 overlap the kernels of
// step i: the copies run on an upload and a download stream owned by the library (one pair per
// device, created on first use), ordered against the caller's stream by events:
//
//   upload i      (upload stream)   after the kernels of step i - 2 have read set i % 2
//   kernels i     (caller's stream) after upload i, and after the read-back of step i - 2 has
//                                   emptied output set i % 2
//   read-back i   (download stream) after kernels i
//
// The call enqueues everything and returns; the caller's stream waits for the last read-back,
// so anything recorded on it after the call (an event, a synchronisation) covers all steps.
// One cudaMemcpyAsync per copy.
#include <mutex>

#include "internal.h"

namespace iamap {
namespace {

constexpr int kMaxDev = 64;

struct CopyStreams {
  cudaStream_t up = nullptr, down = nullptr;
  cudaEvent_t entry = nullptr;
  cudaEvent_t uploaded[2] = {}, computed[2] = {}, downloaded[2] = {};
};

std::mutex g_mutex;
CopyStreams g_streams[kMaxDev];

int copy_streams(CopyStreams** out) {
  int dev = -1;
  IAMAP_CUDA_CHECK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDev)
    return set_error(IAMAP_ERR_UNSUPPORTED, "device index %d beyond %d", dev, kMaxDev);
  std::lock_guard<std::mutex> lock(g_mutex);
  CopyStreams& c = g_streams[dev];
  if (c.up == nullptr) {
    CopyStreams n;
    IAMAP_CUDA_CHECK(cudaStreamCreateWithFlags(&n.up, cudaStreamNonBlocking));
    IAMAP_CUDA_CHECK(cudaStreamCreateWithFlags(&n.down, cudaStreamNonBlocking));
    IAMAP_CUDA_CHECK(cudaEventCreateWithFlags(&n.entry, cudaEventDisableTiming));
    for (int i = 0; i < 2; ++i) {
      IAMAP_CUDA_CHECK(cudaEventCreateWithFlags(&n.uploaded[i], cudaEventDisableTiming));
      IAMAP_CUDA_CHECK(cudaEventCreateWithFlags(&n.computed[i], cudaEventDisableTiming));
      IAMAP_CUDA_CHECK(cudaEventCreateWithFlags(&n.downloaded[i], cudaEventDisableTiming));
    }
    c = n;
  }
  *out = &c;
  return IAMAP_OK;
}

size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }

struct IoSet {
  void* q;
  void* k;
  void* v;
  float* W;
  float* out;
};

struct IoSizes {
  size_t q, v, W, out, set;
};

IoSizes io_sizes(int64_t n, int H_s, int d, int H_r, int H_kv, int d_v) {
  IoSizes z;
  z.q = 2 * (size_t)n * H_s * d;
  z.v = 2 * (size_t)n * H_kv * d_v;
  z.W = 4 * (size_t)H_r * H_s;
  z.out = 4 * (size_t)n * H_r * d_v;
  z.set = 2 * a256(z.q) + a256(z.v) + a256(z.W) + a256(z.out);
  return z;
}

IoSet carve_set(void* io, const IoSizes& z, int s) {
  char* p = static_cast<char*>(io) + (size_t)s * z.set;
  IoSet r;
  r.q = p;
  p += a256(z.q);
  r.k = p;
  p += a256(z.q);
  r.v = p;
  p += a256(z.v);
  r.W = reinterpret_cast<float*>(p);
  p += a256(z.W);
  r.out = reinterpret_cast<float*>(p);
  return r;
}

}  // namespace
}  // namespace iamap

using namespace iamap;

extern "C" size_t iamap_prefill_io_bytes(int64_t n, int H_s, int d, int H_r, int H_kv, int d_v) {
  if (n < 0 || H_s < 1 || d < 1 || H_r < 1 || H_kv < 1 || d_v < 1) return 0;
  return 2 * io_sizes(n, H_s, d, H_r, H_kv, d_v).set;
}

extern "C" int iamap_prefill_steps_host(
    int steps, const void* const* q_host, const void* const* k_host, const void* const* v_host,
    const float* const* W_host, float* const* out_host, const int32_t* cu_seqlens,
    const int32_t* cu_seqlens_host, int num_seqs, int64_t n, int H_s, int d, int H_r, int H_kv,
    int d_v, int B, float tau, int bias_window, float bias_value, float* lse, float* mass,
    uint64_t* headmask_dense, int32_t* row_ptr, int32_t* col_idx, uint64_t* headmask,
    int64_t* val_off, int64_t* counts, void* vals, int64_t vals_capacity_tiles, void* io,
    size_t io_bytes, void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  if (steps < 0) return set_error(IAMAP_ERR_INVALID_ARG, "steps must be >= 0");
  if (steps == 0) return IAMAP_OK;
  if (!q_host || !k_host || !v_host || !W_host || !out_host)
    return set_error(IAMAP_ERR_INVALID_ARG, "null host pointer array");
  for (int i = 0; i < steps; ++i)
    if (!q_host[i] || !k_host[i] || !v_host[i] || !W_host[i] || !out_host[i])
      return set_error(IAMAP_ERR_INVALID_ARG, "null host pointer for step %d", i);
  if (H_kv < 1 || H_r < 1 || H_r % H_kv != 0)
    return set_error(IAMAP_ERR_INVALID_ARG, "H_kv=%d must divide H_r=%d", H_kv, H_r);
  const IoSizes z = io_sizes(n, H_s, d, H_r, H_kv, d_v);
  if (!io || io_bytes < 2 * z.set)
    return set_error(IAMAP_ERR_WORKSPACE, "io buffer of %zu bytes needed, %zu given", 2 * z.set,
                     io_bytes);
  if (reinterpret_cast<uintptr_t>(io) & 255u)
    return set_error(IAMAP_ERR_INVALID_ARG, "io buffer must be 256-byte aligned");
  CopyStreams* cs = nullptr;
  int rc = copy_streams(&cs);
  if (rc) return rc;
  cudaStream_t comp = static_cast<cudaStream_t>(stream);
  // the first upload follows whatever the caller enqueued before this call
  IAMAP_CUDA_CHECK(cudaEventRecord(cs->entry, comp));
  IAMAP_CUDA_CHECK(cudaStreamWaitEvent(cs->up, cs->entry, 0));

  auto upload = [&](int i) -> int {
    const int s = i & 1;
    const IoSet io_s = carve_set(io, z, s);
    if (i >= 2) IAMAP_CUDA_CHECK(cudaStreamWaitEvent(cs->up, cs->computed[s], 0));
    IAMAP_CUDA_CHECK(cudaMemcpyAsync(io_s.q, q_host[i], z.q, cudaMemcpyHostToDevice, cs->up));
    IAMAP_CUDA_CHECK(cudaMemcpyAsync(io_s.k, k_host[i], z.q, cudaMemcpyHostToDevice, cs->up));
    IAMAP_CUDA_CHECK(cudaMemcpyAsync(io_s.v, v_host[i], z.v, cudaMemcpyHostToDevice, cs->up));
    IAMAP_CUDA_CHECK(cudaMemcpyAsync(io_s.W, W_host[i], z.W, cudaMemcpyHostToDevice, cs->up));
    IAMAP_CUDA_CHECK(cudaEventRecord(cs->uploaded[s], cs->up));
    return IAMAP_OK;
  };

  rc = upload(0);
  if (rc) return rc;
  for (int i = 0; i < steps; ++i) {
    const int s = i & 1;
    const IoSet io_s = carve_set(io, z, s);
    if (i + 1 < steps) {
      rc = upload(i + 1);
      if (rc) return rc;
    }
    IAMAP_CUDA_CHECK(cudaStreamWaitEvent(comp, cs->uploaded[s], 0));
    if (i >= 2) IAMAP_CUDA_CHECK(cudaStreamWaitEvent(comp, cs->downloaded[s], 0));
    rc = iamap_compress(io_s.q, io_s.k, cu_seqlens, cu_seqlens_host, num_seqs, n, H_s, d, B, tau,
                        bias_window, bias_value, lse, mass, headmask_dense, row_ptr, col_idx,
                        headmask, val_off, counts, vals, vals_capacity_tiles, ws, ws_bytes, comp);
    if (rc) return rc;
    rc = iamap_mapped_av_gqa(cu_seqlens, cu_seqlens_host, num_seqs, n, B, H_s, row_ptr, col_idx,
                             headmask, val_off, vals, vals_capacity_tiles, io_s.W, H_r, H_kv,
                             io_s.v, d_v, io_s.out, ws, ws_bytes, comp);
    if (rc) return rc;
    IAMAP_CUDA_CHECK(cudaEventRecord(cs->computed[s], comp));
    IAMAP_CUDA_CHECK(cudaStreamWaitEvent(cs->down, cs->computed[s], 0));
    IAMAP_CUDA_CHECK(cudaMemcpyAsync(out_host[i], io_s.out, z.out, cudaMemcpyDeviceToHost,
                                     cs->down));
    IAMAP_CUDA_CHECK(cudaEventRecord(cs->downloaded[s], cs->down));
  }
  // the caller's stream waits for the last read-backs
  IAMAP_CUDA_CHECK(cudaStreamWaitEvent(comp, cs->downloaded[(steps - 1) & 1], 0));
  if (steps >= 2) IAMAP_CUDA_CHECK(cudaStreamWaitEvent(comp, cs->downloaded[steps & 1], 0));
  return IAMAP_OK;
}
