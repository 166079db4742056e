// Host plumbing of libiamap: error messages, the per-device context, sequence planning and the
// device-side scheduling tables shared by the compress and mapped_av kernels.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "tc_utils.cuh"

namespace iamap {

static thread_local char g_last_error[512] = "";

int set_error(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return code;
}

void clear_error() { g_last_error[0] = 0; }

// One context per device index, in a fixed array: a context's address never changes, so a
// pointer returned to one thread stays valid while other threads create other devices' contexts.
constexpr int kMaxDevices = 64;
static std::mutex g_ctx_mutex;
static DeviceContext g_ctx[kMaxDevices];

DeviceContext* device_context() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    set_error(IAMAP_ERR_CUDA, "cudaGetDevice failed");
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    set_error(IAMAP_ERR_UNSUPPORTED, "device index %d beyond %d", dev, kMaxDevices);
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_ctx_mutex);
  DeviceContext& c = g_ctx[dev];
  if (c.status == nullptr) {
    unsigned int* p = nullptr;
    cudaError_t e = cudaMalloc(&p, sizeof(unsigned int));
    if (e != cudaSuccess) {
      set_error(IAMAP_ERR_CUDA, "status word allocation failed: %s", cudaGetErrorString(e));
      return nullptr;
    }
    e = cudaMemset(p, 0, sizeof(unsigned int));
    if (e != cudaSuccess) {
      cudaFree(p);
      set_error(IAMAP_ERR_CUDA, "status word init failed: %s", cudaGetErrorString(e));
      return nullptr;
    }
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    c.device = dev;
    c.status = p;
    c.num_sms = sms;
  }
  return &c;
}

int make_plan(const int32_t* cu_host, int num_seqs, int B, int64_t n, Plan* out) {
  if (!cu_host) return set_error(IAMAP_ERR_INVALID_ARG, "cu_seqlens_host is null");
  if (num_seqs < 1) return set_error(IAMAP_ERR_INVALID_ARG, "num_seqs must be >= 1");
  if (B < 1) return set_error(IAMAP_ERR_INVALID_ARG, "block size must be >= 1");
  if (cu_host[0] != 0) return set_error(IAMAP_ERR_INVALID_ARG, "cu_seqlens[0] must be 0");
  Plan p;
  for (int s = 0; s < num_seqs; ++s) {
    int64_t L = (int64_t)cu_host[s + 1] - cu_host[s];
    if (L < 0) return set_error(IAMAP_ERR_INVALID_ARG, "cu_seqlens decreases at %d", s);
    int64_t nb = (L + B - 1) / B;
    p.num_rowblocks += nb;
    p.num_causal_blocks += nb * (nb + 1) / 2;
    p.num_pairs += (nb + 1) / 2;
    if (nb > p.max_nb) p.max_nb = (int32_t)nb;
  }
  if (n >= 0 && (int64_t)cu_host[num_seqs] != n)
    return set_error(IAMAP_ERR_INVALID_ARG, "cu_seqlens[num_seqs]=%d does not equal n=%lld",
                     cu_host[num_seqs], (long long)n);
  if (p.num_causal_blocks >= (int64_t)INT32_MAX)
    return set_error(IAMAP_ERR_UNSUPPORTED, "more than 2^31 causal blocks");
  *out = p;
  return IAMAP_OK;
}

int make_chunk_plan(const int32_t* cu_k_host, const int32_t* cu_q_host,
                    const int32_t* starts_host, int num_seqs, int B, int64_t n_k, int64_t n_q,
                    Plan* out) {
  if (!cu_k_host || !cu_q_host || !starts_host)
    return set_error(IAMAP_ERR_INVALID_ARG, "cu_k_host, cu_q_host and starts_host are required");
  if (num_seqs < 1) return set_error(IAMAP_ERR_INVALID_ARG, "num_seqs must be >= 1");
  if (B < 1) return set_error(IAMAP_ERR_INVALID_ARG, "block size must be >= 1");
  if (cu_k_host[0] != 0 || cu_q_host[0] != 0)
    return set_error(IAMAP_ERR_INVALID_ARG, "cu_k[0] and cu_q[0] must be 0");
  Plan p;
  for (int s = 0; s < num_seqs; ++s) {
    const int64_t e = (int64_t)cu_k_host[s + 1] - cu_k_host[s];
    const int64_t rows = (int64_t)cu_q_host[s + 1] - cu_q_host[s];
    const int64_t c0 = starts_host[s];
    if (e < 0 || rows < 0) return set_error(IAMAP_ERR_INVALID_ARG, "cu_k or cu_q decreases at %d", s);
    if (c0 < 0 || c0 % B != 0)
      return set_error(IAMAP_ERR_INVALID_ARG, "chunk start %lld of sequence %d is not a "
                       "non-negative multiple of B=%d", (long long)c0, s, B);
    if (c0 + rows != e)
      return set_error(IAMAP_ERR_INVALID_ARG, "sequence %d: a chunk of %lld query rows from %lld "
                       "does not end at the key length %lld", s, (long long)rows, (long long)c0,
                       (long long)e);
    const int64_t nb = (e + B - 1) / B, i0 = c0 / B;
    if (i0 < nb) {
      p.num_rowblocks += nb - i0;
      p.num_causal_blocks += nb * (nb + 1) / 2 - i0 * (i0 + 1) / 2;
      p.num_pairs += (nb + 1) / 2 - i0 / 2;
    }
    if (nb > p.max_nb) p.max_nb = (int32_t)nb;
  }
  if ((int64_t)cu_k_host[num_seqs] != n_k || (int64_t)cu_q_host[num_seqs] != n_q)
    return set_error(IAMAP_ERR_INVALID_ARG, "cu_k / cu_q totals (%d, %d) differ from n_k=%lld, "
                     "n_q=%lld", cu_k_host[num_seqs], cu_q_host[num_seqs], (long long)n_k,
                     (long long)n_q);
  if (p.num_causal_blocks >= (int64_t)INT32_MAX)
    return set_error(IAMAP_ERR_UNSUPPORTED, "more than 2^31 causal blocks");
  *out = p;
  return IAMAP_OK;
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t seq_tables_bytes(int num_seqs, int64_t num_rowblocks) {
  return 3 * align256(sizeof(int32_t) * (size_t)num_seqs) +
         2 * align256(sizeof(int32_t) * (size_t)(num_seqs + 1)) +
         align256(sizeof(int2) * (size_t)(num_rowblocks > 0 ? num_rowblocks : 1)) +
         align256(sizeof(int64_t) * (size_t)(num_rowblocks > 0 ? num_rowblocks : 1)) +
         align256(sizeof(int2) * (size_t)(num_rowblocks > 0 ? num_rowblocks : 1));
}

SeqTables carve_seq_tables(void* ws, int num_seqs, int64_t num_rowblocks) {
  char* p = static_cast<char*>(ws);
  SeqTables t;
  t.nb = reinterpret_cast<int32_t*>(p);
  p += align256(sizeof(int32_t) * (size_t)num_seqs);
  t.rb_start = reinterpret_cast<int32_t*>(p);
  p += align256(sizeof(int32_t) * (size_t)(num_seqs + 1));
  t.cb_start = reinterpret_cast<int32_t*>(p);
  p += align256(sizeof(int32_t) * (size_t)(num_seqs + 1));
  t.items = reinterpret_cast<int2*>(p);
  p += align256(sizeof(int2) * (size_t)(num_rowblocks > 0 ? num_rowblocks : 1));
  t.row_tiles = reinterpret_cast<int64_t*>(p);
  p += align256(sizeof(int64_t) * (size_t)(num_rowblocks > 0 ? num_rowblocks : 1));
  t.pairs = reinterpret_cast<int2*>(p);   // at most num_rowblocks pairs
  p += align256(sizeof(int2) * (size_t)(num_rowblocks > 0 ? num_rowblocks : 1));
  t.I0 = reinterpret_cast<int32_t*>(p);
  p += align256(sizeof(int32_t) * (size_t)num_seqs);
  t.qoff = reinterpret_cast<int32_t*>(p);
  return t;
}

// One CTA. Row blocks are ordered by decreasing causal length (I descending), then by sequence,
// so that the longest rows start first (load balance of the triangular work). A sequence lists
// its row blocks I0[s] .. nb[s] - 1 (I0 = 0 without chunks), and the pairs (E, E + 1), E even,
// that hold at least one of them.
__global__ void build_tables_kernel(const int32_t* __restrict__ cu, int num_seqs, int B,
                                    int32_t max_nb, SeqTables t, const int32_t* __restrict__ cu_q,
                                    const int32_t* __restrict__ starts) {
  if (threadIdx.x == 0) {
    int32_t rb = 0, cb = 0;
    for (int s = 0; s < num_seqs; ++s) {
      int32_t L = cu[s + 1] - cu[s];
      int32_t nb = (L + B - 1) / B;
      int32_t i0 = starts ? starts[s] / B : 0;
      if (i0 > nb) i0 = nb;
      t.nb[s] = nb;
      t.I0[s] = i0;
      t.qoff[s] = starts ? cu_q[s] - starts[s] : cu[s];
      t.rb_start[s] = rb;
      t.cb_start[s] = cb;
      rb += nb - i0;
      cb += nb * (nb + 1) / 2 - i0 * (i0 + 1) / 2;
    }
    t.rb_start[num_seqs] = rb;
    t.cb_start[num_seqs] = cb;
  }
  __syncthreads();
  for (int I = threadIdx.x; I < max_nb; I += blockDim.x) {
    // items with a longer row block come first
    int32_t base = 0;
    for (int s = 0; s < num_seqs; ++s) {
      const int32_t lo = max(t.I0[s], I + 1);
      base += max(0, t.nb[s] - lo);
    }
    int32_t c = 0;
    for (int s = 0; s < num_seqs; ++s)
      if (t.nb[s] > I && I >= t.I0[s]) t.items[base + c++] = make_int2(s, I);
    // pairs (I, I + 1) with I even, in the same order: the pairs after it are those with a
    // larger even first row block
    if ((I & 1) == 0) {
      int32_t pbase = 0;
      for (int s = 0; s < num_seqs; ++s) {
        const int32_t lo = max(I + 2, t.I0[s] & ~1);     // first even block of a later pair
        const int32_t hi = (t.nb[s] - 1) & ~1;           // last even block of the sequence
        pbase += hi >= lo ? (hi - lo) / 2 + 1 : 0;
      }
      int32_t pc = 0;
      for (int s = 0; s < num_seqs; ++s)
        if (t.nb[s] > I && I >= (t.I0[s] & ~1)) t.pairs[pbase + pc++] = make_int2(s, I);
    }
  }
}

int launch_build_tables(const int32_t* cu_seqlens, int num_seqs, int B, int32_t max_nb,
                        SeqTables t, cudaStream_t stream, const int32_t* cu_q,
                        const int32_t* starts) {
  if ((cu_q == nullptr) != (starts == nullptr))
    return set_error(IAMAP_ERR_INVALID_ARG, "chunk tables need both cu_q and starts");
  build_tables_kernel<<<1, 256, 0, stream>>>(cu_seqlens, num_seqs, B, max_nb, t, cu_q, starts);
  IAMAP_LAUNCH_CHECK("build_tables_kernel");
  return IAMAP_OK;
}

}  // namespace iamap

namespace iamap {

// One CTA waits on an mbarrier that nothing arrives on, with the kernels' bounded wait and a
// short limit: the timeout path (status bit, abort flag, orderly return) without a real stall.
__global__ void selftest_timeout_kernel(unsigned int* status, uint64_t limit_ns, int* gave_up) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    tc::mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    tc::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = tc::wait_bar_for(smem_u32(&bar), 0, &abort_flag, status, limit_ns);
    *gave_up = (!ok && abort_flag) ? 1 : 0;
  }
}

}  // namespace iamap

namespace iamap {

int selftest_timeout(int limit_us, int* gave_up_dev, cudaStream_t stream) {
  DeviceContext* c = device_context();
  if (!c) return IAMAP_ERR_CUDA;
  selftest_timeout_kernel<<<1, 32, 0, stream>>>(c->status, (uint64_t)limit_us * 1000ull,
                                                gave_up_dev);
  IAMAP_LAUNCH_CHECK("selftest_timeout_kernel");
  return IAMAP_OK;
}

}  // namespace iamap

using namespace iamap;

extern "C" int iamap_selftest_wait_timeout(int limit_us, int* gave_up, void* stream) {
  clear_error();
  if (limit_us < 1 || limit_us > 1000000 || !gave_up)
    return set_error(IAMAP_ERR_INVALID_ARG, "limit_us must be in [1, 1e6] and gave_up non-null");
  return selftest_timeout(limit_us, gave_up, static_cast<cudaStream_t>(stream));
}

extern "C" int iamap_version(void) { return (0 << 16) | 1; }

extern "C" const char* iamap_last_error(void) { return g_last_error; }

extern "C" int iamap_device_status(void* stream, int* status) {
  clear_error();
  if (!status) return set_error(IAMAP_ERR_INVALID_ARG, "status is null");
  DeviceContext* c = device_context();
  if (!c) return IAMAP_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  IAMAP_CUDA_CHECK(cudaStreamSynchronize(st));
  unsigned int h = 0;
  IAMAP_CUDA_CHECK(cudaMemcpyAsync(&h, c->status, sizeof(h), cudaMemcpyDeviceToHost, st));
  IAMAP_CUDA_CHECK(cudaMemsetAsync(c->status, 0, sizeof(unsigned int), st));
  IAMAP_CUDA_CHECK(cudaStreamSynchronize(st));
  *status = (int)h;
  return IAMAP_OK;
}

extern "C" int iamap_plan(const int32_t* cu_seqlens_host, int num_seqs, int B,
                          int64_t* num_rowblocks, int64_t* num_causal_blocks,
                          int32_t* max_blocks_per_seq) {
  clear_error();
  Plan p;
  int rc = make_plan(cu_seqlens_host, num_seqs, B, -1, &p);
  if (rc) return rc;
  if (num_rowblocks) *num_rowblocks = p.num_rowblocks;
  if (num_causal_blocks) *num_causal_blocks = p.num_causal_blocks;
  if (max_blocks_per_seq) *max_blocks_per_seq = p.max_nb;
  return IAMAP_OK;
}

extern "C" size_t iamap_compress_workspace_bytes(int num_seqs, int64_t num_rowblocks) {
  if (num_seqs < 1 || num_rowblocks < 0) return 0;
  return seq_tables_bytes(num_seqs, num_rowblocks);
}
