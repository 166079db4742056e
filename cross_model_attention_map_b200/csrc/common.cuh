// Shared device helpers and host-side plumbing of libiamap (sm_100a).
#pragma once

#include <cstdint>
#include <cstddef>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/iamap.h"

namespace iamap {

// ------------------------------------------------------------------------------------------------
// Host side: error reporting and per-device context
// ------------------------------------------------------------------------------------------------

int set_error(int code, const char* fmt, ...);   // records the thread-local message, returns code
void clear_error();

// Per-device context: a device status word (IAMAP_DEV_* bits) that kernels OR into.
struct DeviceContext {
  int device = -1;
  unsigned int* status = nullptr;   // device memory, 1 word
  int num_sms = 0;
};
// Returns the context of the current device (created on first use) or nullptr on failure (the
// error is recorded).
DeviceContext* device_context();

#define IAMAP_CUDA_CHECK(call)                                                                 \
  do {                                                                                         \
    cudaError_t _e = (call);                                                                   \
    if (_e != cudaSuccess)                                                                     \
      return ::iamap::set_error(IAMAP_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(_e)); \
  } while (0)

#define IAMAP_LAUNCH_CHECK(what)                                                               \
  do {                                                                                         \
    cudaError_t _e = cudaGetLastError();                                                       \
    if (_e != cudaSuccess)                                                                     \
      return ::iamap::set_error(IAMAP_ERR_CUDA, "launch of %s failed: %s", what,               \
                                cudaGetErrorString(_e));                                       \
  } while (0)

// Scheduling tables placed in the caller's workspace (see iamap_compress_workspace_bytes).
struct SeqTables {
  int32_t* nb;        // [num_seqs]     row blocks of each sequence
  int32_t* rb_start;  // [num_seqs + 1]
  int32_t* cb_start;  // [num_seqs + 1]  (fits int32: checked on the host)
  int2* items;        // [num_rowblocks] (seq, I), longest causal row first
  int64_t* row_tiles; // [num_rowblocks] tiles of each row block (then their exclusive scan)
  int2* pairs;        // [num_pairs] (seq, I0) of the row-block pairs (I0, I0 + 1), I0 even,
                      // longest first
  // Chunked prefill: sequence s contributes only its row blocks I >= I0[s] (its query rows
  // [B * I0[s], L_s)), and the query (and output) row of sequence-local row i is packed at
  // qoff[s] + i. Whole sequences have I0 = 0 and qoff = cu_seqlens[s].
  int32_t* I0;        // [num_seqs]
  int32_t* qoff;      // [num_seqs]
};

// Index of row block I of sequence s among the row blocks listed in the tables.
__device__ __forceinline__ int tab_rb(const SeqTables& t, int s, int I) {
  return t.rb_start[s] + I - t.I0[s];
}
// Index of causal block (I, 0) of sequence s among the causal blocks listed in the tables.
__device__ __forceinline__ int64_t tab_cb(const SeqTables& t, int s, int I) {
  const int64_t i0 = t.I0[s];
  return (int64_t)t.cb_start[s] + (int64_t)I * (I + 1) / 2 - i0 * (i0 + 1) / 2;
}
size_t seq_tables_bytes(int num_seqs, int64_t num_rowblocks);
SeqTables carve_seq_tables(void* ws, int num_seqs, int64_t num_rowblocks);

// Host plan of packed sequences.
struct Plan {
  int64_t num_rowblocks = 0;
  int64_t num_causal_blocks = 0;
  int32_t max_nb = 0;
  int64_t num_pairs = 0;   // sum over sequences of ceil(nb / 2)
};
int make_plan(const int32_t* cu_host, int num_seqs, int B, int64_t n, Plan* out);
// Plan of the chunks of packed sequences: sequence s has keys [0, cu_k[s+1] - cu_k[s]) and query
// rows [starts[s], that length), starts[s] a multiple of B; the query rows are packed by
// cu_q (cu_q[s+1] - cu_q[s] rows each, n_q in all). Only the chunk's row blocks are counted.
int make_chunk_plan(const int32_t* cu_k_host, const int32_t* cu_q_host,
                    const int32_t* starts_host, int num_seqs, int B, int64_t n_k, int64_t n_q,
                    Plan* out);

// Builds SeqTables on the device from cu_seqlens (device), on `stream`. With cu_q and starts
// (device, both non-null) the tables list only each sequence's chunk (see make_chunk_plan).
int launch_build_tables(const int32_t* cu_seqlens, int num_seqs, int B, int32_t max_nb,
                        SeqTables t, cudaStream_t stream, const int32_t* cu_q = nullptr,
                        const int32_t* starts = nullptr);

// ------------------------------------------------------------------------------------------------
// Device side helpers
// ------------------------------------------------------------------------------------------------

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                            uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                                  uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + D, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void raise_status(unsigned int* status, unsigned int bits) {
  if (status) atomicOr(status, bits);
}

}  // namespace iamap
