// extern "C" entry points of the chunked-prefill form and of the sender's own attention output:
// argument validation, the chunk plan and tables, and dispatch to the tensor-core kernels.
//
// A chunk of sequence s is its query rows [starts[s], e_s) with e_s = cu_k[s + 1] - cu_k[s]; it
// attends to the keys [0, e_s) of that sequence, with absolute positions in the causal mask and
// the local bias. starts[s] is a multiple of B, so the chunk's row blocks are the sequence's own
// row blocks starts[s] / B .. ceil(e_s / B) - 1 and every result equals the whole-sequence
// result of those rows (MapFlow news page, the paragraph on the vLLM integration: the fused
// kernel works with chunked prefill). Whole sequences are chunks with starts[s] = 0.
#include <algorithm>

#include "internal.h"

using namespace iamap;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_chunk_common(int B, int H_s, int d) {
  if (B != 64) return set_error(IAMAP_ERR_UNSUPPORTED, "only block size B = 64 is implemented");
  if (H_s < 1 || H_s > 64) return set_error(IAMAP_ERR_UNSUPPORTED, "H_s must be in [1, 64]");
  if (d != 64 && d != 128) return set_error(IAMAP_ERR_UNSUPPORTED, "head dim must be 64 or 128");
  return IAMAP_OK;
}

// Plan and (optionally) device tables of the chunks; the chunk form runs on the tensor-core
// kernels only (at most 256 column blocks per sequence).
int setup_chunk_tables(const int32_t* cu_q, const int32_t* cu_k, const int32_t* starts,
                       const int32_t* cu_q_host, const int32_t* cu_k_host,
                       const int32_t* starts_host, int num_seqs, int64_t n_q, int64_t n_k, int B,
                       void* ws, size_t ws_bytes, cudaStream_t stream, Plan* plan, SeqTables* tab,
                       bool build) {
  int rc = make_chunk_plan(cu_k_host, cu_q_host, starts_host, num_seqs, B, n_k, n_q, plan);
  if (rc) return rc;
  if (!cu_q || !cu_k || !starts)
    return set_error(IAMAP_ERR_INVALID_ARG, "cu_q, cu_k and starts (device) are required");
  const size_t need = seq_tables_bytes(num_seqs, plan->num_rowblocks);
  if (!ws || ws_bytes < need)
    return set_error(IAMAP_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                     ws_bytes);
  *tab = carve_seq_tables(ws, num_seqs, plan->num_rowblocks);
  if (build && plan->num_rowblocks > 0)
    return launch_build_tables(cu_k, num_seqs, B, plan->max_nb, *tab, stream, cu_q, starts);
  return IAMAP_OK;
}

// Stage 1 + stage 2 (+ the sender output) on prepared tables.
int compress_on_tables(CompressArgs& a, const int64_t* counts, void* vals, int64_t cap,
                       cudaStream_t st) {
  int rc = compress_stats_impl(a, st);
  if (rc) return rc;
  a.lse_in = a.lse;
  a.row_ptr_in = a.row_ptr;
  a.col_idx_in = a.col_idx;
  a.headmask_in = a.headmask;
  a.val_off_in = a.val_off;
  a.counts_in = counts;
  a.vals = vals;
  a.capacity = cap;
  return compress_extract_impl(a, st);
}

int check_compress_outputs(float* lse, float* mass, uint64_t* headmask_dense, int32_t* row_ptr,
                           int32_t* col_idx, uint64_t* headmask, int64_t* val_off,
                           int64_t* counts, void* vals, int64_t cap, float tau, int bias_window,
                           const void* v_s, int d_vs, float* o_s) {
  if (!lse || !mass || !headmask_dense || !row_ptr || !col_idx || !headmask || !val_off ||
      !counts || (!vals && cap > 0))
    return set_error(IAMAP_ERR_INVALID_ARG, "null tensor pointer");
  if (cap < 0) return set_error(IAMAP_ERR_INVALID_ARG, "negative capacity");
  if (vals && !aligned16(vals)) return set_error(IAMAP_ERR_INVALID_ARG, "vals must be 16-byte aligned");
  if (!(tau > 0.f)) return set_error(IAMAP_ERR_INVALID_ARG, "tau must be > 0");
  if (bias_window < 0) return set_error(IAMAP_ERR_INVALID_ARG, "bias_window must be >= 0");
  if ((v_s == nullptr) != (o_s == nullptr))
    return set_error(IAMAP_ERR_INVALID_ARG, "v_s and o_s must be given together");
  if (o_s) {
    if (d_vs != 64 && d_vs != 128)
      return set_error(IAMAP_ERR_UNSUPPORTED, "sender value dim d_vs must be 64 or 128");
    if (!aligned16(v_s) || !aligned16(o_s))
      return set_error(IAMAP_ERR_INVALID_ARG, "v_s and o_s must be 16-byte aligned");
  }
  return IAMAP_OK;
}

}  // namespace

extern "C" int iamap_chunk_plan(const int32_t* cu_q_host, const int32_t* cu_k_host,
                                const int32_t* starts_host, int num_seqs, int B,
                                int64_t* num_rowblocks, int64_t* num_causal_blocks,
                                int32_t* max_blocks_per_seq) {
  clear_error();
  if (!cu_q_host || !cu_k_host || !starts_host || num_seqs < 1)
    return set_error(IAMAP_ERR_INVALID_ARG, "null host arrays or num_seqs < 1");
  Plan p;
  int rc = make_chunk_plan(cu_k_host, cu_q_host, starts_host, num_seqs, B, cu_k_host[num_seqs],
                           cu_q_host[num_seqs], &p);
  if (rc) return rc;
  if (num_rowblocks) *num_rowblocks = p.num_rowblocks;
  if (num_causal_blocks) *num_causal_blocks = p.num_causal_blocks;
  if (max_blocks_per_seq) *max_blocks_per_seq = p.max_nb;
  return IAMAP_OK;
}

extern "C" int iamap_compress_chunk(
    const void* q, const void* k, const int32_t* cu_q, const int32_t* cu_k, const int32_t* starts,
    const int32_t* cu_q_host, const int32_t* cu_k_host, const int32_t* starts_host, int num_seqs,
    int64_t n_q, int64_t n_k, int H_s, int d, int B, float tau, int bias_window, float bias_value,
    const void* v_s, int d_vs, float* o_s, float* lse, float* mass, uint64_t* headmask_dense,
    int32_t* row_ptr, int32_t* col_idx, uint64_t* headmask, int64_t* val_off, int64_t* counts,
    void* vals, int64_t vals_capacity_tiles, void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  int rc = check_chunk_common(B, H_s, d);
  if (rc) return rc;
  if (!q || !k) return set_error(IAMAP_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k))
    return set_error(IAMAP_ERR_INVALID_ARG, "q, k must be 16-byte aligned");
  rc = check_compress_outputs(lse, mass, headmask_dense, row_ptr, col_idx, headmask, val_off,
                              counts, vals, vals_capacity_tiles, tau, bias_window, v_s, d_vs, o_s);
  if (rc) return rc;
  DeviceContext* ctx = device_context();
  if (!ctx) return IAMAP_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CompressArgs a;
  rc = setup_chunk_tables(cu_q, cu_k, starts, cu_q_host, cu_k_host, starts_host, num_seqs, n_q,
                          n_k, B, ws, ws_bytes, st, &a.plan, &a.tab, true);
  if (rc) return rc;
  if (!compress_tc_supported(d, a.plan.max_nb))
    return set_error(IAMAP_ERR_UNSUPPORTED, "the chunk form needs sequences of at most 256 "
                     "blocks (%d given)", a.plan.max_nb);
  a.q = q;
  a.k = k;
  a.cu_seqlens = cu_k;
  a.num_seqs = num_seqs;
  a.n = n_q;
  a.n_k = n_k;
  a.H_s = H_s;
  a.d = d;
  a.tau = tau;
  a.bias_window = bias_window;
  a.bias_value = bias_value;
  a.lse = lse;
  a.mass = mass;
  a.headmask_dense = headmask_dense;
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  a.headmask = headmask;
  a.val_off = val_off;
  a.counts = counts;
  a.v_s = v_s;
  a.d_vs = d_vs;
  a.o_s = o_s;
  a.status = ctx->status;
  return compress_on_tables(a, counts, vals, vals_capacity_tiles, st);
}

extern "C" int iamap_compress_with_output(
    const void* q, const void* k, const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
    int num_seqs, int64_t n, int H_s, int d, int B, float tau, int bias_window, float bias_value,
    const void* v_s, int d_vs, float* o_s, float* lse, float* mass, uint64_t* headmask_dense,
    int32_t* row_ptr, int32_t* col_idx, uint64_t* headmask, int64_t* val_off, int64_t* counts,
    void* vals, int64_t vals_capacity_tiles, void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  int rc = check_chunk_common(B, H_s, d);
  if (rc) return rc;
  if (!q || !k || !cu_seqlens) return set_error(IAMAP_ERR_INVALID_ARG, "null tensor pointer");
  if (!v_s || !o_s) return set_error(IAMAP_ERR_INVALID_ARG, "v_s and o_s are required");
  if (!aligned16(q) || !aligned16(k))
    return set_error(IAMAP_ERR_INVALID_ARG, "q, k must be 16-byte aligned");
  rc = check_compress_outputs(lse, mass, headmask_dense, row_ptr, col_idx, headmask, val_off,
                              counts, vals, vals_capacity_tiles, tau, bias_window, v_s, d_vs, o_s);
  if (rc) return rc;
  DeviceContext* ctx = device_context();
  if (!ctx) return IAMAP_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CompressArgs a;
  rc = make_plan(cu_seqlens_host, num_seqs, B, n, &a.plan);
  if (rc) return rc;
  if (!compress_tc_supported(d, a.plan.max_nb))
    return set_error(IAMAP_ERR_UNSUPPORTED, "the sender output needs sequences of at most 256 "
                     "blocks (%d given)", a.plan.max_nb);
  const size_t need = seq_tables_bytes(num_seqs, a.plan.num_rowblocks);
  if (!ws || ws_bytes < need)
    return set_error(IAMAP_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                     ws_bytes);
  a.tab = carve_seq_tables(ws, num_seqs, a.plan.num_rowblocks);
  if (a.plan.num_rowblocks > 0) {
    rc = launch_build_tables(cu_seqlens, num_seqs, B, a.plan.max_nb, a.tab, st);
    if (rc) return rc;
  }
  a.q = q;
  a.k = k;
  a.cu_seqlens = cu_seqlens;
  a.num_seqs = num_seqs;
  a.n = n;
  a.H_s = H_s;
  a.d = d;
  a.tau = tau;
  a.bias_window = bias_window;
  a.bias_value = bias_value;
  a.lse = lse;
  a.mass = mass;
  a.headmask_dense = headmask_dense;
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  a.headmask = headmask;
  a.val_off = val_off;
  a.counts = counts;
  a.v_s = v_s;
  a.d_vs = d_vs;
  a.o_s = o_s;
  a.status = ctx->status;
  return compress_on_tables(a, counts, vals, vals_capacity_tiles, st);
}

extern "C" int iamap_compress_extract_with_output(
    const void* q, const void* k, const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
    int num_seqs, int64_t n, int H_s, int d, int B, int bias_window, float bias_value,
    const void* v_s, int d_vs, float* o_s, const float* lse, const int32_t* row_ptr,
    const int32_t* col_idx, const uint64_t* headmask, const int64_t* val_off,
    const int64_t* counts, void* vals, int64_t vals_capacity_tiles, void* ws, size_t ws_bytes,
    void* stream) {
  clear_error();
  int rc = check_chunk_common(B, H_s, d);
  if (rc) return rc;
  if (!q || !k || !cu_seqlens || !lse || !row_ptr || !col_idx || !headmask || !val_off ||
      !counts || (!vals && vals_capacity_tiles > 0))
    return set_error(IAMAP_ERR_INVALID_ARG, "null tensor pointer");
  if (!v_s || !o_s) return set_error(IAMAP_ERR_INVALID_ARG, "v_s and o_s are required");
  if (d_vs != 64 && d_vs != 128)
    return set_error(IAMAP_ERR_UNSUPPORTED, "sender value dim d_vs must be 64 or 128");
  if (vals_capacity_tiles < 0) return set_error(IAMAP_ERR_INVALID_ARG, "negative capacity");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v_s) || !aligned16(o_s) ||
      (vals && !aligned16(vals)))
    return set_error(IAMAP_ERR_INVALID_ARG, "q, k, v_s, o_s, vals must be 16-byte aligned");
  DeviceContext* ctx = device_context();
  if (!ctx) return IAMAP_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CompressArgs a;
  rc = make_plan(cu_seqlens_host, num_seqs, B, n, &a.plan);
  if (rc) return rc;
  if (!compress_tc_supported(d, a.plan.max_nb))
    return set_error(IAMAP_ERR_UNSUPPORTED, "the sender output needs sequences of at most 256 "
                     "blocks (%d given)", a.plan.max_nb);
  const size_t need = seq_tables_bytes(num_seqs, a.plan.num_rowblocks);
  if (!ws || ws_bytes < need)
    return set_error(IAMAP_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                     ws_bytes);
  a.tab = carve_seq_tables(ws, num_seqs, a.plan.num_rowblocks);
  if (a.plan.num_rowblocks > 0) {
    rc = launch_build_tables(cu_seqlens, num_seqs, B, a.plan.max_nb, a.tab, st);
    if (rc) return rc;
  }
  a.q = q;
  a.k = k;
  a.cu_seqlens = cu_seqlens;
  a.num_seqs = num_seqs;
  a.n = n;
  a.H_s = H_s;
  a.d = d;
  a.bias_window = bias_window;
  a.bias_value = bias_value;
  a.lse_in = lse;
  a.row_ptr_in = row_ptr;
  a.col_idx_in = col_idx;
  a.headmask_in = headmask;
  a.val_off_in = val_off;
  a.counts_in = counts;
  a.vals = vals;
  a.capacity = vals_capacity_tiles;
  a.v_s = v_s;
  a.d_vs = d_vs;
  a.o_s = o_s;
  a.status = ctx->status;
  return compress_extract_impl(a, st);
}

extern "C" int iamap_mapped_av_chunk(
    const int32_t* cu_q, const int32_t* cu_k, const int32_t* starts, const int32_t* cu_q_host,
    const int32_t* cu_k_host, const int32_t* starts_host, int num_seqs, int64_t n_q, int64_t n_k,
    int B, int H_s, const int32_t* row_ptr, const int32_t* col_idx, const uint64_t* headmask,
    const int64_t* val_off, const void* vals, int64_t vals_capacity_tiles, const float* W,
    int H_r, int H_kv, const void* v, int d_v, float* out, void* ws, size_t ws_bytes,
    void* stream) {
  clear_error();
  int rc = check_chunk_common(B, H_s, d_v);
  if (rc) return rc;
  if (H_r < 1) return set_error(IAMAP_ERR_INVALID_ARG, "H_r must be >= 1");
  if (H_kv < 1 || H_r % H_kv != 0)
    return set_error(IAMAP_ERR_INVALID_ARG, "H_kv=%d must divide H_r=%d", H_kv, H_r);
  if (!row_ptr || !col_idx || !headmask || !val_off || !W || !v || !out ||
      (!vals && vals_capacity_tiles > 0))
    return set_error(IAMAP_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(v) || (vals && !aligned16(vals)) || !aligned16(out))
    return set_error(IAMAP_ERR_INVALID_ARG, "v, vals, out must be 16-byte aligned");
  DeviceContext* ctx = device_context();
  if (!ctx) return IAMAP_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MappedAvArgs a;
  rc = setup_chunk_tables(cu_q, cu_k, starts, cu_q_host, cu_k_host, starts_host, num_seqs, n_q,
                          n_k, B, ws, ws_bytes, st, &a.plan, &a.tab, true);
  if (rc) return rc;
  a.cu_seqlens = cu_k;
  a.num_seqs = num_seqs;
  a.n = n_q;
  a.n_k = n_k;
  a.H_s = H_s;
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  a.headmask = headmask;
  a.val_off = val_off;
  a.vals = vals;
  a.capacity = vals_capacity_tiles;
  a.W = W;
  a.H_r = H_r;
  a.H_kv = H_kv;
  a.v = v;
  a.d_v = d_v;
  a.out = out;
  a.status = ctx->status;
  return mapped_av_impl(a, st);
}
