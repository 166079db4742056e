// extern "C" entry points of libiamap: argument validation, planning and dispatch to the kernels.
// Every function returns IAMAP_OK or a negative IAMAP_ERR_* code and records a message for
// iamap_last_error(); no C++ exception crosses this boundary.
#include <algorithm>
#include <vector>

#include "internal.h"

using namespace iamap;

namespace {

constexpr int kMaxSeqBlocks = 512;  // compress: at most 512 row blocks of 64 per sequence

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common(int B, int H_s, int d) {
  if (B != 64) return set_error(IAMAP_ERR_UNSUPPORTED, "only block size B = 64 is implemented");
  if (H_s < 1 || H_s > 64) return set_error(IAMAP_ERR_UNSUPPORTED, "H_s must be in [1, 64]");
  if (d != 64 && d != 128) return set_error(IAMAP_ERR_UNSUPPORTED, "head dim must be 64 or 128");
  return IAMAP_OK;
}

int setup_tables(const int32_t* cu, const int32_t* cu_host, int num_seqs, int64_t n, int B,
                 void* ws, size_t ws_bytes, cudaStream_t stream, Plan* plan, SeqTables* tab,
                 bool build) {
  int rc = make_plan(cu_host, num_seqs, B, n, plan);
  if (rc) return rc;
  if (plan->max_nb > kMaxSeqBlocks)
    return set_error(IAMAP_ERR_UNSUPPORTED, "sequence of %d row blocks exceeds %d",
                     plan->max_nb, kMaxSeqBlocks);
  const size_t need = seq_tables_bytes(num_seqs, plan->num_rowblocks);
  if (!ws || ws_bytes < need)
    return set_error(IAMAP_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                     ws_bytes);
  if (!cu) return set_error(IAMAP_ERR_INVALID_ARG, "cu_seqlens is null");
  *tab = carve_seq_tables(ws, num_seqs, plan->num_rowblocks);
  if (build && plan->num_rowblocks > 0)
    return launch_build_tables(cu, num_seqs, B, plan->max_nb, *tab, stream);
  return IAMAP_OK;
}

}  // namespace

extern "C" int iamap_compress_stats(const void* q, const void* k, const int32_t* cu_seqlens,
                                    const int32_t* cu_seqlens_host, int num_seqs, int64_t n,
                                    int H_s, int d, int B, float tau, int bias_window,
                                    float bias_value, float* lse, float* mass,
                                    uint64_t* headmask_dense, int32_t* row_ptr, int32_t* col_idx,
                                    uint64_t* headmask, int64_t* val_off, int64_t* counts,
                                    void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  int rc = check_common(B, H_s, d);
  if (rc) return rc;
  if (!q || !k || !lse || !mass || !headmask_dense || !row_ptr || !col_idx || !headmask ||
      !val_off || !counts)
    return set_error(IAMAP_ERR_INVALID_ARG, "null tensor pointer");
  if (!(tau > 0.f)) return set_error(IAMAP_ERR_INVALID_ARG, "tau must be > 0");
  if (bias_window < 0) return set_error(IAMAP_ERR_INVALID_ARG, "bias_window must be >= 0");
  if (!aligned16(q) || !aligned16(k)) return set_error(IAMAP_ERR_INVALID_ARG, "q, k must be 16-byte aligned");
  DeviceContext* ctx = device_context();
  if (!ctx) return IAMAP_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CompressArgs a;
  rc = setup_tables(cu_seqlens, cu_seqlens_host, num_seqs, n, B, ws, ws_bytes, st, &a.plan,
                    &a.tab, true);
  if (rc) return rc;
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
  a.status = ctx->status;
  return compress_stats_impl(a, st);
}

static int extract_common(const void* q, const void* k, const int32_t* cu_seqlens,
                          const int32_t* cu_seqlens_host, int num_seqs, int64_t n, int H_s, int d,
                          int B, int bias_window, float bias_value, const float* lse,
                          const int32_t* row_ptr, const int32_t* col_idx,
                          const uint64_t* headmask, const int64_t* val_off, const int64_t* counts,
                          void* vals, int64_t cap, void* ws, size_t ws_bytes, void* stream,
                          bool build_tables) {
  int rc = check_common(B, H_s, d);
  if (rc) return rc;
  if (!q || !k || !lse || !row_ptr || !col_idx || !headmask || !val_off || !counts ||
      (!vals && cap > 0))
    return set_error(IAMAP_ERR_INVALID_ARG, "null tensor pointer");
  if (cap < 0) return set_error(IAMAP_ERR_INVALID_ARG, "negative capacity");
  if (!aligned16(q) || !aligned16(k) || (vals && !aligned16(vals)))
    return set_error(IAMAP_ERR_INVALID_ARG, "q, k, vals must be 16-byte aligned");
  DeviceContext* ctx = device_context();
  if (!ctx) return IAMAP_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CompressArgs a;
  rc = setup_tables(cu_seqlens, cu_seqlens_host, num_seqs, n, B, ws, ws_bytes, st, &a.plan,
                    &a.tab, build_tables);
  if (rc) return rc;
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
  a.capacity = cap;
  a.status = ctx->status;
  return compress_extract_impl(a, st);
}

extern "C" int iamap_compress_extract(const void* q, const void* k, const int32_t* cu_seqlens,
                                      const int32_t* cu_seqlens_host, int num_seqs, int64_t n,
                                      int H_s, int d, int B, int bias_window, float bias_value,
                                      const float* lse, const int32_t* row_ptr,
                                      const int32_t* col_idx, const uint64_t* headmask,
                                      const int64_t* val_off, const int64_t* counts, void* vals,
                                      int64_t vals_capacity_tiles, void* ws, size_t ws_bytes,
                                      void* stream) {
  clear_error();
  return extract_common(q, k, cu_seqlens, cu_seqlens_host, num_seqs, n, H_s, d, B, bias_window,
                        bias_value, lse, row_ptr, col_idx, headmask, val_off, counts, vals,
                        vals_capacity_tiles, ws, ws_bytes, stream, true);
}

extern "C" int iamap_compress(const void* q, const void* k, const int32_t* cu_seqlens,
                              const int32_t* cu_seqlens_host, int num_seqs, int64_t n, int H_s,
                              int d, int B, float tau, int bias_window, float bias_value,
                              float* lse, float* mass, uint64_t* headmask_dense, int32_t* row_ptr,
                              int32_t* col_idx, uint64_t* headmask, int64_t* val_off,
                              int64_t* counts, void* vals, int64_t vals_capacity_tiles, void* ws,
                              size_t ws_bytes, void* stream) {
  int rc = iamap_compress_stats(q, k, cu_seqlens, cu_seqlens_host, num_seqs, n, H_s, d, B, tau,
                                bias_window, bias_value, lse, mass, headmask_dense, row_ptr,
                                col_idx, headmask, val_off, counts, ws, ws_bytes, stream);
  if (rc) return rc;
  // The scheduling tables built by stage 1 are still in the workspace.
  return extract_common(q, k, cu_seqlens, cu_seqlens_host, num_seqs, n, H_s, d, B, bias_window,
                        bias_value, lse, row_ptr, col_idx, headmask, val_off, counts, vals,
                        vals_capacity_tiles, ws, ws_bytes, stream, false);
}

extern "C" int iamap_mapped_av(const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                               int num_seqs, int64_t n, int B, int H_s, const int32_t* row_ptr,
                               const int32_t* col_idx, const uint64_t* headmask,
                               const int64_t* val_off, const void* vals,
                               int64_t vals_capacity_tiles, const float* W, int H_r,
                               const void* v, int d_v, float* out, void* ws, size_t ws_bytes,
                               void* stream) {
  return iamap_mapped_av_gqa(cu_seqlens, cu_seqlens_host, num_seqs, n, B, H_s, row_ptr, col_idx,
                             headmask, val_off, vals, vals_capacity_tiles, W, H_r, H_r, v, d_v,
                             out, ws, ws_bytes, stream);
}

extern "C" int iamap_mapped_av_gqa(const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                                   int num_seqs, int64_t n, int B, int H_s, const int32_t* row_ptr,
                                   const int32_t* col_idx, const uint64_t* headmask,
                                   const int64_t* val_off, const void* vals,
                                   int64_t vals_capacity_tiles, const float* W, int H_r, int H_kv,
                                   const void* v, int d_v, float* out, void* ws, size_t ws_bytes,
                                   void* stream) {
  clear_error();
  int rc = check_common(B, H_s, d_v);
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
  rc = setup_tables(cu_seqlens, cu_seqlens_host, num_seqs, n, B, ws, ws_bytes, st, &a.plan,
                    &a.tab, true);
  if (rc) return rc;
  a.cu_seqlens = cu_seqlens;
  a.num_seqs = num_seqs;
  a.n = n;
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

extern "C" size_t iamap_mapped_av_paged_workspace_bytes(int batch, int H_r, int d_v, int max_ctx,
                                                        int page_size) {
  if (batch < 1 || H_r < 1 || d_v < 1 || max_ctx < 0 || page_size < 1) return 0;
  DeviceContext* ctx = device_context();
  const int sms = ctx ? ctx->num_sms : 148;
  int chunks = 0, ppc = 0;
  paged_split(batch, max_ctx, page_size, sms, &chunks, &ppc);
  return sizeof(float) * (size_t)batch * chunks * H_r * d_v;
}

extern "C" int iamap_mapped_av_paged(const float* p_rows, int ctx_stride, const float* W,
                                     const void* v_pages, int64_t num_pages,
                                     const int32_t* page_table, int max_pages, int page_size,
                                     const int32_t* ctx_lens, const int32_t* ctx_lens_host,
                                     int batch, int H_s, int H_r, int d_v, float* out, void* ws,
                                     size_t ws_bytes, void* stream) {
  return iamap_mapped_av_paged_gqa(p_rows, ctx_stride, W, v_pages, num_pages, page_table,
                                   max_pages, page_size, ctx_lens, ctx_lens_host, batch, H_s, H_r,
                                   H_r, d_v, out, ws, ws_bytes, stream);
}

extern "C" int iamap_mapped_av_paged_gqa(const float* p_rows, int ctx_stride, const float* W,
                                         const void* v_pages, int64_t num_pages,
                                         const int32_t* page_table, int max_pages, int page_size,
                                         const int32_t* ctx_lens, const int32_t* ctx_lens_host,
                                         int batch, int H_s, int H_r, int H_kv, int d_v,
                                         float* out, void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  if (H_kv < 1 || H_r < 1 || H_r % H_kv != 0)
    return set_error(IAMAP_ERR_INVALID_ARG, "H_kv=%d must divide H_r=%d", H_kv, H_r);
  if (!p_rows || !W || !v_pages || !page_table || !ctx_lens || !ctx_lens_host || !out)
    return set_error(IAMAP_ERR_INVALID_ARG, "null pointer");
  if (batch < 1 || H_s < 1 || H_r < 1 || page_size < 1 || max_pages < 0 || num_pages < 0)
    return set_error(IAMAP_ERR_INVALID_ARG, "bad sizes");
  if (d_v % 8 != 0) return set_error(IAMAP_ERR_UNSUPPORTED, "d_v must be a multiple of 8");
  if (!aligned16(v_pages) || !aligned16(out))
    return set_error(IAMAP_ERR_INVALID_ARG, "v_pages and out must be 16-byte aligned");
  int max_ctx = 0;
  for (int b = 0; b < batch; ++b) {
    const int c = ctx_lens_host[b];
    if (c < 0 || c > ctx_stride || (int64_t)c > (int64_t)max_pages * page_size)
      return set_error(IAMAP_ERR_INVALID_ARG, "ctx_lens[%d]=%d exceeds the row or page table", b, c);
    max_ctx = std::max(max_ctx, c);
  }
  DeviceContext* ctx = device_context();
  if (!ctx) return IAMAP_ERR_CUDA;
  PagedArgs a;
  paged_split(batch, max_ctx, page_size, ctx->num_sms, &a.chunks, &a.pages_per_chunk);
  const size_t need = sizeof(float) * (size_t)batch * a.chunks * H_r * d_v;
  if (!ws || ws_bytes < need)
    return set_error(IAMAP_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                     ws_bytes);
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
  a.H_kv = H_kv;
  a.H_s = H_s;
  a.H_r = H_r;
  a.d_v = d_v;
  a.out = out;
  a.partial = static_cast<float*>(ws);
  a.status = ctx->status;
  return mapped_av_paged_impl(a, static_cast<cudaStream_t>(stream));
}

extern "C" size_t iamap_head_match_workspace_bytes(int L_s, int H_small, int L_l, int H_large,
                                                   int n_used) {
  if (L_s < 1 || H_small < 1 || L_l < 1 || H_large < 1 || n_used < 1) return 0;
  return head_match_ws_bytes(L_s, H_small, L_l, H_large, n_used);
}

extern "C" int iamap_head_match(const void* q_small, const void* k_small, int L_s, int H_small,
                                int d_small, const void* q_large, const void* k_large, int L_l,
                                int H_large, int d_large, int n, int n_used, int32_t* argmax,
                                float* sim, void* ws, size_t ws_bytes, void* stream) {
  return iamap_head_match_metric(q_small, k_small, L_s, H_small, d_small, q_large, k_large, L_l,
                                 H_large, d_large, n, n_used, IAMAP_SIM_COSINE, argmax, sim, ws,
                                 ws_bytes, stream);
}

extern "C" int iamap_mapping_consistency(const int32_t* a, const int32_t* b, int n_heads,
                                         int32_t* agree, void* stream) {
  clear_error();
  if (!a || !b || !agree) return set_error(IAMAP_ERR_INVALID_ARG, "null pointer");
  if (n_heads < 1) return set_error(IAMAP_ERR_INVALID_ARG, "n_heads must be >= 1");
  if (!device_context()) return IAMAP_ERR_CUDA;
  return consistency_impl(a, b, n_heads, agree, static_cast<cudaStream_t>(stream));
}

extern "C" int iamap_head_match_metric(const void* q_small, const void* k_small, int L_s,
                                       int H_small, int d_small, const void* q_large,
                                       const void* k_large, int L_l, int H_large, int d_large,
                                       int n, int n_used, int metric, int32_t* argmax, float* sim,
                                       void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  if (metric != IAMAP_SIM_COSINE && metric != IAMAP_SIM_PEARSON && metric != IAMAP_SIM_EUCLIDEAN)
    return set_error(IAMAP_ERR_INVALID_ARG, "unknown similarity metric %d", metric);
  if (!q_small || !k_small || !q_large || !k_large || !argmax)
    return set_error(IAMAP_ERR_INVALID_ARG, "null pointer");
  if (L_s < 1 || H_small < 1 || L_l < 1 || H_large < 1 || n < 1 || n_used < 1 || n_used > n)
    return set_error(IAMAP_ERR_INVALID_ARG, "bad sizes (need 1 <= n_used <= n)");
  if ((d_small != 64 && d_small != 128) || (d_large != 64 && d_large != 128))
    return set_error(IAMAP_ERR_UNSUPPORTED, "head dims must be 64 or 128");
  if (!aligned16(q_small) || !aligned16(k_small) || !aligned16(q_large) || !aligned16(k_large))
    return set_error(IAMAP_ERR_INVALID_ARG, "q, k must be 16-byte aligned");
  const size_t need = head_match_ws_bytes(L_s, H_small, L_l, H_large, n_used);
  if (!ws || ws_bytes < need)
    return set_error(IAMAP_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                     ws_bytes);
  if (!aligned16(ws)) return set_error(IAMAP_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  DeviceContext* ctx = device_context();
  if (!ctx) return IAMAP_ERR_CUDA;
  HeadMatchArgs a;
  a.q_small = q_small;
  a.k_small = k_small;
  a.L_s = L_s;
  a.H_small = H_small;
  a.d_small = d_small;
  a.q_large = q_large;
  a.k_large = k_large;
  a.L_l = L_l;
  a.H_large = H_large;
  a.d_large = d_large;
  a.n = n;
  a.n_used = n_used;
  a.metric = metric;
  a.argmax = argmax;
  a.sim = sim;
  a.ws = ws;
  a.status = ctx->status;
  return head_match_impl(a, static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------------------------------------
// Prefix-hash block index
// ------------------------------------------------------------------------------------------------

namespace {

constexpr int64_t kMaxIndexCapacity = int64_t(1) << 40;
constexpr int kMaxKeyBlock = 4096;

int check_capacity(const void* table_keys, const void* table_vals, int64_t capacity) {
  if (!table_keys || !table_vals) return set_error(IAMAP_ERR_INVALID_ARG, "null table pointer");
  if (capacity < 1 || capacity > kMaxIndexCapacity || (capacity & (capacity - 1)) != 0)
    return set_error(IAMAP_ERR_INVALID_ARG, "capacity must be a power of two in [1, 2^40]");
  return IAMAP_OK;
}

}  // namespace

extern "C" int iamap_prefix_num_keys(const int32_t* cu_seqlens_host, int num_seqs, int B,
                                     int64_t* num_keys) {
  clear_error();
  if (!cu_seqlens_host || !num_keys) return set_error(IAMAP_ERR_INVALID_ARG, "null pointer");
  if (num_seqs < 1 || B < 1) return set_error(IAMAP_ERR_INVALID_ARG, "need num_seqs >= 1, B >= 1");
  if (cu_seqlens_host[0] < 0)
    return set_error(IAMAP_ERR_INVALID_ARG, "cu_seqlens_host[0] must be >= 0");
  int64_t t = 0;
  for (int s = 0; s < num_seqs; ++s) {
    const int64_t L = (int64_t)cu_seqlens_host[s + 1] - cu_seqlens_host[s];
    if (L < 0) return set_error(IAMAP_ERR_INVALID_ARG, "cu_seqlens_host decreases at %d", s);
    t += L / B;
  }
  *num_keys = t;
  return IAMAP_OK;
}

extern "C" int iamap_prefix_keys(const int32_t* tokens, int64_t n, const int32_t* cu_seqlens,
                                 int num_seqs, int B, uint64_t salt, uint64_t* keys,
                                 int64_t keys_capacity, int64_t* key_cu, void* stream) {
  clear_error();
  if (!cu_seqlens || !key_cu) return set_error(IAMAP_ERR_INVALID_ARG, "null pointer");
  if (n < 0 || num_seqs < 1 || keys_capacity < 0)
    return set_error(IAMAP_ERR_INVALID_ARG, "need n >= 0, num_seqs >= 1, keys_capacity >= 0");
  if (n > 0 && !tokens) return set_error(IAMAP_ERR_INVALID_ARG, "tokens is null");
  if (keys_capacity > 0 && !keys) return set_error(IAMAP_ERR_INVALID_ARG, "keys is null");
  if (B < 1 || B > kMaxKeyBlock)
    return set_error(IAMAP_ERR_INVALID_ARG, "B must be in [1, %d]", kMaxKeyBlock);
  return prefix_keys_launch(tokens, n, cu_seqlens, num_seqs, B, salt, keys, keys_capacity, key_cu,
                            static_cast<cudaStream_t>(stream));
}

extern "C" int iamap_prefix_index_clear(uint64_t* table_keys, int64_t* table_vals,
                                        int64_t capacity, void* stream) {
  clear_error();
  int rc = check_capacity(table_keys, table_vals, capacity);
  if (rc) return rc;
  if (!device_context()) return IAMAP_ERR_CUDA;
  return prefix_clear_launch(table_keys, table_vals, capacity, static_cast<cudaStream_t>(stream));
}

extern "C" int iamap_prefix_insert(const uint64_t* keys, const int64_t* values, int64_t count,
                                   uint64_t* table_keys, int64_t* table_vals, int64_t capacity,
                                   int64_t* stored, void* stream) {
  clear_error();
  int rc = check_capacity(table_keys, table_vals, capacity);
  if (rc) return rc;
  if (count < 0 || count > kMaxIndexCapacity)
    return set_error(IAMAP_ERR_INVALID_ARG, "count must be in [0, 2^40]");
  if (count > 0 && (!keys || !values || !stored))
    return set_error(IAMAP_ERR_INVALID_ARG, "null pointer");
  return prefix_insert_launch(keys, values, count, table_keys, table_vals, capacity, stored,
                              static_cast<cudaStream_t>(stream));
}

extern "C" int iamap_prefix_lookup(const uint64_t* keys, int64_t count, const int64_t* key_cu,
                                   int num_seqs, const uint64_t* table_keys,
                                   const int64_t* table_vals, int64_t capacity, int64_t* found,
                                   int32_t* hit_blocks, void* stream) {
  clear_error();
  int rc = check_capacity(table_keys, table_vals, capacity);
  if (rc) return rc;
  if (count < 0 || count > kMaxIndexCapacity)
    return set_error(IAMAP_ERR_INVALID_ARG, "count must be in [0, 2^40]");
  if (count > 0 && (!keys || !found)) return set_error(IAMAP_ERR_INVALID_ARG, "null pointer");
  if ((key_cu == nullptr) != (hit_blocks == nullptr))
    return set_error(IAMAP_ERR_INVALID_ARG, "key_cu and hit_blocks go together");
  if (key_cu && num_seqs < 1) return set_error(IAMAP_ERR_INVALID_ARG, "num_seqs must be >= 1");
  return prefix_lookup_launch(keys, count, key_cu, num_seqs, table_keys, table_vals, capacity,
                              found, hit_blocks, static_cast<cudaStream_t>(stream));
}
