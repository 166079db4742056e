// Internal launch interfaces between the C ABI layer (api.cu) and the kernel files.
#pragma once

#include "common.cuh"

namespace iamap {

struct CompressArgs {
  const void* q = nullptr;
  const void* k = nullptr;
  const int32_t* cu_seqlens = nullptr;
  int num_seqs = 0;
  int64_t n = 0;
  int H_s = 0, d = 0;
  float tau = 1.f;
  int bias_window = 0;
  float bias_value = 0.f;
  Plan plan;
  SeqTables tab;
  // stage 1 outputs
  float* lse = nullptr;
  float* mass = nullptr;
  uint64_t* headmask_dense = nullptr;
  int32_t* row_ptr = nullptr;
  int32_t* col_idx = nullptr;
  uint64_t* headmask = nullptr;
  int64_t* val_off = nullptr;
  int64_t* counts = nullptr;
  // stage 2 inputs / outputs
  const float* lse_in = nullptr;
  const int32_t* row_ptr_in = nullptr;
  const int32_t* col_idx_in = nullptr;
  const uint64_t* headmask_in = nullptr;
  const int64_t* val_off_in = nullptr;
  const int64_t* counts_in = nullptr;
  void* vals = nullptr;
  int64_t capacity = 0;
  unsigned int* status = nullptr;
  // head_match's use of the tensor-core kernels (compress_tc.cu): sequences at token offsets
  // tok0[s] of q/k tensors holding n_tok tokens (lse and rows are indexed by the packed
  // cu_seqlens), statistics without masses (mass == nullptr), and the dense head-major output
  // with per-head sums and squared norms.
  const int32_t* tok0 = nullptr;
  int64_t n_tok = 0;
  // Chunked prefill: k holds n_k key tokens packed by cu_seqlens (the keys [0, e) of every
  // sequence), q the n query rows of the chunks (SeqTables::qoff); 0 = q and k alike.
  int64_t n_k = 0;
  // Sender output (extract only): v_s bf16 [n_k, H_s, d_vs] packed like k; o_s fp32
  // [n, H_s, d_vs] packed like q. Null: no sender output.
  const void* v_s = nullptr;
  int d_vs = 0;
  float* o_s = nullptr;
  int dense = 0;
  int64_t dense_tiles = 0;
  float* norm2 = nullptr;
  float* sum1 = nullptr;
};

int compress_stats_impl(const CompressArgs& a, cudaStream_t stream);
int compress_extract_impl(const CompressArgs& a, cudaStream_t stream);
size_t compress_stats_smem(int d, int max_nb);
// Tensor-core forms (compress_tc.cu), used when supported: d of 64 or 128, at most 256 column
// blocks per sequence.
bool compress_tc_supported(int d, int max_nb);
int compress_stats_tc_launch(const CompressArgs& a, cudaStream_t stream);
int compress_extract_tc_launch(const CompressArgs& a, cudaStream_t stream);
size_t compress_extract_smem(int d, int max_nb);

struct MappedAvArgs {
  const int32_t* cu_seqlens = nullptr;
  int num_seqs = 0;
  int64_t n = 0;
  int H_s = 0;
  Plan plan;
  SeqTables tab;
  const int32_t* row_ptr = nullptr;
  const int32_t* col_idx = nullptr;
  const uint64_t* headmask = nullptr;
  const int64_t* val_off = nullptr;
  const void* vals = nullptr;
  int64_t capacity = 0;
  const float* W = nullptr;
  int H_r = 0;
  int H_kv = 0;   // value heads; 0 = H_r
  const void* v = nullptr;
  int d_v = 0;
  float* out = nullptr;
  unsigned int* status = nullptr;
  // Chunked prefill: v holds n_k tokens packed by cu_seqlens (the keys of every sequence), out
  // the n query rows of the chunks (SeqTables::qoff); 0 = v and out alike.
  int64_t n_k = 0;
  // Several mapped layers in one launch: sequence s uses the mixing matrix W + (s / seqs_per_w)
  // * H_r * H_s (0 = one W for every sequence).
  int seqs_per_w = 0;
};
int mapped_av_impl(const MappedAvArgs& a, cudaStream_t stream);
// Tensor-core, cluster-cooperative form (mapped_av_tc.cu); used when supported.
bool mapped_av_tc_supported(int H_s, int H_r, int d_v);
int mapped_av_tc_impl(const MappedAvArgs& a, cudaStream_t stream);

struct PagedArgs {
  const float* p_rows = nullptr;
  int ctx_stride = 0;
  const float* W = nullptr;
  const void* v_pages = nullptr;
  int64_t num_pages = 0;
  const int32_t* page_table = nullptr;
  int max_pages = 0;
  int page_size = 0;
  const int32_t* ctx_lens = nullptr;
  int max_ctx = 0;
  int batch = 0, H_s = 0, H_r = 0, d_v = 0;
  int H_kv = 0;   // value heads of the page pool; 0 = H_r
  float* out = nullptr;
  float* partial = nullptr;  // [batch][chunks][H_r][d_v]
  int chunks = 0;            // chunks per sequence
  int pages_per_chunk = 0;
  unsigned int* status = nullptr;
};
void paged_split(int batch, int max_ctx, int page_size, int num_sms, int* chunks,
                 int* pages_per_chunk);
int mapped_av_paged_impl(const PagedArgs& a, cudaStream_t stream);

struct HeadMatchArgs {
  const void* q_small = nullptr;
  const void* k_small = nullptr;
  int L_s = 0, H_small = 0, d_small = 0;
  const void* q_large = nullptr;
  const void* k_large = nullptr;
  int L_l = 0, H_large = 0, d_large = 0;
  int n = 0, n_used = 0;
  int metric = 0;   // IAMAP_SIM_*
  int32_t* argmax = nullptr;
  float* sim = nullptr;
  void* ws = nullptr;
  unsigned int* status = nullptr;
};
size_t head_match_ws_bytes(int L_s, int H_small, int L_l, int H_large, int n_used);
int head_match_impl(const HeadMatchArgs& a, cudaStream_t stream);
int consistency_impl(const int32_t* a, const int32_t* b, int n, int32_t* agree,
                     cudaStream_t stream);

// Prefix-hash block index (prefix_index.cu).
int prefix_keys_launch(const int32_t* tokens, int64_t n, const int32_t* cu, int num_seqs, int B,
                       uint64_t salt, uint64_t* keys, int64_t keys_capacity, int64_t* key_cu,
                       cudaStream_t stream);
int prefix_clear_launch(uint64_t* table_keys, int64_t* table_vals, int64_t capacity,
                        cudaStream_t stream);
int prefix_insert_launch(const uint64_t* keys, const int64_t* values, int64_t count,
                         uint64_t* table_keys, int64_t* table_vals, int64_t capacity,
                         int64_t* stored, cudaStream_t stream);
int prefix_lookup_launch(const uint64_t* keys, int64_t count, const int64_t* key_cu,
                         int num_seqs, const uint64_t* table_keys, const int64_t* table_vals,
                         int64_t capacity, int64_t* found, int32_t* hit_blocks,
                         cudaStream_t stream);

}  // namespace iamap
