/*
 * iamap.h -- C ABI of the cross-model attention-map reuse library (libiamap.so, sm_100a).
 *
 * The library computes, on one NVIDIA B200, the hot path of reusing one model's attention map in
 * another model's attention output:
 *
 *   compress     a sender model's causal softmax attention, per head, turned into a block-sparse
 *                (BSR) map: first block-level probability mass, then the extraction of the blocks
 *                kept by cumulative mass, with no dense n x n matrix ever formed.
 *                ("PKU MapFlow: cross-model attention map reuse" news page, storage-and-execution
 *                part, first component.)
 *   mapped_av    for every kept block, mix the sender heads by an H_r x H_s matrix W on chip,
 *                multiply by the receiver's V and accumulate the output, with no dense receiver
 *                map. (Same page, third component; the head mapping as a learned linear
 *                combination of sender heads is in its layer/head-mapping paragraph.)
 *   mapped_av_paged  the decode form: one query row per sequence, sender rows given, V in a paged
 *                cache. ("IAM: Efficient Inference through Attention Mapping between
 *                Different-scale LLMs" notes, Method section 4, decode bullet.) The sender rows
 *                themselves: iamap_sender_rows (the small model's softmax row, paged keys).
 *   head_match   IAM's calibration: cosine similarity of flattened causal attention maps of every
 *                large-model head with every small-model head, then the most similar small head
 *                per large head. (IAM notes, Method sections 1 and 4.) Variants: Pearson and
 *                Euclidean similarity (section 1), the agreement count of two mappings
 *                (section 3).
 *   *_gqa        mapped_av / mapped_av_paged with grouped receiver values: H_kv value heads,
 *                receiver head r reads value head r / (H_r / H_kv).
 *   *_layers     several mapped layer pairs per launch (layer-major stacked tensors).
 *   prefill_steps_host  end-to-end steps on host-resident inputs, the copies overlapping the
 *                kernels of neighbouring steps.
 *   compress_with_output, *_chunk  the sender's own attention output fused into compress, and
 *                the chunked-prefill form of compress and mapped_av (query rows of a chunk
 *                against all earlier keys). (MapFlow news page: the sender runs its own
 *                attention; the fused kernel works with chunked prefill.)
 *   prefix index the prefix-hash index of stored map blocks: chained FNV-1a-64 keys of every full
 *                block of a prompt, insert of (key, location) pairs into a device hash table,
 *                lookup of a prompt's blocks and of its longest cached prefix. (MapFlow news
 *                page, storage-and-execution part, second component.)
 *   iamap_selftest_wait_timeout  exercises the bounded-wait failure path on the GPU.
 *   iamap_selftest_exp2  evaluates the FMA-pipe exponential that the compress kernels can use
 *                beside the MUFU one, for accuracy tests.
 *
 * Conventions (all entry points):
 *   - Return 0 (IAMAP_OK) or a negative IAMAP_ERR_* code; iamap_last_error() gives a
 *     thread-local message for the last failure. No C++ exception crosses this boundary.
 *   - Tensor pointers are DEVICE pointers owned by the caller unless the name ends in _host.
 *     The library never frees or keeps them. bf16 tensors are passed as void* (IEEE bfloat16).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). Work is enqueued
 *     asynchronously on it; no entry point synchronises the stream except iamap_device_status.
 *   - The library keeps one lazily created context per device: a device status word that kernels
 *     set on a detected error (capacity exceeded, bounded wait expired, malformed index). Read and
 *     clear it with iamap_device_status.
 *   - Only block size B = 64 is implemented for the maps (IAMAP_ERR_UNSUPPORTED otherwise; the
 *     prefix index takes any B in 1..4096). Head dims d, d_v must be 64 or 128. Sender heads
 *     H_s <= 64 (one bit per head in the head masks).
 *
 * Layouts:
 *   q, k      bf16 [n, H_s, d]     token-major, packed sequences (cu_seqlens, int32 [S+1])
 *   v         bf16 [n, H_r, d_v]   ([n, H_kv, d_v] for the *_gqa entry points)
 *   W         fp32 [H_r, H_s]      row r mixes the sender heads for receiver head r
 *   lse       fp32 [H_s, n]        natural-log row log-sum-exp of the sender's scaled logits
 *   Causal blocks: sequence s has nb_s = ceil(L_s / B) row blocks; row block I has column blocks
 *   J = 0..I. Global row-block index rb = rb_start[s] + I; causal-block index
 *   cb = cb_start[s] + I*(I+1)/2 + J (both enumerations sequence-major, as iamap_plan reports).
 *   mass      fp32 [H_s, num_causal_blocks]  summed probability of each (head, causal block)
 *   headmask_dense u64 [num_causal_blocks]   bit h set = sender head h keeps that block
 *   BSR (union over heads, per row block, column blocks ascending):
 *     row_ptr  int32 [num_rowblocks + 1]
 *     col_idx  int32 [nnz_blocks]   column-block index J (local to the sequence)
 *     headmask u64   [nnz_blocks]   present sender heads
 *     val_off  int64 [nnz_blocks]   first tile of the block; a block with k present heads
 *                                   occupies tiles [val_off, val_off + k)
 *     vals     bf16  [tiles, B, B]  probabilities, interleaved by row within a block: row i of the
 *                                   head of rank t (t-th present head in increasing order) is at
 *                                   element (val_off*B + i*k + t) * B; causally masked entries and
 *                                   rows past the sequence end are 0
 *   out       fp32 [n, H_r, d_v]
 */
#ifndef IAMAP_H
#define IAMAP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define IAMAP_OK                0
#define IAMAP_ERR_INVALID_ARG  (-1)   /* null pointer, bad size or shape */
#define IAMAP_ERR_UNSUPPORTED  (-2)   /* valid but not implemented (B != 64, d not 64/128, ...) */
#define IAMAP_ERR_CAPACITY     (-3)   /* an output buffer is too small for the data */
#define IAMAP_ERR_CUDA         (-4)   /* a CUDA runtime call or launch failed */
#define IAMAP_ERR_TIMEOUT      (-5)   /* a bounded device-side wait expired */
#define IAMAP_ERR_WORKSPACE    (-6)   /* workspace pointer null or smaller than required */

/* Device status bits (iamap_device_status). */
#define IAMAP_DEV_CAPACITY   1
#define IAMAP_DEV_TIMEOUT    2
#define IAMAP_DEV_BAD_INDEX  4

/* Similarity of flattened attention maps for head matching (IAM notes, method section 1, which
 * compares cosine similarity, Minkowski distance and the Pearson correlation). */
#define IAMAP_SIM_COSINE     0   /* a.b / (|a| |b|) */
#define IAMAP_SIM_PEARSON    1   /* cosine of a - mean(a) and b - mean(b) over the n_used^2 entries */
#define IAMAP_SIM_EUCLIDEAN  2   /* -|a - b| (Minkowski distance with p = 2, negated: larger = closer) */

/* Library version, (major << 16) | minor. */
int iamap_version(void);

/* Thread-local message of the last failed call on this thread ("" if none). */
const char* iamap_last_error(void);

/*
 * Synchronise `stream`, then read and clear the device status word of the current device.
 * *status receives a bitwise OR of IAMAP_DEV_* (0 = no device-side error since the last read).
 * Returns IAMAP_ERR_CUDA if the synchronisation itself reports an error.
 */
int iamap_device_status(void* stream, int* status);

/*
 * Planning (host only, no device work). From the host copy of cu_seqlens, report the number of
 * row blocks, of causal blocks, and the largest row-block count of any sequence.
 * Errors: IAMAP_ERR_INVALID_ARG if cu_seqlens_host is null, num_seqs < 1, B < 1, or the offsets
 * decrease.
 */
int iamap_plan(const int32_t* cu_seqlens_host, int num_seqs, int B, int64_t* num_rowblocks,
               int64_t* num_causal_blocks, int32_t* max_blocks_per_seq);

/* Workspace bytes needed by iamap_compress_stats / _extract / iamap_compress / iamap_mapped_av
 * (scheduling tables). */
size_t iamap_compress_workspace_bytes(int num_seqs, int64_t num_rowblocks);

/*
 * Compress, stage 1 (block-level statistics and the kept sets).
 * For every sender head h and row block: the row-wise log-sum-exp of the scaled causal logits
 * s_ij = q_i.k_j / sqrt(d) (+ bias_value when 0 <= i - j < bias_window; window 0 = no bias),
 * the probability mass of every causal column block, and the kept set: the shortest prefix of
 * the column blocks sorted by decreasing mass (ties: lower J) whose cumulative mass reaches
 * tau * (valid rows of the block); tau >= 1 keeps every causal block. Then the union BSR index
 * (row_ptr, col_idx, headmask, val_off) and counts[0] = nnz_blocks, counts[1] = nnz_tiles.
 * col_idx / headmask / val_off must hold num_causal_blocks entries (the nnz is data-dependent).
 * Outputs lse, mass, headmask_dense, row_ptr, col_idx, headmask, val_off, counts are written in
 * full. The only input read on the host is cu_seqlens_host (the same values as cu_seqlens).
 */
int iamap_compress_stats(const void* q, const void* k, const int32_t* cu_seqlens,
                         const int32_t* cu_seqlens_host, int num_seqs, int64_t n, int H_s, int d,
                         int B, float tau, int bias_window, float bias_value,
                         float* lse, float* mass, uint64_t* headmask_dense, int32_t* row_ptr,
                         int32_t* col_idx, uint64_t* headmask, int64_t* val_off, int64_t* counts,
                         void* ws, size_t ws_bytes, void* stream);

/*
 * Compress, stage 2 (extraction of the kept blocks). Recomputes each kept (head, row block,
 * column block) tile of probabilities exp(s_ij - lse_i) from q, k and stage 1's lse, and writes
 * it as bf16 at its BSR position (row-interleaved within the block, see Layouts). A stored block
 * that does not fit below vals_capacity_tiles is not written and sets IAMAP_DEV_CAPACITY in the
 * device status. After the last tile the call also zero-fills up to 64 further tiles that fit in
 * the capacity (mapped_av may read that far).
 */
int iamap_compress_extract(const void* q, const void* k, const int32_t* cu_seqlens,
                           const int32_t* cu_seqlens_host, int num_seqs, int64_t n, int H_s, int d,
                           int B, int bias_window, float bias_value, const float* lse,
                           const int32_t* row_ptr, const int32_t* col_idx, const uint64_t* headmask,
                           const int64_t* val_off, const int64_t* counts, void* vals,
                           int64_t vals_capacity_tiles, void* ws, size_t ws_bytes, void* stream);

/*
 * Compress, both stages back to back on `stream`, with no host synchronisation (the tile count
 * stays on the device; a shortfall of vals_capacity_tiles is reported through the device status).
 */
int iamap_compress(const void* q, const void* k, const int32_t* cu_seqlens,
                   const int32_t* cu_seqlens_host, int num_seqs, int64_t n, int H_s, int d, int B,
                   float tau, int bias_window, float bias_value, float* lse, float* mass,
                   uint64_t* headmask_dense, int32_t* row_ptr, int32_t* col_idx, uint64_t* headmask,
                   int64_t* val_off, int64_t* counts, void* vals, int64_t vals_capacity_tiles,
                   void* ws, size_t ws_bytes, void* stream);

/*
 * Mapped attention output: for each row block and each stored column block J,
 *   P_r = sum_s W[r, s] * Pt_s   (absent heads contribute 0; no renormalisation),
 *   out_r[rows of the block] += P_r . V_r[rows of J],
 * for all receiver heads r < H_r; `out` is overwritten. vals_capacity_tiles bounds every tile
 * read (indices beyond it set IAMAP_DEV_BAD_INDEX).
 */
int iamap_mapped_av(const int32_t* cu_seqlens, const int32_t* cu_seqlens_host, int num_seqs,
                    int64_t n, int B, int H_s, const int32_t* row_ptr, const int32_t* col_idx,
                    const uint64_t* headmask, const int64_t* val_off, const void* vals,
                    int64_t vals_capacity_tiles, const float* W, int H_r, const void* v, int d_v,
                    float* out, void* ws, size_t ws_bytes, void* stream);

/*
 * mapped_av with grouped receiver values (grouped-query attention in the receiver): v is bf16
 * [n, H_kv, d_v] and receiver head r reads value head r / (H_r / H_kv). H_kv must divide H_r
 * (IAMAP_ERR_INVALID_ARG otherwise); H_kv = H_r is iamap_mapped_av.
 */
int iamap_mapped_av_gqa(const int32_t* cu_seqlens, const int32_t* cu_seqlens_host, int num_seqs,
                        int64_t n, int B, int H_s, const int32_t* row_ptr, const int32_t* col_idx,
                        const uint64_t* headmask, const int64_t* val_off, const void* vals,
                        int64_t vals_capacity_tiles, const float* W, int H_r, int H_kv,
                        const void* v, int d_v, float* out, void* ws, size_t ws_bytes,
                        void* stream);

/*
 * Compress with the sender's own attention output. As iamap_compress (stages 1 and 2), and in
 * the same pass over the keys the sender output O_s[i, h] = sum_{j <= i} p_h(i, j) V_s[j, h]
 * with the probabilities p of the map before any block is dropped (the bf16-rounded values the
 * stored tiles hold). The sender runs its own attention while its map is recorded for the
 * receiver ("PKU MapFlow" news page, the paragraphs on the attention map as the shared state).
 *   v_s   bf16 [n, H_s, d_vs]  the sender's values, d_vs 64 or 128, 16-byte aligned
 *   o_s   fp32 [n, H_s, d_vs]  written in full
 * Sequences may hold at most 256 blocks of 64 (IAMAP_ERR_UNSUPPORTED otherwise). The workspace
 * is iamap_compress_workspace_bytes(num_seqs, num_rowblocks). Other arguments and outputs as
 * iamap_compress.
 */
int iamap_compress_with_output(const void* q, const void* k, const int32_t* cu_seqlens,
                               const int32_t* cu_seqlens_host, int num_seqs, int64_t n, int H_s,
                               int d, int B, float tau, int bias_window, float bias_value,
                               const void* v_s, int d_vs, float* o_s, float* lse, float* mass,
                               uint64_t* headmask_dense, int32_t* row_ptr, int32_t* col_idx,
                               uint64_t* headmask, int64_t* val_off, int64_t* counts, void* vals,
                               int64_t vals_capacity_tiles, void* ws, size_t ws_bytes,
                               void* stream);

/*
 * Compress stage 2 with the sender's own attention output: as iamap_compress_extract (on the
 * outputs of iamap_compress_stats), and in the same pass the sender output o_s of
 * iamap_compress_with_output. Lets a caller read the tile count after stage 1 and allocate the
 * value buffer exactly. Sequences may hold at most 256 blocks of 64.
 */
int iamap_compress_extract_with_output(const void* q, const void* k, const int32_t* cu_seqlens,
                                       const int32_t* cu_seqlens_host, int num_seqs, int64_t n,
                                       int H_s, int d, int B, int bias_window, float bias_value,
                                       const void* v_s, int d_vs, float* o_s, const float* lse,
                                       const int32_t* row_ptr, const int32_t* col_idx,
                                       const uint64_t* headmask, const int64_t* val_off,
                                       const int64_t* counts, void* vals,
                                       int64_t vals_capacity_tiles, void* ws, size_t ws_bytes,
                                       void* stream);

/*
 * Several mapped layer pairs in one launch per stage ("PKU MapFlow" news page, the layer/head-
 * mapping paragraph: receiver layers paired with sender layers). num_layers = L pairs over the
 * same packed sequences (cu_seqlens, n tokens, S = num_seqs): the layers' tensors are stacked
 * layer-major,
 *   q, k  bf16 [L, n, H_s, d]       v  bf16 [L, n, H_kv, d_v]      W  fp32 [L, H_r, H_s]
 *   out   fp32 [L, n, H_r, d_v]
 * and the batch is read as L copies of the sequences: sequence (l, s) = stacked sequence
 * l * S + s at rows l * n + cu_seqlens[s]. Every other output is that of iamap_compress /
 * iamap_mapped_av on the stacked batch (lse [H_s, L * n], mass [H_s, L * num_causal_blocks],
 * the BSR index over L * num_rowblocks row blocks; iamap_layers_plan reports the stacked
 * counts). Layer l of mapped_av mixes with W[l]. Workspace: iamap_layers_workspace_bytes with
 * the stacked row-block count.
 */
int iamap_layers_plan(const int32_t* cu_seqlens_host, int num_seqs, int num_layers, int B,
                      int64_t* num_rowblocks, int64_t* num_causal_blocks,
                      int32_t* max_blocks_per_seq);
size_t iamap_layers_workspace_bytes(int num_seqs, int num_layers, int64_t num_rowblocks);
int iamap_compress_layers(const void* q, const void* k, const int32_t* cu_seqlens,
                          const int32_t* cu_seqlens_host, int num_seqs, int64_t n,
                          int num_layers, int H_s, int d, int B, float tau, int bias_window,
                          float bias_value, float* lse, float* mass, uint64_t* headmask_dense,
                          int32_t* row_ptr, int32_t* col_idx, uint64_t* headmask,
                          int64_t* val_off, int64_t* counts, void* vals,
                          int64_t vals_capacity_tiles, void* ws, size_t ws_bytes, void* stream);
int iamap_mapped_av_layers(const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                           int num_seqs, int64_t n, int num_layers, int B, int H_s,
                           const int32_t* row_ptr, const int32_t* col_idx,
                           const uint64_t* headmask, const int64_t* val_off, const void* vals,
                           int64_t vals_capacity_tiles, const float* W, int H_r, int H_kv,
                           const void* v, int d_v, float* out, void* ws, size_t ws_bytes,
                           void* stream);

/*
 * Chunked prefill ("PKU MapFlow" news page, the paragraph on the vLLM integration: the fused
 * kernel works with chunked prefill). Sequence s of a batch has keys [0, e_s), e_s =
 * cu_k[s+1] - cu_k[s], and a chunk of query rows [starts[s], e_s); starts[s] is a multiple of
 * B (0 = the whole sequence). The chunk attends to all keys [0, e_s) with absolute positions in
 * the causal mask and the local bias, so its results equal the whole-sequence results of those
 * rows. Its row blocks are the sequence's own row blocks I = starts[s]/B .. ceil(e_s/B) - 1.
 *   q        bf16 [n_q, H_s, d]    the chunks' query rows, packed by cu_q (int32 [S+1],
 *                                  cu_q[s+1] - cu_q[s] = e_s - starts[s])
 *   k        bf16 [n_k, H_s, d]    the keys [0, e_s) of every sequence, packed by cu_k
 *   starts   int32 [S]             chunk starts (device); *_host: the same values on the host
 * Chunk layouts: the listed row blocks are the chunks' row blocks, sequence-major, and the causal
 * blocks (I, J <= I) of those row blocks; iamap_chunk_plan reports their numbers. lse is
 * [H_s, n_q] (packed query rows), mass [H_s, num_causal_blocks], the BSR index has
 * num_rowblocks + 1 row pointers; col_idx stays the sequence-local column block J.
 */
int iamap_chunk_plan(const int32_t* cu_q_host, const int32_t* cu_k_host,
                     const int32_t* starts_host, int num_seqs, int B, int64_t* num_rowblocks,
                     int64_t* num_causal_blocks, int32_t* max_blocks_per_seq);

/*
 * Compress of a batch of chunks (stages 1 and 2 in one call, as iamap_compress), optionally with
 * the sender output of the chunk rows: v_s bf16 [n_k, H_s, d_vs] packed like k, o_s fp32
 * [n_q, H_s, d_vs] (both NULL: no sender output). Sequences may hold at most 256 blocks of 64.
 * Workspace: iamap_compress_workspace_bytes(num_seqs, num_rowblocks of the chunk plan).
 * Errors as iamap_compress; IAMAP_ERR_INVALID_ARG if a start is not a multiple of B or a chunk
 * does not end at its key length.
 */
int iamap_compress_chunk(const void* q, const void* k, const int32_t* cu_q, const int32_t* cu_k,
                         const int32_t* starts, const int32_t* cu_q_host,
                         const int32_t* cu_k_host, const int32_t* starts_host, int num_seqs,
                         int64_t n_q, int64_t n_k, int H_s, int d, int B, float tau,
                         int bias_window, float bias_value, const void* v_s, int d_vs,
                         float* o_s, float* lse, float* mass, uint64_t* headmask_dense,
                         int32_t* row_ptr, int32_t* col_idx, uint64_t* headmask,
                         int64_t* val_off, int64_t* counts, void* vals,
                         int64_t vals_capacity_tiles, void* ws, size_t ws_bytes, void* stream);

/*
 * mapped_av of a batch of chunks: out fp32 [n_q, H_r, d_v] (the chunk rows, packed by cu_q) from
 * the chunk BSR map of iamap_compress_chunk and the receiver's values v bf16 [n_k, H_kv, d_v]
 * packed like the keys (grouped values as iamap_mapped_av_gqa; H_kv = H_r for one value head per
 * receiver head).
 */
int iamap_mapped_av_chunk(const int32_t* cu_q, const int32_t* cu_k, const int32_t* starts,
                          const int32_t* cu_q_host, const int32_t* cu_k_host,
                          const int32_t* starts_host, int num_seqs, int64_t n_q, int64_t n_k,
                          int B, int H_s, const int32_t* row_ptr, const int32_t* col_idx,
                          const uint64_t* headmask, const int64_t* val_off, const void* vals,
                          int64_t vals_capacity_tiles, const float* W, int H_r, int H_kv,
                          const void* v, int d_v, float* out, void* ws, size_t ws_bytes,
                          void* stream);

/*
 * End-to-end prefill steps from host memory. For each step i < steps: upload q_host[i],
 * k_host[i] (bf16 [n, H_s, d]), v_host[i] (bf16 [n, H_kv, d_v]) and W_host[i] (fp32 [H_r, H_s]),
 * run iamap_compress and iamap_mapped_av_gqa on them, and read the output back into out_host[i]
 * (fp32 [n, H_r, d_v]). The host buffers should be pinned (page-locked): pageable memory works
 * but its copies do not overlap the kernels.
 *   io    device buffer of iamap_prefill_io_bytes bytes, 256-byte aligned: two sets of device
 *         inputs and outputs, so that the upload of step i + 1 and the read-back of step i - 1
 *         overlap the kernels of step i. The copies run on an upload and a download stream that
 *         the library creates once per device; events order them against `stream`, on which the
 *         kernels run. One cudaMemcpyAsync per copy.
 *   lse .. vals_capacity_tiles, ws   the compress buffers and workspace, as for iamap_compress
 *         (reused by every step).
 * Enqueues everything and returns; `stream` then waits for the last read-back, so an event
 * recorded or a synchronisation made on `stream` after the call covers every step. Errors as
 * iamap_compress / iamap_mapped_av_gqa, and IAMAP_ERR_WORKSPACE if io is too small.
 */
size_t iamap_prefill_io_bytes(int64_t n, int H_s, int d, int H_r, int H_kv, int d_v);
int iamap_prefill_steps_host(int steps, const void* const* q_host, const void* const* k_host,
                             const void* const* v_host, const float* const* W_host,
                             float* const* out_host, const int32_t* cu_seqlens,
                             const int32_t* cu_seqlens_host, int num_seqs, int64_t n, int H_s,
                             int d, int H_r, int H_kv, int d_v, int B, float tau, int bias_window,
                             float bias_value, float* lse, float* mass, uint64_t* headmask_dense,
                             int32_t* row_ptr, int32_t* col_idx, uint64_t* headmask,
                             int64_t* val_off, int64_t* counts, void* vals,
                             int64_t vals_capacity_tiles, void* io, size_t io_bytes, void* ws,
                             size_t ws_bytes, void* stream);

/*
 * The small model's attention row of a decode step, the row a mapped layer reuses (IAM notes,
 * Method section 4, decode bullet): p[b, h, j] = softmax over j < ctx_lens[b] of
 * q[b, h] . k[b, j, h] / sqrt(d), keys in a paged cache.
 *   q        bf16 [batch, H_s, d]                   (d a multiple of 8, at most 128)
 *   k_pages  bf16 [num_pages, page_size, H_s, d]    16-byte aligned; key j of sequence b is
 *            row j % page_size of page page_table[b, j / page_size]
 *   p_rows   fp32 [batch, H_s, ctx_stride]          written in full (zeros at j >= ctx_lens[b])
 *   ws       iamap_sender_rows_workspace_bytes bytes (per-chunk partial sums)
 * A page index outside [0, num_pages) makes that key's probability 0 and sets
 * IAMAP_DEV_BAD_INDEX. The result feeds iamap_mapped_av_paged as its p_rows.
 */
size_t iamap_sender_rows_workspace_bytes(int batch, int H_s, int ctx_stride);
int iamap_sender_rows(const void* q, const void* k_pages, int64_t num_pages,
                      const int32_t* page_table, int max_pages, int page_size,
                      const int32_t* ctx_lens, const int32_t* ctx_lens_host, int batch, int H_s,
                      int d, float* p_rows, int ctx_stride, void* ws, size_t ws_bytes,
                      void* stream);

/*
 * Decode step on a mapped layer: one query row per sequence b.
 *   out[b, r, :] = sum_{j < ctx_lens[b]} (sum_s W[r, s] * p_rows[b, s, j]) * V[b, j, r, :]
 * p_rows  fp32 [batch, H_s, ctx_stride]  the sender's attention rows
 * v_pages bf16 [num_pages, page_size, H_r, d_v]; token j of sequence b lives in page
 *         page_table[b * max_pages + j / page_size], slot j % page_size.
 * out     fp32 [batch, H_r, d_v]. ws: iamap_mapped_av_paged_workspace_bytes bytes (split partial
 * sums). Page indices outside [0, num_pages) set IAMAP_DEV_BAD_INDEX and are skipped.
 */
size_t iamap_mapped_av_paged_workspace_bytes(int batch, int H_r, int d_v, int max_ctx,
                                             int page_size);
int iamap_mapped_av_paged(const float* p_rows, int ctx_stride, const float* W,
                          const void* v_pages, int64_t num_pages, const int32_t* page_table,
                          int max_pages, int page_size, const int32_t* ctx_lens,
                          const int32_t* ctx_lens_host, int batch, int H_s, int H_r, int d_v,
                          float* out, void* ws, size_t ws_bytes, void* stream);

/*
 * Decode step with grouped receiver values: v_pages bf16 [num_pages, page_size, H_kv, d_v];
 * receiver head r reads value head r / (H_r / H_kv). H_kv must divide H_r. The workspace is
 * that of iamap_mapped_av_paged for the same H_r.
 */
int iamap_mapped_av_paged_gqa(const float* p_rows, int ctx_stride, const float* W,
                              const void* v_pages, int64_t num_pages, const int32_t* page_table,
                              int max_pages, int page_size, const int32_t* ctx_lens,
                              const int32_t* ctx_lens_host, int batch, int H_s, int H_r, int H_kv,
                              int d_v, float* out, void* ws, size_t ws_bytes, void* stream);

/*
 * The paged decode step of iamap_mapped_av_paged for callers that cannot allocate device memory
 * when they call: for example a serving engine that reserved nearly all GPU memory for its KV
 * cache at start-up, or one that forbids cudaMalloc on its decode loop because cudaMalloc
 * synchronises the device. The pages have no counterpart of this entry point; it exists only
 * for such callers. Same arguments and result as iamap_mapped_av_paged, minus the workspace:
 * the split partial sums live in a fixed 16 MiB device array inside the library. The call itself
 * allocates nothing (no cudaMalloc, no cudaFree, no status word), with one exception:
 *   - Under CUDA's lazy module loading (the default) the array, and the decode kernels, are
 *     loaded onto a device by the FIRST call on that device, which therefore takes 16 MiB of
 *     device memory (plus the kernels' code) and may synchronise. Make that first call at
 *     start-up, before reserving the rest of the GPU's memory and before any stream capture;
 *     the device then holds the array until the process exits.
 *   - The array's device address is looked up (cudaGetSymbolAddress) per device and current
 *     context, so a call from another context, or after cudaDeviceReset, looks it up again.
 *   - A call whose partial sums (batch x chunks x H_r x d_v floats) exceed 16 MiB returns
 *     IAMAP_ERR_CAPACITY and launches nothing.
 *   - All calls on a device share the array (it keeps the last call's contents; every value read
 *     is first written by the same call). Calls that overlap on the GPU race on it: order them
 *     on one stream.
 *   - Out-of-range page indices are skipped and not reported (there is no status word).
 */
int iamap_mapped_av_paged_noalloc(const float* p_rows, int ctx_stride, const float* W,
                                  const void* v_pages, int64_t num_pages,
                                  const int32_t* page_table, int max_pages, int page_size,
                                  const int32_t* ctx_lens, const int32_t* ctx_lens_host, int batch,
                                  int H_s, int H_r, int d_v, float* out, void* stream);

/*
 * Failure-detection self-test: one CTA waits, with the kernels' bounded mbarrier wait but a limit
 * of limit_us microseconds (1 .. 1e6), on a barrier that nothing arrives on. The wait gives up:
 * IAMAP_DEV_TIMEOUT is raised in the device status and *gave_up (device int) becomes 1. The
 * context stays usable. Asynchronous on stream.
 */
int iamap_selftest_wait_timeout(int limit_us, int* gave_up, void* stream);

/*
 * Exponential self-test: y_fma[k] = 2^x[k] by the FMA-pipe method of the compress kernels (exact
 * base-2 argument reduction 2^x = 2^n 2^f, n = rint(x), then a degree-5 minimax polynomial for
 * 2^f on [-1/2, 1/2]; inputs below -126 give 2^-126) and y_mufu[k] = 2^x[k] by ex2.approx.ftz on
 * the MUFU unit, for n elements (device fp32 arrays, n >= 0; elements are evaluated in pairs as
 * in the kernels). Meant for x <= 0, the range the softmax passes use. Asynchronous on stream.
 */
int iamap_selftest_exp2(const float* x, float* y_fma, float* y_mufu, int64_t n, void* stream);

/*
 * Head matching (calibration). q_small / k_small bf16 [L_s, n, H_small, d_small];
 * q_large / k_large bf16 [L_l, n, H_large, d_large]. Each head's map is the causal softmax of
 * q k^T / sqrt(d) over the first n_used tokens (n_used <= n; the prompt truncation tau_t).
 * sim (optional, may be NULL) fp32 [L_l * H_large, L_s * H_small]: cosine of the flattened maps.
 * argmax int32 [L_l * H_large]: the small head (layer * H_small + head) of highest cosine,
 * lowest index on ties. ws: iamap_head_match_workspace_bytes bytes (the bf16 maps, norms and
 * the similarity accumulator).
 */
size_t iamap_head_match_workspace_bytes(int L_s, int H_small, int L_l, int H_large, int n_used);
int iamap_head_match(const void* q_small, const void* k_small, int L_s, int H_small, int d_small,
                     const void* q_large, const void* k_large, int L_l, int H_large, int d_large,
                     int n, int n_used, int32_t* argmax, float* sim, void* ws, size_t ws_bytes,
                     void* stream);

/*
 * Head matching with another similarity: as iamap_head_match, with metric one of IAMAP_SIM_*.
 * sim then holds that metric (for IAMAP_SIM_EUCLIDEAN the negated distance) and argmax its
 * largest value per large head. The workspace is the same. An unknown metric returns
 * IAMAP_ERR_INVALID_ARG.
 */
int iamap_head_match_metric(const void* q_small, const void* k_small, int L_s, int H_small,
                            int d_small, const void* q_large, const void* k_large, int L_l,
                            int H_large, int d_large, int n, int n_used, int metric,
                            int32_t* argmax, float* sim, void* ws, size_t ws_bytes, void* stream);

/*
 * Mapping consistency (IAM notes, method section 3: the mapping found at prefill holds during
 * decode). a, b: int32 device arrays of n_heads small-head indices, e.g. the argmax of
 * iamap_head_match on the prompt and on a longer prefix. *agree (device int32) receives the
 * number of positions where they are equal; the consistency rate is agree / n_heads.
 * Asynchronous on stream.
 */
int iamap_mapping_consistency(const int32_t* a, const int32_t* b, int n_heads, int32_t* agree,
                              void* stream);

/*
 * Structure check of a block-sparse map on the host (e.g. one read back from storage or from
 * another process before mapped_av uses it). All pointers are HOST pointers; nothing is written
 * except *bad_block. The map is valid when, for every row block I of every sequence:
 * row_ptr starts at 0 and does not decrease; the column blocks of a row block ascend strictly
 * and lie in 0..I; each head mask is non-zero with bits only below H_s; and each block's tiles
 * [val_off, val_off + popcount(mask)) lie in [0, vals_capacity_tiles).
 * Returns IAMAP_OK, IAMAP_ERR_INVALID_ARG (bad structure or arguments) or IAMAP_ERR_CAPACITY
 * (tiles outside the buffer); *bad_block (if non-null) receives the first offending block, or
 * -1. iamap_last_error names the violation.
 */
int iamap_bsr_check_host(const int32_t* cu_seqlens_host, int num_seqs, int B, int H_s,
                         const int32_t* row_ptr, const int32_t* col_idx, const uint64_t* headmask,
                         const int64_t* val_off, int64_t vals_capacity_tiles,
                         int64_t* bad_block);

/* ---------------------------------------------------------------------------------------------
 * Prefix-hash block index ("PKU MapFlow: cross-model attention map reuse" news page, storage-
 * and-execution part, second component: stored map blocks are located through a prefix hash
 * index whose keys carry the preceding context; one sender state can serve several receivers).
 *
 * Block b of a packed sequence is tokens [b*B, (b+1)*B) (full blocks only; with B = 64 these are
 * the map's row blocks). Its digest is FNV-1a-64 (offset basis 0xcbf29ce484222325, prime
 * 0x100000001b3) of its token ids as 4-byte little-endian integers; its prefix key is the
 * FNV-1a-64 state after absorbing, from `salt`, the 8-byte little-endian digests of blocks 0..b.
 * The key therefore changes with any token before the block's end. Pick one salt per sender
 * layer (or model) so that entries of different layers never share a key.
 *
 * The index is an open-addressing table owned by the caller: table_keys (uint64) and table_vals
 * (int64 locations, e.g. the first tile of the row block's stored blocks), `capacity` entries,
 * capacity a power of two in [1, 2^40]. The all-ones key marks an empty slot and is never stored.
 * A key lives within min(capacity, 1024) slots of its home slot (linear probing); keep the load
 * factor below about 0.7. Entries are never removed (clear the table to start over). Inserts and
 * lookups on one table must be ordered (same stream, or events): they are not atomic with
 * respect to each other.
 * ------------------------------------------------------------------------------------------- */

/*
 * Number of prefix keys (full blocks) of packed sequences, from host cu_seqlens.
 * Errors: IAMAP_ERR_INVALID_ARG for a null pointer, num_seqs < 1, B < 1 or decreasing offsets.
 */
int iamap_prefix_num_keys(const int32_t* cu_seqlens_host, int num_seqs, int B,
                          int64_t* num_keys);

/*
 * Prefix keys of every full block of the packed sequences.
 *   tokens      int32 [n] device, token ids packed by cu_seqlens
 *   cu_seqlens  int32 [num_seqs + 1] device
 *   B           tokens per block, 1 .. 4096
 *   keys        uint64 [keys_capacity] device: sequence s's keys at key_cu[s] .. key_cu[s+1]-1
 *   key_cu      int64 [num_seqs + 1] device: offsets of each sequence's keys
 * Device-side: offsets outside [0, n] set IAMAP_DEV_BAD_INDEX (the sequence gets no keys); keys
 * past keys_capacity are not written and set IAMAP_DEV_CAPACITY. Asynchronous on stream.
 */
int iamap_prefix_keys(const int32_t* tokens, int64_t n, const int32_t* cu_seqlens, int num_seqs,
                      int B, uint64_t salt, uint64_t* keys, int64_t keys_capacity,
                      int64_t* key_cu, void* stream);

/* Empties the table: every key all ones, every location -1. Asynchronous on stream. */
int iamap_prefix_index_clear(uint64_t* table_keys, int64_t* table_vals, int64_t capacity,
                             void* stream);

/*
 * Inserts count (key, location) pairs, keeping the present location of a key that is already
 * in the table (the first writer wins; among equal keys of one call, one of them). stored
 * (int64 [count] device) receives, per pair, the location now associated with its key, or -1 for
 * the reserved empty key and for a pair that found no slot (then IAMAP_DEV_CAPACITY is set).
 * keys and values are device arrays of count entries. Asynchronous on stream.
 */
int iamap_prefix_insert(const uint64_t* keys, const int64_t* values, int64_t count,
                        uint64_t* table_keys, int64_t* table_vals, int64_t capacity,
                        int64_t* stored, void* stream);

/*
 * Looks up count keys: found (int64 [count] device) receives each key's location or -1. With
 * key_cu (int64 [num_seqs + 1] device, as written by iamap_prefix_keys) and hit_blocks (int32
 * [num_seqs] device) both non-null, hit_blocks[s] receives the number of leading blocks of
 * sequence s that were found: its longest cached prefix in blocks. Then only the keys inside
 * the sequences' ranges are looked up (all of them when key_cu comes from iamap_prefix_keys).
 * key_cu offsets outside [0, count] set IAMAP_DEV_BAD_INDEX (that sequence reports 0 and its
 * found entries are not written). Asynchronous on stream.
 */
int iamap_prefix_lookup(const uint64_t* keys, int64_t count, const int64_t* key_cu, int num_seqs,
                        const uint64_t* table_keys, const int64_t* table_vals, int64_t capacity,
                        int64_t* found, int32_t* hit_blocks, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* IAMAP_H */
