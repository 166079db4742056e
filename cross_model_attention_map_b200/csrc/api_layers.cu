// extern "C" entry points that run several mapped layers in one launch per stage.
//
// A layer mapping pairs several receiver layers with sender layers ("PKU MapFlow" news page, the
// layer/head-mapping paragraph); each pair runs compress on its sender layer and mapped_av with
// its own W and receiver values. Here num_layers such pairs over the same packed sequences run
// together: the layers' tensors are stacked layer-major ([L, n, ...] = [L * n, ...]) and the
// batch is the L copies of the sequences, sequence (l, s) at packed rows l * n + cu_seqlens[s].
// Every kernel then sees one packed batch of L * S sequences (one table build, one grid per
// stage); only mapped_av needs to know the layer of a sequence, for its W.
#include <vector>

#include "internal.h"

using namespace iamap;

namespace {

size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }

__global__ void layers_cu_kernel(const int32_t* __restrict__ cu, int S, int L, int n,
                                 int32_t* __restrict__ cu_l) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= L * S; i += gridDim.x * blockDim.x) {
    const int l = i / S, s = i - l * S;
    cu_l[i] = l < L ? l * n + cu[s] : L * n;
  }
}

// Host copy of the stacked batch's offsets, and its plan.
int layers_plan(const int32_t* cu_host, int num_seqs, int num_layers, int64_t n, int B,
                std::vector<int32_t>* cu_l, Plan* plan) {
  if (!cu_host) return set_error(IAMAP_ERR_INVALID_ARG, "cu_seqlens_host is null");
  if (num_seqs < 1 || num_layers < 1)
    return set_error(IAMAP_ERR_INVALID_ARG, "num_seqs and num_layers must be >= 1");
  if (n < 0 || (int64_t)cu_host[num_seqs] != n)
    return set_error(IAMAP_ERR_INVALID_ARG, "cu_seqlens[num_seqs] does not equal n");
  if ((int64_t)num_layers * n >= (int64_t)INT32_MAX)
    return set_error(IAMAP_ERR_UNSUPPORTED, "num_layers * n beyond 2^31 rows");
  cu_l->assign((size_t)num_layers * num_seqs + 1, 0);
  for (int l = 0; l < num_layers; ++l)
    for (int s = 0; s < num_seqs; ++s)
      (*cu_l)[(size_t)l * num_seqs + s] = (int32_t)(l * n + cu_host[s]);
  (*cu_l)[(size_t)num_layers * num_seqs] = (int32_t)(num_layers * n);
  return make_plan(cu_l->data(), num_layers * num_seqs, B, num_layers * n, plan);
}

// The stacked offsets on the device, at the start of the workspace; the scheduling tables after.
int layers_setup(const int32_t* cu, int num_seqs, int num_layers, int64_t n, int B,
                 const std::vector<int32_t>& cu_l, const Plan& plan, void* ws, size_t ws_bytes,
                 cudaStream_t st, int32_t** cu_dev, SeqTables* tab, bool build_tables) {
  if (!cu) return set_error(IAMAP_ERR_INVALID_ARG, "cu_seqlens is null");
  const int S = num_layers * num_seqs;
  const size_t head = a256(sizeof(int32_t) * (cu_l.size()));
  const size_t need = head + seq_tables_bytes(S, plan.num_rowblocks);
  if (!ws || ws_bytes < need)
    return set_error(IAMAP_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                     ws_bytes);
  *cu_dev = static_cast<int32_t*>(ws);
  layers_cu_kernel<<<(S + 256) / 256, 256, 0, st>>>(cu, num_seqs, num_layers, (int)n, *cu_dev);
  IAMAP_LAUNCH_CHECK("layers_cu_kernel");
  *tab = carve_seq_tables(static_cast<char*>(ws) + head, S, plan.num_rowblocks);
  if (build_tables && plan.num_rowblocks > 0)
    return launch_build_tables(*cu_dev, S, B, plan.max_nb, *tab, st);
  return IAMAP_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int iamap_layers_plan(const int32_t* cu_seqlens_host, int num_seqs, int num_layers,
                                 int B, int64_t* num_rowblocks, int64_t* num_causal_blocks,
                                 int32_t* max_blocks_per_seq) {
  clear_error();
  if (!cu_seqlens_host || num_seqs < 1)
    return set_error(IAMAP_ERR_INVALID_ARG, "null host array or num_seqs < 1");
  std::vector<int32_t> cu_l;
  Plan p;
  int rc = layers_plan(cu_seqlens_host, num_seqs, num_layers, cu_seqlens_host[num_seqs], B,
                       &cu_l, &p);
  if (rc) return rc;
  if (num_rowblocks) *num_rowblocks = p.num_rowblocks;
  if (num_causal_blocks) *num_causal_blocks = p.num_causal_blocks;
  if (max_blocks_per_seq) *max_blocks_per_seq = p.max_nb;
  return IAMAP_OK;
}

extern "C" size_t iamap_layers_workspace_bytes(int num_seqs, int num_layers,
                                               int64_t num_rowblocks) {
  if (num_seqs < 1 || num_layers < 1 || num_rowblocks < 0) return 0;
  const int S = num_layers * num_seqs;
  return a256(sizeof(int32_t) * (size_t)(S + 1)) + seq_tables_bytes(S, num_rowblocks);
}

extern "C" int iamap_compress_layers(
    const void* q, const void* k, const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
    int num_seqs, int64_t n, int num_layers, int H_s, int d, int B, float tau, int bias_window,
    float bias_value, float* lse, float* mass, uint64_t* headmask_dense, int32_t* row_ptr,
    int32_t* col_idx, uint64_t* headmask, int64_t* val_off, int64_t* counts, void* vals,
    int64_t vals_capacity_tiles, void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  std::vector<int32_t> cu_l;
  Plan plan;
  int rc = layers_plan(cu_seqlens_host, num_seqs, num_layers, n, B, &cu_l, &plan);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!device_context()) return IAMAP_ERR_CUDA;
  int32_t* cu_dev = nullptr;
  SeqTables tab;
  rc = layers_setup(cu_seqlens, num_seqs, num_layers, n, B, cu_l, plan, ws, ws_bytes, st,
                    &cu_dev, &tab, false);
  if (rc) return rc;
  const size_t head = a256(sizeof(int32_t) * cu_l.size());
  // the stacked batch is an ordinary packed batch: the single-layer entry point does the rest
  return iamap_compress(q, k, cu_dev, cu_l.data(), num_layers * num_seqs, num_layers * n, H_s,
                        d, B, tau, bias_window, bias_value, lse, mass, headmask_dense, row_ptr,
                        col_idx, headmask, val_off, counts, vals, vals_capacity_tiles,
                        static_cast<char*>(ws) + head, ws_bytes - head, stream);
}

extern "C" int iamap_mapped_av_layers(
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_host, int num_seqs, int64_t n,
    int num_layers, int B, int H_s, const int32_t* row_ptr, const int32_t* col_idx,
    const uint64_t* headmask, const int64_t* val_off, const void* vals,
    int64_t vals_capacity_tiles, const float* W, int H_r, int H_kv, const void* v, int d_v,
    float* out, void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  if (B != 64) return set_error(IAMAP_ERR_UNSUPPORTED, "only block size B = 64 is implemented");
  if (H_s < 1 || H_s > 64) return set_error(IAMAP_ERR_UNSUPPORTED, "H_s must be in [1, 64]");
  if (d_v != 64 && d_v != 128) return set_error(IAMAP_ERR_UNSUPPORTED, "d_v must be 64 or 128");
  if (H_r < 1) return set_error(IAMAP_ERR_INVALID_ARG, "H_r must be >= 1");
  if (H_kv < 1 || H_r % H_kv != 0)
    return set_error(IAMAP_ERR_INVALID_ARG, "H_kv=%d must divide H_r=%d", H_kv, H_r);
  if (!row_ptr || !col_idx || !headmask || !val_off || !W || !v || !out ||
      (!vals && vals_capacity_tiles > 0))
    return set_error(IAMAP_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(v) || (vals && !aligned16(vals)) || !aligned16(out))
    return set_error(IAMAP_ERR_INVALID_ARG, "v, vals, out must be 16-byte aligned");
  std::vector<int32_t> cu_l;
  Plan plan;
  int rc = layers_plan(cu_seqlens_host, num_seqs, num_layers, n, B, &cu_l, &plan);
  if (rc) return rc;
  DeviceContext* ctx = device_context();
  if (!ctx) return IAMAP_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MappedAvArgs a;
  int32_t* cu_dev = nullptr;
  rc = layers_setup(cu_seqlens, num_seqs, num_layers, n, B, cu_l, plan, ws, ws_bytes, st,
                    &cu_dev, &a.tab, true);
  if (rc) return rc;
  a.plan = plan;
  a.cu_seqlens = cu_dev;
  a.num_seqs = num_layers * num_seqs;
  a.n = num_layers * n;
  a.H_s = H_s;
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  a.headmask = headmask;
  a.val_off = val_off;
  a.vals = vals;
  a.capacity = vals_capacity_tiles;
  a.W = W;
  a.seqs_per_w = num_seqs;
  a.H_r = H_r;
  a.H_kv = H_kv;
  a.v = v;
  a.d_v = d_v;
  a.out = out;
  a.status = ctx->status;
  return mapped_av_impl(a, st);
}
