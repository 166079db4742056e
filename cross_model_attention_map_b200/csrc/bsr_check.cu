// Host-side structure check of a block-sparse map (BSR, union over sender heads), for maps that
// come from storage or another process (a prefix cache) before mapped_av reads them. Only reads
// host copies; no device work.
#include <cstdint>
#include <vector>

#include "common.cuh"

using namespace iamap;

extern "C" int iamap_bsr_check_host(const int32_t* cu_seqlens_host, int num_seqs, int B, int H_s,
                                    const int32_t* row_ptr, const int32_t* col_idx,
                                    const uint64_t* headmask, const int64_t* val_off,
                                    int64_t vals_capacity_tiles, int64_t* bad_block) {
  clear_error();
  if (bad_block) *bad_block = -1;
  Plan plan;
  int rc = make_plan(cu_seqlens_host, num_seqs, B, -1, &plan);
  if (rc) return rc;
  if (H_s < 1 || H_s > 64) return set_error(IAMAP_ERR_INVALID_ARG, "H_s must be in [1, 64]");
  if (!row_ptr) return set_error(IAMAP_ERR_INVALID_ARG, "row_ptr is null");
  if (vals_capacity_tiles < 0) return set_error(IAMAP_ERR_INVALID_ARG, "negative capacity");
  if (row_ptr[0] != 0)
    return set_error(IAMAP_ERR_INVALID_ARG, "row_ptr[0] = %d, not 0", row_ptr[0]);
  const uint64_t head_bits = H_s == 64 ? ~0ull : ((1ull << H_s) - 1ull);
  int64_t rb = 0;
  for (int s = 0; s < num_seqs; ++s) {
    const int64_t L = (int64_t)cu_seqlens_host[s + 1] - cu_seqlens_host[s];
    const int64_t nb = (L + B - 1) / B;
    for (int64_t I = 0; I < nb; ++I, ++rb) {
      const int64_t lo = row_ptr[rb], hi = row_ptr[rb + 1];
      if (hi < lo)
        return set_error(IAMAP_ERR_INVALID_ARG, "row_ptr decreases at row block %lld",
                         (long long)rb);
      if (hi > lo && (!col_idx || !headmask || !val_off))
        return set_error(IAMAP_ERR_INVALID_ARG, "null col_idx, headmask or val_off");
      for (int64_t b = lo; b < hi; ++b) {
        if (bad_block) *bad_block = b;
        const int64_t J = col_idx[b];
        if (J < 0 || J > I)
          return set_error(IAMAP_ERR_INVALID_ARG,
                           "block %lld: column block %lld outside 0..%lld (row block %lld)",
                           (long long)b, (long long)J, (long long)I, (long long)I);
        if (b > lo && J <= col_idx[b - 1])
          return set_error(IAMAP_ERR_INVALID_ARG, "block %lld: column blocks not ascending",
                           (long long)b);
        const uint64_t m = headmask[b];
        if (m == 0 || (m & ~head_bits))
          return set_error(IAMAP_ERR_INVALID_ARG, "block %lld: head mask %llx not in 1..2^%d-1",
                           (long long)b, (unsigned long long)m, H_s);
        const int64_t k = __builtin_popcountll(m);
        if (val_off[b] < 0)
          return set_error(IAMAP_ERR_INVALID_ARG, "block %lld: negative tile offset %lld",
                           (long long)b, (long long)val_off[b]);
        if (val_off[b] > vals_capacity_tiles - k)
          return set_error(IAMAP_ERR_CAPACITY,
                           "block %lld: tiles [%lld, %lld) outside the %lld-tile value buffer",
                           (long long)b, (long long)val_off[b], (long long)(val_off[b] + k),
                           (long long)vals_capacity_tiles);
      }
    }
  }
  if (bad_block) *bad_block = -1;
  return IAMAP_OK;
}
