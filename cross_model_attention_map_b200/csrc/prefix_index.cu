// Prefix-hash block index: locating a sender's stored map blocks by the tokens that precede them.
//
// "PKU MapFlow: cross-model attention map reuse" news page, storage-and-execution part, second
// component: the cached sparse blocks are found through a prefix hash index whose keys carry the
// preceding context, so that a receiver locates the blocks of its prompt; one sender state can
// serve several downstream models. The page fixes no hash or layout; this file implements:
//
// * block b of a packed sequence = tokens [b*B, (b+1)*B) (full blocks only, aligned with the
//   map's row blocks);
// * digest c_b = FNV-1a-64 of the block's token ids as 4-byte little-endian integers (the
//   Fowler/Noll/Vo hash, FNV-1a variant: offset basis 0xcbf29ce484222325, prime 0x100000001b3,
//   XOR each octet into the state, then multiply modulo 2^64);
// * prefix key k_b = the FNV-1a-64 state after absorbing, from a caller-chosen salt, the 8-byte
//   little-endian digests c_0 .. c_b: the key depends on every token before the block's end;
// * an open-addressing table (keys uint64, all ones = empty; values int64 locations) with linear
//   probing from Fibonacci hashing (multiply by 2^64 / golden ratio, keep the top log2(capacity)
//   bits). Insert keeps the first location of a key; lookup returns it or -1.
//
// Kernels (integer work, a few bytes per token: latency-bound at prompt sizes):
//   1. prefix_keys_kernel   one CTA per sequence: digests of up to 256 blocks in parallel (one
//                           thread per block, 4*B bytes each), then one thread chains them.
//   2. insert_claim_kernel  one thread per key: claims an empty slot with atomicCAS, or finds the
//                           key's slot; writes the slot index.
//   3. insert_publish_kernel the location now stored at each key's slot (a separate launch, so
//                           every claimer's location is visible to duplicates of its key).
//   4. lookup_kernel        one CTA per sequence (or per 4096-key chunk): found locations and the
//                           number of leading hits (the longest cached prefix, in blocks).
// Probing is bounded: a key lives within min(capacity, 1024) slots of its home slot. An insert
// that finds neither the key nor an empty slot in that window fails (location -1) and raises
// IAMAP_DEV_CAPACITY; a lookup stops at the first empty slot or the window's end. Keep the load
// factor below about 0.7 and the window is never exhausted in practice.
#include <algorithm>

#include "internal.h"

namespace iamap {

namespace {

constexpr uint64_t kFnvOffset = 0xcbf29ce484222325ull;
constexpr uint64_t kFnvPrime = 0x100000001b3ull;
constexpr uint64_t kEmptyKey = ~0ull;
constexpr uint64_t kFibMul = 0x9e3779b97f4a7c15ull;   // 2^64 / golden ratio, odd
constexpr int kKeyThreads = 256;
constexpr int kLookupThreads = 256;
constexpr int64_t kFlatSegment = 4096;
constexpr int64_t kMaxProbes = 1024;

__device__ __forceinline__ uint64_t fnv_absorb_u32(uint64_t h, uint32_t w) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    h ^= (w >> (8 * i)) & 0xffu;
    h *= kFnvPrime;
  }
  return h;
}

__device__ __forceinline__ uint64_t fnv_absorb_u64(uint64_t h, uint64_t w) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    h ^= (w >> (8 * i)) & 0xffu;
    h *= kFnvPrime;
  }
  return h;
}

__device__ __forceinline__ uint64_t home_slot(uint64_t key, int log2cap) {
  return log2cap == 0 ? 0ull : (key * kFibMul) >> (64 - log2cap);
}

// Sum over a CTA of one int64 per thread (blockDim.x a multiple of 32, at most 1024).
__device__ int64_t block_sum(int64_t v, int64_t* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  int64_t t = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
  __syncthreads();
  return t;
}

__device__ int64_t block_min(int64_t v, int64_t* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, (int64_t)__shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  int64_t t = red[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) t = min(t, red[w]);
  __syncthreads();
  return t;
}

// Valid [a, b) of sequence s, or an empty range (with IAMAP_DEV_BAD_INDEX) when cu_seqlens
// does not describe a range inside the n tokens.
__device__ __forceinline__ void seq_range(const int32_t* cu, int s, int64_t n, int64_t* a,
                                          int64_t* b, bool* bad) {
  const int64_t x = cu[s], y = cu[s + 1];
  *bad = x < 0 || y < x || y > n;
  *a = *bad ? 0 : x;
  *b = *bad ? 0 : y;
}

__global__ void __launch_bounds__(kKeyThreads) prefix_keys_kernel(
    const int32_t* __restrict__ tokens, int64_t n, const int32_t* __restrict__ cu, int B,
    uint64_t salt, uint64_t* __restrict__ keys, int64_t keys_capacity,
    int64_t* __restrict__ key_cu, unsigned int* status) {
  __shared__ uint64_t dig[kKeyThreads];
  __shared__ int64_t red[kKeyThreads / 32];
  const int s = blockIdx.x;

  // offset of this sequence's keys: full blocks of the sequences before it
  int64_t before = 0;
  for (int t = threadIdx.x; t < s; t += blockDim.x) {
    int64_t a, b;
    bool bad;
    seq_range(cu, t, n, &a, &b, &bad);
    before += (b - a) / B;
  }
  const int64_t off = block_sum(before, red);
  int64_t a, b;
  bool bad;
  seq_range(cu, s, n, &a, &b, &bad);
  const int64_t nfull = (b - a) / B;
  if (threadIdx.x == 0) {
    if (bad) raise_status(status, IAMAP_DEV_BAD_INDEX);
    if (off + nfull > keys_capacity) raise_status(status, IAMAP_DEV_CAPACITY);
    key_cu[s + 1] = off + nfull;
    if (s == 0) key_cu[0] = 0;
  }

  uint64_t h = salt;   // chain state, carried by thread 0 across chunks
  for (int64_t c0 = 0; c0 < nfull; c0 += kKeyThreads) {
    const int64_t blk = c0 + threadIdx.x;
    if (blk < nfull) {
      const int32_t* p = tokens + a + blk * B;
      uint64_t d = kFnvOffset;
      for (int j = 0; j < B; ++j) d = fnv_absorb_u32(d, (uint32_t)__ldg(p + j));
      dig[threadIdx.x] = d;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      const int m = (int)min((int64_t)kKeyThreads, nfull - c0);
      for (int i = 0; i < m; ++i) {
        h = fnv_absorb_u64(h, dig[i]);
        const int64_t at = off + c0 + i;
        if (at < keys_capacity) keys[at] = h;
      }
    }
    __syncthreads();
  }
}

__global__ void insert_claim_kernel(const uint64_t* __restrict__ keys,
                                    const int64_t* __restrict__ values, int64_t count,
                                    unsigned long long* table_keys, int64_t* table_vals,
                                    int log2cap, int64_t probes, int64_t* slot_out,
                                    unsigned int* status) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= count) return;
  const uint64_t key = keys[i];
  int64_t slot = -1;
  if (key != kEmptyKey) {
    const uint64_t mask = (1ull << log2cap) - 1ull;
    uint64_t pos = home_slot(key, log2cap);
    for (int64_t probe = 0; probe < probes; ++probe) {
      const unsigned long long cur =
          atomicCAS(table_keys + pos, (unsigned long long)kEmptyKey, (unsigned long long)key);
      if (cur == kEmptyKey) {          // claimed: this item's location becomes the key's
        table_vals[pos] = values[i];
        slot = (int64_t)pos;
        break;
      }
      if (cur == key) {                // present (earlier insert or a duplicate in this batch)
        slot = (int64_t)pos;
        break;
      }
      pos = (pos + 1) & mask;
    }
    if (slot < 0) raise_status(status, IAMAP_DEV_CAPACITY);
  }
  slot_out[i] = slot;
}

__global__ void insert_publish_kernel(int64_t count, const int64_t* __restrict__ table_vals,
                                      int64_t* stored) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= count) return;
  const int64_t slot = stored[i];
  stored[i] = slot >= 0 ? table_vals[slot] : -1;
}

// Segment s: keys [key_cu[s], key_cu[s+1]) when key_cu is given, else [s*4096, ...) capped at
// count. Writes found[] for the segment and, with key_cu, hit_blocks[s] = leading hits.
__global__ void __launch_bounds__(kLookupThreads) lookup_kernel(
    const uint64_t* __restrict__ keys, int64_t count, const int64_t* __restrict__ key_cu,
    const uint64_t* __restrict__ table_keys, const int64_t* __restrict__ table_vals, int log2cap,
    int64_t probes, int64_t* __restrict__ found, int32_t* __restrict__ hit_blocks,
    unsigned int* status) {
  __shared__ int64_t red[kLookupThreads / 32];
  const int s = blockIdx.x;
  int64_t lo, hi;
  bool bad = false;
  if (key_cu) {
    lo = key_cu[s];
    hi = key_cu[s + 1];
    bad = lo < 0 || hi < lo || hi > count;
    if (bad) lo = hi = 0;
  } else {
    lo = (int64_t)s * kFlatSegment;
    hi = min(count, lo + kFlatSegment);
  }
  const uint64_t mask = (1ull << log2cap) - 1ull;
  int64_t first_miss = hi;
  for (int64_t i = lo + threadIdx.x; i < hi; i += blockDim.x) {
    const uint64_t key = keys[i];
    int64_t v = -1;
    if (key != kEmptyKey) {
      uint64_t pos = home_slot(key, log2cap);
      for (int64_t probe = 0; probe < probes; ++probe) {
        const uint64_t cur = table_keys[pos];
        if (cur == key) {
          v = table_vals[pos];
          break;
        }
        if (cur == kEmptyKey) break;
        pos = (pos + 1) & mask;
      }
    }
    found[i] = v;
    if (v < 0) first_miss = min(first_miss, i);
  }
  if (key_cu && hit_blocks) {
    const int64_t m = block_min(first_miss, red);
    if (threadIdx.x == 0) {
      if (bad) raise_status(status, IAMAP_DEV_BAD_INDEX);
      hit_blocks[s] = (int32_t)(m - lo);
    }
  }
}

int log2_exact(int64_t x) {
  int l = 0;
  while ((int64_t(1) << l) < x) ++l;
  return l;
}

}  // namespace

int prefix_keys_launch(const int32_t* tokens, int64_t n, const int32_t* cu, int num_seqs, int B,
                       uint64_t salt, uint64_t* keys, int64_t keys_capacity, int64_t* key_cu,
                       cudaStream_t stream) {
  DeviceContext* c = device_context();
  if (!c) return IAMAP_ERR_CUDA;
  prefix_keys_kernel<<<num_seqs, kKeyThreads, 0, stream>>>(tokens, n, cu, B, salt, keys,
                                                           keys_capacity, key_cu, c->status);
  IAMAP_LAUNCH_CHECK("prefix_keys_kernel");
  return IAMAP_OK;
}

int prefix_clear_launch(uint64_t* table_keys, int64_t* table_vals, int64_t capacity,
                        cudaStream_t stream) {
  // all-ones bytes: the empty key, and location -1
  IAMAP_CUDA_CHECK(cudaMemsetAsync(table_keys, 0xff, (size_t)capacity * sizeof(uint64_t), stream));
  IAMAP_CUDA_CHECK(cudaMemsetAsync(table_vals, 0xff, (size_t)capacity * sizeof(int64_t), stream));
  return IAMAP_OK;
}

int prefix_insert_launch(const uint64_t* keys, const int64_t* values, int64_t count,
                         uint64_t* table_keys, int64_t* table_vals, int64_t capacity,
                         int64_t* stored, cudaStream_t stream) {
  DeviceContext* c = device_context();
  if (!c) return IAMAP_ERR_CUDA;
  if (count == 0) return IAMAP_OK;
  const int threads = 256;
  const unsigned blocks = (unsigned)((count + threads - 1) / threads);
  const int l2 = log2_exact(capacity);
  insert_claim_kernel<<<blocks, threads, 0, stream>>>(
      keys, values, count, reinterpret_cast<unsigned long long*>(table_keys), table_vals, l2,
      std::min(capacity, kMaxProbes), stored, c->status);
  IAMAP_LAUNCH_CHECK("insert_claim_kernel");
  insert_publish_kernel<<<blocks, threads, 0, stream>>>(count, table_vals, stored);
  IAMAP_LAUNCH_CHECK("insert_publish_kernel");
  return IAMAP_OK;
}

int prefix_lookup_launch(const uint64_t* keys, int64_t count, const int64_t* key_cu,
                         int num_seqs, const uint64_t* table_keys, const int64_t* table_vals,
                         int64_t capacity, int64_t* found, int32_t* hit_blocks,
                         cudaStream_t stream) {
  DeviceContext* c = device_context();
  if (!c) return IAMAP_ERR_CUDA;
  const int64_t segs = key_cu ? num_seqs : (count + kFlatSegment - 1) / kFlatSegment;
  if (segs == 0) return IAMAP_OK;
  lookup_kernel<<<(unsigned)segs, kLookupThreads, 0, stream>>>(
      keys, count, key_cu, table_keys, table_vals, log2_exact(capacity),
      std::min(capacity, kMaxProbes), found, hit_blocks, c->status);
  IAMAP_LAUNCH_CHECK("lookup_kernel");
  return IAMAP_OK;
}

}  // namespace iamap
