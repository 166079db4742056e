"""CPU oracle of the prefix-hash block index (exact integer arithmetic in Python ints).

TEST INFRASTRUCTURE ONLY. Imported by ``tests/`` and ``bench.py``'s reference leg; never by the
product path. It shares no code with the CUDA library and imports nothing from this repository.

Source:

[MapFlow-C2]  "PKU MapFlow: cross-model attention map reuse" news page, "storage and execution"
              part, second component: the sparse blocks left by different layers and positions
              differ in number; they are found through a prefix hash index whose keys carry the
              preceding context, so that a receiver model can locate the cached blocks of its
              prompt; one sender state can serve several downstream models.
[FNV]         the Fowler/Noll/Vo hash, 64-bit FNV-1a variant, as published by its authors (IETF
              draft "The FNV Non-Cryptographic Hash Algorithm"): the state starts at the offset
              basis 0xcbf29ce484222325, and each octet is XORed into the state, which is then
              multiplied by the prime 0x100000001b3 modulo 2**64.

The page fixes no hash function, block size or table layout. The readings used here:

* blocks are the map's row blocks: B consecutive tokens of one packed sequence, starting at a
  multiple of B; only full blocks are indexed, because a partial last block changes once the
  sequence grows;
* the digest of block b is FNV-1a-64 of its B token ids as 4-byte little-endian integers;
* the prefix key of block b continues FNV-1a-64 from the state ``salt`` over the 8-byte
  little-endian digests of blocks 0 .. b; with salt = the FNV offset basis it is FNV-1a-64 of the
  concatenated digests. A caller picks the salt per sender layer (or model), so entries of
  different layers never share a key;
* the index maps a key to one int64 location (where the row block's stored map blocks are);
  inserting a key that is present keeps the present location (first writer wins) and returns it;
* the all-ones 64-bit key is reserved as "empty" and is never stored (a 2**-64 event);
* a lookup of a sequence reports its number of leading full blocks whose keys are present: the
  longest cached prefix, in blocks.

Parity status: pinned by ``tests/test_prefix_index_oracle.py`` against the published FNV-1a-64
test vectors (``tests/golden/fnv1a64.json``) and against brute-force token-prefix comparison
that uses no hashing.
"""

from __future__ import annotations

import numpy as np

FNV64_OFFSET = 0xCBF29CE484222325
FNV64_PRIME = 0x100000001B3
MASK64 = (1 << 64) - 1
EMPTY_KEY = MASK64
MISSING = -1

__all__ = ["FNV64_OFFSET", "FNV64_PRIME", "EMPTY_KEY", "MISSING", "fnv1a64", "block_digests",
           "prefix_keys", "PrefixIndex", "prefix_hits", "num_full_blocks"]


def fnv1a64(data: bytes, state: int = FNV64_OFFSET) -> int:
    """[FNV] FNV-1a-64 of `data`, continued from `state` (the offset basis for a fresh hash)."""
    h = state
    for octet in data:
        h ^= octet
        h = (h * FNV64_PRIME) & MASK64
    return h


def _le_int32(tokens) -> bytes:
    return b"".join(int(t).to_bytes(4, "little", signed=True) for t in tokens)


def num_full_blocks(seqlens, B: int):
    return [int(L) // B for L in seqlens]


def block_digests(tokens: np.ndarray, cu_seqlens, B: int):
    """Per sequence, the list of digests of its full blocks ([MapFlow-C2] reading: FNV-1a-64 of
    the block's token ids, 4-byte little-endian)."""
    out = []
    for s in range(len(cu_seqlens) - 1):
        a, b = int(cu_seqlens[s]), int(cu_seqlens[s + 1])
        out.append([fnv1a64(_le_int32(tokens[a + j * B: a + (j + 1) * B]))
                    for j in range((b - a) // B)])
    return out


def prefix_keys(tokens: np.ndarray, cu_seqlens, B: int, salt: int = FNV64_OFFSET):
    """Prefix keys of every full block, packed sequence after sequence, and their per-sequence
    offsets: (keys uint64 [sum of full blocks], key_cu int64 [num_seqs + 1]).

    [MapFlow-C2] the key of a block carries its whole preceding context: the FNV-1a-64 state
    after absorbing, from `salt`, the little-endian digests of the sequence's blocks up to it."""
    keys, key_cu = [], [0]
    for digs in block_digests(tokens, cu_seqlens, B):
        h = salt & MASK64
        for c in digs:
            h = fnv1a64(c.to_bytes(8, "little"), h)
            keys.append(h)
        key_cu.append(len(keys))
    return np.array(keys, dtype=np.uint64), np.array(key_cu, dtype=np.int64)


class PrefixIndex:
    """[MapFlow-C2] the index as a mapping from prefix key to location (a Python dict)."""

    def __init__(self):
        self.table = {}

    def insert(self, keys, values):
        """Insert-if-absent, in the given order; returns, per item, the location now associated
        with its key (MISSING for the reserved empty key)."""
        stored = np.empty(len(keys), dtype=np.int64)
        for i, (k, v) in enumerate(zip(keys, values)):
            k = int(k)
            if k == EMPTY_KEY:
                stored[i] = MISSING
                continue
            if k not in self.table:
                self.table[k] = int(v)
            stored[i] = self.table[k]
        return stored

    def lookup(self, keys):
        return np.array([MISSING if int(k) == EMPTY_KEY else self.table.get(int(k), MISSING)
                         for k in keys], dtype=np.int64)


def prefix_hits(found: np.ndarray, key_cu) -> np.ndarray:
    """Per sequence, the number of leading blocks whose lookup found a location."""
    hits = []
    for s in range(len(key_cu) - 1):
        a, b = int(key_cu[s]), int(key_cu[s + 1])
        j = 0
        while a + j < b and found[a + j] != MISSING:
            j += 1
        hits.append(j)
    return np.array(hits, dtype=np.int32)
