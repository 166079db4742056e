"""Buffer management around the C ABI for one mapped prefill layer (allocation and calls only).

``PrefillLayer`` owns the device buffers of one (sender layer, receiver layer) pair with fixed
packed sequence lengths and runs the hot path through libiamap:

    compress(q, k)          -> lse, block masses, BSR index and bf16 tiles (no host sync)
    mapped_av(W, v)         -> out [n, H_r, d_v]
    step(q, k, W, v)        -> both

The value buffer is sized for the worst case (every head keeps every causal block) unless a
capacity is given, so the step needs no host synchronisation.
"""

from __future__ import annotations

import torch

from . import iamap as C


class PrefillLayer:
    def __init__(self, seqlens, H_s, d, H_r, d_v, tau, bias_window=0, bias_value=0.0, B=64,
                 capacity_tiles=None, device="cuda", H_kv=None):
        self.seqlens = [int(x) for x in seqlens]
        self.num_seqs = len(self.seqlens)
        cu = [0]
        for L in self.seqlens:
            cu.append(cu[-1] + L)
        self.cu_host = torch.tensor(cu, dtype=torch.int32)
        self.cu = self.cu_host.to(device)
        self.n = cu[-1]
        self.H_s, self.d, self.H_r, self.d_v, self.B = H_s, d, H_r, d_v, B
        self.H_kv = H_r if H_kv is None else int(H_kv)   # receiver value heads (grouped if < H_r)
        self.tau, self.bias_window, self.bias_value = float(tau), int(bias_window), float(bias_value)
        self.nrb, self.ncb, self.max_nb = C.iamap_plan(self.cu_host, self.num_seqs, B)
        self.bufs = C.alloc_compress_outputs(self.n, H_s, self.nrb, self.ncb, device)
        cap = H_s * self.ncb if capacity_tiles is None else int(capacity_tiles)
        self.capacity = cap
        self.vals = torch.empty(max(cap, 1), B, B, dtype=torch.bfloat16, device=device)
        self.ws = C.alloc_workspace(C.iamap_compress_workspace_bytes(self.num_seqs, self.nrb),
                                    device)
        self.out = torch.empty(self.n, H_r, d_v, dtype=torch.float32, device=device)

    def compress(self, q, k, stream=None):
        b = self.bufs
        C.iamap_compress(q, k, self.cu, self.cu_host, self.num_seqs, self.n, self.H_s, self.d,
                         self.B, self.tau, self.bias_window, self.bias_value, b["lse"], b["mass"],
                         b["headmask_dense"], b["row_ptr"], b["col_idx"], b["headmask"],
                         b["val_off"], b["counts"], self.vals, self.capacity, self.ws, stream)

    def mapped_av(self, W, v, stream=None, out=None):
        b = self.bufs
        out = self.out if out is None else out
        C.iamap_mapped_av_gqa(self.cu, self.cu_host, self.num_seqs, self.n, self.B, self.H_s,
                              b["row_ptr"], b["col_idx"], b["headmask"], b["val_off"], self.vals,
                              self.capacity, W, self.H_r, self.H_kv, v, self.d_v, out, self.ws,
                              stream)
        return out

    def step(self, q, k, W, v, stream=None, out=None):
        self.compress(q, k, stream)
        return self.mapped_av(W, v, stream, out)

    def compress_with_output(self, q, k, v_s, o_s, stream=None):
        """compress plus the sender's own attention output o_s [n, H_s, d_vs] from its values
        v_s [n, H_s, d_vs] (same pass over the keys)."""
        b = self.bufs
        C.iamap_compress_with_output(q, k, self.cu, self.cu_host, self.num_seqs, self.n,
                                     self.H_s, self.d, self.B, self.tau, self.bias_window,
                                     self.bias_value, v_s, int(v_s.shape[2]), o_s, b["lse"],
                                     b["mass"], b["headmask_dense"], b["row_ptr"], b["col_idx"],
                                     b["headmask"], b["val_off"], b["counts"], self.vals,
                                     self.capacity, self.ws, stream)
        return o_s

    def counts(self):
        """(nnz_blocks, nnz_tiles) -- synchronises."""
        c = self.bufs["counts"].cpu()
        return int(c[0]), int(c[1])


class ChunkPrefillLayer:
    """Buffers of one chunked-prefill step of a mapped layer pair: the query rows
    [starts[s], ends[s]) of every sequence s against its keys [0, ends[s]) (earlier chunks'
    keys and values cached). starts[s] is a multiple of B. Optionally (d_vs given) the sender's
    own attention output of the chunk rows is produced with the map.

        compress(q, k, v_s=None) -> lse, masses, BSR map of the chunk rows (+ o_s)
        mapped_av(W, v)          -> out [n_q, H_r, d_v]

    q holds the chunk rows packed by cu_q; k, v (and v_s) hold rows [0, ends[s]) packed by cu_k.
    """

    def __init__(self, starts, ends, H_s, d, H_r, d_v, tau, bias_window=0, bias_value=0.0, B=64,
                 capacity_tiles=None, device="cuda", H_kv=None, d_vs=None):
        self.starts = [int(x) for x in starts]
        self.ends = [int(x) for x in ends]
        self.num_seqs = len(self.starts)
        cu_q, cu_k = [0], [0]
        for c0, e in zip(self.starts, self.ends):
            cu_q.append(cu_q[-1] + e - c0)
            cu_k.append(cu_k[-1] + e)
        self.cu_q_host = torch.tensor(cu_q, dtype=torch.int32)
        self.cu_k_host = torch.tensor(cu_k, dtype=torch.int32)
        self.starts_host = torch.tensor(self.starts, dtype=torch.int32)
        self.cu_q = self.cu_q_host.to(device)
        self.cu_k = self.cu_k_host.to(device)
        self.starts_dev = self.starts_host.to(device)
        self.n_q, self.n_k = cu_q[-1], cu_k[-1]
        self.H_s, self.d, self.H_r, self.d_v, self.B = H_s, d, H_r, d_v, B
        self.H_kv = H_r if H_kv is None else int(H_kv)
        self.tau, self.bias_window, self.bias_value = float(tau), int(bias_window), float(bias_value)
        self.nrb, self.ncb, self.max_nb = C.iamap_chunk_plan(self.cu_q_host, self.cu_k_host,
                                                             self.starts_host, self.num_seqs, B)
        self.bufs = C.alloc_compress_outputs(self.n_q, H_s, self.nrb, self.ncb, device)
        cap = H_s * self.ncb if capacity_tiles is None else int(capacity_tiles)
        self.capacity = cap
        self.vals = torch.empty(max(cap, 1), B, B, dtype=torch.bfloat16, device=device)
        self.ws = C.alloc_workspace(C.iamap_compress_workspace_bytes(self.num_seqs, self.nrb),
                                    device)
        self.out = torch.empty(self.n_q, H_r, d_v, dtype=torch.float32, device=device)
        self.d_vs = None if d_vs is None else int(d_vs)
        self.o_s = (None if d_vs is None else
                    torch.empty(self.n_q, H_s, self.d_vs, dtype=torch.float32, device=device))

    def compress(self, q, k, v_s=None, stream=None):
        b = self.bufs
        C.iamap_compress_chunk(q, k, self.cu_q, self.cu_k, self.starts_dev, self.cu_q_host,
                               self.cu_k_host, self.starts_host, self.num_seqs, self.n_q,
                               self.n_k, self.H_s, self.d, self.B, self.tau, self.bias_window,
                               self.bias_value, v_s, self.d_vs or 0,
                               self.o_s if v_s is not None else None, b["lse"], b["mass"],
                               b["headmask_dense"], b["row_ptr"], b["col_idx"], b["headmask"],
                               b["val_off"], b["counts"], self.vals, self.capacity, self.ws,
                               stream)

    def mapped_av(self, W, v, stream=None, out=None):
        b = self.bufs
        out = self.out if out is None else out
        C.iamap_mapped_av_chunk(self.cu_q, self.cu_k, self.starts_dev, self.cu_q_host,
                                self.cu_k_host, self.starts_host, self.num_seqs, self.n_q,
                                self.n_k, self.B, self.H_s, b["row_ptr"], b["col_idx"],
                                b["headmask"], b["val_off"], self.vals, self.capacity, W,
                                self.H_r, self.H_kv, v, self.d_v, out, self.ws, stream)
        return out

    def step(self, q, k, W, v, v_s=None, stream=None, out=None):
        self.compress(q, k, v_s, stream)
        return self.mapped_av(W, v, stream, out)

    def counts(self):
        """(nnz_blocks, nnz_tiles) -- synchronises."""
        c = self.bufs["counts"].cpu()
        return int(c[0]), int(c[1])


class DecodeStep:
    """Buffers of one paged decode step on a mapped layer."""

    def __init__(self, batch, H_s, H_r, d_v, ctx_lens_host, ctx_stride, max_pages, page_size,
                 num_pages, device="cuda", H_kv=None):
        self.batch, self.H_s, self.H_r, self.d_v = batch, H_s, H_r, d_v
        self.H_kv = H_r if H_kv is None else int(H_kv)
        self.ctx_lens_host = torch.as_tensor(ctx_lens_host, dtype=torch.int32).cpu()
        self.ctx_lens = self.ctx_lens_host.to(device)
        self.ctx_stride, self.max_pages, self.page_size = ctx_stride, max_pages, page_size
        self.num_pages = num_pages
        max_ctx = int(self.ctx_lens_host.max())
        self.ws = C.alloc_workspace(
            C.iamap_mapped_av_paged_workspace_bytes(batch, H_r, d_v, max_ctx, page_size), device)
        self.out = torch.empty(batch, H_r, d_v, dtype=torch.float32, device=device)

    def run(self, p_rows, W, v_pages, page_table, stream=None):
        C.iamap_mapped_av_paged_gqa(p_rows, self.ctx_stride, W, v_pages, self.num_pages,
                                    page_table, self.max_pages, self.page_size, self.ctx_lens,
                                    self.ctx_lens_host, self.batch, self.H_s, self.H_r, self.H_kv,
                                    self.d_v, self.out, self.ws, stream)
        return self.out


class HeadMatch:
    """Buffers of one head-matching calibration."""

    def __init__(self, L_s, H_small, d_small, L_l, H_large, d_large, n, n_used=None,
                 want_sim=True, device="cuda", metric="cosine"):
        self.dims = (L_s, H_small, d_small, L_l, H_large, d_large)
        self.metric = C.SIM_METRICS[metric]
        self.n = n
        self.n_used = n if n_used is None else int(n_used)
        self.ws = C.alloc_workspace(
            C.iamap_head_match_workspace_bytes(L_s, H_small, L_l, H_large, self.n_used), device)
        self.argmax = torch.empty(L_l * H_large, dtype=torch.int32, device=device)
        self.sim = (torch.empty(L_l * H_large, L_s * H_small, dtype=torch.float32, device=device)
                    if want_sim else None)

    def run(self, q_small, k_small, q_large, k_large, stream=None):
        L_s, H_small, d_small, L_l, H_large, d_large = self.dims
        C.iamap_head_match_metric(q_small, k_small, L_s, H_small, d_small, q_large, k_large,
                                  L_l, H_large, d_large, self.n, self.n_used, self.metric,
                                  self.argmax, self.sim, self.ws, stream)
        return self.argmax, self.sim


def mapping_consistency(argmax_a, argmax_b, stream=None):
    """Number of large heads (device int32 tensor of one element) that two head mappings send to
    the same small head; divide by the head count for the consistency rate."""
    agree = torch.zeros(1, dtype=torch.int32, device=argmax_a.device)
    C.iamap_mapping_consistency(argmax_a, argmax_b, argmax_a.numel(), agree, stream)
    return agree


class PrefixIndex:
    """A device prefix-hash index of stored map blocks: `capacity` slots (a power of two) of
    uint64 keys (carried as int64 tensors) and int64 locations, keys made with `salt` (one salt
    per sender layer or model)."""

    def __init__(self, capacity, B=64, salt=0xCBF29CE484222325, device="cuda"):
        self.capacity, self.B, self.salt = int(capacity), int(B), int(salt)
        self.table_keys = torch.empty(self.capacity, dtype=torch.int64, device=device)
        self.table_vals = torch.empty(self.capacity, dtype=torch.int64, device=device)
        self.device = device
        self.clear()

    def clear(self, stream=None):
        C.iamap_prefix_index_clear(self.table_keys, self.table_vals, self.capacity, stream)

    def keys(self, tokens, cu_seqlens, cu_seqlens_host, stream=None):
        """(keys int64 [num_keys], key_cu int64 [num_seqs + 1]) of packed prompts."""
        num_seqs = len(cu_seqlens_host) - 1
        nk = C.iamap_prefix_num_keys(cu_seqlens_host, num_seqs, self.B)
        keys = torch.empty(max(nk, 1), dtype=torch.int64, device=self.device)
        key_cu = torch.empty(num_seqs + 1, dtype=torch.int64, device=self.device)
        C.iamap_prefix_keys(tokens, tokens.numel(), cu_seqlens, num_seqs, self.B, self.salt, keys,
                            nk, key_cu, stream)
        return keys[:nk], key_cu

    def insert(self, keys, values, stream=None):
        """Locations now stored for `keys` (int64 [count]); -1 where no slot was found."""
        stored = torch.empty(max(keys.numel(), 1), dtype=torch.int64, device=self.device)
        C.iamap_prefix_insert(keys, values, keys.numel(), self.table_keys, self.table_vals,
                              self.capacity, stored, stream)
        return stored[:keys.numel()]

    def lookup(self, keys, key_cu=None, stream=None):
        """(found int64 [count], hit_blocks int32 [num_seqs] or None)."""
        found = torch.empty(max(keys.numel(), 1), dtype=torch.int64, device=self.device)
        hits = None
        num_seqs = 0
        if key_cu is not None:
            num_seqs = key_cu.numel() - 1
            hits = torch.empty(num_seqs, dtype=torch.int32, device=self.device)
        C.iamap_prefix_lookup(keys, keys.numel(), key_cu, num_seqs, self.table_keys,
                              self.table_vals, self.capacity, found, hits, stream)
        return found[:keys.numel()], hits


# ------------------------------------------------------------------------------------------------
# Several GPUs: head matching split by large layers, prefill split by sequence
# ------------------------------------------------------------------------------------------------

def shard_range(total, world, rank):
    """[lo, hi) of `total` items given to `rank` of `world`: contiguous blocks of
    ceil(total / world), the last ones possibly short or empty."""
    per = -(-total // world)
    lo = min(total, rank * per)
    return lo, min(total, lo + per)


def causal_blocks(L, B=64):
    """Causal (row block, column block) pairs of a sequence of L tokens: its share of the work of
    compress and mapped_av."""
    nb = -(-int(L) // B)
    return nb * (nb + 1) // 2


def shard_sequences(seqlens, world, B=64):
    """Packed sequences -> ranks for a prefill split by sequence (no collective on the path).
    Longest-processing-time-first: sequences by decreasing causal blocks (ties: lower index)
    go to the rank with the least work so far (ties: lower rank). The most loaded rank then has
    at most (4/3 - 1/(3 world)) times the optimum. Returns per-rank lists of sequence indices in
    increasing order."""
    work = [0] * world
    out = [[] for _ in range(world)]
    order = sorted(range(len(seqlens)), key=lambda s: (-causal_blocks(seqlens[s], B), s))
    for s in order:
        r = min(range(world), key=lambda x: (work[x], x))
        out[r].append(s)
        work[r] += causal_blocks(seqlens[s], B)
    return [sorted(x) for x in out]


def gather_head_mapping(local_argmax, L_l, H_large, group=None):
    """All ranks' head mappings of their large-layer shards ([hi - lo, H_large] int32 on this
    rank's device, shards from shard_range) -> the full [L_l, H_large] mapping on every rank, with
    one all_gather of int32 (the only collective of a sharded calibration)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    per = -(-L_l // world)
    pad = torch.zeros(per, H_large, dtype=torch.int32, device=local_argmax.device)
    pad[:local_argmax.shape[0]] = local_argmax.view(-1, H_large)
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat(parts, dim=0)[:L_l]


class HostPrefillPipeline:
    """Prefill steps of one PrefillLayer on host-resident (pinned) inputs through the library's
    own host-buffer entry point (iamap_prefill_steps_host): every step uploads its q, k, v, W and
    reads its output back, and the upload of the next step and the read-back of the previous one
    overlap the current step's kernels (two device sets of inputs and outputs in `io`; the
    library's upload and download streams, ordered by events against the compute stream)."""

    def __init__(self, layer, device="cuda"):
        self.layer = layer
        L = layer
        self.io = C.alloc_workspace(C.iamap_prefill_io_bytes(L.n, L.H_s, L.d, L.H_r, L.H_kv,
                                                             L.d_v), device)

    def bytes_per_step(self):
        """(host-to-device, device-to-host) bytes of one step."""
        L = self.layer
        h2d = 2 * 2 * L.n * L.H_s * L.d + 2 * L.n * L.H_kv * L.d_v + 4 * L.H_r * L.H_s
        return h2d, 4 * L.n * L.H_r * L.d_v

    def run(self, host_inputs, host_outputs, stream=None):
        """host_inputs[i] = (q, k, v, W) pinned CPU tensors of step i; host_outputs[i] the pinned
        CPU tensor receiving its output (entries may repeat: a buffer is written in step order).
        Enqueues every step (the first upload follows everything enqueued on `stream` before)
        and returns the event recorded on `stream` after the last read-back."""
        comp = torch.cuda.current_stream() if stream is None else stream
        L = self.layer
        b = L.bufs
        if host_inputs:
            qs, ks, vs, Ws = (list(x) for x in zip(*host_inputs))
            C.iamap_prefill_steps_host(qs, ks, vs, Ws, list(host_outputs), L.cu, L.cu_host,
                                       L.num_seqs, L.n, L.H_s, L.d, L.H_r, L.H_kv, L.d_v, L.B,
                                       L.tau, L.bias_window, L.bias_value, b["lse"], b["mass"],
                                       b["headmask_dense"], b["row_ptr"], b["col_idx"],
                                       b["headmask"], b["val_off"], b["counts"], L.vals,
                                       L.capacity, self.io, L.ws, comp)
        done = torch.cuda.Event(enable_timing=True)
        done.record(comp)
        return done
