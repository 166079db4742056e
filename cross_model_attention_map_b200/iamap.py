"""Python binding of libiamap (ctypes): argument marshalling only.

Every function here has the name and argument order of the C entry point in include/iamap.h.
Tensors are torch tensors on the current CUDA device (their data pointers are passed); the CUDA
stream is torch's current stream unless one is given. Nothing is computed in Python: every step
runs in the library's kernels. If libiamap.so is missing or fails to load, importing this module
raises ImportError -- there is no fallback.

Small helpers (``alloc_*``) allocate output buffers with torch in the shapes the C ABI documents.
"""

from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libiamap.so")

if not os.path.exists(_LIB_PATH):
    raise ImportError("libiamap.so not found at %s: build it with "
                      "`python -m cross_model_attention_map_b200.build`" % _LIB_PATH)
try:
    _lib = ctypes.CDLL(_LIB_PATH)
except OSError as e:  # pragma: no cover - exercised only on broken installs
    raise ImportError("libiamap.so failed to load: %s" % e) from e

LIB_PATH = _LIB_PATH

IAMAP_OK = 0
IAMAP_DEV_CAPACITY = 1
IAMAP_DEV_TIMEOUT = 2
IAMAP_DEV_BAD_INDEX = 4

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_F = ctypes.c_float
_SZ = ctypes.c_size_t
_U64 = ctypes.c_uint64

_SIGS = {
    "iamap_version": (_I, []),
    "iamap_last_error": (ctypes.c_char_p, []),
    "iamap_device_status": (_I, [_P, ctypes.POINTER(_I)]),
    "iamap_plan": (_I, [_P, _I, _I, ctypes.POINTER(_I64), ctypes.POINTER(_I64),
                        ctypes.POINTER(ctypes.c_int32)]),
    "iamap_compress_workspace_bytes": (_SZ, [_I, _I64]),
    "iamap_compress_stats": (_I, [_P, _P, _P, _P, _I, _I64, _I, _I, _I, _F, _I, _F,
                                  _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "iamap_compress_extract": (_I, [_P, _P, _P, _P, _I, _I64, _I, _I, _I, _I, _F,
                                    _P, _P, _P, _P, _P, _P, _P, _I64, _P, _SZ, _P]),
    "iamap_compress": (_I, [_P, _P, _P, _P, _I, _I64, _I, _I, _I, _F, _I, _F,
                            _P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _P, _SZ, _P]),
    "iamap_mapped_av": (_I, [_P, _P, _I, _I64, _I, _I, _P, _P, _P, _P, _P, _I64, _P, _I, _P,
                             _I, _P, _P, _SZ, _P]),
    "iamap_mapped_av_gqa": (_I, [_P, _P, _I, _I64, _I, _I, _P, _P, _P, _P, _P, _I64, _P, _I, _I,
                                 _P, _I, _P, _P, _SZ, _P]),
    "iamap_mapped_av_paged_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I]),
    "iamap_mapped_av_paged_gqa": (_I, [_P, _I, _P, _P, _I64, _P, _I, _I, _P, _P, _I, _I, _I, _I,
                                       _I, _P, _P, _SZ, _P]),
    "iamap_mapped_av_paged": (_I, [_P, _I, _P, _P, _I64, _P, _I, _I, _P, _P, _I, _I, _I, _I,
                                   _P, _P, _SZ, _P]),
    "iamap_mapped_av_paged_noalloc": (_I, [_P, _I, _P, _P, _I64, _P, _I, _I, _P, _P, _I, _I, _I,
                                           _I, _P, _P]),
    "iamap_head_match_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I]),
    "iamap_head_match": (_I, [_P, _P, _I, _I, _I, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _SZ,
                              _P]),
    "iamap_head_match_metric": (_I, [_P, _P, _I, _I, _I, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P,
                                     _P, _SZ, _P]),
    "iamap_mapping_consistency": (_I, [_P, _P, _I, _P, _P]),
    "iamap_selftest_wait_timeout": (_I, [_I, _P, _P]),
    "iamap_selftest_exp2": (_I, [_P, _P, _P, _I64, _P]),
    "iamap_prefix_num_keys": (_I, [_P, _I, _I, ctypes.POINTER(_I64)]),
    "iamap_bsr_check_host": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _I64,
                                  ctypes.POINTER(_I64)]),
    "iamap_prefix_keys": (_I, [_P, _I64, _P, _I, _I, _U64, _P, _I64, _P, _P]),
    "iamap_prefix_index_clear": (_I, [_P, _P, _I64, _P]),
    "iamap_prefix_insert": (_I, [_P, _P, _I64, _P, _P, _I64, _P, _P]),
    "iamap_prefix_lookup": (_I, [_P, _I64, _P, _I, _P, _P, _I64, _P, _P, _P]),
    "iamap_prefill_io_bytes": (_SZ, [_I64, _I, _I, _I, _I, _I]),
    "iamap_prefill_steps_host": (_I, [_I, _P, _P, _P, _P, _P, _P, _P, _I, _I64, _I, _I, _I, _I,
                                      _I, _I, _F, _I, _F, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                      _I64, _P, _SZ, _P, _SZ, _P]),
    "iamap_compress_with_output": (_I, [_P, _P, _P, _P, _I, _I64, _I, _I, _I, _F, _I, _F,
                                        _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I64,
                                        _P, _SZ, _P]),
    "iamap_compress_extract_with_output": (_I, [_P, _P, _P, _P, _I, _I64, _I, _I, _I, _I, _F,
                                                _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _P,
                                                _SZ, _P]),
    "iamap_sender_rows_workspace_bytes": (_SZ, [_I, _I, _I]),
    "iamap_sender_rows": (_I, [_P, _P, _I64, _P, _I, _I, _P, _P, _I, _I, _I, _P, _I, _P, _SZ,
                               _P]),
    "iamap_layers_plan": (_I, [_P, _I, _I, _I, ctypes.POINTER(_I64), ctypes.POINTER(_I64),
                               ctypes.POINTER(ctypes.c_int32)]),
    "iamap_layers_workspace_bytes": (_SZ, [_I, _I, _I64]),
    "iamap_compress_layers": (_I, [_P, _P, _P, _P, _I, _I64, _I, _I, _I, _I, _F, _I, _F, _P, _P,
                                   _P, _P, _P, _P, _P, _P, _P, _I64, _P, _SZ, _P]),
    "iamap_mapped_av_layers": (_I, [_P, _P, _I, _I64, _I, _I, _I, _P, _P, _P, _P, _P, _I64, _P,
                                    _I, _I, _P, _I, _P, _P, _SZ, _P]),
    "iamap_chunk_plan": (_I, [_P, _P, _P, _I, _I, ctypes.POINTER(_I64), ctypes.POINTER(_I64),
                              ctypes.POINTER(ctypes.c_int32)]),
    "iamap_compress_chunk": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I64, _I64, _I, _I, _I,
                                  _F, _I, _F, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                  _I64, _P, _SZ, _P]),
    "iamap_mapped_av_chunk": (_I, [_P, _P, _P, _P, _P, _P, _I, _I64, _I64, _I, _I, _P, _P, _P,
                                   _P, _P, _I64, _P, _I, _I, _P, _I, _P, _P, _SZ, _P]),
}

EXPORTED = tuple(_SIGS)

for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class IamapError(RuntimeError):
    def __init__(self, fn, code):
        msg = _lib.iamap_last_error().decode(errors="replace")
        super().__init__("%s returned %d: %s" % (fn, code, msg))
        self.code = code


def _check(fn, rc):
    if rc != IAMAP_OK:
        raise IamapError(fn, rc)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _host_i32(a):
    """Host int32 buffer (numpy array, list or CPU tensor) -> (ctypes pointer, keep-alive)."""
    t = torch.as_tensor(a, dtype=torch.int32).cpu().contiguous()
    return ctypes.c_void_p(t.data_ptr()), t


# ------------------------------------------------------------------------------------------------

def iamap_version() -> int:
    return _lib.iamap_version()


def iamap_last_error() -> str:
    return _lib.iamap_last_error().decode(errors="replace")


def iamap_device_status(stream=None) -> int:
    st = _I(0)
    _check("iamap_device_status", _lib.iamap_device_status(_stream(stream), ctypes.byref(st)))
    return st.value


def iamap_plan(cu_seqlens_host, num_seqs, B):
    p, keep = _host_i32(cu_seqlens_host)
    nrb, ncb, mx = _I64(0), _I64(0), ctypes.c_int32(0)
    _check("iamap_plan", _lib.iamap_plan(p, num_seqs, B, ctypes.byref(nrb), ctypes.byref(ncb),
                                         ctypes.byref(mx)))
    del keep
    return nrb.value, ncb.value, mx.value


def iamap_compress_workspace_bytes(num_seqs, num_rowblocks) -> int:
    return _lib.iamap_compress_workspace_bytes(num_seqs, num_rowblocks)


def iamap_compress_stats(q, k, cu_seqlens, cu_seqlens_host, num_seqs, n, H_s, d, B, tau,
                         bias_window, bias_value, lse, mass, headmask_dense, row_ptr, col_idx,
                         headmask, val_off, counts, ws, stream=None):
    cp, keep = _host_i32(cu_seqlens_host)
    _check("iamap_compress_stats", _lib.iamap_compress_stats(
        _ptr(q), _ptr(k), _ptr(cu_seqlens), cp, num_seqs, n, H_s, d, B, tau, bias_window,
        bias_value, _ptr(lse), _ptr(mass), _ptr(headmask_dense), _ptr(row_ptr), _ptr(col_idx),
        _ptr(headmask), _ptr(val_off), _ptr(counts), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))
    del keep


def iamap_compress_extract(q, k, cu_seqlens, cu_seqlens_host, num_seqs, n, H_s, d, B,
                           bias_window, bias_value, lse, row_ptr, col_idx, headmask, val_off,
                           counts, vals, vals_capacity_tiles, ws, stream=None):
    cp, keep = _host_i32(cu_seqlens_host)
    _check("iamap_compress_extract", _lib.iamap_compress_extract(
        _ptr(q), _ptr(k), _ptr(cu_seqlens), cp, num_seqs, n, H_s, d, B, bias_window, bias_value,
        _ptr(lse), _ptr(row_ptr), _ptr(col_idx), _ptr(headmask), _ptr(val_off), _ptr(counts),
        _ptr(vals), vals_capacity_tiles, _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))
    del keep


def iamap_compress(q, k, cu_seqlens, cu_seqlens_host, num_seqs, n, H_s, d, B, tau, bias_window,
                   bias_value, lse, mass, headmask_dense, row_ptr, col_idx, headmask, val_off,
                   counts, vals, vals_capacity_tiles, ws, stream=None):
    cp, keep = _host_i32(cu_seqlens_host)
    _check("iamap_compress", _lib.iamap_compress(
        _ptr(q), _ptr(k), _ptr(cu_seqlens), cp, num_seqs, n, H_s, d, B, tau, bias_window,
        bias_value, _ptr(lse), _ptr(mass), _ptr(headmask_dense), _ptr(row_ptr), _ptr(col_idx),
        _ptr(headmask), _ptr(val_off), _ptr(counts), _ptr(vals), vals_capacity_tiles, _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    del keep


def iamap_mapped_av(cu_seqlens, cu_seqlens_host, num_seqs, n, B, H_s, row_ptr, col_idx, headmask,
                    val_off, vals, vals_capacity_tiles, W, H_r, v, d_v, out, ws, stream=None):
    cp, keep = _host_i32(cu_seqlens_host)
    _check("iamap_mapped_av", _lib.iamap_mapped_av(
        _ptr(cu_seqlens), cp, num_seqs, n, B, H_s, _ptr(row_ptr), _ptr(col_idx), _ptr(headmask),
        _ptr(val_off), _ptr(vals), vals_capacity_tiles, _ptr(W), H_r, _ptr(v), d_v, _ptr(out),
        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))
    del keep


def iamap_compress_with_output(q, k, cu_seqlens, cu_seqlens_host, num_seqs, n, H_s, d, B, tau,
                               bias_window, bias_value, v_s, d_vs, o_s, lse, mass,
                               headmask_dense, row_ptr, col_idx, headmask, val_off, counts, vals,
                               vals_capacity_tiles, ws, stream=None):
    cp, keep = _host_i32(cu_seqlens_host)
    _check("iamap_compress_with_output", _lib.iamap_compress_with_output(
        _ptr(q), _ptr(k), _ptr(cu_seqlens), cp, num_seqs, n, H_s, d, B, tau, bias_window,
        bias_value, _ptr(v_s), d_vs, _ptr(o_s), _ptr(lse), _ptr(mass), _ptr(headmask_dense),
        _ptr(row_ptr), _ptr(col_idx), _ptr(headmask), _ptr(val_off), _ptr(counts), _ptr(vals),
        vals_capacity_tiles, _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))
    del keep


def iamap_prefill_io_bytes(n, H_s, d, H_r, H_kv, d_v) -> int:
    return _lib.iamap_prefill_io_bytes(n, H_s, d, H_r, H_kv, d_v)


def _host_ptrs(tensors):
    """ctypes array of the data pointers of host tensors (pinned CPU tensors)."""
    for t in tensors:
        if t.is_cuda:
            raise ValueError("host buffers expected")
    return (ctypes.c_void_p * len(tensors))(*[t.data_ptr() for t in tensors])


def iamap_prefill_steps_host(q_host, k_host, v_host, W_host, out_host, cu_seqlens,
                             cu_seqlens_host, num_seqs, n, H_s, d, H_r, H_kv, d_v, B, tau,
                             bias_window, bias_value, lse, mass, headmask_dense, row_ptr, col_idx,
                             headmask, val_off, counts, vals, vals_capacity_tiles, io, ws,
                             stream=None):
    """q_host .. out_host: lists (one entry per step) of CPU tensors (pinned for overlap)."""
    steps = len(q_host)
    if not (len(k_host) == len(v_host) == len(W_host) == len(out_host) == steps):
        raise ValueError("one host buffer of each kind per step")
    arrs = [_host_ptrs(x) for x in (q_host, k_host, v_host, W_host, out_host)]
    cp, keep = _host_i32(cu_seqlens_host)
    _check("iamap_prefill_steps_host", _lib.iamap_prefill_steps_host(
        steps, *[ctypes.cast(a, ctypes.c_void_p) for a in arrs], _ptr(cu_seqlens), cp, num_seqs,
        n, H_s, d, H_r, H_kv, d_v, B, tau, bias_window, bias_value, _ptr(lse), _ptr(mass),
        _ptr(headmask_dense), _ptr(row_ptr), _ptr(col_idx), _ptr(headmask), _ptr(val_off),
        _ptr(counts), _ptr(vals), vals_capacity_tiles, _ptr(io), io.numel() * io.element_size(),
        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))
    del keep, arrs


def iamap_compress_extract_with_output(q, k, cu_seqlens, cu_seqlens_host, num_seqs, n, H_s, d,
                                       B, bias_window, bias_value, v_s, d_vs, o_s, lse, row_ptr,
                                       col_idx, headmask, val_off, counts, vals,
                                       vals_capacity_tiles, ws, stream=None):
    cp, keep = _host_i32(cu_seqlens_host)
    _check("iamap_compress_extract_with_output", _lib.iamap_compress_extract_with_output(
        _ptr(q), _ptr(k), _ptr(cu_seqlens), cp, num_seqs, n, H_s, d, B, bias_window, bias_value,
        _ptr(v_s), d_vs, _ptr(o_s), _ptr(lse), _ptr(row_ptr), _ptr(col_idx), _ptr(headmask),
        _ptr(val_off), _ptr(counts), _ptr(vals), vals_capacity_tiles, _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    del keep


def iamap_sender_rows_workspace_bytes(batch, H_s, ctx_stride) -> int:
    return _lib.iamap_sender_rows_workspace_bytes(batch, H_s, ctx_stride)


def iamap_sender_rows(q, k_pages, num_pages, page_table, max_pages, page_size, ctx_lens,
                      ctx_lens_host, batch, H_s, d, p_rows, ctx_stride, ws, stream=None):
    cp, keep = _host_i32(ctx_lens_host)
    _check("iamap_sender_rows", _lib.iamap_sender_rows(
        _ptr(q), _ptr(k_pages), num_pages, _ptr(page_table), max_pages, page_size,
        _ptr(ctx_lens), cp, batch, H_s, d, _ptr(p_rows), ctx_stride, _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    del keep


def iamap_layers_plan(cu_seqlens_host, num_seqs, num_layers, B):
    cp, keep = _host_i32(cu_seqlens_host)
    nrb, ncb, mx = _I64(0), _I64(0), ctypes.c_int32(0)
    _check("iamap_layers_plan", _lib.iamap_layers_plan(cp, num_seqs, num_layers, B,
                                                       ctypes.byref(nrb), ctypes.byref(ncb),
                                                       ctypes.byref(mx)))
    del keep
    return nrb.value, ncb.value, mx.value


def iamap_layers_workspace_bytes(num_seqs, num_layers, num_rowblocks) -> int:
    return _lib.iamap_layers_workspace_bytes(num_seqs, num_layers, num_rowblocks)


def iamap_compress_layers(q, k, cu_seqlens, cu_seqlens_host, num_seqs, n, num_layers, H_s, d, B,
                          tau, bias_window, bias_value, lse, mass, headmask_dense, row_ptr,
                          col_idx, headmask, val_off, counts, vals, vals_capacity_tiles, ws,
                          stream=None):
    cp, keep = _host_i32(cu_seqlens_host)
    _check("iamap_compress_layers", _lib.iamap_compress_layers(
        _ptr(q), _ptr(k), _ptr(cu_seqlens), cp, num_seqs, n, num_layers, H_s, d, B, tau,
        bias_window, bias_value, _ptr(lse), _ptr(mass), _ptr(headmask_dense), _ptr(row_ptr),
        _ptr(col_idx), _ptr(headmask), _ptr(val_off), _ptr(counts), _ptr(vals),
        vals_capacity_tiles, _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))
    del keep


def iamap_mapped_av_layers(cu_seqlens, cu_seqlens_host, num_seqs, n, num_layers, B, H_s, row_ptr,
                           col_idx, headmask, val_off, vals, vals_capacity_tiles, W, H_r, H_kv, v,
                           d_v, out, ws, stream=None):
    cp, keep = _host_i32(cu_seqlens_host)
    _check("iamap_mapped_av_layers", _lib.iamap_mapped_av_layers(
        _ptr(cu_seqlens), cp, num_seqs, n, num_layers, B, H_s, _ptr(row_ptr), _ptr(col_idx),
        _ptr(headmask), _ptr(val_off), _ptr(vals), vals_capacity_tiles, _ptr(W), H_r, H_kv,
        _ptr(v), d_v, _ptr(out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))
    del keep


def iamap_chunk_plan(cu_q_host, cu_k_host, starts_host, num_seqs, B):
    qp, kq = _host_i32(cu_q_host)
    kp, kk = _host_i32(cu_k_host)
    sp, ks = _host_i32(starts_host)
    nrb, ncb, mx = _I64(0), _I64(0), ctypes.c_int32(0)
    _check("iamap_chunk_plan", _lib.iamap_chunk_plan(qp, kp, sp, num_seqs, B, ctypes.byref(nrb),
                                                     ctypes.byref(ncb), ctypes.byref(mx)))
    del kq, kk, ks
    return nrb.value, ncb.value, mx.value


def iamap_compress_chunk(q, k, cu_q, cu_k, starts, cu_q_host, cu_k_host, starts_host, num_seqs,
                         n_q, n_k, H_s, d, B, tau, bias_window, bias_value, v_s, d_vs, o_s, lse,
                         mass, headmask_dense, row_ptr, col_idx, headmask, val_off, counts, vals,
                         vals_capacity_tiles, ws, stream=None):
    qp, kq = _host_i32(cu_q_host)
    kp, kk = _host_i32(cu_k_host)
    sp, ks = _host_i32(starts_host)
    _check("iamap_compress_chunk", _lib.iamap_compress_chunk(
        _ptr(q), _ptr(k), _ptr(cu_q), _ptr(cu_k), _ptr(starts), qp, kp, sp, num_seqs, n_q, n_k,
        H_s, d, B, tau, bias_window, bias_value, _ptr(v_s), d_vs, _ptr(o_s), _ptr(lse),
        _ptr(mass), _ptr(headmask_dense), _ptr(row_ptr), _ptr(col_idx), _ptr(headmask),
        _ptr(val_off), _ptr(counts), _ptr(vals), vals_capacity_tiles, _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    del kq, kk, ks


def iamap_mapped_av_chunk(cu_q, cu_k, starts, cu_q_host, cu_k_host, starts_host, num_seqs, n_q,
                          n_k, B, H_s, row_ptr, col_idx, headmask, val_off, vals,
                          vals_capacity_tiles, W, H_r, H_kv, v, d_v, out, ws, stream=None):
    qp, kq = _host_i32(cu_q_host)
    kp, kk = _host_i32(cu_k_host)
    sp, ks = _host_i32(starts_host)
    _check("iamap_mapped_av_chunk", _lib.iamap_mapped_av_chunk(
        _ptr(cu_q), _ptr(cu_k), _ptr(starts), qp, kp, sp, num_seqs, n_q, n_k, B, H_s,
        _ptr(row_ptr), _ptr(col_idx), _ptr(headmask), _ptr(val_off), _ptr(vals),
        vals_capacity_tiles, _ptr(W), H_r, H_kv, _ptr(v), d_v, _ptr(out), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    del kq, kk, ks


def iamap_mapped_av_paged_workspace_bytes(batch, H_r, d_v, max_ctx, page_size) -> int:
    return _lib.iamap_mapped_av_paged_workspace_bytes(batch, H_r, d_v, max_ctx, page_size)


def iamap_mapped_av_gqa(cu_seqlens, cu_seqlens_host, num_seqs, n, B, H_s, row_ptr, col_idx,
                        headmask, val_off, vals, vals_capacity_tiles, W, H_r, H_kv, v, d_v, out, ws,
                        stream=None):
    cp, keep = _host_i32(cu_seqlens_host)
    _check("iamap_mapped_av_gqa", _lib.iamap_mapped_av_gqa(
        _ptr(cu_seqlens), cp, num_seqs, n, B, H_s, _ptr(row_ptr), _ptr(col_idx), _ptr(headmask),
        _ptr(val_off), _ptr(vals), vals_capacity_tiles, _ptr(W), H_r, H_kv, _ptr(v), d_v,
        _ptr(out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))
    del keep


def iamap_mapped_av_paged_gqa(p_rows, ctx_stride, W, v_pages, num_pages, page_table, max_pages,
                              page_size, ctx_lens, ctx_lens_host, batch, H_s, H_r, H_kv, d_v, out,
                              ws, stream=None):
    cp, keep = _host_i32(ctx_lens_host)
    _check("iamap_mapped_av_paged_gqa", _lib.iamap_mapped_av_paged_gqa(
        _ptr(p_rows), ctx_stride, _ptr(W), _ptr(v_pages), num_pages, _ptr(page_table), max_pages,
        page_size, _ptr(ctx_lens), cp, batch, H_s, H_r, H_kv, d_v, _ptr(out), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    del keep


def iamap_mapped_av_paged(p_rows, ctx_stride, W, v_pages, num_pages, page_table, max_pages,
                          page_size, ctx_lens, ctx_lens_host, batch, H_s, H_r, d_v, out, ws,
                          stream=None):
    cp, keep = _host_i32(ctx_lens_host)
    _check("iamap_mapped_av_paged", _lib.iamap_mapped_av_paged(
        _ptr(p_rows), ctx_stride, _ptr(W), _ptr(v_pages), num_pages, _ptr(page_table), max_pages,
        page_size, _ptr(ctx_lens), cp, batch, H_s, H_r, d_v, _ptr(out), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    del keep


def iamap_mapped_av_paged_noalloc(p_rows, ctx_stride, W, v_pages, num_pages, page_table,
                                  max_pages, page_size, ctx_lens, ctx_lens_host, batch, H_s, H_r,
                                  d_v, out, stream=None):
    """The decode step without a workspace, for callers that cannot allocate device memory at
    call time (the partial sums live in a fixed 16 MiB array inside the library)."""
    cp, keep = _host_i32(ctx_lens_host)
    _check("iamap_mapped_av_paged_noalloc", _lib.iamap_mapped_av_paged_noalloc(
        _ptr(p_rows), ctx_stride, _ptr(W), _ptr(v_pages), num_pages, _ptr(page_table), max_pages,
        page_size, _ptr(ctx_lens), cp, batch, H_s, H_r, d_v, _ptr(out), _stream(stream)))
    del keep


def iamap_head_match_workspace_bytes(L_s, H_small, L_l, H_large, n_used) -> int:
    return _lib.iamap_head_match_workspace_bytes(L_s, H_small, L_l, H_large, n_used)


IAMAP_SIM_COSINE, IAMAP_SIM_PEARSON, IAMAP_SIM_EUCLIDEAN = 0, 1, 2
SIM_METRICS = {"cosine": IAMAP_SIM_COSINE, "pearson": IAMAP_SIM_PEARSON,
               "euclidean": IAMAP_SIM_EUCLIDEAN}


def iamap_head_match_metric(q_small, k_small, L_s, H_small, d_small, q_large, k_large, L_l,
                            H_large, d_large, n, n_used, metric, argmax, sim, ws, stream=None):
    _check("iamap_head_match_metric", _lib.iamap_head_match_metric(
        _ptr(q_small), _ptr(k_small), L_s, H_small, d_small, _ptr(q_large), _ptr(k_large), L_l,
        H_large, d_large, n, n_used, metric, _ptr(argmax), _ptr(sim), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def iamap_selftest_wait_timeout(limit_us, gave_up, stream=None):
    _check("iamap_selftest_wait_timeout", _lib.iamap_selftest_wait_timeout(
        limit_us, _ptr(gave_up), _stream(stream)))


def iamap_selftest_exp2(x, y_fma, y_mufu, n, stream=None):
    _check("iamap_selftest_exp2", _lib.iamap_selftest_exp2(
        _ptr(x), _ptr(y_fma), _ptr(y_mufu), n, _stream(stream)))


def iamap_mapping_consistency(a, b, n_heads, agree, stream=None):
    _check("iamap_mapping_consistency", _lib.iamap_mapping_consistency(
        _ptr(a), _ptr(b), n_heads, _ptr(agree), _stream(stream)))


def iamap_head_match(q_small, k_small, L_s, H_small, d_small, q_large, k_large, L_l, H_large,
                     d_large, n, n_used, argmax, sim, ws, stream=None):
    _check("iamap_head_match", _lib.iamap_head_match(
        _ptr(q_small), _ptr(k_small), L_s, H_small, d_small, _ptr(q_large), _ptr(k_large), L_l,
        H_large, d_large, n, n_used, _ptr(argmax), _ptr(sim), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def iamap_bsr_check_host(cu_seqlens_host, num_seqs, B, H_s, row_ptr, col_idx, headmask, val_off,
                         vals_capacity_tiles):
    """Host structure check of a block-sparse map (host arrays or CPU tensors). Returns
    (status, first offending block or -1, message); does not raise on an invalid map."""
    def host(a, dtype):
        t = torch.as_tensor(a).cpu().contiguous()
        return t.view(dtype) if t.dtype.itemsize == dtype.itemsize else t.to(dtype)
    cu, _k0 = _host_i32(cu_seqlens_host)
    rp, ci = host(row_ptr, torch.int32), host(col_idx, torch.int32)
    hm, vo = host(headmask, torch.int64), host(val_off, torch.int64)
    bad = _I64(-1)
    rc = _lib.iamap_bsr_check_host(cu, num_seqs, B, H_s, _ptr(rp), _ptr(ci), _ptr(hm), _ptr(vo),
                                   vals_capacity_tiles, ctypes.byref(bad))
    return rc, bad.value, iamap_last_error()


def iamap_prefix_num_keys(cu_seqlens_host, num_seqs, B) -> int:
    cu, _keep = _host_i32(cu_seqlens_host)
    out = _I64(0)
    _check("iamap_prefix_num_keys", _lib.iamap_prefix_num_keys(cu, num_seqs, B,
                                                               ctypes.byref(out)))
    return out.value


def iamap_prefix_keys(tokens, n, cu_seqlens, num_seqs, B, salt, keys, keys_capacity, key_cu,
                      stream=None):
    """keys: a uint64 buffer carried as an int64 tensor (same bits)."""
    _check("iamap_prefix_keys", _lib.iamap_prefix_keys(
        _ptr(tokens), n, _ptr(cu_seqlens), num_seqs, B, int(salt) & (2**64 - 1), _ptr(keys),
        keys_capacity, _ptr(key_cu), _stream(stream)))


def iamap_prefix_index_clear(table_keys, table_vals, capacity, stream=None):
    _check("iamap_prefix_index_clear", _lib.iamap_prefix_index_clear(
        _ptr(table_keys), _ptr(table_vals), capacity, _stream(stream)))


def iamap_prefix_insert(keys, values, count, table_keys, table_vals, capacity, stored,
                        stream=None):
    _check("iamap_prefix_insert", _lib.iamap_prefix_insert(
        _ptr(keys), _ptr(values), count, _ptr(table_keys), _ptr(table_vals), capacity,
        _ptr(stored), _stream(stream)))


def iamap_prefix_lookup(keys, count, key_cu, num_seqs, table_keys, table_vals, capacity, found,
                        hit_blocks, stream=None):
    _check("iamap_prefix_lookup", _lib.iamap_prefix_lookup(
        _ptr(keys), count, _ptr(key_cu), num_seqs, _ptr(table_keys), _ptr(table_vals), capacity,
        _ptr(found), _ptr(hit_blocks), _stream(stream)))


# ------------------------------------------------------------------------------------------------
# Buffer helpers (torch allocations in the documented shapes)
# ------------------------------------------------------------------------------------------------

def alloc_compress_outputs(n, H_s, num_rowblocks, num_causal_blocks, device="cuda"):
    """lse, mass, headmask_dense, row_ptr, col_idx, headmask, val_off, counts."""
    i64 = torch.int64
    return dict(
        lse=torch.empty(H_s, n, dtype=torch.float32, device=device),
        mass=torch.empty(H_s, num_causal_blocks, dtype=torch.float32, device=device),
        headmask_dense=torch.empty(num_causal_blocks, dtype=i64, device=device),
        row_ptr=torch.empty(num_rowblocks + 1, dtype=torch.int32, device=device),
        col_idx=torch.empty(max(num_causal_blocks, 1), dtype=torch.int32, device=device),
        headmask=torch.empty(max(num_causal_blocks, 1), dtype=i64, device=device),
        val_off=torch.empty(max(num_causal_blocks, 1), dtype=i64, device=device),
        counts=torch.zeros(2, dtype=i64, device=device),
    )


def alloc_workspace(nbytes, device="cuda"):
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
