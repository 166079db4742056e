"""Helpers shared by the GPU parity tests: workload upload, readback of the compress outputs,
and the comparison rules (tolerances of the benchmark description)."""

from __future__ import annotations

import os

import numpy as np
import torch

import oracle as O

# Output tolerance: relative Frobenius <= 5e-3 and max abs <= 2e-2 * max|O_ref| (bf16 operands,
# fp32 accumulation).
REL_FRO = 5e-3
MAX_ABS_FRAC = 2e-2
# lse (natural log, fp32 with ex2/lg2.approx): |err| <= 2e-4.
LSE_ATOL = 2e-4
# block masses normalised by the block's rows: |err| <= 2e-5 (fp32 sums of up to 4096 terms).
MASS_NORM_ATOL = 2e-5


def bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def upload_prefill(wl, device="cuda"):
    return (bf16(wl.q, device), bf16(wl.k, device), bf16(wl.v, device),
            torch.from_numpy(wl.W).to(device))


def gpu_kept(layer) -> np.ndarray:
    """[H_s, num_causal_blocks] bool from the dense head masks."""
    hm = layer.bufs["headmask_dense"].cpu().numpy().view(np.uint64)
    sh = np.arange(layer.H_s, dtype=np.uint64)[:, None]
    return ((hm[None, :] >> sh) & np.uint64(1)).astype(bool)


def check_output(o_gpu: np.ndarray, o_ref: np.ndarray, what=""):
    err = o_gpu.astype(np.float64) - o_ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(o_ref), 1e-300)
    mx = np.abs(err).max() / max(np.abs(o_ref).max(), 1e-300)
    assert rel <= REL_FRO, "%s relative Frobenius error %.3e > %.1e" % (what, rel, REL_FRO)
    assert mx <= MAX_ABS_FRAC, "%s max abs error %.3e of max|O| > %.1e" % (what, mx, MAX_ABS_FRAC)
    return rel, mx


def compare_kept(kept_gpu: np.ndarray, kept_ref: np.ndarray, near: np.ndarray, report=True):
    """Bit-exact outside near-threshold blocks; returns the number of (near-threshold) flips.
    The counts of compared, near and flipped blocks go to the end-of-run report."""
    diff = kept_gpu != kept_ref
    bad = diff & ~near
    assert not bad.any(), "kept sets differ outside near-threshold blocks at %s" % (
        list(zip(*np.nonzero(bad)))[:10],)
    flips = int(diff.sum())
    if report:
        import conftest
        name = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
        conftest.KEPT_REPORT.append((name, int(kept_ref.size), int(near.sum()), flips))
    return flips


def check_kept_invariants(kept, mass_norm, tau, eps=1e-5):
    """The cumulative-mass choice of every (head, row block), checked on a kept set with the
    given normalised masses [H, blocks of the row block]: the kept mass reaches tau, dropping the
    smallest kept block falls below it, and no dropped block outweighs a kept one."""
    if tau >= 1.0:
        assert kept.all()
        return
    km = (mass_norm * kept).sum(axis=1)
    assert (km >= tau - eps).all(), "kept mass below tau: %s" % (km.min(),)
    mn = np.where(kept, mass_norm, np.inf).min(axis=1)
    assert (km - mn < tau + eps).all(), "kept set is not minimal"
    mx = np.where(~kept, mass_norm, -np.inf).max(axis=1)
    assert (mx <= mn + eps).all(), "a dropped block outweighs a kept one"


def bsr_readback(layer):
    b = layer.bufs
    nnz, tiles = layer.counts()
    row_ptr = b["row_ptr"].cpu().numpy()
    col_idx = b["col_idx"].cpu().numpy()[:nnz]
    headmask = b["headmask"].cpu().numpy().view(np.uint64)[:nnz]
    val_off = b["val_off"].cpu().numpy()[:nnz]
    return row_ptr, col_idx, headmask, val_off, tiles


def head_tile(vals, val_off_u, k, rank):
    """[64, 64] tile of head rank `rank` in a stored block of k present heads: the block's values
    are interleaved by row, row i of rank t at line i * k + t."""
    blk = vals[int(val_off_u) * 64:(int(val_off_u) + k) * 64]
    return blk.reshape(64, k, 64)[:, rank, :]


def check_bsr_structure(layer, kept_gpu, lay):
    """The union index the GPU wrote equals the union of its own per-head kept sets."""
    row_ptr, col_idx, headmask, val_off, tiles = bsr_readback(layer)
    r_ref, c_ref, h_ref, v_ref, t_ref = O.union_bsr(kept_gpu, lay)
    np.testing.assert_array_equal(row_ptr, r_ref)
    np.testing.assert_array_equal(col_idx, c_ref)
    np.testing.assert_array_equal(headmask, h_ref)
    np.testing.assert_array_equal(val_off, v_ref)
    assert tiles == t_ref
    return row_ptr, col_idx, headmask, val_off
