"""The host structure check of block-sparse maps (no GPU): maps built by the oracle pass; each
kind of corruption is reported at the first offending block."""

import numpy as np
import pytest

import oracle as O
from synth import make_prefill


@pytest.fixture(scope="module")
def lib():
    from cross_model_attention_map_b200 import build
    build.build()
    from cross_model_attention_map_b200 import iamap
    return iamap


@pytest.fixture(scope="module")
def bsr():
    wl = make_prefill([150, 64, 0, 90], H_s=3, d=16, H_r=2, d_v=8, B=64, tau=0.9, seed=13)
    res = O.compress(wl)
    row_ptr, col_idx, headmask, val_off, tiles = O.union_bsr(res.kept, res.layout)
    return wl, row_ptr, col_idx, headmask, val_off, tiles


def _check(lib, wl, rp, ci, hm, vo, cap):
    return lib.iamap_bsr_check_host(wl.cu_seqlens, len(wl.seqlens), wl.B, wl.H_s, rp, ci,
                                    hm.view(np.int64), vo, cap)


def test_oracle_maps_pass(lib, bsr):
    wl, rp, ci, hm, vo, tiles = bsr
    assert len(ci) > 0
    assert _check(lib, wl, rp, ci, hm, vo, tiles)[:2] == (0, -1)
    # keep-all maps of a ragged batch pass too
    wl1 = make_prefill([65, 1, 200], H_s=64, d=16, H_r=1, d_v=8, B=64, tau=1.0, seed=14)
    r1 = O.compress(wl1)
    rp1, ci1, hm1, vo1, t1 = O.union_bsr(r1.kept, r1.layout)
    assert int(hm1[0]) == 2**64 - 1
    assert _check(lib, wl1, rp1, ci1, hm1, vo1, t1)[:2] == (0, -1)


@pytest.mark.parametrize("what", ["row_ptr", "col_range", "col_order", "mask_zero", "mask_bits",
                                  "val_neg", "val_cap"])
def test_corruptions_are_reported(lib, bsr, what):
    wl, rp, ci, hm, vo, tiles = bsr
    rp, ci, hm, vo = rp.copy(), ci.copy(), hm.copy(), vo.copy()
    cap = tiles
    # the first row block of sequence 0 that stores two or more blocks (its local index is I)
    I = next(i for i in range(3) if int(rp[i + 1]) - int(rp[i]) >= 2)
    first = int(rp[I])
    if what == "row_ptr":
        rp[I + 1] = rp[I] - 1
        b = -1
    elif what == "col_range":
        ci[first] = I + 1      # row block I may only reach column block I
        b = first
    elif what == "col_order":
        ci[first], ci[first + 1] = ci[first + 1], ci[first]
        b = first + 1
    elif what == "mask_zero":
        hm[first] = 0
        b = first
    elif what == "mask_bits":
        hm[first] |= np.uint64(1 << 3)   # head 3 of 3
        b = first
    elif what == "val_neg":
        vo[first] = -1
        b = first
    else:
        cap = tiles - 1        # the last block's last tile no longer fits
        b = len(ci) - 1
    rc, bad, msg = _check(lib, wl, rp, ci, hm, vo, cap)
    assert rc == (-3 if what == "val_cap" else -1), (rc, msg)
    assert msg
    if b >= 0:
        assert bad == b, (bad, b, msg)


def test_bad_arguments(lib, bsr):
    wl, rp, ci, hm, vo, tiles = bsr
    assert lib.iamap_bsr_check_host(wl.cu_seqlens, 4, 64, 65, rp, ci, hm.view(np.int64), vo,
                                    tiles)[0] == -1
    assert lib.iamap_bsr_check_host(wl.cu_seqlens, 4, 64, 3, rp, ci, hm.view(np.int64), vo,
                                    -1)[0] == -1
    bad_rp = rp.copy()
    bad_rp[0] = 1
    assert lib.iamap_bsr_check_host(wl.cu_seqlens, 4, 64, 3, bad_rp, ci, hm.view(np.int64), vo,
                                    tiles)[0] == -1
