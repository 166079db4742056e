"""The allocation-free decode entry point (iamap_mapped_av_paged_noalloc).

Some callers cannot allocate device memory when they call the library: a serving engine that
reserved nearly all GPU memory for its KV cache at start-up, or one that forbids cudaMalloc on
its decode loop because it synchronises the device. For them the library keeps the decode
kernel's partial sums in a fixed device array instead of a caller workspace. This test calls that
entry point through the C ABI twice in a row (different inputs, so stale contents of the shared
array would show) and checks each result against the float64 oracle of the paged decode and against
iamap_mapped_av_paged with a workspace, within the output tolerance of the other parity tests. The
file is named to be collected last.
"""

import numpy as np
import pytest
import torch

import oracle as O
from synth import make_decode

from _gpu_common import bf16, check_output

pytestmark = pytest.mark.gpu


def _inputs(dw):
    return (torch.from_numpy(dw.p_rows).cuda(), torch.from_numpy(dw.W).cuda(), bf16(dw.v_pages),
            torch.from_numpy(dw.page_table).cuda(),
            torch.from_numpy(dw.ctx_lens).cuda())


def _with_workspace(C, dw, p, W, vp, pt, cl):
    out = torch.empty(dw.batch, dw.H_r, dw.d_v, dtype=torch.float32, device="cuda")
    ws = C.alloc_workspace(C.iamap_mapped_av_paged_workspace_bytes(
        dw.batch, dw.H_r, dw.d_v, int(dw.ctx_lens.max()), dw.page_size))
    C.iamap_mapped_av_paged(p, dw.p_rows.shape[2], W, vp, dw.v_pages.shape[0], pt,
                            dw.page_table.shape[1], dw.page_size, cl, dw.ctx_lens, dw.batch,
                            dw.H_s, dw.H_r, dw.d_v, out, ws)
    return out


def _no_alloc(C, dw, p, W, vp, pt, cl):
    out = torch.empty(dw.batch, dw.H_r, dw.d_v, dtype=torch.float32, device="cuda")
    C.iamap_mapped_av_paged_noalloc(p, dw.p_rows.shape[2], W, vp, dw.v_pages.shape[0], pt,
                                    dw.page_table.shape[1], dw.page_size, cl, dw.ctx_lens,
                                    dw.batch, dw.H_s, dw.H_r, dw.d_v, out)
    return out


def test_no_alloc_decode_matches_oracle_and_workspace_entry_point():
    from cross_model_attention_map_b200 import iamap as C
    cases = [make_decode(seed=41),                                     # batch 4, context 8704
             make_decode(batch=3, ctx=500, H_s=5, H_r=16, d_v=128, page_size=16,
                         ctx_lens=[500, 37, 260], seed=42)]
    for dw in cases:                                                   # two calls in a row
        args = _inputs(dw)
        got = _no_alloc(C, dw, *args)
        ref = _with_workspace(C, dw, *args)
        torch.cuda.synchronize()
        check_output(got.cpu().numpy(), O.mapped_av_paged(dw), "no-alloc decode vs oracle")
        check_output(got.cpu().numpy(), ref.cpu().numpy().astype(np.float64), "no-alloc decode")


def test_no_alloc_rejects_oversized_split():
    """64 sequences of 4096 tokens with 128 receiver heads of 128 dims need more split partial sums
    than the fixed array holds: refused on the host, before any launch (the small tensors passed
    here are never read)."""
    from cross_model_attention_map_b200 import iamap as C
    batch, ctx, ps, H_r, d_v = 64, 4096, 16, 128, 128
    dummy = torch.zeros(64, dtype=torch.float32, device="cuda")
    vp = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    pt = torch.zeros(64, dtype=torch.int32, device="cuda")
    out = torch.empty(64, dtype=torch.float32, device="cuda")
    with pytest.raises(C.IamapError) as e:
        C.iamap_mapped_av_paged_noalloc(dummy, ctx, dummy, vp, batch * ctx // ps, pt, ctx // ps,
                                        ps, pt, [ctx] * batch, batch, 2, H_r, d_v, out)
    assert e.value.code == -3
    assert "16777216" in C.iamap_last_error()
