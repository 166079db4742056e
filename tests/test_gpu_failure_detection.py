"""Failure detection on the GPU without a fault: a bounded mbarrier wait that nothing completes
gives up after its limit, raises IAMAP_DEV_TIMEOUT in the device status (read on the host), and
leaves the context usable."""

import time

import numpy as np
import pytest
import torch

import oracle as O
from synth import make_decode

from _gpu_common import bf16, check_output

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C():
    from cross_model_attention_map_b200 import iamap
    return iamap


def test_bounded_wait_gives_up_and_reports(C):
    assert C.iamap_device_status() == 0
    gave_up = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.time()
    C.iamap_selftest_wait_timeout(20000, gave_up)     # 20 ms limit
    torch.cuda.synchronize()
    assert time.time() - t0 < 5.0
    assert int(gave_up.item()) == 1
    st = C.iamap_device_status()
    assert st & C.IAMAP_DEV_TIMEOUT
    assert C.iamap_device_status() == 0                 # the read clears it
    # the context still runs kernels correctly
    from cross_model_attention_map_b200.runner import DecodeStep
    dw = make_decode(batch=2, ctx=100, H_s=3, H_r=8, d_v=64, page_size=16, seed=61)
    step = DecodeStep(dw.batch, dw.H_s, dw.H_r, dw.d_v, dw.ctx_lens, dw.p_rows.shape[2],
                      dw.page_table.shape[1], dw.page_size, dw.v_pages.shape[0])
    out = step.run(torch.from_numpy(dw.p_rows).cuda(), torch.from_numpy(dw.W).cuda(),
                   bf16(dw.v_pages), torch.from_numpy(dw.page_table).cuda())
    torch.cuda.synchronize()
    check_output(out.cpu().numpy(), O.mapped_av_paged(dw), "decode after a timeout")
    assert C.iamap_device_status() == 0


def test_selftest_rejects_bad_limits(C):
    gave_up = torch.zeros(1, dtype=torch.int32, device="cuda")
    for bad in (0, -5, 2_000_000):
        with pytest.raises(C.IamapError):
            C.iamap_selftest_wait_timeout(bad, gave_up)
