"""GPU parity of several mapped layer pairs in one launch per stage (iamap_compress_layers,
iamap_mapped_av_layers) through the C ABI: every layer's results equal the single-layer calls on
that layer's tensors bit for bit, and the float64 oracle of each layer within the tolerances."""

import numpy as np
import pytest
import torch

import oracle as O
from synth import make_prefill

from _gpu_common import bf16, check_output, compare_kept

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("seqlens,H_s,H_r,H_kv,d,tau,bias", [
    ([300, 70, 1], 5, 14, 14, 64, 0.9, (0, 0.0)),      # tensor-core mapped_av (4-CTA clusters)
    ([260, 90], 4, 40, 8, 64, 0.9, (0, 0.0)),          # H_r > 32: the CUDA-core mapped_av
    ([500], 6, 8, 8, 128, 0.95, (128, 2.0)),           # d = 128, local bias, CUDA-core mapped_av
])
def test_layers_in_one_launch(seqlens, H_s, H_r, H_kv, d, tau, bias):
    from cross_model_attention_map_b200 import iamap as C
    from cross_model_attention_map_b200.runner import PrefillLayer
    L = 3
    wls = [make_prefill(seqlens, H_s=H_s, d=d, H_r=H_r, d_v=d, B=64, tau=tau, std=1.5,
                        sink=True, bias_window=bias[0], bias_value=bias[1], seed=90 + l,
                        H_kv=H_kv) for l in range(L)]
    n, S = wls[0].n, len(seqlens)
    q = bf16(np.concatenate([w.q for w in wls]))
    k = bf16(np.concatenate([w.k for w in wls]))
    v = bf16(np.concatenate([w.v for w in wls]))
    W = torch.from_numpy(np.stack([w.W for w in wls])).cuda()
    cu_host = wls[0].cu_seqlens
    cu = torch.from_numpy(cu_host).cuda()
    nrb, ncb, _ = C.iamap_layers_plan(cu_host, S, L, 64)
    one_nrb, one_ncb, _ = C.iamap_plan(cu_host, S, 64)
    assert (nrb, ncb) == (L * one_nrb, L * one_ncb)
    bufs = C.alloc_compress_outputs(L * n, H_s, nrb, ncb)
    cap = H_s * ncb
    vals = torch.empty(cap, 64, 64, dtype=torch.bfloat16, device="cuda")
    ws = C.alloc_workspace(C.iamap_layers_workspace_bytes(S, L, nrb))
    out = torch.empty(L * n, H_r, d, dtype=torch.float32, device="cuda")
    C.iamap_compress_layers(q, k, cu, cu_host, S, n, L, H_s, d, 64, tau, bias[0], bias[1],
                            bufs["lse"], bufs["mass"], bufs["headmask_dense"], bufs["row_ptr"],
                            bufs["col_idx"], bufs["headmask"], bufs["val_off"], bufs["counts"],
                            vals, cap, ws)
    C.iamap_mapped_av_layers(cu, cu_host, S, n, L, 64, H_s, bufs["row_ptr"], bufs["col_idx"],
                             bufs["headmask"], bufs["val_off"], vals, cap, W, H_r, H_kv, v, d,
                             out, ws)
    torch.cuda.synchronize()
    assert C.iamap_device_status() == 0
    hm = bufs["headmask_dense"].cpu().numpy().view(np.uint64)
    kept_all = ((hm[None, :] >> np.arange(H_s, dtype=np.uint64)[:, None]) & np.uint64(1)).astype(bool)
    for l, w in enumerate(wls):
        single = PrefillLayer(w.seqlens, H_s, d, H_r, d, tau, bias[0], bias[1], H_kv=H_kv)
        single.step(bf16(w.q), bf16(w.k), torch.from_numpy(w.W).cuda(), bf16(w.v))
        torch.cuda.synchronize()
        rows = slice(l * n, (l + 1) * n)
        blocks = slice(l * one_ncb, (l + 1) * one_ncb)
        assert torch.equal(bufs["lse"][:, rows], single.bufs["lse"])
        assert torch.equal(bufs["mass"][:, blocks], single.bufs["mass"])
        assert torch.equal(bufs["headmask_dense"][blocks], single.bufs["headmask_dense"])
        assert torch.equal(out[rows], single.out)
        ref = O.compress(w)
        kept = kept_all[:, blocks]
        compare_kept(kept, ref.kept, ref.near)
        check_output(out[rows].cpu().numpy(), O.mapped_av(w, kept), "layer %d" % l)
