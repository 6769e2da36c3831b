"""Routing heat statistics on the GPU, through the C ABI.

The cycleuser.org page "本地部署Qwen3.8-Flash-Next模型的两条路线…", section
"硬件形态决定了各自的走法", ranks experts by routing heat to choose which to
cache. Here moe_options.heat (device uint32 [E]) accumulates how often each
expert was picked over calls; every routing call adds its T k picks. The
counts are integer atomics, so they must equal a host bincount of the
returned indices exactly, on the fused decode kernel over many steps, on the
prefill path and on moe_route alone.
"""
import numpy as np
import pytest

from bit_quantized_moe_gemv_b200 import workload as wlm
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


def _run(case, steps):
    import torch

    from bit_quantized_moe_gemv_b200 import _lib as L
    from bit_quantized_moe_gemv_b200.device import bf16_tensor
    wl = case
    lay = wlm.gen_layer(wl)
    dev = pu.upload_layer(lay)
    bias, stride = wlm.gen_bias(wl)
    b = pu.bias_tensor(bias)
    ws = L.new_workspace(wl.T, wl.H, wl.I, wl.E, wl.k)
    heat = torch.zeros(wl.E, dtype=torch.int32, device="cuda")
    picks = []
    for s in range(steps):
        x = bf16_tensor(wlm.gen_x(wl, step=s))
        idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
        w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
        out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
        L.layer(x, wl.I, wl.E, wl.k, dev["w_router"], b, stride, dev["experts"].table, dev["shared"].table, idx, w,
                out, ws, heat=heat)
        picks.append(idx.cpu().numpy().ravel())
        # the same routing again through moe_route: its picks count as well
        idx2 = torch.empty_like(idx)
        L.route(x, dev["w_router"], b, stride, wl.k, idx2, w, ws, heat=heat)
        picks.append(idx2.cpu().numpy().ravel())
    torch.cuda.synchronize()
    assert L.get_status(ws) == 0
    return heat.cpu().numpy(), np.bincount(np.concatenate(picks), minlength=wl.E)


def test_heat_counts_on_the_fused_decode_path():
    got, ref = _run(wlm.Workload("heat_decode", T=2, H=1024, I=512, E=64, k=6, zipf_s=1.1, seed=61), steps=25)
    np.testing.assert_array_equal(got, ref)
    assert got.sum() == 25 * 2 * 2 * 6


def test_heat_counts_on_the_prefill_path():
    got, ref = _run(wlm.Workload("heat_prefill", T=300, H=512, I=256, E=128, k=4, zipf_s=0.9, seed=62), steps=2)
    np.testing.assert_array_equal(got, ref)
