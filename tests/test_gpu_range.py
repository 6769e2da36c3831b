"""Activations outside the fp16 range, on the GPU against the fp64 oracle.

The tensor-core operands are fp16, whose range ends at 65504, while the bf16
activations the boundary accepts reach about 3e38. Every path therefore
scales its fp16 operands by exact powers of two and undoes the scaling on
the fp32 results: the fused decode kernel per token for x and per expert and
token for the SwiGLU output h (from its largest |h|), the tcgen05 prefill
path per row for x and by a matching factor for h, and the general kernels
compute in fp32 throughout. Inputs: N(0, 300^2) activations with a few
+-1e4 outlier channels per token (h then reaches ~1e6, far beyond fp16), and
the same pattern scaled to 1e6 (x itself beyond fp16). Outputs must meet the
same tolerance as ordinary inputs.
"""
import numpy as np
import pytest

import oracle
from bit_quantized_moe_gemv_b200 import workload as wlm
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

CASES = {
    "fused_int4_T2": wlm.Workload("rng_fused_T2", T=2, H=1024, I=512, E=64, k=6, zipf_s=1.1, seed=51),
    "fused_int2_int8_T4": wlm.Workload("rng_fused_T4", T=4, H=1024, I=512, E=32, k=4, zipf_s=0.8, seed=52,
                                       routed_qtypes=((0, None, wlm.Q_INT2_ASYM_G16),),
                                       shared_qtype=wlm.Q_INT8_PER_CHANNEL),
    "tc_mixed_T300": wlm.Workload("rng_tc", T=300, H=512, I=256, E=16, k=4, zipf_s=1.0, seed=53,
                                  routed_qtypes=((0, 6, wlm.Q_INT4_SYM_G32), (6, 11, wlm.Q_INT2_ASYM_G16),
                                                 (11, None, wlm.Q_INT8_PER_CHANNEL)),
                                  shared_qtype=wlm.Q_INT8_PER_CHANNEL),
    "general_T37": wlm.Workload("rng_general", T=37, H=192, I=128, E=24, k=3, seed=54),
}


@pytest.fixture(scope="module")
def L():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_quantized_moe_gemv_b200 import build
    build.build()
    from bit_quantized_moe_gemv_b200 import _lib
    return _lib


def _large_x(wl, scale):
    rng = np.random.default_rng(7000 + wl.seed)
    x = rng.standard_normal((wl.T, wl.H)) * 300.0
    for t in range(wl.T):
        ch = rng.choice(wl.H, 4, replace=False)
        x[t, ch] = rng.choice([-1.0, 1.0], 4) * 1e4
    return wlm.f32_to_bf16_bits((x * (scale / 300.0)).astype(np.float32))


@pytest.mark.parametrize("scale", [300.0, 1e6], ids=["n300_outliers1e4", "n1e6_outliers3e7"])
@pytest.mark.parametrize("case", list(CASES))
def test_large_activations_match_oracle(L, case, scale):
    import torch

    from bit_quantized_moe_gemv_b200.device import bf16_bits, bf16_tensor
    wl = CASES[case]
    lay = wlm.gen_layer(wl)
    dev = pu.upload_layer(lay)
    bias, stride = wlm.gen_bias(wl)
    xb = _large_x(wl, scale)
    x = bf16_tensor(xb)
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    lg = torch.empty((wl.T, wl.E), dtype=torch.float32, device="cuda")
    out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    ws = L.new_workspace(wl.T, wl.H, wl.I, wl.E, wl.k)
    L.layer(x, wl.I, wl.E, wl.k, dev["w_router"], pu.bias_tensor(bias), stride, dev["experts"].table,
            dev["shared"].table, idx, w, out, ws, logits=lg)
    torch.cuda.synchronize()
    assert L.get_status(ws) == 0
    gi, gw = idx.cpu().numpy(), w.cpu().numpy()
    pu.check_routing(gi, gw, lg.cpu().numpy(), xb, lay.w_router, bias, wl.k)
    ref = oracle.moe_layer(xb, lay.w_router, bias, wl.k, lay.experts, lay.shared,
                           routing=(gi, pu.oracle_gates_for(oracle.router_logits(xb, lay.w_router, bias), gi)))
    got = pu.bf16_to_f64(bf16_bits(out))
    assert np.all(np.isfinite(got))
    pu.assert_close(got, ref["out"], f"{case} x{scale:g}")
    if case == "tc_mixed_T300":
        # the four-call path too: moe_expert_ffn's bf16 rows on the same routing
        E, k, H = wl.E, wl.k, wl.H
        counts = torch.empty(E, dtype=torch.int32, device="cuda")
        offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        perm = torch.empty(wl.T * k, dtype=torch.int32, device="cuda")
        inv = torch.empty(wl.T * k, dtype=torch.int32, device="cuda")
        L.dispatch(idx, E, counts, offsets, perm, inv, ws)
        y = torch.empty((wl.T * k, H), dtype=torch.bfloat16, device="cuda")
        L.expert_ffn(x, wl.I, k, E, perm, offsets, counts, dev["experts"].table, y, ws)
        torch.cuda.synchronize()
        assert L.get_status(ws) == 0
        y_ref = oracle.expert_rows(xb, perm.cpu().numpy(), offsets.cpu().numpy(), k, lay.experts)
        pu.assert_close(pu.bf16_to_f64(bf16_bits(y)), y_ref, f"{case} y_perm x{scale:g}")
