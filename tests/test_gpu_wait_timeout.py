"""A bounded device wait that runs out, on the GPU, through the C ABI.

Every wait of the fused decode launch (the grid counter on the logits, each
expert's readiness counter) has a cycle budget. moe_set_wait_cycles(0) makes
any wait that is not met at its first check give up: the launch must end on
its own (no hang, no fault), leave MOE_ERR_TIMEOUT in the workspace's status
word, and leave the workspace's counters clear, so that after
moe_reset_status and the default budget the next call on the same workspace
matches the oracle. The failure is made without faulting the GPU: nothing
but the budget changes.
"""
import numpy as np
import pytest

import oracle
from bit_quantized_moe_gemv_b200 import workload as wlm
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

MOE_ERR_TIMEOUT = 6


def test_expired_wait_reports_timeout_then_next_call_matches_oracle():
    import torch
    assert torch.cuda.is_available()
    from bit_quantized_moe_gemv_b200 import _lib as L
    from bit_quantized_moe_gemv_b200.device import bf16_bits, bf16_tensor

    wl = wlm.Workload("wait_budget", T=2, H=1024, I=512, E=64, k=6, zipf_s=1.1, seed=21)
    lay = wlm.gen_layer(wl)
    dev = pu.upload_layer(lay)
    bias, stride = wlm.gen_bias(wl)
    b = pu.bias_tensor(bias)
    xb = wlm.gen_x(wl)
    x = bf16_tensor(xb)
    ws = L.new_workspace(wl.T, wl.H, wl.I, wl.E, wl.k)
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")

    def call():
        L.layer(x, wl.I, wl.E, wl.k, dev["w_router"], b, stride, dev["experts"].table, dev["shared"].table, idx, w,
                out, ws)
        torch.cuda.synchronize()

    prev = L.set_wait_cycles(0)
    try:
        call()  # the host call itself succeeds: the failure is reported by the device
        assert L.get_status(ws) == MOE_ERR_TIMEOUT
    finally:
        assert L.set_wait_cycles(-1) == 0
    assert L.set_wait_cycles(-1) == prev  # the default is back
    L.reset_status(ws)
    out.zero_()
    call()
    assert L.get_status(ws) == 0
    gi, gw = idx.cpu().numpy(), w.cpu().numpy()
    ref = oracle.moe_layer(xb, lay.w_router, bias, wl.k, lay.experts, lay.shared)
    np.testing.assert_array_equal(gi, ref["idx"])
    np.testing.assert_allclose(gw, ref["w"], rtol=1e-5, atol=1e-6)
    pu.assert_close(pu.bf16_to_f64(bf16_bits(out)), ref["out"], "after an expired wait")
