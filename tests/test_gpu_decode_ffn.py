"""moe_expert_ffn at decode sizes, on the GPU against the fp64 oracle.

At 1 <= T <= 4 tokens (H and I multiples of 256 up to 2048) the standalone
expert call runs the fused decode kernel's expert phases on the routing it
is given (the dispatch arrays): streamed int4/int2/int8 weights, mma.sync on
dequantised fragments, every dispatched row's output rounded once to bf16.
These cases run it at the full decode shapes (512 experts, top-10, H = 2048,
I = 768) for one token and for a four-token verification batch, compare
every row with the oracle's expert rows, and check that inconsistent
dispatch counts are refused on the device with MOE_ERR_DEVICE_FAULT and no
row written.
"""
import numpy as np
import pytest

import oracle
from bit_quantized_moe_gemv_b200 import workload as wlm
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_quantized_moe_gemv_b200 import build
    build.build()
    from bit_quantized_moe_gemv_b200 import _lib
    return _lib


def _route_dispatch(L, wl, dev, xb, bias, stride, ws):
    import torch
    from bit_quantized_moe_gemv_b200.device import bf16_tensor
    T, k, E = wl.T, wl.k, wl.E
    x = bf16_tensor(xb)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    L.route(x, dev["w_router"], pu.bias_tensor(bias), stride, k, idx, w, ws)
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    L.dispatch(idx, E, counts, offsets, perm, inv, ws)
    return x, idx, counts, offsets, perm


@pytest.mark.parametrize("name", ["decode1", "verify4"])
def test_expert_ffn_decode_rows_match_oracle(L, name):
    import torch
    from bit_quantized_moe_gemv_b200.device import bf16_bits
    wl = wlm.WORKLOADS[name]
    lay = wlm.gen_layer(wl)
    dev = pu.upload_layer(lay)
    bias, stride = wlm.gen_bias(wl)
    ws = L.new_workspace(wl.T, wl.H, wl.I, wl.E, wl.k)
    for step in range(3):
        xb = wlm.gen_x(wl, step=step)
        x, idx, counts, offsets, perm = _route_dispatch(L, wl, dev, xb, bias, stride, ws)
        y = torch.empty((wl.T * wl.k, wl.H), dtype=torch.bfloat16, device="cuda")
        L.expert_ffn(x, wl.I, wl.k, wl.E, perm, offsets, counts, dev["experts"].table, y, ws)
        torch.cuda.synchronize()
        assert L.get_status(ws) == 0
        y_ref = oracle.expert_rows(xb, perm.cpu().numpy(), offsets.cpu().numpy(), wl.k, lay.experts)
        pu.assert_close(pu.bf16_to_f64(bf16_bits(y)), y_ref, f"{name} step {step} y_perm")


def test_expert_ffn_decode_bad_counts_flag_fault(L):
    import torch
    from bit_quantized_moe_gemv_b200.device import bf16_bits
    wl = wlm.WORKLOADS["decode1"]
    lay = wlm.gen_layer(wl)
    dev = pu.upload_layer(lay)
    bias, stride = wlm.gen_bias(wl)
    ws = L.new_workspace(wl.T, wl.H, wl.I, wl.E, wl.k)
    xb = wlm.gen_x(wl)
    x, idx, counts, offsets, perm = _route_dispatch(L, wl, dev, xb, bias, stride, ws)
    torch.cuda.synchronize()
    # one expert claims more rows than there are tokens: refused on the device
    bad = counts.clone()
    bad[int(torch.nonzero(counts == 0)[0])] = wl.T + 1
    y = torch.full((wl.T * wl.k, wl.H), 7.0, dtype=torch.bfloat16, device="cuda")
    before = bf16_bits(y)
    L.expert_ffn(x, wl.I, wl.k, wl.E, perm, offsets, bad, dev["experts"].table, y, ws)
    torch.cuda.synchronize()
    assert L.get_status(ws) == 5
    np.testing.assert_array_equal(bf16_bits(y), before)
