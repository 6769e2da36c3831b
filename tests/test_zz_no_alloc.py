"""moe_layer_decode_noalloc against moe_layer and the oracle, through the C ABI.

The no-allocation entry point serves callers that cannot allocate device
memory themselves: a host that owns every allocation and hands a kernel
library only inputs and outputs (a plugin slot in another runtime, a process
held to a fixed device-memory budget). It runs the same fused decode kernel
as moe_layer with its scratch in a device array inside the library, so on
the same inputs its outputs must be bit-identical to moe_layer's, on two
calls in a row (the second call reuses the array the first one left behind).
One call is also checked against the fp64 oracle. This file is collected
last on purpose.
"""
import numpy as np
import pytest

import oracle
from bit_quantized_moe_gemv_b200 import workload as wlm
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


def test_noalloc_matches_moe_layer_two_calls():
    import torch
    assert torch.cuda.is_available()
    from bit_quantized_moe_gemv_b200 import _lib as L
    from bit_quantized_moe_gemv_b200.device import bf16_bits, bf16_tensor

    wl = wlm.Workload("noalloc_decode", T=3, H=1024, I=512, E=64, k=8, zipf_s=1.1, seed=11,
                      routed_qtypes=((0, 32, wlm.Q_INT4_SYM_G32), (32, None, wlm.Q_INT2_ASYM_G16)),
                      shared_qtype=wlm.Q_INT8_PER_CHANNEL)
    lay = wlm.gen_layer(wl)
    dev = pu.upload_layer(lay)
    bias, stride = wlm.gen_bias(wl)
    b = pu.bias_tensor(bias)
    ws = L.new_workspace(wl.T, wl.H, wl.I, wl.E, wl.k)

    def buffers():
        return (torch.full((wl.T, wl.k), -1, dtype=torch.int32, device="cuda"),
                torch.full((wl.T, wl.k), -1.0, dtype=torch.float32, device="cuda"),
                torch.full((wl.T, wl.E), -1.0, dtype=torch.float32, device="cuda"),
                torch.zeros((wl.T, wl.H), dtype=torch.bfloat16, device="cuda"))

    for step in range(2):
        xb = wlm.gen_x(wl, step=step)
        x = bf16_tensor(xb)
        r_idx, r_w, r_lg, r_out = buffers()
        L.layer(x, wl.I, wl.E, wl.k, dev["w_router"], b, stride, dev["experts"].table, dev["shared"].table,
                r_idx, r_w, r_out, ws, logits=r_lg)
        idx, w, lg, out = buffers()
        L.layer_decode_noalloc(x, wl.I, wl.E, wl.k, dev["w_router"], b, stride, dev["experts"].table,
                               dev["shared"].table, idx, w, out, logits=lg)
        torch.cuda.synchronize()
        assert L.get_status(ws) == 0  # moe_layer's own status word (the no-alloc one lives in the library)
        # the same kernel on the same inputs: every output bit for bit
        np.testing.assert_array_equal(idx.cpu().numpy(), r_idx.cpu().numpy())
        np.testing.assert_array_equal(w.cpu().numpy().view(np.uint32), r_w.cpu().numpy().view(np.uint32))
        np.testing.assert_array_equal(lg.cpu().numpy().view(np.uint32), r_lg.cpu().numpy().view(np.uint32))
        np.testing.assert_array_equal(bf16_bits(out), bf16_bits(r_out))
        if step == 1:
            # and against the oracle: routing exactly (on the device's fp32
            # logits; against the fp64 logits outside near-ties), outputs
            # within the float tolerance
            gi, gw = idx.cpu().numpy(), w.cpu().numpy()
            pu.check_routing(gi, gw, lg.cpu().numpy(), xb, lay.w_router, bias, wl.k)
            ref = oracle.moe_layer(xb, lay.w_router, bias, wl.k, lay.experts, lay.shared,
                                   routing=(gi, pu.oracle_gates_for(oracle.router_logits(xb, lay.w_router, bias), gi)))
            pu.assert_close(pu.bf16_to_f64(bf16_bits(out)), ref["out"], "no-alloc out vs oracle")


def test_noalloc_rejects_sizes_beyond_its_limits():
    from bit_quantized_moe_gemv_b200 import _lib as L
    lib = L.LIB
    # T = 5 exceeds the 4-token limit; E = 2048 and k = 17 exceed theirs.
    args = (None, None, 0, None, None, None, None, None, None, None, None)
    assert lib.moe_layer_decode_noalloc(None, 5, 1024, 512, 64, 8, *args) == 2
    assert lib.moe_layer_decode_noalloc(None, 1, 1024, 512, 2048, 8, *args) == 2
    assert lib.moe_layer_decode_noalloc(None, 1, 1024, 512, 64, 17, *args) == 2
