"""moe_layer_decode_noalloc against moe_layer, through the C ABI.

The no-allocation entry point serves callers whose host code cannot allocate
device memory (a host that owns every allocation and passes only inputs and
outputs): it runs the fused decode step with scratch kept in a device array
inside the library. Its output must match moe_layer's on the same inputs, on
two calls in a row (the second call reuses the array the first one left
behind). This file is collected last on purpose.
"""
import numpy as np
import pytest

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
    for step in range(2):
        x = bf16_tensor(wlm.gen_x(wl, step=step))
        ref_idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
        ref_w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
        ref_out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
        L.layer(x, wl.I, wl.E, wl.k, dev["w_router"], b, stride, dev["experts"].table, dev["shared"].table,
                ref_idx, ref_w, ref_out, ws)
        idx = torch.full((wl.T, wl.k), -1, dtype=torch.int32, device="cuda")
        w = torch.zeros((wl.T, wl.k), dtype=torch.float32, device="cuda")
        out = torch.zeros((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
        L.layer_decode_noalloc(x, wl.I, wl.E, wl.k, dev["w_router"], b, stride, dev["experts"].table,
                               dev["shared"].table, idx, w, out)
        torch.cuda.synchronize()
        assert L.get_status(ws) == 0
        np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx.cpu().numpy())
        np.testing.assert_allclose(w.cpu().numpy(), ref_w.cpu().numpy(), rtol=1e-6, atol=1e-7)
        pu.assert_close(pu.bf16_to_f64(bf16_bits(out)), pu.bf16_to_f64(bf16_bits(ref_out)), f"call {step}")


def test_noalloc_rejects_sizes_beyond_its_limits():
    from bit_quantized_moe_gemv_b200 import _lib as L
    lib = L.LIB
    # T = 5 exceeds the 4-token limit; E = 2048 and k = 17 exceed theirs.
    assert lib.moe_layer_decode_noalloc(None, 5, 1024, 512, 64, 8, None, None, 0, None, None, None, None, None,
                                        None) == 2
    assert lib.moe_layer_decode_noalloc(None, 1, 1024, 512, 2048, 8, None, None, 0, None, None, None, None, None,
                                        None) == 2
    assert lib.moe_layer_decode_noalloc(None, 1, 1024, 512, 64, 17, None, None, 0, None, None, None, None, None,
                                        None) == 2
