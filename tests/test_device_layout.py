"""Host-side layout of uploaded weights, on CPU.

`DeviceExperts` packs every part of every expert (codes, scales, mins) into
one buffer, each part 256-byte aligned, and writes a table of `moe_expert`
descriptors pointing into it; `BlockExperts` points descriptors into stacked
tensors drawn on the device. Built here on CPU tensors, every descriptor must
carry the matrix's shape and format and point at exactly that matrix's bytes.
The device-side draw of the 48-layer stack must follow the same value recipe
as the host generator.
"""
import ctypes

import numpy as np
import torch

from bit_quantized_moe_gemv_b200 import _lib
from bit_quantized_moe_gemv_b200 import workload as wlm
from bit_quantized_moe_gemv_b200.device import BlockExperts, DeviceExperts


def _read(base_tensor, ptr, nbytes):
    off = ptr - base_tensor.data_ptr()
    assert 0 <= off and off + nbytes <= base_tensor.numel()
    return base_tensor[off:off + nbytes].numpy()


def test_device_experts_descriptors_point_at_their_bytes():
    wl = wlm.Workload("layout", T=1, H=256, I=128, E=6, k=2, seed=5,
                      routed_qtypes=((0, 2, wlm.Q_INT4_SYM_G32), (2, 4, wlm.Q_INT2_ASYM_G16),
                                     (4, None, wlm.Q_INT8_PER_CHANNEL)))
    lay = wlm.gen_layer(wl, with_shared=False)
    dx = DeviceExperts(lay.experts, "cpu")
    assert dx.table.numel() == wl.E * ctypes.sizeof(_lib.ExpertC)
    for e, ex in enumerate(lay.experts):
        d = dx.descriptor(e)
        for name in ("gate", "up", "down"):
            qm, dm = getattr(ex, name), getattr(d, name)
            assert (dm.qtype, dm.rows, dm.cols, dm.group) == (qm.qtype, qm.rows, qm.cols, wlm.qtype_group(qm.qtype))
            for ptr in (dm.codes, dm.scales) + ((dm.mins,) if qm.mins is not None else ()):
                assert (ptr - dx.buffer.data_ptr()) % 256 == 0
            np.testing.assert_array_equal(_read(dx.buffer, dm.codes, qm.codes.nbytes), qm.codes.reshape(-1))
            sc = np.ascontiguousarray(qm.scales, dtype=np.float16).view(np.uint8).reshape(-1)
            np.testing.assert_array_equal(_read(dx.buffer, dm.scales, sc.size), sc)
            if qm.mins is None:
                assert dm.mins is None
            else:
                mn = np.ascontiguousarray(qm.mins, dtype=np.float16).view(np.uint8).reshape(-1)
                np.testing.assert_array_equal(_read(dx.buffer, dm.mins, mn.size), mn)


def test_block_experts_descriptors_point_into_the_stacks():
    wl = wlm.Workload("block", T=4, H=256, I=128, E=4, k=2, seed=6,
                      routed_qtypes=((0, None, wlm.Q_INT2_ASYM_G16),), shared_qtype=wlm.Q_INT8_PER_CHANNEL)
    d = wlm.draw_layer_device(wl, 0, device="cpu")
    bx = BlockExperts(d["qtype"], d["gu"], d["dn"], wl.I, wl.H, device="cpu")
    raw = bx.table.numpy().tobytes()
    size = ctypes.sizeof(_lib.ExpertC)
    for e in range(wl.E):
        ex = _lib.ExpertC.from_buffer_copy(raw[e * size:(e + 1) * size])
        for name, j in (("gate", 0), ("up", 1), ("down", None)):
            dm = getattr(ex, name)
            codes = d["gu"][0][e, j] if j is not None else d["dn"][0][e]
            scales = d["gu"][1][e, j] if j is not None else d["dn"][1][e]
            mins = d["gu"][2][e, j] if j is not None else d["dn"][2][e]
            assert dm.codes == codes.data_ptr() and dm.scales == scales.data_ptr() and dm.mins == mins.data_ptr()
            assert (dm.rows, dm.cols) == ((wl.I, wl.H) if j is not None else (wl.H, wl.I))
            assert dm.qtype == wlm.Q_INT2_ASYM_G16 and dm.group == 16


def test_device_draw_follows_the_value_recipe():
    wl = wlm.WORKLOADS["decode48"]
    small = wlm.Workload("draw", T=4, H=512, I=256, E=8, k=2, seed=7, routed_qtypes=wl.routed_qtypes,
                         shared_qtype=wl.shared_qtype)
    d = wlm.draw_layer_device(small, 0, device="cpu")
    c, s, m = d["gu"]
    assert c.shape == (8, 2, 256, 512 // 4) and c.dtype == torch.uint8
    assert s.shape == m.shape == (8, 2, 256, 512 // 16)
    s64, m64 = s.double(), m.double()
    assert s64.min() >= 0.01 - 1e-5 and s64.max() <= 0.04 + 1e-4
    assert bool((m64 <= -s64 * (1 - 1e-3)).all()) and bool((m64 >= -2 * s64 * (1 + 1e-3)).all())
    assert set(torch.unique(c & 3).tolist()) == {0, 1, 2, 3}
    sc, ss, sm = d["sdn"]
    assert sc.shape == (1, 512, 256) and sm is None and ss.shape == (1, 512)
    q = sc.view(torch.int8)
    assert int(q.min()) >= -127 and int(q.max()) <= 127
    assert 0.005 / 16 - 1e-6 <= float(ss.double().min()) and float(ss.double().max()) <= 0.02 / 16 + 1e-6
    wr = d["w_router"]
    assert wr.shape == (8, 512) and abs(float(wr.std()) - 0.02) < 0.003
    d2 = wlm.draw_layer_device(small, 0, device="cpu")
    assert torch.equal(d2["gu"][0], c) and not torch.equal(wlm.draw_layer_device(small, 1, device="cpu")["gu"][0], c)
