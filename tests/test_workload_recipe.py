"""The seeded input recipe and the algorithmic byte counts, on CPU.

The roofline figures divide algorithmic bytes by time, so the byte counts are
pinned here against sizes worked out by hand from the packing (codes, fp16
scales, fp16 mins), independently of `qmatrix_nbytes`. The generator is
checked for what the input recipe promises: bf16 rounding to nearest even,
per-array determinism, value ranges, the Zipf prior and the share of
uniformly routed rows.
"""
import math

import numpy as np
import pytest

from bit_quantized_moe_gemv_b200 import workload as wlm

W = wlm.WORKLOADS


def _hand_bytes(kind, rows, cols):
    """Bytes of one packed [rows, cols] matrix, counted per row by hand."""
    if kind == "int4":  # 2 codes per byte, one fp16 scale per 32 inputs
        return rows * (cols // 2 + (cols // 32) * 2)
    if kind == "int2":  # 4 codes per byte, fp16 scale + fp16 min per 16 inputs
        return rows * (cols // 4 + (cols // 16) * 4)
    if kind == "int8":  # 1 code per byte, one fp16 scale per row
        return rows * (cols + 2)
    raise ValueError(kind)


def test_expert_bytes_by_hand():
    # H = 2048, I = 768: gate and up are [768, 2048], down is [2048, 768]
    assert _hand_bytes("int4", 768, 2048) == 884_736 and _hand_bytes("int4", 2048, 768) == 884_736
    int4_expert = 3 * 884_736
    assert int4_expert == 2_654_208
    assert W["decode1"].k == 10
    assert wlm.per_token_layer_bytes(W["decode1"]) == 11 * int4_expert + 4 * 512 * 2048 == 33_390_592
    int2_expert = 2 * _hand_bytes("int2", 768, 2048) + _hand_bytes("int2", 2048, 768)
    int8_shared = 2 * _hand_bytes("int8", 768, 2048) + _hand_bytes("int8", 2048, 768)
    assert int2_expert == 2_359_296 and int8_shared == 4_725_760
    # decode48: one step of 4 tokens streams each DISTINCT routed expert once
    assert wlm.per_token_layer_bytes(W["decode48"], unique_experts=23) == 23 * int2_expert + int8_shared + 4 * 512 * 2048


@pytest.mark.parametrize("qtype,kind", [(wlm.Q_INT4_SYM_G32, "int4"), (wlm.Q_INT2_ASYM_G16, "int2"),
                                        (wlm.Q_INT8_PER_CHANNEL, "int8")])
@pytest.mark.parametrize("rows,cols", [(768, 2048), (2048, 768), (64, 256)])
def test_generated_arrays_have_the_counted_bytes(qtype, kind, rows, cols):
    q = wlm.gen_qmatrix(W["tiny"], 0, 3, "gate", qtype, rows, cols)
    got = q.codes.nbytes + q.scales.nbytes + (0 if q.mins is None else q.mins.nbytes)
    assert got == _hand_bytes(kind, rows, cols) == q.nbytes
    assert q.codes.dtype == np.uint8 and q.codes.flags.c_contiguous
    assert q.scales.dtype == np.float16


def test_bf16_rounding_is_nearest_even():
    one = np.float32(1.0)
    vals = np.array([one, one + np.float32(2.0 ** -8), one + np.float32(3 * 2.0 ** -8),
                     one + np.float32(2.0 ** -8 + 2.0 ** -20), -np.float32(1.0) - np.float32(2.0 ** -8),
                     np.float32(3.0e38), np.float32(0.0)], dtype=np.float32)
    bits = wlm.f32_to_bf16_bits(vals)
    # 1 + half an ulp ties to 1 (even); 1 + 1.5 ulp ties up to 1 + 2 ulp (even);
    # just above half an ulp rounds up; the sign is kept.
    assert bits.tolist() == [0x3F80, 0x3F80, 0x3F82, 0x3F81, 0xBF80, 0x7F62, 0x0000]


def test_generation_is_deterministic_and_per_array():
    wl = W["tiny"]
    a, b = wlm.gen_expert(wl, 0, 5), wlm.gen_expert(wl, 0, 5)
    for m in ("gate", "up", "down"):
        np.testing.assert_array_equal(getattr(a, m).codes, getattr(b, m).codes)
        np.testing.assert_array_equal(getattr(a, m).scales, getattr(b, m).scales)
    c = wlm.gen_expert(wl, 0, 6)
    assert not np.array_equal(a.gate.codes, c.gate.codes)
    assert not np.array_equal(a.gate.codes, a.up.codes)
    assert not np.array_equal(wlm.gen_x(wl, step=0), wlm.gen_x(wl, step=1))
    np.testing.assert_array_equal(wlm.gen_x(wl, step=2), wlm.gen_x(wl, step=2))


def test_value_ranges_follow_the_recipe():
    wl = W["tiny"]
    q4 = wlm.gen_qmatrix(wl, 0, 0, "gate", wlm.Q_INT4_SYM_G32, 256, 512)
    s = q4.scales.astype(np.float64)
    assert s.min() >= 0.005 - 1e-5 and s.max() <= 0.02 + 1e-5
    nib = np.concatenate([q4.codes & 15, q4.codes >> 4]).ravel()
    assert set(np.unique(nib).tolist()) == set(range(16))
    q2 = wlm.gen_qmatrix(wl, 0, 0, "up", wlm.Q_INT2_ASYM_G16, 256, 512)
    s2, m2 = q2.scales.astype(np.float64), q2.mins.astype(np.float64)
    assert s2.min() >= 0.01 - 1e-5 and s2.max() <= 0.04 + 1e-4
    assert np.all(m2 <= -s2 * (1 - 1e-3)) and np.all(m2 >= -2 * s2 * (1 + 1e-3))
    q8 = wlm.gen_qmatrix(wl, 0, 0, "down", wlm.Q_INT8_PER_CHANNEL, 256, 512)
    c8 = q8.codes.view(np.int8)
    assert c8.min() >= -127 and c8.max() <= 127 and q8.mins is None
    x = wlm.gen_x(W["decode1"], step=0, T=64).view(np.uint16).astype(np.uint32) << 16
    xf = x.view(np.float32).astype(np.float64)
    assert abs(xf.mean()) < 0.05 and abs(xf.std() - 1.0) < 0.05
    wr = wlm.gen_router(wl)
    assert wr.shape == (wl.E, wl.H) and wr.dtype == np.float32 and abs(wr.std() - 0.02) < 0.002


def test_zipf_prior_and_uniform_rows():
    b, stride = wlm.gen_bias(W["decode1"])
    assert stride == 0 and b.shape == (512,)
    np.testing.assert_allclose(b, [-1.1 * math.log(e + 1) for e in range(512)], rtol=1e-6, atol=1e-6)
    assert b[0] == 0.0 and np.all(np.diff(b) < 0)
    wl = W["prefill32k"]
    T = 2000
    b, stride = wlm.gen_bias(wl, T=T)
    assert stride == wl.E and b.shape == (T, wl.E)
    zero_rows = np.all(b == 0.0, axis=1)
    assert zero_rows.sum() == round(0.05 * T)
    prior = np.array([-1.2 * math.log(e + 1) for e in range(wl.E)])
    np.testing.assert_allclose(b[~zero_rows], np.broadcast_to(prior, (T - zero_rows.sum(), wl.E)), rtol=1e-6,
                               atol=1e-6)


def test_mixed_precision_layout_of_the_long_prefill():
    wl = W["prefill32k"]
    assert [wl.expert_qtype(e) for e in (0, 255, 256, 511)] == [wlm.Q_INT4_SYM_G32] * 2 + [wlm.Q_INT2_ASYM_G16] * 2
    assert wl.shared_qtype == wlm.Q_INT8_PER_CHANNEL
    with pytest.raises(ValueError):
        wl.expert_qtype(-1)
