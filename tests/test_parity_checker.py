"""The parity checks themselves, on CPU.

The GPU parity tests accept a device result through `assert_close` (the
float tolerance) and `check_routing` (bit-exact indices, with near-ties
handled). Here both are fed a simulated device result built from the fp64
oracle: a faithful one must pass, and each planted mistake (slots out of
order, a perturbed gate, a logit off by more than the fp32 rounding bound,
an output off by more than the tolerance) must fail. A near-tie, where
either expert is a correct pick, must be accepted both ways.
"""
import numpy as np
import pytest

import oracle
from bit_quantized_moe_gemv_b200 import workload as wlm
from tests.parity_util import MAX_ABS_RMS, REL_L2, assert_close, check_routing, near_tie_tau, oracle_gates_for

T, K = 8, 2


def _case():
    wl = wlm.WORKLOADS["tiny"]
    x = wlm.gen_x(wl, step=0, T=T)
    wr = wlm.gen_router(wl).copy()
    bias = np.zeros((T, wl.E), np.float32)
    # token 0: expert 0 first, experts 3 and 9 tied exactly for the second slot
    wr[9] = wr[3]
    bias[0, 0] = 4.0
    bias[0, 3] = bias[0, 9] = 2.0
    return x, wr, bias


def _device(x, wr, bias, logits32=None):
    """A simulated device result: fp32 logits, the top-k on them, fp32 gates."""
    gl = (oracle.router_logits(x, wr, bias).astype(np.float32) if logits32 is None else logits32).astype(np.float64)
    idx = oracle.topk_order(gl, K)
    w = oracle_gates_for(gl, idx).astype(np.float32)
    return idx, w, gl.astype(np.float32)


def _untied_token(x, wr, bias):
    l64 = oracle.router_logits(x, wr, bias)
    tau = near_tie_tau(x, wr, bias)
    for t in range(1, T):
        s = -np.sort(-l64[t])[:K + 2]
        if np.all(s[:-1] - s[1:] > 1e3 * tau[t]):
            return t, l64, tau
    pytest.fail("no well-separated token in the case")


def test_faithful_device_result_passes():
    x, wr, bias = _case()
    idx, w, gl = _device(x, wr, bias)
    n_tied, _ = check_routing(idx, w, gl, x, wr, bias, K)
    assert n_tied >= 1  # token 0


def test_near_tie_accepts_either_expert():
    x, wr, bias = _case()
    _, _, gl = _device(x, wr, bias)
    assert gl[0, 3] == gl[0, 9]
    gl = gl.copy()
    gl[0, 9] = np.nextafter(gl[0, 9], np.float32(np.inf))  # the device's rounding favours expert 9
    idx, w, gl = _device(x, wr, bias, logits32=gl)
    assert idx[0].tolist() == [0, 9]
    check_routing(idx, w, gl, x, wr, bias, K)


def test_slots_out_of_order_fail():
    x, wr, bias = _case()
    idx, w, gl = _device(x, wr, bias)
    idx = idx.copy()
    idx[2] = idx[2][::-1]
    with pytest.raises(AssertionError):
        check_routing(idx, w, gl, x, wr, bias, K)


def test_perturbed_gate_fails():
    x, wr, bias = _case()
    idx, w, gl = _device(x, wr, bias)
    w = w.copy()
    w[3, 0] += 1e-4
    with pytest.raises(AssertionError):
        check_routing(idx, w, gl, x, wr, bias, K)


def test_logit_error_beyond_the_rounding_bound_fails():
    x, wr, bias = _case()
    t, l64, tau = _untied_token(x, wr, bias)
    third = oracle.topk_order(l64, K + 1)[t, K]
    _, _, gl = _device(x, wr, bias)
    gl = gl.copy()
    gl[t, third] += np.float32(l64[t].max() - l64[t, third] + 1.0)  # a wrong dot product promotes it
    idx, w, gl = _device(x, wr, bias, logits32=gl)
    assert third in idx[t].tolist()
    with pytest.raises(AssertionError):
        check_routing(idx, w, gl, x, wr, bias, K)


def test_tolerance_accepts_rounding_and_rejects_errors():
    rng = np.random.default_rng(7)
    ref = rng.standard_normal((16, 256))
    rms = np.sqrt(np.mean(ref ** 2))
    assert_close(ref + 1e-4 * rms * rng.standard_normal(ref.shape), ref)
    spike = ref.copy()
    spike[5, 17] += 1.5 * MAX_ABS_RMS * rms  # one element beyond the max-abs bound
    with pytest.raises(AssertionError):
        assert_close(spike, ref)
    with pytest.raises(AssertionError):
        assert_close(ref * (1 + 2 * REL_L2), ref)  # a uniform 1 % scale error
    nan = ref.copy()
    nan[0, 0] = np.nan
    with pytest.raises(AssertionError):
        assert_close(nan, ref)
    with pytest.raises(AssertionError):
        assert_close(ref[:, :-1], ref)


def test_correctly_rounded_bf16_passes_even_with_outliers():
    # heavy-tailed reference: a few elements far beyond 10 x rms, where the
    # bf16 rounding alone exceeds 2e-2 x rms; the exact values rounded to
    # bf16 must still pass, and an error of one more bf16 ulp must not
    from tests.parity_util import bf16_half_ulp, round_bf16
    rng = np.random.default_rng(7)
    ref = rng.standard_normal((64, 256))
    ref[3, 5], ref[9, 100] = 60.0 + 0.3, -45.0 - 0.17
    assert_close(round_bf16(ref), ref)
    bad = round_bf16(ref)
    bad[3, 5] += 2 * bf16_half_ulp(ref[3, 5]) + MAX_ABS_RMS * np.sqrt(np.mean(ref ** 2))
    with pytest.raises(AssertionError):
        assert_close(bad, ref)


def test_error_accumulator_matches_whole_array_check():
    from tests.parity_util import ErrorAccumulator, round_bf16
    rng = np.random.default_rng(8)
    ref = rng.standard_normal((40, 64)) * 3
    got = round_bf16(ref + 1e-3 * rng.standard_normal(ref.shape))
    acc = ErrorAccumulator("pieces")
    for i in range(0, 40, 7):
        acc.add(got[i:i + 7], ref[i:i + 7])
    rel, mx = acc.check()
    rel2, mx2 = assert_close(got, ref)
    assert abs(rel - rel2) < 1e-12 and abs(mx - mx2) < 1e-12
    got[17, 3] += 0.5  # one planted wrong element
    acc = ErrorAccumulator("pieces")
    for i in range(0, 40, 7):
        acc.add(got[i:i + 7], ref[i:i + 7])
    with pytest.raises(AssertionError):
        acc.check()


def test_every_row_check_catches_one_wrong_row():
    import oracle
    from bit_quantized_moe_gemv_b200 import workload as wlm
    from tests.parity_util import check_every_row
    wl = wlm.WORKLOADS["tiny"]
    lay, xb = wlm.gen_layer(wl), wlm.gen_x(wl)
    bias, _ = wlm.gen_bias(wl)
    r = oracle.moe_layer(xb, lay.w_router, bias, wl.k, lay.experts, lay.shared)
    f2b = lambda a: wlm.f32_to_bf16_bits(np.asarray(a, np.float32))  # noqa: E731
    y, out = f2b(r["y_perm"]), f2b(r["out"])
    check_every_row(xb, lay.w_router, bias, wl.k, lay.experts, lay.shared, r["idx"], r["perm_src"], r["offsets"],
                    y, out)
    y_bad = y.copy()
    y_bad[5] = f2b(r["y_perm"][5] * 1.05)  # one row 5 % off
    with pytest.raises(AssertionError):
        check_every_row(xb, lay.w_router, bias, wl.k, lay.experts, lay.shared, r["idx"], r["perm_src"],
                        r["offsets"], y_bad, out)
