"""GPU parity of every step against the fp64 oracle, through the C ABI.

Integer outputs (top-k indices, counts, offsets, permutations) must be
bit-exact; floating outputs must be within rel L2 <= 5e-3 and max abs <=
2e-2 x rms of the oracle. Small cases are compared element by element over
all outputs; the full-size workloads on sampled tokens/rows.
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


def _small_mixed():
    return wlm.Workload("small_mixed", T=19, H=128, I=64, E=12, k=3, zipf_s=0.5, uniform_frac=0.3,
                        routed_qtypes=((0, 4, wlm.Q_INT4_SYM_G32), (4, 8, wlm.Q_INT2_ASYM_G16),
                                       (8, None, wlm.Q_INT8_PER_CHANNEL)),
                        shared_qtype=wlm.Q_INT8_PER_CHANNEL, seed=3)


SMALL = {
    "tiny": wlm.WORKLOADS["tiny"],
    # decode-sized batches that take the fused single-launch path (T <= 4)
    "fused_mixed_T3": wlm.Workload("fused_mixed_T3", T=3, H=512, I=256, E=32, k=4, zipf_s=0.8, seed=7,
                                   routed_qtypes=((0, 10, wlm.Q_INT4_SYM_G32), (10, 20, wlm.Q_INT2_ASYM_G16),
                                                  (20, None, wlm.Q_INT8_PER_CHANNEL)),
                                   shared_qtype=wlm.Q_INT8_PER_CHANNEL),
    "fused_int4_T1": wlm.Workload("fused_int4_T1", T=1, H=1024, I=512, E=64, k=6, zipf_s=1.1, seed=8),
    "fused_int2_T4": wlm.Workload("fused_int2_T4", T=4, H=1536, I=512, E=24, k=5, seed=9,
                                  routed_qtypes=((0, None, wlm.Q_INT2_ASYM_G16),), shared_qtype=wlm.Q_INT4_SYM_G32),
    # several router quarter-rows per CTA (E * H / 512 well above the SM count)
    "fused_router_rows_T2": wlm.Workload("fused_router_rows_T2", T=2, H=1024, I=512, E=384, k=8, zipf_s=0.9,
                                         seed=16),
    "small_mixed": _small_mixed(),
    "k_equals_E": wlm.Workload("k_equals_E", T=5, H=128, I=64, E=16, k=16, seed=4),
    # batches > 4 tokens with H, I multiples of 128 take the tcgen05 grouped GEMM
    "tc_int4": wlm.Workload("tc_int4", T=200, H=256, I=256, E=8, k=2, zipf_s=0.5, seed=12),
    "tc_mixed": wlm.Workload("tc_mixed", T=300, H=512, I=384, E=16, k=4, zipf_s=1.0, uniform_frac=0.1, seed=13,
                             routed_qtypes=((0, 6, wlm.Q_INT4_SYM_G32), (6, 11, wlm.Q_INT2_ASYM_G16),
                                            (11, None, wlm.Q_INT8_PER_CHANNEL)),
                             shared_qtype=wlm.Q_INT8_PER_CHANNEL),
    # E a multiple of 128 and T > 4: the tensor-core router (three-way bf16 split of W_r)
    "tc_router": wlm.Workload("tc_router", T=300, H=512, I=256, E=128, k=4, zipf_s=0.9, seed=15),
    "tc_skew": wlm.Workload("tc_skew", T=1000, H=256, I=128, E=64, k=3, zipf_s=2.0, seed=14),
    # groups of 5, 3 and 2 row tiles (and the shared expert's 5) paired into
    # 256-token tiles, each with a partial last tile; H / 128 odd, so the down
    # GEMM's last 256-row weight block holds one 128-row tile
    "tc_wide_odd_h": wlm.Workload("tc_wide_odd_h", T=600, H=384, I=256, E=10, k=2, zipf_s=0.8, seed=20,
                                  routed_qtypes=((0, 7, wlm.Q_INT4_SYM_G32), (7, None, wlm.Q_INT2_ASYM_G16))),
    # a handful of tokens on the tcgen05 path: every expert (and the shared
    # one) on the mma.sync GEMV path; then a mix where the int2/int8 experts
    # and the int8 shared expert take the dequantising GEMM beside it
    "tc_few_tokens": wlm.Workload("tc_few_tokens", T=12, H=256, I=256, E=16, k=4, zipf_s=0.5, seed=21),
    "tc_few_tokens_mixed": wlm.Workload("tc_few_tokens_mixed", T=9, H=384, I=128, E=12, k=3, zipf_s=0.3, seed=22,
                                        routed_qtypes=((0, 5, wlm.Q_INT4_SYM_G32), (5, 9, wlm.Q_INT2_ASYM_G16),
                                                       (9, None, wlm.Q_INT8_PER_CHANNEL)),
                                        shared_qtype=wlm.Q_INT8_PER_CHANNEL),
    "k1_ragged": wlm.Workload("k1_ragged", T=37, H=192, I=128, E=40, k=1, zipf_s=0.3, seed=6,
                              shared_qtype=wlm.Q_INT2_ASYM_G16),
    # 256 routed experts (the pages' Coder variant keeps half of the 512) on
    # each expert path: the fused decode kernel, the tcgen05 grouped GEMM
    # (H, I multiples of 128) and the general kernels (H = 192)
    "e256_fused_T2": wlm.Workload("e256_fused_T2", T=2, H=2048, I=768, E=256, k=10, zipf_s=1.1, seed=17),
    "e256_tc": wlm.Workload("e256_tc", T=300, H=512, I=256, E=256, k=8, zipf_s=1.0, seed=18),
    "e256_simt": wlm.Workload("e256_simt", T=37, H=192, I=128, E=256, k=8, zipf_s=0.8, seed=19,
                              shared_qtype=wlm.Q_INT8_PER_CHANNEL),
}


def _run_steps(L, wl, lay, dev, xb, bias, stride, ws):
    """Run route/dispatch/expert_ffn/combine separately; return host results."""
    import torch
    T, k, E, H, I = wl.T, wl.k, wl.E, wl.H, wl.I
    from bit_quantized_moe_gemv_b200.device import bf16_bits, bf16_tensor
    x = bf16_tensor(xb)
    b = pu.bias_tensor(bias)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    logits = torch.empty((T, E), dtype=torch.float32, device="cuda")
    L.route(x, dev["w_router"], b, stride, k, idx, w, ws, logits=logits)
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    L.dispatch(idx, E, counts, offsets, perm, inv, ws)
    y_perm = torch.empty((T * k, H), dtype=torch.bfloat16, device="cuda")
    L.expert_ffn(x, I, k, E, perm, offsets, counts, dev["experts"].table, y_perm, ws)
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    L.combine(y_perm, inv, w, I, x, dev["shared"].table if dev["shared"] else None, out, ws)
    torch.cuda.synchronize()
    assert L.get_status(ws) == 0
    return dict(idx=idx.cpu().numpy(), w=w.cpu().numpy(), logits=logits.cpu().numpy(), counts=counts.cpu().numpy(),
                offsets=offsets.cpu().numpy(), perm=perm.cpu().numpy(), inv=inv.cpu().numpy(),
                y_perm=bf16_bits(y_perm), out=bf16_bits(out))


@pytest.mark.parametrize("name", list(SMALL))
def test_steps_small_all_outputs(L, name):
    wl = SMALL[name]
    lay = wlm.gen_layer(wl)
    dev = pu.upload_layer(lay)
    xb = wlm.gen_x(wl)
    bias, stride = wlm.gen_bias(wl)
    ws = L.new_workspace(wl.T, wl.H, wl.I, wl.E, wl.k)
    g = _run_steps(L, wl, lay, dev, xb, bias, stride, ws)
    ntied, logits64 = pu.check_routing(g["idx"], g["w"], g["logits"], xb, lay.w_router, bias, wl.k)
    assert ntied == 0
    counts, offsets, perm, inv = oracle.dispatch(g["idx"], wl.E)
    np.testing.assert_array_equal(g["counts"], counts)
    np.testing.assert_array_equal(g["offsets"], offsets)
    np.testing.assert_array_equal(g["perm"], perm)
    np.testing.assert_array_equal(g["inv"], inv)
    y_ref = oracle.expert_rows(xb, perm, offsets, wl.k, lay.experts)
    pu.assert_close(pu.bf16_to_f64(g["y_perm"]), y_ref, "y_perm")
    # The four-call path defines y_perm as bf16: compare with the oracle's rows
    # rounded the same way (moe_layer keeps them in fp32; see test_layer_small).
    sy = oracle.shared_rows(xb, lay.shared)
    ref_out = oracle.combine(pu.round_bf16(y_ref), inv, oracle_gates(xb, lay, bias, g["idx"]), wl.k, sy)
    pu.assert_close(pu.bf16_to_f64(g["out"]), ref_out, "out")
    # combine alone: oracle combine on the device's own y_perm and gates
    sy = oracle.shared_rows(xb, lay.shared)
    comb = oracle.combine(pu.bf16_to_f64(g["y_perm"]), g["inv"], g["w"].astype(np.float64), wl.k, sy)
    pu.assert_close(pu.bf16_to_f64(g["out"]), comb, "combine")


def oracle_gates(xb, lay, bias, idx):
    return pu.oracle_gates_for(oracle.router_logits(xb, lay.w_router, bias), idx)


def _layer_call(L, wl, dev, xb, bias, stride, ws, with_logits=False):
    import torch

    from bit_quantized_moe_gemv_b200.device import bf16_bits, bf16_tensor
    x = bf16_tensor(xb)
    idx = torch.empty((x.shape[0], wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((x.shape[0], wl.k), dtype=torch.float32, device="cuda")
    out = torch.empty((x.shape[0], wl.H), dtype=torch.bfloat16, device="cuda")
    lg = torch.full((x.shape[0], wl.E), float("nan"), dtype=torch.float32, device="cuda") if with_logits else None
    L.layer(x, wl.I, wl.E, wl.k, dev["w_router"], pu.bias_tensor(bias), stride, dev["experts"].table,
            dev["shared"].table if dev["shared"] else None, idx, w, out, ws, logits=lg)
    torch.cuda.synchronize()
    assert L.get_status(ws) == 0
    if with_logits:
        return idx.cpu().numpy(), w.cpu().numpy(), bf16_bits(out), lg.cpu().numpy()
    return idx.cpu().numpy(), w.cpu().numpy(), bf16_bits(out)


@pytest.mark.parametrize("name", list(SMALL))
def test_layer_small(L, name):
    wl = SMALL[name]
    lay = wlm.gen_layer(wl)
    dev = pu.upload_layer(lay)
    xb = wlm.gen_x(wl)
    bias, stride = wlm.gen_bias(wl)
    ws = L.new_workspace(wl.T, wl.H, wl.I, wl.E, wl.k)
    idx, w, out, lg = _layer_call(L, wl, dev, xb, bias, stride, ws, with_logits=True)
    ref = oracle.moe_layer(xb, lay.w_router, bias, wl.k, lay.experts, lay.shared)
    ntied, _ = pu.check_routing(idx, w, lg, xb, lay.w_router, bias, wl.k)
    assert ntied == 0
    np.testing.assert_array_equal(idx, ref["idx"])
    np.testing.assert_allclose(w, ref["w"], rtol=1e-5, atol=1e-6)
    pu.assert_close(pu.bf16_to_f64(out), ref["out"])
    # determinism: a second call gives identical bits
    idx2, w2, out2 = _layer_call(L, wl, dev, xb, bias, stride, ws)
    np.testing.assert_array_equal(out2, out)
    np.testing.assert_array_equal(w2, w)


def _check_sampled_tokens(wl, lay, xb, bias, stride, idx, w, out, tokens):
    """Outputs of the given tokens against the oracle. The routing must have
    been checked first (pu.check_routing): the oracle evaluates the device's
    picks, which equal its own except on flagged near-ties, where they are a
    valid top-k within the fp32 rounding bound."""
    cache = oracle.DequantCache(lay.experts, capacity=256)
    sh = tuple(oracle.dequant_qm(m) for m in (lay.shared.gate, lay.shared.up, lay.shared.down))
    logits64 = oracle.router_logits(xb[tokens], lay.w_router, bias[tokens] if stride else bias)
    for n, t in enumerate(tokens):
        brow = bias[t] if stride else bias
        # same expert set as the device (identical except on flagged near-ties)
        gates = pu.oracle_gates_for(logits64[n:n + 1], idx[t:t + 1])[0]
        _, _, ref = oracle.moe_token(xb[t], lay.w_router, brow, wl.k, cache, sh, routing=(idx[t], gates))
        pu.assert_close(pu.bf16_to_f64(out[t]), ref, f"token {t}")
        np.testing.assert_allclose(w[t], gates, rtol=1e-5, atol=1e-6)


def test_layer_decode1_steps(L):
    wl = wlm.WORKLOADS["decode1"]
    lay = wlm.gen_layer(wl)
    dev = pu.upload_layer(lay)
    bias, stride = wlm.gen_bias(wl)
    ws = L.new_workspace(wl.T, wl.H, wl.I, wl.E, wl.k)
    for step in range(6):
        xb = wlm.gen_x(wl, step=step)
        idx, w, out, lg = _layer_call(L, wl, dev, xb, bias, stride, ws, with_logits=True)
        # selection exactly on the device's fp32 logits; against the fp64
        # oracle bit for bit unless flagged, else a valid top-k within tau
        pu.check_routing(idx, w, lg, xb, lay.w_router, bias, wl.k)
        _check_sampled_tokens(wl, lay, xb, bias, stride, idx, w, out, [0])


def test_layer_verify4_steps(L):
    """A speculative-decoding verification batch (4 tokens of one sequence,
    the decode1 layer) through the fused decode kernel: routing exact against
    the oracle (outside near-ties), every token's output within tolerance."""
    wl = wlm.WORKLOADS["verify4"]
    lay = wlm.gen_layer(wl)
    dev = pu.upload_layer(lay)
    bias, stride = wlm.gen_bias(wl)
    ws = L.new_workspace(wl.T, wl.H, wl.I, wl.E, wl.k)
    for step in range(3):
        xb = wlm.gen_x(wl, step=step)
        idx, w, out, lg = _layer_call(L, wl, dev, xb, bias, stride, ws, with_logits=True)
        pu.check_routing(idx, w, lg, xb, lay.w_router, bias, wl.k)
        _check_sampled_tokens(wl, lay, xb, bias, stride, idx, w, out, list(range(wl.T)))


@pytest.mark.parametrize("name", ["prefill8k", "prefill32k"])
def test_prefill_full_routing_dispatch_every_output(L, name):
    import torch

    from bit_quantized_moe_gemv_b200.device import bf16_tensor
    wl = wlm.WORKLOADS[name]
    lay = wlm.gen_layer(wl)
    dev = pu.upload_layer(lay)
    xb = wlm.gen_x(wl)
    bias, stride = wlm.gen_bias(wl)
    ws = L.new_workspace(wl.T, wl.H, wl.I, wl.E, wl.k)
    x = bf16_tensor(xb)
    T, k, E = wl.T, wl.k, wl.E
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    logits = torch.empty((T, E), dtype=torch.float32, device="cuda")
    L.route(x, dev["w_router"], pu.bias_tensor(bias), stride, k, idx, w, ws, logits=logits)
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    L.dispatch(idx, E, counts, offsets, perm, inv, ws)
    torch.cuda.synchronize()
    gi = idx.cpu().numpy()
    ntied, _ = pu.check_routing(gi, w.cpu().numpy(), logits.cpu().numpy(), xb, lay.w_router, bias, k)
    print(f"{name}: {ntied} of {T} tokens have a near-tie within tau among their top-{k + 1} logits")
    assert ntied <= T // 50
    c, o, p, v = oracle.dispatch(gi, E)
    np.testing.assert_array_equal(counts.cpu().numpy(), c)
    np.testing.assert_array_equal(offsets.cpu().numpy(), o)
    np.testing.assert_array_equal(perm.cpu().numpy(), p)
    np.testing.assert_array_equal(inv.cpu().numpy(), v)
    # the expert FFN alone: every dispatched row (bf16 y_perm)
    from bit_quantized_moe_gemv_b200.device import bf16_bits
    y_perm = torch.empty((T * k, wl.H), dtype=torch.bfloat16, device="cuda")
    L.expert_ffn(x, wl.I, k, E, perm, offsets, counts, dev["experts"].table, y_perm, ws)
    # whole layer through moe_layer: every output token
    out_idx, out_w, out, out_lg = _layer_call(L, wl, dev, xb, bias, stride, ws, with_logits=True)
    np.testing.assert_array_equal(out_idx, gi)
    np.testing.assert_array_equal(out_lg.view(np.uint32), logits.cpu().numpy().view(np.uint32))
    (ry, my), (ro, mo) = pu.check_every_row(xb, lay.w_router, bias, k, lay.experts, lay.shared, gi,
                                            perm.cpu().numpy(), offsets.cpu().numpy(), bf16_bits(y_perm), out)
    print(f"{name}: y_perm rel {ry:.2e} max/rms {my:.2e}; out rel {ro:.2e} max/rms {mo:.2e}")
    # and a few tokens through the per-token oracle path (moe_token)
    rng = np.random.default_rng(0)
    tokens = sorted(set([0, T - 1] + rng.choice(T, 6, replace=False).tolist()))
    _check_sampled_tokens(wl, lay, xb, bias, stride, out_idx, out_w, out, tokens)


def test_decode48_two_layers(L):
    wl = wlm.WORKLOADS["decode48"]
    for layer in (0, 47):
        lay = wlm.gen_layer(wl, layer)
        dev = pu.upload_layer(lay)
        bias, stride = wlm.gen_bias(wl)
        ws = L.new_workspace(wl.T, wl.H, wl.I, wl.E, wl.k)
        for step in (0, 199):
            xb = wlm.gen_x(wl, step=step, layer=layer)
            idx, w, out, lg = _layer_call(L, wl, dev, xb, bias, stride, ws, with_logits=True)
            pu.check_routing(idx, w, lg, xb, lay.w_router, bias, wl.k)
            _check_sampled_tokens(wl, lay, xb, bias, stride, idx, w, out, list(range(wl.T)))


def test_dispatch_invalid_id_flags_device_fault(L):
    import torch
    E, T, k = 8, 3, 2
    ids = torch.tensor([[0, 1], [8, 2], [3, 1]], dtype=torch.int32, device="cuda")
    ws = L.new_workspace(T, 64, 64, E, k)
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    L.dispatch(ids, E, counts, offsets, perm, inv, ws)
    assert L.get_status(ws) == 5
    assert inv.cpu().numpy()[2] == -1
    assert counts.cpu().numpy().sum() == 5 and offsets.cpu().numpy()[-1] == 5
    L.reset_status(ws)
    assert L.get_status(ws) == 0


def test_bad_descriptor_flags_device_fault(L):
    import torch
    wl = SMALL["tiny"]
    lay = wlm.gen_layer(wl)
    dev = pu.upload_layer(lay)
    # corrupt every routed expert's gate qtype (first int32 of each descriptor)
    tab = dev["experts"].table.view(torch.int32).view(wl.E, -1)
    tab[:, 0] = 9
    xb = wlm.gen_x(wl)
    bias, stride = wlm.gen_bias(wl)
    ws = L.new_workspace(wl.T, wl.H, wl.I, wl.E, wl.k)
    from bit_quantized_moe_gemv_b200.device import bf16_tensor
    x = bf16_tensor(xb)
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    L.layer(x, wl.I, wl.E, wl.k, dev["w_router"], pu.bias_tensor(bias), stride, dev["experts"].table,
            dev["shared"].table, idx, w, out, ws)
    assert L.get_status(ws) == 5


def test_zero_tokens_is_noop(L):
    import torch
    ws = L.new_workspace(0, 128, 64, 8, 2)
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    counts = torch.full((8,), 3, dtype=torch.int32, device="cuda")
    offsets = torch.full((9,), 3, dtype=torch.int32, device="cuda")
    idx = torch.empty((0, 2), dtype=torch.int32, device="cuda")
    L.dispatch(idx, 8, counts, offsets, torch.empty(0, dtype=torch.int32, device="cuda"),
               torch.empty(0, dtype=torch.int32, device="cuda"), ws)
    torch.cuda.synchronize()
    assert counts.cpu().numpy().tolist() == [0] * 8 and offsets.cpu().numpy().tolist() == [0] * 9
    assert L.get_status(ws) == 0
    del x
