"""Pins of the fp64 oracle against values fixed by the pages' structure and by
mathematics, never against the oracle itself.

* dequantisation: hand-computed bit patterns (tests/golden/dequant_vectors.txt);
* routing: closed-form softmax/top-k cases (tests/golden/routing_closed_form.txt),
  brute force over every k-subset, invariants (gates sum to 1, sorted);
* dispatch: a library stable sort and bincount;
* SwiGLU expert: a closed-form case (tests/golden/swiglu_expert_closed_form.txt);
* the whole layer: dense evaluation of every expert on every token masked by the
  renormalised gates, with weights unpacked bit by bit through np.unpackbits.

Structure cited throughout: the telli.sh page "Strata 与 Qwen3.8-Flash-Next：如何在
个人电脑上运行 180B 级模型", section "稀疏架构创造了机会" (E routed experts per
layer, k routed + 1 shared active per token).
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle
from bit_quantized_moe_gemv_b200 import workload as wlm

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
QT = {"int4": oracle.INT4_SYM_G32, "int2": oracle.INT2_ASYM_G16, "int8": oracle.INT8_PER_CHANNEL}


# ------------------------------------------------------------ fixture parsing
def _records(name):
    blocks, cur = [], []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.rstrip("\n")
        if line.startswith("#"):
            continue
        if not line.strip():
            if cur:
                blocks.append(cur)
                cur = []
            continue
        cur.append(line)
    if cur:
        blocks.append(cur)
    return blocks


def _dequant_cases():
    out = []
    for b in _records("dequant_vectors.txt"):
        qt, rows, cols = b[0].split()
        kv = dict(l.split(":", 1) for l in b[1:])
        codes = np.array([int(h, 16) for h in kv["codes"].split()], dtype=np.uint8)
        scales = np.array([float(v) for v in kv["scales"].split()], dtype=np.float16)
        mins = None if kv["mins"].strip() == "-" else np.array([float(v) for v in kv["mins"].split()], dtype=np.float16)
        expect = np.array([float(v) for v in kv["expect"].split()]).reshape(int(rows), int(cols))
        out.append((QT[qt], int(rows), int(cols), codes, scales, mins, expect))
    return out


@pytest.mark.parametrize("case", _dequant_cases(), ids=lambda c: f"q{c[0]}_{c[1]}x{c[2]}")
def test_dequant_golden(case):
    qt, rows, cols, codes, scales, mins, expect = case
    got = oracle.dequant(qt, rows, cols, codes, scales, mins)
    np.testing.assert_array_equal(got, expect)


def _parse_logits(tok):
    if tok.startswith("-ln"):
        return -math.log(float(tok[3:]))
    if tok.startswith("ln"):
        return math.log(float(tok[2:]))
    return float(tok)


def _routing_cases():
    cases = []
    for line in open(os.path.join(GOLDEN, "routing_closed_form.txt")):
        if line.startswith("#") or not line.strip():
            continue
        k, logits, idx, w = [p.strip() for p in line.split("|")]
        cases.append((int(k), [_parse_logits(t) for t in logits.split()], [int(v) for v in idx.split()],
                      [float(v) for v in w.split()]))
    return cases


@pytest.mark.parametrize("case", _routing_cases())
def test_routing_closed_form(case):
    k, logits, idx_exp, w_exp = case
    E, H = len(logits), 8
    x = np.zeros((1, H), dtype=np.float32)
    x[0, 0] = 1.0
    w_r = np.zeros((E, H), dtype=np.float64)
    w_r[:, 0] = logits  # kept in float64 so the logits are exact
    _, idx, w = oracle.route(wlm.f32_to_bf16_bits(x), w_r, np.zeros(E), k)
    assert idx[0].tolist() == idx_exp
    np.testing.assert_allclose(w[0], w_exp, rtol=0, atol=1e-15)


def _routing_bias_cases():
    cases = []
    for line in open(os.path.join(GOLDEN, "routing_bias_closed_form.txt")):
        if line.startswith("#") or not line.strip():
            continue
        k, r, b, idx, w = [p.strip() for p in line.split("|")]
        rows = lambda f, conv: [[conv(v) for v in part.split()] for part in f.split(";")]  # noqa: E731
        cases.append((int(k), [_parse_logits(t) for t in r.split()], rows(b, _parse_logits), rows(idx, int),
                      rows(w, float)))
    return cases


@pytest.mark.parametrize("case", _routing_bias_cases())
def test_routing_bias_closed_form(case):
    """The bias enters the logit: it moves the selection and the gates
    (hand-worked values in tests/golden/routing_bias_closed_form.txt)."""
    k, r, bias_rows, idx_exp, w_exp = case
    E, H, T = len(r), 8, len(idx_exp)
    x = np.zeros((T, H), dtype=np.float32)
    x[:, 0] = 1.0
    w_r = np.zeros((E, H), dtype=np.float64)
    w_r[:, 0] = r
    bias = np.asarray(bias_rows[0] if len(bias_rows) == 1 else bias_rows, dtype=np.float64)
    _, idx, w = oracle.route(wlm.f32_to_bf16_bits(x), w_r, bias, k)
    assert idx.tolist() == idx_exp
    np.testing.assert_allclose(w, np.asarray(w_exp), rtol=0, atol=1e-15)


def _variant_cases(kind):
    cases = []
    for line in open(os.path.join(GOLDEN, "router_variants_closed_form.txt")):
        if line.startswith("#") or not line.strip():
            continue
        parts = [p.strip() for p in line.split("|")]
        if parts[0] != kind:
            continue
        if kind == "sel":
            cases.append((int(parts[1]), [_parse_logits(t) for t in parts[2].split()],
                          [_parse_logits(t) for t in parts[3].split()], [int(v) for v in parts[4].split()],
                          [float(v) for v in parts[5].split()]))
        else:
            cases.append((_parse_logits(parts[1]), float(parts[2])))
    return cases


@pytest.mark.parametrize("case", _variant_cases("sel"))
def test_bias_selection_only_closed_form(case):
    """The bias picks the experts; the gates come from the unbiased logits
    (hand-worked values in tests/golden/router_variants_closed_form.txt)."""
    k, r, b, idx_exp, w_exp = case
    E, H = len(r), 8
    x = np.zeros((1, H), dtype=np.float32)
    x[0, 0] = 1.0
    w_r = np.zeros((E, H), dtype=np.float64)
    w_r[:, 0] = r
    logits, idx, w = oracle.route(wlm.f32_to_bf16_bits(x), w_r, np.asarray(b), k, bias_selection_only=True)
    assert idx[0].tolist() == idx_exp
    np.testing.assert_allclose(w[0], w_exp, rtol=0, atol=1e-15)
    np.testing.assert_allclose(logits[0], np.asarray(r) + np.asarray(b), rtol=0, atol=1e-15)  # biased logits


@pytest.mark.parametrize("case", _variant_cases("gate"))
def test_shared_gate_closed_form(case):
    gx, expect = case
    x = np.zeros((1, 8), dtype=np.float32)
    x[0, 0] = 1.0
    g = np.zeros(8)
    g[0] = gx
    np.testing.assert_allclose(oracle.shared_gate(wlm.f32_to_bf16_bits(x), g), [expect], rtol=0, atol=1e-15)


def test_sigmoid_gated_shared_expert_through_the_layer():
    """The closed-form expert as both the routed pick (gate 1, k = 1) and the
    shared expert with sigma(g . x) = 3/4: the output is 1.75 times its y."""
    ex, _, y_exp = _closed_form_fixture()
    zero = _closed_form_fixture()[0]
    zero.down = _int4_matrix_from_q(np.zeros((32, 32), dtype=np.int32), 0.125)
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, 0] = 1.0
    xb = wlm.f32_to_bf16_bits(x)
    w_r = np.zeros((2, 32))
    w_r[1, 0] = 0.5
    g = np.zeros(32)
    g[0] = math.log(3.0)
    r = oracle.moe_layer(xb, w_r, np.zeros(2), 1, [zero, ex], shared=ex, shared_gate_w=g)
    n = len(y_exp)  # the fixture's nonzero outputs; the rest are exactly 0
    np.testing.assert_allclose(r["out"][0, :n], 1.75 * np.asarray(y_exp), rtol=0, atol=1e-12)
    assert np.all(r["out"][0, n:] == 0.0)
    cache = oracle.DequantCache([zero, ex])
    sh = tuple(oracle.dequant_qm(m) for m in (ex.gate, ex.up, ex.down))
    _, _, out_t = oracle.moe_token(xb[0], w_r, np.zeros(2), 1, cache, sh, shared_gate_w=g)
    np.testing.assert_allclose(out_t, r["out"][0], rtol=0, atol=1e-12)


def test_routing_k1_gate_is_exactly_one():
    rng = np.random.default_rng(3)
    x = wlm.f32_to_bf16_bits(rng.standard_normal((5, 64)).astype(np.float32))
    _, _, w = oracle.route(x, rng.standard_normal((9, 64)) * 0.1, np.zeros(9), 1)
    assert np.all(w == 1.0)


@pytest.mark.parametrize("k", [1, 2, 3, 5, 8])
def test_topk_equals_brute_force_subsets(k):
    rng = np.random.default_rng(100 + k)
    E, H, T = 8, 32, 40
    x = wlm.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    w_r = rng.standard_normal((E, H)) * 0.3
    b = rng.standard_normal(E) * 0.5
    logits, idx, w = oracle.route(x, w_r, b, k)
    for t in range(T):
        best = max(itertools.combinations(range(E), k), key=lambda s: sum(logits[t, e] for e in s))
        assert set(idx[t].tolist()) == set(best)
        sel = logits[t, idx[t]]
        assert np.all(np.diff(sel) <= 0)
    assert np.allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(np.diff(w, axis=1) <= 0)


def test_topk_k_equals_E_selects_all():
    rng = np.random.default_rng(7)
    x = wlm.f32_to_bf16_bits(rng.standard_normal((3, 16)).astype(np.float32))
    _, idx, w = oracle.route(x, rng.standard_normal((6, 16)), np.zeros(6), 6)
    for t in range(3):
        assert sorted(idx[t].tolist()) == list(range(6))


def test_dispatch_matches_stable_sort():
    rng = np.random.default_rng(11)
    T, k, E = 300, 4, 37
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, inv = oracle.dispatch(idx, E)
    flat = idx.reshape(-1)
    np.testing.assert_array_equal(counts, np.bincount(flat, minlength=E))
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
    np.testing.assert_array_equal(perm, np.argsort(flat, kind="stable"))
    np.testing.assert_array_equal(inv[perm], np.arange(T * k))
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) > 0) and np.all(flat[seg] == e)


def test_dispatch_empty_and_degenerate():
    counts, offsets, perm, inv = oracle.dispatch(np.zeros((0, 3), dtype=np.int32), 5)
    assert counts.tolist() == [0] * 5 and offsets.tolist() == [0] * 6 and perm.size == 0
    counts, offsets, perm, inv = oracle.dispatch(np.zeros((4, 1), dtype=np.int32), 3)
    assert counts.tolist() == [4, 0, 0] and perm.tolist() == [0, 1, 2, 3]


# ------------------------------------------------------------ SwiGLU closed form
def _int4_matrix_from_q(q: np.ndarray, scale: float):
    """Pack an int4 matrix (test-side encoder: code = q + 8, low nibble first)."""
    rows, cols = q.shape
    c = (q + 8).astype(np.uint8)
    codes = (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    scales = np.full((rows, cols // 32), scale, dtype=np.float16)
    return wlm.QMatrix(wlm.Q_INT4_SYM_G32, rows, cols, codes, scales, None)


def _closed_form_fixture():
    kv = {}
    for line in open(os.path.join(GOLDEN, "swiglu_expert_closed_form.txt")):
        if line.startswith("#") or ":" not in line:
            continue
        key, v = line.split(":", 1)
        kv[key.strip()] = v.strip()
    H = I = 32
    qg = np.zeros((I, H), dtype=np.int32)
    qg[:3, 0] = [int(v) for v in kv["gate_q_col0"].split()]
    qu = np.zeros((I, H), dtype=np.int32)
    qu[:3, 0] = [int(v) for v in kv["up_q_col0"].split()]
    qd = np.zeros((H, I), dtype=np.int32)
    for n, row in enumerate(kv["down_q"].split("|")):
        qd[n, :3] = [int(v) for v in row.split()]
    ex = wlm.Expert(_int4_matrix_from_q(qg, float(kv["gate_scale"])), _int4_matrix_from_q(qu, float(kv["up_scale"])),
                    _int4_matrix_from_q(qd, float(kv["down_scale"])))
    return ex, [float(v) for v in kv["expect_h"].split()], [float(v) for v in kv["expect_y"].split()]


def test_swiglu_expert_closed_form():
    ex, h_exp, y_exp = _closed_form_fixture()
    x = np.zeros((1, 32))
    x[0, 0] = 1.0
    h, y = oracle.expert_forward(oracle.dequant_qm(ex.gate), oracle.dequant_qm(ex.up), oracle.dequant_qm(ex.down), x)
    np.testing.assert_allclose(h[0, :3], h_exp, rtol=1e-15)
    assert np.all(h[0, 3:] == 0)
    np.testing.assert_allclose(y[0, :4], y_exp, rtol=1e-15)
    assert np.all(y[0, 4:] == 0)


def test_layer_closed_form_through_routing():
    """One token, two routed experts, k=1: the chosen expert's closed-form y comes
    out with gate exactly 1; adding the same expert as shared doubles it."""
    ex, _, y_exp = _closed_form_fixture()
    zero = _closed_form_fixture()[0]
    zero.down = _int4_matrix_from_q(np.zeros((32, 32), dtype=np.int32), 0.125)
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, 0] = 1.0
    xb = wlm.f32_to_bf16_bits(x)
    w_r = np.zeros((2, 32))
    w_r[1, 0] = 0.5  # expert 1 wins
    r = oracle.moe_layer(xb, w_r, np.zeros(2), 1, [zero, ex], shared=None)
    assert r["idx"].tolist() == [[1]]
    np.testing.assert_allclose(r["out"][0, :4], y_exp, rtol=1e-15)
    r2 = oracle.moe_layer(xb, w_r, np.zeros(2), 1, [zero, ex], shared=ex)
    np.testing.assert_allclose(r2["out"][0, :4], 2 * np.array(y_exp), rtol=1e-15)


# ------------------------------------------------------------ dense brute force
def _unpack_bits(qm):
    """Independent bit-level unpacking via np.unpackbits (LSB first)."""
    rows, cols = qm.rows, qm.cols
    bits = np.unpackbits(np.asarray(qm.codes, dtype=np.uint8).reshape(rows, -1), axis=1, bitorder="little")
    kcol = np.arange(cols)
    if qm.qtype == wlm.Q_INT4_SYM_G32:
        b = bits.reshape(rows, cols, 4)
        c = (b * np.array([1, 2, 4, 8])).sum(axis=2).astype(np.float64)
        return (c - 8) * np.asarray(qm.scales, dtype=np.float64)[:, kcol // 32]
    if qm.qtype == wlm.Q_INT2_ASYM_G16:
        b = bits.reshape(rows, cols, 2)
        c = (b * np.array([1, 2])).sum(axis=2).astype(np.float64)
        s = np.asarray(qm.scales, dtype=np.float64)[:, kcol // 16]
        m = np.asarray(qm.mins, dtype=np.float64)[:, kcol // 16]
        return c * s + m
    b = bits.reshape(rows, cols, 8)
    c = (b * np.array([1, 2, 4, 8, 16, 32, 64, -128])).sum(axis=2).astype(np.float64)
    return c * np.asarray(qm.scales, dtype=np.float64)[:, None]


def _dense_layer(xb, w_r, bias, k, experts, shared):
    x = ((xb.astype(np.uint32) << 16).view(np.float32)).astype(np.float64)
    logits = x @ np.asarray(w_r, np.float64).T + np.asarray(bias, np.float64)
    T, E = logits.shape
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    mask = np.zeros_like(p)
    for t in range(T):
        mask[t, np.argsort(-logits[t], kind="stable")[:k]] = 1.0
    m = p * mask
    m /= m.sum(axis=1, keepdims=True)
    out = np.zeros_like(x)
    for e in range(E):
        wg, wu, wd = (_unpack_bits(q) for q in (experts[e].gate, experts[e].up, experts[e].down))
        g, u = x @ wg.T, x @ wu.T
        out += m[:, e:e + 1] * (((g / (1 + np.exp(-g))) * u) @ wd.T)
    if shared is not None:
        wg, wu, wd = (_unpack_bits(q) for q in (shared.gate, shared.up, shared.down))
        g, u = x @ wg.T, x @ wu.T
        out += ((g / (1 + np.exp(-g))) * u) @ wd.T
    return out


def _mixed_small():
    return wlm.Workload("mixed_small", T=9, H=64, I=32, E=8, k=3, zipf_s=0.7, uniform_frac=0.34,
                        routed_qtypes=((0, 3, wlm.Q_INT4_SYM_G32), (3, 6, wlm.Q_INT2_ASYM_G16),
                                       (6, None, wlm.Q_INT8_PER_CHANNEL)),
                        shared_qtype=wlm.Q_INT2_ASYM_G16, seed=5)


@pytest.mark.parametrize("wl", [wlm.WORKLOADS["tiny"], _mixed_small()], ids=lambda w: w.name)
def test_sparse_oracle_equals_dense_masked(wl):
    lay = wlm.gen_layer(wl)
    xb = wlm.gen_x(wl)
    bias, _ = wlm.gen_bias(wl)
    r = oracle.moe_layer(xb, lay.w_router, bias, wl.k, lay.experts, lay.shared)
    dense = _dense_layer(xb, lay.w_router, bias, wl.k, lay.experts, lay.shared)
    np.testing.assert_allclose(r["out"], dense, rtol=1e-12, atol=1e-12 * np.abs(dense).max())
    assert np.allclose(r["w"].sum(axis=1), 1.0, atol=1e-12)


def test_moe_token_matches_moe_layer():
    wl = _mixed_small()
    lay = wlm.gen_layer(wl)
    xb = wlm.gen_x(wl)
    bias, stride = wlm.gen_bias(wl)
    r = oracle.moe_layer(xb, lay.w_router, bias, wl.k, lay.experts, lay.shared)
    cache = oracle.DequantCache(lay.experts)
    sh = tuple(oracle.dequant_qm(m) for m in (lay.shared.gate, lay.shared.up, lay.shared.down))
    for t in range(wl.T):
        brow = bias[t] if stride else bias
        idx, w, out = oracle.moe_token(xb[t], lay.w_router, brow, wl.k, cache, sh)
        assert idx.tolist() == r["idx"][t].tolist()
        np.testing.assert_allclose(out, r["out"][t], rtol=1e-12, atol=1e-14)
