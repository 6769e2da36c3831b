"""Plant plausible mistakes in the oracle (on the CPU, via monkeypatching) and
check that at least one pin fails for each. Shows the pins have teeth."""
import numpy as np
import pytest

import oracle
from oracle import moe_oracle as mo
from tests import test_oracle_pins as pins


def _swapped_nibbles(qtype, rows, cols, codes, scales, mins=None):
    if qtype == mo.INT4_SYM_G32:
        codes = np.asarray(codes, dtype=np.uint8)
        codes = ((codes >> 4) | (codes << 4)).astype(np.uint8)
    return ORIG_DEQUANT(qtype, rows, cols, codes, scales, mins)


def _offset7(qtype, rows, cols, codes, scales, mins=None):
    w = ORIG_DEQUANT(qtype, rows, cols, codes, scales, mins)
    if qtype == mo.INT4_SYM_G32:
        w = w + np.repeat(np.asarray(scales, np.float64).reshape(rows, -1), 32, axis=1)
    return w


def _int2_msb_first(qtype, rows, cols, codes, scales, mins=None):
    if qtype == mo.INT2_ASYM_G16:
        c = np.asarray(codes, dtype=np.uint8)
        c = (((c & 0x03) << 6) | ((c & 0x0C) << 2) | ((c & 0x30) >> 2) | ((c & 0xC0) >> 6)).astype(np.uint8)
        codes = c
    return ORIG_DEQUANT(qtype, rows, cols, codes, scales, mins)


ORIG_DEQUANT = mo.dequant


def _silu_on_up(wg, wu, wd, x):
    g, u = x @ wg.T, x @ wu.T
    h = mo.silu(u) * g
    return h, h @ wd.T


def _down_transposed(wg, wu, wd, x):
    g, u = x @ wg.T, x @ wu.T
    h = mo.silu(g) * u
    return h, h @ wd  # uses W_d untransposed (only shape-valid when square)


def _softmax_free_gates(x_bits, w_router, bias, k, bias_selection_only=False):
    logits = mo.router_logits(x_bits, w_router, bias)
    idx = mo.topk_order(logits, k)
    sel = np.take_along_axis(logits, idx.astype(np.int64), axis=1)
    return logits, idx, sel / sel.sum(axis=1, keepdims=True)


def _ties_to_higher_index(logits, k):
    T, E = logits.shape
    out = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        out[t] = np.lexsort((-np.arange(E), -logits[t]))[:k]
    return out


ORIG_DISPATCH = mo.dispatch
ORIG_COMBINE = mo.combine
ORIG_ROUTE = mo.route


def _int8_unsigned(qtype, rows, cols, codes, scales, mins=None):
    if qtype == mo.INT8_PER_CHANNEL:
        q = np.asarray(codes, dtype=np.uint8).astype(np.float64).reshape(rows, cols)
        return q * np.asarray(scales, np.float64).reshape(rows, 1)
    return ORIG_DEQUANT(qtype, rows, cols, codes, scales, mins)


def _int4_group16(qtype, rows, cols, codes, scales, mins=None):
    w = ORIG_DEQUANT(qtype, rows, cols, codes, scales, mins)
    if qtype == mo.INT4_SYM_G32:
        s = np.asarray(scales, np.float64).reshape(rows, -1)
        k = np.arange(cols)
        w = w / s[:, k // 32] * s[:, np.minimum(k // 16, s.shape[1] - 1)]
    return w


def _sigmoid_for_silu(wg, wu, wd, x):
    g, u = x @ wg.T, x @ wu.T
    h = (1.0 / (1.0 + np.exp(-g))) * u
    return h, h @ wd.T


def _gates_not_renormalised(x_bits, w_router, bias, k, bias_selection_only=False):
    logits, idx, _ = ORIG_ROUTE(x_bits, w_router, bias, k)
    p = mo.softmax(logits)
    return logits, idx, np.take_along_axis(p, idx.astype(np.int64), axis=1)


def _bias_only_selects(x_bits, w_router, bias, k, bias_selection_only=False):
    logits, idx, _ = ORIG_ROUTE(x_bits, w_router, bias, k)
    p = mo.softmax(logits - np.asarray(bias, np.float64))
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    return logits, idx, sel / sel.sum(axis=1, keepdims=True)


def _bias_only_gates(x_bits, w_router, bias, k, bias_selection_only=False):
    """Selection on the unbiased logits, gates from the biased softmax."""
    logits = mo.router_logits(x_bits, w_router, bias)
    idx = mo.topk_order(logits - np.asarray(bias, np.float64), k)
    p = mo.softmax(logits)
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    return logits, idx, sel / sel.sum(axis=1, keepdims=True)


def _selection_only_ignored(x_bits, w_router, bias, k, bias_selection_only=False):
    """The variant flag dropped: gates always from the biased logits."""
    return ORIG_ROUTE(x_bits, w_router, bias, k, False)


def _shared_gate_without_sigmoid(x_bits, gate_w):
    return mo.bf16_bits_to_f64(x_bits) @ np.asarray(gate_w, dtype=np.float64)


def _dispatch_descending(idx, E):
    counts, offsets, perm, inv = ORIG_DISPATCH(idx, E)
    perm = perm.copy()
    for e in range(E):
        perm[offsets[e]:offsets[e + 1]] = perm[offsets[e]:offsets[e + 1]][::-1]
    inv = np.empty_like(inv)
    inv[perm] = np.arange(perm.size, dtype=inv.dtype)
    return counts, offsets, perm, inv


def _dispatch_inclusive_offsets(idx, E):
    counts, offsets, perm, inv = ORIG_DISPATCH(idx, E)
    return counts, np.concatenate([np.cumsum(counts), [offsets[-1]]]).astype(offsets.dtype), perm, inv


def _combine_without_shared(y_perm, inv_perm, w, k, shared_y=None):
    return ORIG_COMBINE(y_perm, inv_perm, w, k, None)


def _combine_unweighted(y_perm, inv_perm, w, k, shared_y=None):
    return ORIG_COMBINE(y_perm, inv_perm, np.ones_like(np.asarray(w, np.float64)), k, shared_y)


def _combine_slots_transposed(y_perm, inv_perm, w, k, shared_y=None):
    T = np.asarray(w).shape[0]
    inv = np.asarray(inv_perm).reshape(k, T).T.reshape(-1)
    return ORIG_COMBINE(y_perm, inv, w, k, shared_y)


def _expert_rows_token_mod_k(x_bits, perm_src, offsets, k, experts, rows=None, cache=None):
    x = mo.bf16_bits_to_f64(x_bits)
    n = int(np.asarray(offsets)[-1])
    rows = np.arange(n) if rows is None else np.asarray(rows)
    owner = np.searchsorted(np.asarray(offsets), rows, side="right") - 1
    y = np.zeros((rows.size, x.shape[1]))
    for i, r in enumerate(rows):
        ex = experts[int(owner[i])]
        wg, wu, wd = (mo.dequant_qm(m) for m in (ex.gate, ex.up, ex.down))
        _, y[i] = mo.expert_forward(wg, wu, wd, x[int(perm_src[r]) % k][None])
    return y


def _pins_pass():
    """Run every pin; True only if all of them pass."""
    try:
        for case in pins._dequant_cases():
            pins.test_dequant_golden(case)
        for case in pins._routing_cases():
            pins.test_routing_closed_form(case)
        for case in pins._routing_bias_cases():
            pins.test_routing_bias_closed_form(case)
        for case in pins._variant_cases("sel"):
            pins.test_bias_selection_only_closed_form(case)
        for case in pins._variant_cases("gate"):
            pins.test_shared_gate_closed_form(case)
        pins.test_sigmoid_gated_shared_expert_through_the_layer()
        pins.test_swiglu_expert_closed_form()
        pins.test_layer_closed_form_through_routing()
        for k in (1, 2, 3):
            pins.test_topk_equals_brute_force_subsets(k)
        pins.test_dispatch_matches_stable_sort()
        pins.test_dispatch_empty_and_degenerate()
        pins.test_sparse_oracle_equals_dense_masked(pins.wlm.WORKLOADS["tiny"])
        pins.test_sparse_oracle_equals_dense_masked(pins._mixed_small())
    except AssertionError:  # a value comparison failed (a crash would propagate and fail the test)
        return False
    return True


@pytest.mark.parametrize("target,mutant", [
    ("dequant", _swapped_nibbles),
    ("dequant", _offset7),
    ("dequant", _int2_msb_first),
    ("expert_forward", _silu_on_up),
    ("expert_forward", _down_transposed),
    ("route", _softmax_free_gates),
    ("topk_order", _ties_to_higher_index),
    ("dequant", _int8_unsigned),
    ("dequant", _int4_group16),
    ("expert_forward", _sigmoid_for_silu),
    ("route", _gates_not_renormalised),
    ("route", _bias_only_selects),
    ("route", _bias_only_gates),
    ("route", _selection_only_ignored),
    ("shared_gate", _shared_gate_without_sigmoid),
    ("dispatch", _dispatch_descending),
    ("dispatch", _dispatch_inclusive_offsets),
    ("combine", _combine_without_shared),
    ("combine", _combine_unweighted),
    ("combine", _combine_slots_transposed),
    ("expert_rows", _expert_rows_token_mod_k),
])
def test_planted_mistake_is_caught(monkeypatch, target, mutant):
    assert _pins_pass()
    monkeypatch.setattr(mo, target, mutant)
    monkeypatch.setattr(oracle, target, mutant)
    assert not _pins_pass(), f"a planted mistake in {target} went unnoticed"


@pytest.mark.parametrize("mutant", [_bias_only_selects, _bias_only_gates])
def test_bias_golden_alone_catches_bias_mistakes(monkeypatch, mutant):
    """The hand-worked bias fixture pins the bias term by itself, without the
    dense evaluation (which restates the same logit formula)."""
    monkeypatch.setattr(mo, "route", mutant)
    monkeypatch.setattr(oracle, "route", mutant)
    failed = False
    for case in pins._routing_bias_cases():
        try:
            pins.test_routing_bias_closed_form(case)
        except AssertionError:
            failed = True
    assert failed
