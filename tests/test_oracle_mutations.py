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


def _softmax_free_gates(x_bits, w_router, bias, k):
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


def _pins_pass():
    """Run every pin; True only if all of them pass."""
    try:
        for case in pins._dequant_cases():
            pins.test_dequant_golden(case)
        for case in pins._routing_cases():
            pins.test_routing_closed_form(case)
        pins.test_swiglu_expert_closed_form()
        pins.test_layer_closed_form_through_routing()
        for k in (1, 2, 3):
            pins.test_topk_equals_brute_force_subsets(k)
    except (AssertionError, ValueError):
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
])
def test_planted_mistake_is_caught(monkeypatch, target, mutant):
    assert _pins_pass()
    monkeypatch.setattr(mo, target, mutant)
    monkeypatch.setattr(oracle, target, mutant)
    assert not _pins_pass(), f"a planted mistake in {target} went unnoticed"
