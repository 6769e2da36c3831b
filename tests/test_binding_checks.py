"""Argument checks of the Python binding, on CPU.

The C ABI sees only pointers, so the binding checks what it cannot: device,
contiguity, element type and minimum sizes of every tensor argument. Here the
library is replaced by a recorder and the device check is turned off, so the
binding runs on CPU tensors: the argument patterns the tests, the bench and
smoke() use must pass, and malformed ones must raise before any call.
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_quantized_moe_gemv_b200 import _lib
from bit_quantized_moe_gemv_b200 import workload as wlm
from bit_quantized_moe_gemv_b200.device import DeviceExperts, bf16_tensor


class _Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append(name)
            return 0
        return fn


@pytest.fixture
def rec(monkeypatch):
    r = _Recorder()
    monkeypatch.setattr(_lib, "LIB", r)
    monkeypatch.setattr(_lib, "REQUIRE_CUDA", False)
    return r


@pytest.fixture(scope="module")
def tiny():
    wl = wlm.WORKLOADS["tiny"]
    lay = wlm.gen_layer(wl)
    return wl, lay, DeviceExperts(lay.experts, "cpu"), DeviceExperts([lay.shared], "cpu")


def _i32(*shape):
    return torch.empty(shape, dtype=torch.int32)


def _f32(*shape):
    return torch.empty(shape, dtype=torch.float32)


def _bf16(*shape):
    return torch.empty(shape, dtype=torch.bfloat16)


def _ws():
    return torch.empty(4096, dtype=torch.uint8)


def test_four_calls_and_layer_accept_the_test_patterns(rec, tiny):
    wl, lay, ex, sh = tiny
    T, k, E, H, I = wl.T, wl.k, wl.E, wl.H, wl.I
    x = bf16_tensor(wlm.gen_x(wl), "cpu")
    w_r = torch.from_numpy(lay.w_router)
    for bias, stride in ((torch.zeros(E), 0), (torch.zeros(T, E), E), (None, 0)):
        _lib.route(x, w_r, bias, stride, k, _i32(T, k), _f32(T, k), _ws(), logits=_f32(T, E), stream=0)
        _lib.layer(x, I, E, k, w_r, bias, stride, ex.table, sh.table, _i32(T, k), _f32(T, k), _bf16(T, H), _ws(),
                   stream=0)
        _lib.layer(x, I, E, k, w_r, bias, stride, ex.table, sh.table, _i32(T, k), _f32(T, k), _bf16(T, H), _ws(),
                   stream=0, logits=_f32(T, E))
        _lib.layer_decode_noalloc(x, I, E, k, w_r, bias, stride, ex.table, None, _i32(T, k), _f32(T, k),
                                  _bf16(T, H), stream=0, logits=_f32(T, E))
    _lib.dispatch(_i32(T, k), E, _i32(E), _i32(E + 1), _i32(T * k), _i32(T * k), _ws(), stream=0)
    _lib.expert_ffn(x, I, k, E, _i32(T * k), _i32(E + 1), _i32(E), ex.table, _bf16(T * k, H), _ws(), stream=0)
    _lib.combine(_bf16(T * k, H), _i32(T * k), _f32(T, k), I, x, sh.table, _bf16(T, H), _ws(), stream=0)
    _lib.combine(_bf16(T * k, H), _i32(T * k), _f32(T, k), I, None, None, _bf16(T, H), _ws(), stream=0)
    _lib.reset_status(_ws(), stream=0)
    assert rec.calls.count("moe_route") == 3 and rec.calls.count("moe_layer") == 6
    assert rec.calls.count("moe_combine") == 2 and "moe_reset_status" in rec.calls


def test_slices_of_stacked_step_buffers_pass(rec, tiny):
    # the bench keeps every step's tensors in one buffer and passes [s] / [s, layer] slices
    wl, lay, ex, sh = tiny
    T, k, E, H, I = wl.T, wl.k, wl.E, wl.H, wl.I
    xs = _bf16(3, 2, T, H)
    idx, gw, out = _i32(3, 2, T, k), _f32(3, 2, T, k), _bf16(3, 2, T, H)
    _lib.layer(xs[1, 1], I, E, k, torch.from_numpy(lay.w_router), torch.zeros(E), 0, ex.table, sh.table, idx[1, 1],
               gw[1, 1], out[1, 1], _ws(), stream=0)
    assert rec.calls == ["moe_layer"]


def test_zero_tokens_pass(rec):
    _lib.dispatch(_i32(0, 2), 8, _i32(8), _i32(9), _i32(0), _i32(0), _ws(), stream=0)
    assert rec.calls == ["moe_dispatch"]


@pytest.mark.parametrize("case", ["transposed_x", "f32_x", "short_out", "short_counts", "stride_below_E",
                                  "short_bias", "no_table", "short_table", "router_width", "i64_idx", "no_ws",
                                  "short_logits"])
def test_malformed_arguments_raise_before_the_call(rec, tiny, case):
    wl, lay, ex, sh = tiny
    T, k, E, H, I = wl.T, wl.k, wl.E, wl.H, wl.I
    a = dict(x=bf16_tensor(wlm.gen_x(wl), "cpu"), w_router=torch.from_numpy(lay.w_router), bias=torch.zeros(E),
             stride=0, table=ex.table, idx=_i32(T, k), w=_f32(T, k), out=_bf16(T, H), ws=_ws(), logits=None)
    if case == "transposed_x":
        a["x"] = _bf16(H, T).t()
    elif case == "f32_x":
        a["x"] = _f32(T, H)
    elif case == "short_out":
        a["out"] = _bf16(T - 1, H)
    elif case == "stride_below_E":
        a["bias"], a["stride"] = torch.zeros(T, E), E - 1
    elif case == "short_bias":
        a["bias"], a["stride"] = torch.zeros(T - 1, E), E
    elif case == "no_table":
        a["table"] = None
    elif case == "short_table":
        a["table"] = ex.table[:-1]
    elif case == "router_width":
        a["w_router"] = _f32(E, H + 1)
    elif case == "i64_idx":
        a["idx"] = torch.empty((T, k), dtype=torch.int64)
    elif case == "no_ws":
        a["ws"] = None
    elif case == "short_logits":
        a["logits"] = _f32(T, E - 1)
    if case == "short_counts":
        with pytest.raises((ValueError, TypeError)):
            _lib.dispatch(_i32(T, k), E, _i32(E - 1), _i32(E + 1), _i32(T * k), _i32(T * k), _ws(), stream=0)
    else:
        with pytest.raises((ValueError, TypeError, AttributeError)):
            _lib.layer(a["x"], I, E, k, a["w_router"], a["bias"], a["stride"], a["table"], sh.table, a["idx"], a["w"],
                       a["out"], a["ws"], stream=0, logits=a["logits"])
    assert rec.calls == []


def test_host_tensors_are_refused(monkeypatch):
    monkeypatch.setattr(_lib, "LIB", _Recorder())
    with pytest.raises(ValueError, match="CUDA"):
        _lib.dispatch(_i32(2, 2), 4, _i32(4), _i32(5), _i32(4), _i32(4), _ws(), stream=0)


def test_descriptor_size_matches_the_table_stride(tiny):
    wl, _, ex, _ = tiny
    assert ex.table.numel() == wl.E * ctypes.sizeof(_lib.ExpertC)
    assert ctypes.sizeof(_lib.ExpertC) == 3 * ctypes.sizeof(_lib.QMatrixC)
    assert np.dtype(np.uint8).itemsize == ex.table.element_size()
