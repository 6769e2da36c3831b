"""ctypes binding of libmoe_b200.so (include/moe.h).

Argument marshalling only: every function takes torch tensors (device
memory) or plain integers, passes their addresses and sizes to the C ABI and
turns a non-zero status into a MoeError. No step of the MoE computation runs
here. If the library is missing this module raises at import: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

from . import build as _build

c_i32, c_i64, c_sz, c_vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE_TOO_SMALL",
                4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_FAULT", 6: "MOE_ERR_TIMEOUT"}

# Every symbol include/moe.h declares (checked by the CPU test suite).
EXPORTS = ("moe_workspace_size", "moe_route", "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_layer",
           "moe_layer_decode_noalloc", "moe_reset_status", "moe_get_status", "moe_launch_count",
           "moe_status_string")


class QMatrixC(ctypes.Structure):
    _fields_ = [("qtype", c_i32), ("rows", c_i32), ("cols", c_i32), ("group", c_i32),
                ("codes", c_vp), ("scales", c_vp), ("mins", c_vp)]


class ExpertC(ctypes.Structure):
    _fields_ = [("gate", QMatrixC), ("up", QMatrixC), ("down", QMatrixC)]


class MoeError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} returned {STATUS_NAMES.get(status, status)}: {status_string(status)}")


def _load():
    path = _build.LIB
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m bit_quantized_moe_gemv_b200.build` "
                          "(there is no fallback implementation)")
    lib = ctypes.CDLL(path)
    sig = {
        "moe_workspace_size": (c_sz, [c_i32] * 5),
        "moe_route": (c_i32, [c_vp, c_i32, c_i32, c_vp, c_i32, c_vp, c_i64, c_i32, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
        "moe_dispatch": (c_i32, [c_vp, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
        "moe_expert_ffn": (c_i32, [c_vp, c_i32, c_i32, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz,
                                   c_vp]),
        "moe_combine": (c_i32, [c_vp, c_vp, c_vp, c_i32, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
        "moe_layer": (c_i32, [c_vp, c_i32, c_i32, c_i32, c_i32, c_i32, c_vp, c_vp, c_i64, c_vp, c_vp, c_vp, c_vp,
                              c_vp, c_vp, c_sz, c_vp]),
        "moe_layer_decode_noalloc": (c_i32, [c_vp, c_i32, c_i32, c_i32, c_i32, c_i32, c_vp, c_vp, c_i64, c_vp,
                                             c_vp, c_vp, c_vp, c_vp, c_vp]),
        "moe_reset_status": (c_i32, [c_vp, c_vp]),
        "moe_get_status": (c_i32, [c_vp, c_vp, ctypes.POINTER(c_i32)]),
        "moe_launch_count": (ctypes.c_uint64, []),
        "moe_status_string": (ctypes.c_char_p, [c_i32]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    return lib


LIB = _load()


def launch_count() -> int:
    """Kernels this library has launched in this process (host-side count)."""
    return int(LIB.moe_launch_count())


def status_string(st: int) -> str:
    return LIB.moe_status_string(int(st)).decode()


def _check(fn, st):
    if st != MOE_OK:
        raise MoeError(fn, st)


def _p(t):
    """Address of a tensor (None -> NULL)."""
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def workspace_size(T, H, I, E, k) -> int:
    return int(LIB.moe_workspace_size(T, H, I, E, k))


def new_workspace(T, H, I, E, k, device="cuda"):
    """Allocate a workspace (torch uint8) and clear its status word."""
    import torch
    n = workspace_size(T, H, I, E, k)
    if n == 0:
        raise MoeError("moe_workspace_size", 1)
    ws = torch.empty(n + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + n]
    reset_status(ws)
    return ws


def route(x, w_router, bias, bias_row_stride, k, topk_idx, topk_w, ws, logits=None, stream=None):
    T, H = x.shape
    E = w_router.shape[0]
    _check("moe_route", LIB.moe_route(_p(x), T, H, _p(w_router), E, _p(bias), bias_row_stride, k, _p(topk_idx),
                                      _p(topk_w), _p(logits), _p(ws), ws.numel(), _stream(stream)))


def dispatch(topk_idx, E, counts, offsets, perm_src, inv_perm, ws, stream=None):
    T, k = topk_idx.shape
    _check("moe_dispatch", LIB.moe_dispatch(_p(topk_idx), T, k, E, _p(counts), _p(offsets), _p(perm_src),
                                            _p(inv_perm), _p(ws), ws.numel(), _stream(stream)))


def expert_ffn(x, I, k, E, perm_src, offsets, counts, experts_table, y_perm, ws, stream=None):
    T, H = x.shape
    _check("moe_expert_ffn", LIB.moe_expert_ffn(_p(x), T, H, I, k, E, _p(perm_src), _p(offsets), _p(counts),
                                                _p(experts_table), _p(y_perm), _p(ws), ws.numel(), _stream(stream)))


def combine(y_perm, inv_perm, topk_w, I, x, shared_table, out, ws, stream=None):
    T, k = topk_w.shape
    H = out.shape[1]
    _check("moe_combine", LIB.moe_combine(_p(y_perm), _p(inv_perm), _p(topk_w), T, H, I, k, _p(x), _p(shared_table),
                                          _p(out), _p(ws), ws.numel(), _stream(stream)))


def layer(x, I, E, k, w_router, bias, bias_row_stride, experts_table, shared_table, topk_idx, topk_w, out, ws,
          stream=None):
    T, H = x.shape
    _check("moe_layer", LIB.moe_layer(_p(x), T, H, I, E, k, _p(w_router), _p(bias), bias_row_stride,
                                      _p(experts_table), _p(shared_table), _p(topk_idx), _p(topk_w), _p(out), _p(ws),
                                      ws.numel(), _stream(stream)))


def layer_decode_noalloc(x, I, E, k, w_router, bias, bias_row_stride, experts_table, shared_table, topk_idx,
                         topk_w, out, stream=None):
    """moe_layer_decode_noalloc: the fused decode step without a workspace."""
    T, H = x.shape
    _check("moe_layer_decode_noalloc",
           LIB.moe_layer_decode_noalloc(_p(x), T, H, I, E, k, _p(w_router), _p(bias), bias_row_stride,
                                        _p(experts_table), _p(shared_table), _p(topk_idx), _p(topk_w), _p(out),
                                        _stream(stream)))


def reset_status(ws, stream=None):
    _check("moe_reset_status", LIB.moe_reset_status(_p(ws), _stream(stream)))


def get_status(ws, stream=None) -> int:
    v = c_i32(0)
    _check("moe_get_status", LIB.moe_get_status(_p(ws), _stream(stream), ctypes.byref(v)))
    return int(v.value)
