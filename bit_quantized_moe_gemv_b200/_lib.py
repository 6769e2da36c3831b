"""ctypes binding of libmoe_b200.so (include/moe.h).

Argument marshalling only: every function takes torch tensors (device
memory) or plain integers, checks what the C ABI cannot see (each tensor is
on a CUDA device, contiguous, of the element type the header names and large
enough for the call), passes addresses and sizes to the C ABI and turns a
non-zero status into a MoeError. No step of the MoE computation runs
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
           "moe_set_wait_cycles", "moe_status_string")


class QMatrixC(ctypes.Structure):
    _fields_ = [("qtype", c_i32), ("rows", c_i32), ("cols", c_i32), ("group", c_i32),
                ("codes", c_vp), ("scales", c_vp), ("mins", c_vp)]


class ExpertC(ctypes.Structure):
    _fields_ = [("gate", QMatrixC), ("up", QMatrixC), ("down", QMatrixC)]


class OptionsC(ctypes.Structure):
    _fields_ = [("flags", ctypes.c_uint32), ("shared_gate", c_vp), ("heat", c_vp)]


MOE_BIAS_SELECTION_ONLY = 1


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
        "moe_route": (c_i32, [c_vp, c_i32, c_i32, c_vp, c_i32, c_vp, c_i64, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz,
                              c_vp]),
        "moe_dispatch": (c_i32, [c_vp, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
        "moe_expert_ffn": (c_i32, [c_vp, c_i32, c_i32, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz,
                                   c_vp]),
        "moe_combine": (c_i32, [c_vp, c_vp, c_vp, c_i32, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz,
                                c_vp]),
        "moe_layer": (c_i32, [c_vp, c_i32, c_i32, c_i32, c_i32, c_i32, c_vp, c_vp, c_i64, c_vp, c_vp, c_vp, c_vp,
                              c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
        "moe_layer_decode_noalloc": (c_i32, [c_vp, c_i32, c_i32, c_i32, c_i32, c_i32, c_vp, c_vp, c_i64, c_vp,
                                             c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
        "moe_reset_status": (c_i32, [c_vp, c_vp]),
        "moe_get_status": (c_i32, [c_vp, c_vp, ctypes.POINTER(c_i32)]),
        "moe_launch_count": (ctypes.c_uint64, []),
        "moe_set_wait_cycles": (c_i64, [c_i64]),
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


def set_wait_cycles(cycles: int) -> int:
    """Budget of every bounded wait of later fused decode launches (testing
    the failure path); negative restores the default. Returns the previous."""
    return int(LIB.moe_set_wait_cycles(int(cycles)))


def status_string(st: int) -> str:
    return LIB.moe_status_string(int(st)).decode()


def _check(fn, st):
    if st != MOE_OK:
        raise MoeError(fn, st)


# Device-tensor arguments must live on a CUDA device (a CPU test of these
# checks turns this off; no call reaches the library that way).
REQUIRE_CUDA = True

_KINDS = {  # element kind in include/moe.h -> accepted torch dtype names
    "bf16": ("bfloat16", "int16", "uint16"),  # bf16 bit patterns
    "f32": ("float32",),
    "i32": ("int32",),
    "u8": ("uint8",),
}


def _dev(t, name, kind, numel=0, optional=False):
    """Address of a device-tensor argument after the checks the C ABI cannot
    make: a CUDA tensor, contiguous, of the element type the header names and
    holding at least the `numel` elements the call touches. None is passed as
    NULL only where the header allows it."""
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name}: required (the call takes no NULL here)")
    if REQUIRE_CUDA and not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor, got one on {t.device}")
    if str(t.dtype).replace("torch.", "") not in _KINDS[kind]:
        raise TypeError(f"{name}: dtype {t.dtype} where the call takes {kind}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{name}: {t.numel()} elements, the call needs {numel}")
    return ctypes.c_void_p(t.data_ptr())


def _table(t, name, n, optional=False):
    """A device array of n moe_expert descriptors (uint8 bytes)."""
    return _dev(t, name, "u8", n * ctypes.sizeof(ExpertC), optional)


def _ws(ws):
    return _dev(ws, "ws", "u8")


def _bias(bias, T, E, stride):
    if stride < 0 or (stride > 0 and stride < E):
        raise ValueError(f"bias_row_stride {stride}: 0 (one row for all tokens) or at least E = {E}")
    return _dev(bias, "bias", "f32", E if stride == 0 or T == 0 else (T - 1) * stride + E, optional=True)


def _shape2(t, name, cols=None):
    if t.dim() != 2 or (cols is not None and t.shape[1] != cols):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected [rows, {cols if cols is not None else 'cols'}]")
    return t.shape


def _opts(H, bias_selection_only=False, shared_gate=None, heat=None, E=0):
    """The moe_options of a call (None = the defaults: NULL). shared_gate is a
    device fp32 [H] tensor, heat a device int32/uint32 [E] counter tensor the
    call adds its picks to; the struct is read on the host during the call."""
    if not bias_selection_only and shared_gate is None and heat is None:
        return None
    g = _dev(shared_gate, "shared_gate", "f32", H, optional=True)
    hp = _dev(heat, "heat", "i32", E, optional=True)
    return ctypes.byref(OptionsC(MOE_BIAS_SELECTION_ONLY if bias_selection_only else 0, g, hp))


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


def route(x, w_router, bias, bias_row_stride, k, topk_idx, topk_w, ws, logits=None, stream=None,
          bias_selection_only=False, heat=None):
    T, H = _shape2(x, "x")
    E = _shape2(w_router, "w_router", H)[0]
    _check("moe_route", LIB.moe_route(_dev(x, "x", "bf16"), T, H, _dev(w_router, "w_router", "f32"), E,
                                      _bias(bias, T, E, bias_row_stride), bias_row_stride, k,
                                      _dev(topk_idx, "topk_idx", "i32", T * k), _dev(topk_w, "topk_w", "f32", T * k),
                                      _dev(logits, "logits", "f32", T * E, optional=True),
                                      _opts(H, bias_selection_only, heat=heat, E=E), _ws(ws), ws.numel(),
                                      _stream(stream)))


def dispatch(topk_idx, E, counts, offsets, perm_src, inv_perm, ws, stream=None):
    T, k = _shape2(topk_idx, "topk_idx")
    _check("moe_dispatch", LIB.moe_dispatch(_dev(topk_idx, "topk_idx", "i32"), T, k, E,
                                            _dev(counts, "counts", "i32", E), _dev(offsets, "offsets", "i32", E + 1),
                                            _dev(perm_src, "perm_src", "i32", T * k),
                                            _dev(inv_perm, "inv_perm", "i32", T * k), _ws(ws), ws.numel(),
                                            _stream(stream)))


def expert_ffn(x, I, k, E, perm_src, offsets, counts, experts_table, y_perm, ws, stream=None):
    T, H = _shape2(x, "x")
    _check("moe_expert_ffn", LIB.moe_expert_ffn(_dev(x, "x", "bf16"), T, H, I, k, E,
                                                _dev(perm_src, "perm_src", "i32", T * k),
                                                _dev(offsets, "offsets", "i32", E + 1), _dev(counts, "counts", "i32", E),
                                                _table(experts_table, "experts_table", E),
                                                _dev(y_perm, "y_perm", "bf16", T * k * H), _ws(ws), ws.numel(),
                                                _stream(stream)))


def combine(y_perm, inv_perm, topk_w, I, x, shared_table, out, ws, stream=None, shared_gate=None):
    T, k = _shape2(topk_w, "topk_w")
    H = _shape2(out, "out")[1]
    _check("moe_combine", LIB.moe_combine(_dev(y_perm, "y_perm", "bf16", T * k * H),
                                          _dev(inv_perm, "inv_perm", "i32", T * k), _dev(topk_w, "topk_w", "f32"),
                                          T, H, I, k, _dev(x, "x", "bf16", T * H, optional=shared_table is None),
                                          _table(shared_table, "shared_table", 1, optional=True),
                                          _dev(out, "out", "bf16", T * H), _opts(H, shared_gate=shared_gate), _ws(ws),
                                          ws.numel(), _stream(stream)))


def layer(x, I, E, k, w_router, bias, bias_row_stride, experts_table, shared_table, topk_idx, topk_w, out, ws,
          stream=None, logits=None, bias_selection_only=False, shared_gate=None, heat=None):
    T, H = _shape2(x, "x")
    _shape2(w_router, "w_router", H)
    _check("moe_layer", LIB.moe_layer(_dev(x, "x", "bf16"), T, H, I, E, k, _dev(w_router, "w_router", "f32", E * H),
                                      _bias(bias, T, E, bias_row_stride), bias_row_stride,
                                      _table(experts_table, "experts_table", E),
                                      _table(shared_table, "shared_table", 1, optional=True),
                                      _dev(topk_idx, "topk_idx", "i32", T * k), _dev(topk_w, "topk_w", "f32", T * k),
                                      _dev(logits, "logits", "f32", T * E, optional=True),
                                      _dev(out, "out", "bf16", T * H),
                                      _opts(H, bias_selection_only, shared_gate, heat, E), _ws(ws), ws.numel(),
                                      _stream(stream)))


def layer_decode_noalloc(x, I, E, k, w_router, bias, bias_row_stride, experts_table, shared_table, topk_idx,
                         topk_w, out, stream=None, logits=None, bias_selection_only=False, shared_gate=None,
                         heat=None):
    """moe_layer_decode_noalloc: the fused decode step without a workspace."""
    T, H = _shape2(x, "x")
    _shape2(w_router, "w_router", H)
    _check("moe_layer_decode_noalloc",
           LIB.moe_layer_decode_noalloc(_dev(x, "x", "bf16"), T, H, I, E, k, _dev(w_router, "w_router", "f32", E * H),
                                        _bias(bias, T, E, bias_row_stride), bias_row_stride,
                                        _table(experts_table, "experts_table", E),
                                        _table(shared_table, "shared_table", 1, optional=True),
                                        _dev(topk_idx, "topk_idx", "i32", T * k),
                                        _dev(topk_w, "topk_w", "f32", T * k),
                                        _dev(logits, "logits", "f32", T * E, optional=True),
                                        _dev(out, "out", "bf16", T * H),
                                        _opts(H, bias_selection_only, shared_gate, heat, E), _stream(stream)))


def reset_status(ws, stream=None):
    _check("moe_reset_status", LIB.moe_reset_status(_ws(ws), _stream(stream)))


def get_status(ws, stream=None) -> int:
    v = c_i32(0)
    _check("moe_get_status", LIB.moe_get_status(_ws(ws), _stream(stream), ctypes.byref(v)))
    return int(v.value)
