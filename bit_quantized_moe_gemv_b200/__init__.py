"""B200-native routed-MoE FFN step with block-quantised low-bit experts.

The compute runs in hand-written CUDA kernels for sm_100a behind a C-ABI
shared library (include/moe.h). `bit_quantized_moe_gemv_b200.lib` is the thin
ctypes binding to it; importing this package does not load the library, so
the pure-host pieces (workload generators) work without a GPU.
"""
__all__ = ["workload", "lib"]


def __getattr__(name):
    if name == "lib":
        from . import _lib as lib
        return lib
    raise AttributeError(name)
