"""Host-only checks of the C ABI: the library loads on a machine without a GPU,
exports every symbol include/moe.h declares, its struct layout matches the
ctypes binding, and argument checks reject bad calls before any CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    from bit_quantized_moe_gemv_b200 import build
    build.build()
    from bit_quantized_moe_gemv_b200 import _lib
    return _lib


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", src)))


def test_header_declares_the_binding_exports(lib):
    assert _declared() == sorted(lib.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib._build.LIB], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (moe_\w+)", out))
    for name in _declared():
        assert name in exported, name
        assert hasattr(lib.LIB, name)


def test_struct_layout_matches_c(tmp_path, lib):
    c = tmp_path / "layout.c"
    c.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "moe.h"\nint main(void){'
                 'printf("%zu %zu %zu %zu %zu %zu\\n", sizeof(moe_qmatrix), sizeof(moe_expert),'
                 'offsetof(moe_qmatrix, codes), offsetof(moe_qmatrix, mins), offsetof(moe_expert, up),'
                 'offsetof(moe_expert, down)); return 0;}\n')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(c), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()]
    Q, X = lib.QMatrixC, lib.ExpertC
    assert got == [ctypes.sizeof(Q), ctypes.sizeof(X), Q.codes.offset, Q.mins.offset, X.up.offset, X.down.offset]


def test_workspace_size_limits(lib):
    assert lib.workspace_size(4, 256, 128, 16, 2) > 0
    assert lib.workspace_size(8192, 2048, 768, 512, 10) > 8192 * 10 * 2048 * 2
    for bad in [(4, 250, 128, 16, 2), (4, 256, 100, 16, 2), (4, 256, 128, 16, 17), (4, 256, 128, 2048, 2),
                (-1, 256, 128, 16, 2), (4, 256, 128, 0, 1), (4, 256, 128, 100, 65)]:
        assert lib.workspace_size(*bad) == 0, bad


def test_status_strings(lib):
    for st in range(7):
        assert len(lib.status_string(st)) > 0
    assert lib.status_string(99) == "unknown status"


def test_host_argument_checks_without_gpu(lib):
    L = lib.LIB
    # Null activations with T > 0: rejected before any CUDA call.
    assert L.moe_route(None, 4, 256, None, 16, None, 0, 2, None, None, None, None, None, 0, None) == 1
    # k > E.
    assert L.moe_route(None, 4, 256, None, 4, None, 0, 5, None, None, None, None, None, 0, None) == 1
    # Bad bias stride (nonzero but < E).
    assert L.moe_layer(None, 4, 256, 128, 16, 2, None, None, 3, None, None, None, None, None, None, None, None, 0, None) == 1
    assert L.moe_dispatch(None, 4, 2, 0, None, None, None, None, None, 0, None) == 1
    assert L.moe_expert_ffn(None, 4, 256, 100, 2, 16, None, None, None, None, None, None, 0, None) == 1
    assert L.moe_combine(None, None, None, 4, 256, 128, 2, None, None, None, None, None, 0, None) == 1
    assert L.moe_reset_status(None, None) == 1
    v = ctypes.c_int32(7)
    assert L.moe_get_status(None, None, ctypes.byref(v)) == 1
    # Misaligned workspace pointer.
    assert L.moe_reset_status(ctypes.c_void_p(0x1001), None) == 1
    # T = 0 is a no-op that succeeds without touching the device.
    assert L.moe_route(None, 0, 256, None, 16, None, 0, 2, None, None, None, None, None, 0, None) == 0
    assert L.moe_layer(None, 0, 256, 128, 16, 2, None, None, 0, None, None, None, None, None, None, None, None, 0, None) == 0


def test_wait_budget_setter_round_trip(lib):
    default = lib.set_wait_cycles(12345)
    assert default == 2000000000
    assert lib.set_wait_cycles(-1) == 12345
    assert lib.set_wait_cycles(-1) == default
