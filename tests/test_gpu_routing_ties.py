"""Exact ties in the routing, on the GPU, through the C ABI.

The pages fix no tie rule; this library's reading is that the k picks are
ordered by descending logit and equal logits go to the lower expert index
(the selection of the telli.sh page "Strata 与 Qwen3.8-Flash-Next：如何在个人电脑上
运行 180B 级模型", section "稀疏架构创造了机会": k of E routed experts per token).
Exact ties are made on purpose, so that the expected picks are known without
any tolerance:
  * W_r = 0 and b = 0: every logit is exactly 0, so the picks are 0..k-1
    and every gate is 1/k;
  * duplicated router rows with equal bias: their logits are computed by the
    same arithmetic and are bit-identical, so each tied group must come out
    in ascending index order, and a group cut by the k-th place must keep its
    lowest indices.
Every router path runs: the fused decode kernel (moe_layer, T <= 4), the
decode GEMV router (moe_route, T <= 8), the tensor-core router (T > 8, E a
multiple of 128) and the general tiled router (T > 8, other E); the prefill
moe_layer (T > 4) routes through the latter two.
"""
import numpy as np
import pytest

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


# (name, T, H, I, E, k, call): call "layer" = moe_layer, "route" = moe_route
PATHS = [
    ("fused_decode", 2, 1024, 512, 512, 10, "layer"),
    ("gemv_router", 3, 512, 256, 64, 8, "route"),
    ("tc_router", 20, 512, 256, 128, 8, "route"),
    ("tiled_router", 20, 256, 128, 40, 6, "route"),
    ("prefill_layer_tc", 20, 512, 256, 128, 8, "layer"),
    ("prefill_layer_tiled", 20, 256, 128, 40, 6, "layer"),
]


def _run(L, name, T, H, I, E, k, call, w_router, bias, xb):
    import torch

    from bit_quantized_moe_gemv_b200.device import bf16_tensor
    x = bf16_tensor(xb)
    wr = torch.from_numpy(np.ascontiguousarray(w_router, dtype=np.float32)).cuda()
    b = pu.bias_tensor(bias)
    idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), -1.0, dtype=torch.float32, device="cuda")
    lg = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda")
    ws = L.new_workspace(T, H, I, E, k)
    if call == "route":
        L.route(x, wr, b, 0, k, idx, w, ws, logits=lg)
    else:
        wl = wlm.Workload(f"ties_{name}", T=T, H=H, I=I, E=E, k=k, seed=5)
        dev = pu.upload_layer(wlm.gen_layer(wl))
        out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
        L.layer(x, I, E, k, wr, b, 0, dev["experts"].table, dev["shared"].table, idx, w, out, ws, logits=lg)
    torch.cuda.synchronize()
    assert L.get_status(ws) == 0
    return idx.cpu().numpy(), w.cpu().numpy(), lg.cpu().numpy()


@pytest.mark.parametrize("path", PATHS, ids=[p[0] for p in PATHS])
def test_all_zero_router_picks_first_k_with_equal_gates(L, path):
    name, T, H, I, E, k, call = path
    rng = np.random.default_rng(31)
    xb = wlm.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    idx, w, lg = _run(L, name, T, H, I, E, k, call, np.zeros((E, H)), np.zeros(E), xb)
    assert np.all(lg == 0.0)
    np.testing.assert_array_equal(idx, np.tile(np.arange(k, dtype=np.int32), (T, 1)))
    # softmax of k equal logits: each gate is 1/k, to the last fp32 ulp
    one_over_k = np.float32(1.0) / np.float32(k)
    assert np.all(np.abs(w - one_over_k) <= np.spacing(one_over_k)), w


@pytest.mark.parametrize("path", PATHS, ids=[p[0] for p in PATHS])
def test_duplicated_router_rows_resolve_to_lower_index(L, path):
    name, T, H, I, E, k, call = path
    rng = np.random.default_rng(32)
    xb = wlm.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    w_r = (rng.standard_normal((E, H)) * 0.02).astype(np.float32)
    bias = np.zeros(E, dtype=np.float32)
    # two tied groups far above the rest (random rows give |logit| < ~5):
    # ids spread over the whole range so the decode kernel's 32-logit
    # chunks each hold part of a group
    top = sorted({3, E // 2 + 1, E - 2})
    mid = sorted({1, E // 4 + 3, (3 * E) // 4, E - 1} - set(top))
    w_r[top] = w_r[top[0]]
    w_r[mid] = w_r[mid[0]]
    bias[top] = 40.0
    bias[mid] = 20.0
    idx, w, lg = _run(L, name, T, H, I, E, k, call, w_r, bias, xb)
    for t in range(T):
        assert len(set(lg[t, top].tolist())) == 1 and len(set(lg[t, mid].tolist())) == 1, "duplicates must tie exactly"
    n = min(k, len(top) + len(mid))
    for t in range(T):
        assert idx[t, :n].tolist() == (top + mid)[:n], (t, idx[t])
        # equal logits give bit-identical gates
        assert len(set(w[t, :len(top)].tolist())) == 1
        assert len(set(w[t, len(top):n].tolist())) == 1
    # the whole selection: the oracle's top-k on the device's own logits, and
    # a valid top-k of the fp64 logits (every token here has exact ties)
    pu.check_routing(idx, w, lg, xb, w_r, bias, k)
