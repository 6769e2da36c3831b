"""Router variants on the GPU against the fp64 oracle, through the C ABI.

Two readings of what the pages leave open about the router and the shared
expert (the telli.sh page "Strata 与 Qwen3.8-Flash-Next：如何在个人电脑上运行 180B
级模型", section "稀疏架构创造了机会", names both without their functions):
  * MOE_BIAS_SELECTION_ONLY: the bias picks the experts, the gates are the
    softmax of the unbiased logits renormalised over the picks;
  * a sigmoid-gated shared expert: its output is scaled by sigma(g . x).
Each runs on every path of moe_layer (the fused decode kernel, the tcgen05
prefill path, the general kernels) and on the four-call composition, with
the same bars as the default router: routing exact on the device's logits
and equal to the fp64 oracle's outside near-ties, outputs within the float
tolerance.
"""
import numpy as np
import pytest

import oracle
from bit_quantized_moe_gemv_b200 import workload as wlm
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

CASES = {
    "fused_T2": wlm.Workload("var_fused_T2", T=2, H=1024, I=512, E=64, k=6, zipf_s=1.1, seed=41),
    "fused_e256_T1": wlm.Workload("var_fused_e256", T=1, H=2048, I=768, E=256, k=8, zipf_s=1.1, seed=42),
    "tc_T300": wlm.Workload("var_tc", T=300, H=512, I=256, E=128, k=4, zipf_s=0.9, seed=43),
    "simt_T37": wlm.Workload("var_simt", T=37, H=192, I=128, E=40, k=3, zipf_s=0.6, seed=45,
                             shared_qtype=wlm.Q_INT8_PER_CHANNEL),
}
VARIANTS = {"selection_only": (True, False), "shared_gate": (False, True), "both": (True, True)}


@pytest.fixture(scope="module")
def L():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_quantized_moe_gemv_b200 import build
    build.build()
    from bit_quantized_moe_gemv_b200 import _lib
    return _lib


def _gate_vector(wl):
    rng = np.random.default_rng(1000 + wl.seed)
    return (rng.standard_normal(wl.H) * 0.02).astype(np.float32)


@pytest.mark.parametrize("variant", list(VARIANTS))
@pytest.mark.parametrize("case", list(CASES))
def test_layer_variant_matches_oracle(L, case, variant):
    import torch

    from bit_quantized_moe_gemv_b200.device import bf16_bits, bf16_tensor
    sel_only, gated = VARIANTS[variant]
    wl = CASES[case]
    lay = wlm.gen_layer(wl)
    dev = pu.upload_layer(lay)
    bias, stride = wlm.gen_bias(wl)
    xb = wlm.gen_x(wl)
    g = _gate_vector(wl) if gated else None
    x = bf16_tensor(xb)
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    lg = torch.empty((wl.T, wl.E), dtype=torch.float32, device="cuda")
    out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    ws = L.new_workspace(wl.T, wl.H, wl.I, wl.E, wl.k)
    L.layer(x, wl.I, wl.E, wl.k, dev["w_router"], pu.bias_tensor(bias), stride, dev["experts"].table,
            dev["shared"].table, idx, w, out, ws, logits=lg, bias_selection_only=sel_only,
            shared_gate=torch.from_numpy(g).cuda() if gated else None)
    torch.cuda.synchronize()
    assert L.get_status(ws) == 0
    gi, gw = idx.cpu().numpy(), w.cpu().numpy()
    pu.check_routing(gi, gw, lg.cpu().numpy(), xb, lay.w_router, bias, wl.k, bias_selection_only=sel_only)
    # oracle on the device's picks (equal to its own outside near-ties), gates
    # from the fp64 logits of the variant
    gate_logits = oracle.router_logits(xb, lay.w_router, np.zeros(1) if sel_only else bias)
    ref = oracle.moe_layer(xb, lay.w_router, bias, wl.k, lay.experts, lay.shared,
                           routing=(gi, pu.oracle_gates_for(gate_logits, gi)), bias_selection_only=sel_only,
                           shared_gate_w=g)
    np.testing.assert_allclose(gw, pu.oracle_gates_for(gate_logits, gi), rtol=1e-5, atol=1e-6)
    pu.assert_close(pu.bf16_to_f64(bf16_bits(out)), ref["out"], f"{case}/{variant}")


@pytest.mark.parametrize("case", ["fused_T2", "tc_T300"])
def test_four_calls_with_variants_match_oracle(L, case):
    """moe_route with the selection-only bias, then dispatch, experts, and
    moe_combine with the gated shared expert."""
    import torch

    from bit_quantized_moe_gemv_b200.device import bf16_bits, bf16_tensor
    wl = CASES[case]
    lay = wlm.gen_layer(wl)
    dev = pu.upload_layer(lay)
    bias, stride = wlm.gen_bias(wl)
    xb = wlm.gen_x(wl)
    g = _gate_vector(wl)
    T, k, E, H = wl.T, wl.k, wl.E, wl.H
    x = bf16_tensor(xb)
    ws = L.new_workspace(T, H, wl.I, E, k)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    lg = torch.empty((T, E), dtype=torch.float32, device="cuda")
    L.route(x, dev["w_router"], pu.bias_tensor(bias), stride, k, idx, w, ws, logits=lg, bias_selection_only=True)
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    L.dispatch(idx, E, counts, offsets, perm, inv, ws)
    y = torch.empty((T * k, H), dtype=torch.bfloat16, device="cuda")
    L.expert_ffn(x, wl.I, k, E, perm, offsets, counts, dev["experts"].table, y, ws)
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    L.combine(y, inv, w, wl.I, x, dev["shared"].table, out, ws, shared_gate=torch.from_numpy(g).cuda())
    torch.cuda.synchronize()
    assert L.get_status(ws) == 0
    gi, gw = idx.cpu().numpy(), w.cpu().numpy()
    pu.check_routing(gi, gw, lg.cpu().numpy(), xb, lay.w_router, bias, k, bias_selection_only=True)
    # combine on the device's own rows and gates: the gated shared expert
    sy = oracle.shared_rows(xb, lay.shared) * oracle.shared_gate(xb, g)[:, None]
    comb = oracle.combine(pu.bf16_to_f64(bf16_bits(y)), inv.cpu().numpy(), gw.astype(np.float64), k, sy)
    pu.assert_close(pu.bf16_to_f64(bf16_bits(out)), comb, f"{case} combine")
