"""Helpers shared by the GPU parity tests: tolerance checks, routing agreement
with near-tie handling, and device upload of seeded workloads."""
from __future__ import annotations

import numpy as np

import oracle

# Float tolerance for bf16 activations with fp32 accumulation.
REL_L2 = 5e-3
MAX_ABS_RMS = 2e-2


def bf16_half_ulp(ref):
    """Half a bf16 ulp at each |ref| (8 significant bits): the largest error
    of a correctly rounded bf16 value of ref."""
    a = np.abs(np.asarray(ref, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.ldexp(1.0, (e - 8).astype(np.int64)), 0.0)


def _excess(err, ref, out_bf16):
    """Per-element error beyond the output format's own rounding."""
    a = np.abs(err)
    return np.maximum(a - bf16_half_ulp(ref), 0.0) if out_bf16 else a


def assert_close(got, ref, what="output", out_bf16=True):
    """The stated float tolerance: rel L2 <= 5e-3 and max abs <= 2e-2 x rms.

    Outputs stored as bf16 (the default) cannot be nearer to the exact value
    than half a bf16 ulp: an element beyond ~10 x rms would fail the max-abs
    bound by its rounding alone. So the max-abs bound applies to the error
    beyond that half ulp (a correctly rounded exact result always passes);
    rel L2 counts the whole error."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    rms = np.sqrt(np.mean(ref ** 2))
    err = got - ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300)
    mx = _excess(err, ref, out_bf16).max() if err.size else 0.0
    assert rel <= REL_L2, f"{what}: rel L2 {rel:.3e} > {REL_L2}"
    assert mx <= MAX_ABS_RMS * rms, f"{what}: max abs {mx:.3e} > {MAX_ABS_RMS} x rms {rms:.3e}"
    return rel, mx / max(rms, 1e-300)


def round_bf16(a):
    """Round float64 values to bf16 (nearest even), returned as float64."""
    f = np.asarray(a, dtype=np.float64).astype(np.float32)  # exact enough: bf16 keeps 8 of fp32's 24 bits
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint32) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def bf16_to_f64(bits):
    return oracle.bf16_bits_to_f64(bits)


def near_tie_tau(x_bits, w_router, bias):
    """Per-token tie tolerance: 64 ulp(fp32) of the largest sum |W x| + |b|."""
    x = np.abs(bf16_to_f64(x_bits))
    a = x @ np.abs(np.asarray(w_router, np.float64)).T + np.abs(np.asarray(bias, np.float64))
    return 64.0 * 2.0 ** -24 * a.max(axis=1)


def oracle_gates_for(logits64, idx):
    """Renormalised softmax gates of the given picks, from fp64 logits."""
    p = oracle.softmax(logits64)
    sel = np.take_along_axis(p, np.asarray(idx, np.int64), axis=1)
    return sel / sel.sum(axis=1, keepdims=True)


def check_routing(gpu_idx, gpu_w, gpu_logits, x_bits, w_router, bias, k, bias_selection_only=False):
    """Routing parity.

    1. The selection logic, exactly: the oracle's top-k and gates evaluated on
       the device's own fp32 logits give the device's indices bit for bit and
       its gates within a few fp32 ulps.
    2. Against the fp64 oracle logits: identical indices on every token whose
       top-(k+1) logits are separated by more than the fp32 rounding bound tau;
       on near-tied tokens, the device's picks are a valid top-k within tau.
    Returns (number of near-tied tokens, oracle fp64 logits).
    """
    gpu_idx = np.asarray(gpu_idx)
    T = gpu_idx.shape[0]
    gl = np.asarray(gpu_logits, dtype=np.float64)
    ref_idx_on_gpu_logits = oracle.topk_order(gl, k)
    np.testing.assert_array_equal(gpu_idx, ref_idx_on_gpu_logits)
    # gates: on the device's logits, less the bias when it only selects
    # (fp32 logit - bias differs from the device's own unbiased fp32 logit by
    # at most an ulp of the biased one, hence the looser bound there)
    gate_logits = gl - np.asarray(bias, np.float64) if bias_selection_only else gl
    np.testing.assert_allclose(gpu_w, oracle_gates_for(gate_logits, gpu_idx),
                               rtol=2e-5 if bias_selection_only else 2e-6, atol=1e-7)
    logits64 = oracle.router_logits(x_bits, w_router, bias)
    ref_idx = oracle.topk_order(logits64, k)
    tau = near_tie_tau(x_bits, w_router, bias)
    srt = -np.sort(-logits64, axis=1)[:, :k + 1]
    gaps = srt[:, :-1] - srt[:, 1:] if srt.shape[1] > k else srt[:, :-1] - srt[:, 1:]
    tied = (gaps < tau[:, None]).any(axis=1)
    for t in range(T):
        if not tied[t]:
            assert gpu_idx[t].tolist() == ref_idx[t].tolist(), f"token {t}: {gpu_idx[t]} vs {ref_idx[t]}"
        else:
            sel = gpu_idx[t]
            assert len(set(sel.tolist())) == k
            kth = srt[t, k - 1]
            assert np.all(logits64[t, sel] >= kth - tau[t])
            assert np.all(np.diff(logits64[t, sel]) <= tau[t])
    return int(tied.sum()), logits64


def upload_layer(lay, device="cuda"):
    """Device copies of a workload.LayerInputs (router, routed + shared experts)."""
    import torch

    from bit_quantized_moe_gemv_b200.device import DeviceExperts
    d = dict(
        w_router=torch.from_numpy(lay.w_router).to(device),
        experts=DeviceExperts(lay.experts, device),
        shared=DeviceExperts([lay.shared], device) if lay.shared is not None else None,
    )
    return d


def bias_tensor(bias, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bias, dtype=np.float32)).to(device)


class ErrorAccumulator:
    """assert_close over data seen in pieces: accumulates the squared error,
    the squared reference and the largest error, then applies the same two
    bounds (rel L2 and max abs against the rms of the whole reference)."""

    def __init__(self, what, out_bf16=True):
        self.what, self.out_bf16 = what, out_bf16
        self.se, self.sr, self.mx, self.n = 0.0, 0.0, 0.0, 0
        self.worst = None  # (excess, got, ref) of the worst element so far

    def add(self, got, ref):
        got = np.asarray(got, dtype=np.float64)
        ref = np.asarray(ref, dtype=np.float64)
        assert got.shape == ref.shape, (got.shape, ref.shape)
        assert np.all(np.isfinite(got)), f"{self.what}: non-finite values"
        err = got - ref
        self.se += float(np.sum(err * err))
        self.sr += float(np.sum(ref * ref))
        if err.size:
            ex = _excess(err, ref, self.out_bf16)
            i = int(np.argmax(ex))
            if self.worst is None or ex.flat[i] > self.worst[0]:
                self.worst = (float(ex.flat[i]), float(got.flat[i]), float(ref.flat[i]))
            self.mx = max(self.mx, float(ex.flat[i]))
        self.n += ref.size

    def check(self):
        rms = np.sqrt(self.sr / max(self.n, 1))
        rel = np.sqrt(self.se) / max(np.sqrt(self.sr), 1e-300)
        assert rel <= REL_L2, f"{self.what}: rel L2 {rel:.3e} > {REL_L2}"
        assert self.mx <= MAX_ABS_RMS * rms, (f"{self.what}: max abs {self.mx:.3e} > {MAX_ABS_RMS} x rms {rms:.3e} "
                                              f"(worst: got {self.worst[1]!r}, oracle {self.worst[2]!r})")
        return rel, self.mx / max(rms, 1e-300)


def check_every_row(xb, w_router, bias, k, experts, shared, idx, perm, offsets, y_perm_bits, out_bits,
                    shared_chunk=2048):
    """Every dispatched row and every output token of a step against the
    oracle, one expert at a time (a whole prefill step's fp64 rows would not
    fit in host memory at once).

    y_perm_bits: the device's bf16 rows in dispatch order (moe_expert_ffn);
    out_bits: the device's bf16 layer output (moe_layer). The routing must
    have been checked already (check_routing); the oracle evaluates the
    device's picks with gates from the fp64 logits.
    Returns ((rel, max/rms) of y_perm, (rel, max/rms) of out)."""
    x = bf16_to_f64(xb)
    T, H = x.shape
    gates = oracle_gates_for(oracle.router_logits(xb, w_router, bias), idx)
    perm = np.asarray(perm, dtype=np.int64)
    offsets = np.asarray(offsets, dtype=np.int64)
    out_ref = np.zeros((T, H), dtype=np.float64)
    acc_y = ErrorAccumulator("y_perm (every row)")
    for e in range(len(experts)):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r0 == r1:
            continue
        wg, wu, wd = (oracle.dequant_qm(m) for m in (experts[e].gate, experts[e].up, experts[e].down))
        src = perm[r0:r1]
        toks, slots = src // k, src % k
        _, y = oracle.expert_forward(wg, wu, wd, x[toks])
        acc_y.add(bf16_to_f64(y_perm_bits[r0:r1]), y)
        out_ref[toks] += gates[toks, slots][:, None] * y  # a token picks an expert at most once
    if shared is not None:
        sg, su, sd = (oracle.dequant_qm(m) for m in (shared.gate, shared.up, shared.down))
        for c0 in range(0, T, shared_chunk):
            out_ref[c0:c0 + shared_chunk] += oracle.expert_forward(sg, su, sd, x[c0:c0 + shared_chunk])[1]
    acc_o = ErrorAccumulator("out (every token)")
    acc_o.add(bf16_to_f64(out_bits), out_ref)
    return acc_y.check(), acc_o.check()
