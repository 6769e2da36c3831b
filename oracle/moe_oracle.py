"""fp64 CPU oracle of the routed-MoE FFN step.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, links or runs
this module: only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline
leg (and its `--impl reference` arm) may call it. It shares no code, header,
table or constant generator with the CUDA library; both sides only consume
the same seeded arrays from bit_quantized_moe_gemv_b200.workload.

What it computes (one MoE block of a Qwen3.8-Flash-Next-style layer):
  the telli.sh page "Strata 与 Qwen3.8-Flash-Next：如何在个人电脑上运行 180B 级模型",
  section "稀疏架构创造了机会", fixes the structure: every layer has 512 routed
  experts, each token activates 10 of them plus one shared expert. The
  cycleuser.org page "本地部署Qwen3.8-Flash-Next模型的两条路线…", section
  "硬件形态决定了各自的走法", places the router and the shared expert beside
  the routed experts and quantises experts to 2-3 bits (section
  "精度和内存占用": 4 bits in the other engine). The pages do not print the
  router function, the activation or any bit layout; the readings below are
  the plainest ones consistent with them and with the workload definition:

  1. logits   l[t,e] = sum_h W_r[e,h] x[t,h] + b[t,e]
  2. p[t,:]   = softmax over all E logits
  3. S_t      = the k experts first in the order (l descending, index ascending)
  4. w[t,j]   = p[t,S_j] / sum_j' p[t,S_j']            (renormalised gates)
  5. dispatch: stable counting sort of the (t, j) pairs by expert
  6. expert e on token t: g = W_g x, u = W_u x, h = silu(g) * u,
     silu(z) = z / (1 + exp(-z)), y = W_d h            (SwiGLU FFN)
  7. out[t]   = sum_j w[t,j] y_{S_j}(x_t) + shared(x_t) (shared expert ungated)

Two router variants, both readings of what the pages leave open (they name a
router and a shared expert but not their functions), off by default:
  * bias for selection only: S_t is chosen on the biased logits (step 3) but
    the gates of step 4 come from the softmax of the unbiased logits W_r x;
  * sigmoid-gated shared expert: step 7 adds sigma(g . x_t) * shared(x_t)
    for a gate vector g [H] instead of shared(x_t).

Every quantity is float64 and nothing is rounded between steps.
Quantised weight formats (codes row-major [N, K*bits/8], groups along K):
  int4_sym_g32:      element 2i in the low nibble of byte i, 2i+1 in the high
                     nibble; q = c - 8; w = q * scale[n, k // 32]
  int2_asym_g16:     element 4i+m in bits 2m..2m+1 of byte i; w = c *
                     scale[n, k // 16] + min[n, k // 16]
  int8_per_channel:  two's-complement byte q; w = q * scale[n]
"""
from __future__ import annotations

import numpy as np

INT4_SYM_G32 = 1
INT2_ASYM_G16 = 2
INT8_PER_CHANNEL = 3


# ---------------------------------------------------------------- formats
def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64 (exact: bf16 is the top half of fp32)."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


def dequant(qtype: int, rows: int, cols: int, codes, scales, mins=None) -> np.ndarray:
    """Dequantise one packed matrix to float64 [rows, cols]."""
    codes = np.asarray(codes, dtype=np.uint8).reshape(rows, -1)
    s = np.asarray(scales).astype(np.float64)
    if qtype == INT4_SYM_G32:
        c = np.empty((rows, cols), dtype=np.float64)
        c[:, 0::2] = codes & 0x0F
        c[:, 1::2] = codes >> 4
        q = c - 8.0
        return q * np.repeat(s.reshape(rows, cols // 32), 32, axis=1)
    if qtype == INT2_ASYM_G16:
        c = np.empty((rows, cols), dtype=np.float64)
        for m in range(4):
            c[:, m::4] = (codes >> (2 * m)) & 0x3
        m16 = np.asarray(mins).astype(np.float64).reshape(rows, cols // 16)
        return c * np.repeat(s.reshape(rows, cols // 16), 16, axis=1) + np.repeat(m16, 16, axis=1)
    if qtype == INT8_PER_CHANNEL:
        q = codes.view(np.int8).astype(np.float64).reshape(rows, cols)
        return q * s.reshape(rows, 1)
    raise ValueError(f"unknown qtype {qtype}")


def dequant_qm(qm) -> np.ndarray:
    """Dequantise an object with fields qtype, rows, cols, codes, scales, mins."""
    return dequant(qm.qtype, qm.rows, qm.cols, qm.codes, qm.scales, qm.mins)


# ---------------------------------------------------------------- routing
def router_logits(x_bits: np.ndarray, w_router: np.ndarray, bias: np.ndarray) -> np.ndarray:
    """Step 1: l = x W_r^T + b in float64. bias is [E] or [T, E]."""
    x = bf16_bits_to_f64(x_bits)
    return x @ np.asarray(w_router, dtype=np.float64).T + np.asarray(bias, dtype=np.float64)


def softmax(logits: np.ndarray) -> np.ndarray:
    """Step 2: softmax over the last axis."""
    z = np.exp(logits - logits.max(axis=-1, keepdims=True))
    return z / z.sum(axis=-1, keepdims=True)


def topk_order(logits: np.ndarray, k: int) -> np.ndarray:
    """Step 3: per row, the first k expert ids in (logit desc, index asc) order."""
    T, E = logits.shape
    out = np.empty((T, k), dtype=np.int32)
    idx = np.arange(E)
    for t in range(T):
        order = np.lexsort((idx, -logits[t]))  # primary key -logit, then index
        out[t] = order[:k]
    return out


def route(x_bits, w_router, bias, k, bias_selection_only=False):
    """Steps 1-4. Returns (logits [T,E], idx int32 [T,k], w float64 [T,k]).

    logits are the biased logits the selection is made on. With
    bias_selection_only the gates are the softmax of the unbiased logits,
    renormalised over the same picks."""
    logits = router_logits(x_bits, w_router, bias)
    idx = topk_order(logits, k)
    gate_logits = router_logits(x_bits, w_router, np.zeros(1)) if bias_selection_only else logits
    p = softmax(gate_logits)
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    w = sel / sel.sum(axis=1, keepdims=True)
    return logits, idx, w


def shared_gate(x_bits, gate_w):
    """Weight of the shared expert in the sigmoid-gated variant: sigma(g . x)
    per token, sigma(z) = 1 / (1 + exp(-z))."""
    z = bf16_bits_to_f64(x_bits) @ np.asarray(gate_w, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-z))


# ---------------------------------------------------------------- dispatch
def dispatch(idx: np.ndarray, E: int):
    """Step 5: stable counting sort of the T*k (token, slot) pairs by expert.

    Returns counts [E], offsets [E+1] (exclusive prefix sum), perm_src [T*k]
    (perm_src[r] = t*k + j of the pair placed at row r; inside one expert,
    rows follow ascending t*k + j) and inv_perm [T*k] (inv_perm[t*k+j] = r).
    """
    flat = np.asarray(idx, dtype=np.int64).reshape(-1)
    counts = np.zeros(E, dtype=np.int64)
    for e in flat:
        counts[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    cursor = offsets[:-1].copy()
    perm_src = np.empty(flat.size, dtype=np.int64)
    inv_perm = np.empty(flat.size, dtype=np.int64)
    for p, e in enumerate(flat):  # ascending pair index -> stable
        r = cursor[e]
        perm_src[r] = p
        inv_perm[p] = r
        cursor[e] += 1
    return (counts.astype(np.int32), offsets.astype(np.int32),
            perm_src.astype(np.int32), inv_perm.astype(np.int32))


# ---------------------------------------------------------------- experts
def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def expert_forward(wg: np.ndarray, wu: np.ndarray, wd: np.ndarray, xrows: np.ndarray):
    """Step 6 on dequantised weights: xrows [n, H] float64 -> (h [n, I], y [n, H])."""
    g = xrows @ wg.T
    u = xrows @ wu.T
    h = silu(g) * u
    return h, h @ wd.T


class DequantCache:
    """Dequantises experts on first use (a full layer in fp64 would not fit)."""

    def __init__(self, experts, capacity: int = 64):
        self.experts = experts
        self.capacity = capacity
        self._cache: dict = {}

    def get(self, e):
        if e not in self._cache:
            if len(self._cache) >= self.capacity:
                self._cache.pop(next(iter(self._cache)))
            ex = self.experts[e]
            self._cache[e] = (dequant_qm(ex.gate), dequant_qm(ex.up), dequant_qm(ex.down))
        return self._cache[e]


def expert_rows(x_bits, perm_src, offsets, k, experts, rows=None, cache=None):
    """Routed expert outputs y_perm[r] for the permuted rows r (all rows by default).

    Row r belongs to the expert e with offsets[e] <= r < offsets[e+1] and reads
    token perm_src[r] // k.
    """
    x = bf16_bits_to_f64(x_bits)
    offsets = np.asarray(offsets, dtype=np.int64)
    n = int(offsets[-1])
    rows = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    cache = cache or DequantCache(experts)
    owner = np.searchsorted(offsets, rows, side="right") - 1
    y = np.zeros((rows.size, x.shape[1]), dtype=np.float64)
    for e in np.unique(owner):
        sel = np.nonzero(owner == e)[0]
        toks = np.asarray(perm_src, dtype=np.int64)[rows[sel]] // k
        wg, wu, wd = cache.get(int(e))
        _, y[sel] = expert_forward(wg, wu, wd, x[toks])
    return y


def shared_rows(x_bits, shared, tokens=None):
    """Shared-expert output for the given tokens (all by default)."""
    x = bf16_bits_to_f64(x_bits)
    tokens = np.arange(x.shape[0]) if tokens is None else np.asarray(tokens)
    _, y = expert_forward(dequant_qm(shared.gate), dequant_qm(shared.up), dequant_qm(shared.down), x[tokens])
    return y


def combine(y_perm, inv_perm, w, k, shared_y=None):
    """Step 7: out[t] = sum_j w[t,j] y_perm[inv_perm[t*k+j]] (+ shared_y[t])."""
    w = np.asarray(w, dtype=np.float64)
    T = w.shape[0]
    inv = np.asarray(inv_perm, dtype=np.int64).reshape(T, k)
    out = np.zeros((T, y_perm.shape[1]), dtype=np.float64)
    for j in range(k):
        out += w[:, j:j + 1] * y_perm[inv[:, j]]
    if shared_y is not None:
        out += shared_y
    return out


def moe_layer(x_bits, w_router, bias, k, experts, shared=None, routing=None, bias_selection_only=False,
              shared_gate_w=None):
    """Steps 1-7 for all tokens.

    routing, if given, is (idx, w) to use instead of the oracle's own routing
    (used where the fp32 router of the device legitimately resolves a near-tie
    differently). bias_selection_only and shared_gate_w select the router
    variants (module docstring). Returns dict with logits, idx, w, counts,
    offsets, perm_src, inv_perm, y_perm, out.
    """
    E = len(experts)
    logits, idx, w = route(x_bits, w_router, bias, k, bias_selection_only)
    if routing is not None:
        idx, w = routing
    counts, offsets, perm_src, inv_perm = dispatch(idx, E)
    y_perm = expert_rows(x_bits, perm_src, offsets, k, experts)
    sy = shared_rows(x_bits, shared) if shared is not None else None
    if sy is not None and shared_gate_w is not None:
        sy = sy * shared_gate(x_bits, shared_gate_w)[:, None]
    out = combine(y_perm, inv_perm, w, k, sy)
    return dict(logits=logits, idx=idx, w=w, counts=counts, offsets=offsets, perm_src=perm_src,
                inv_perm=inv_perm, y_perm=y_perm, out=out)


def moe_token(x_bits_row, w_router, bias_row, k, cache, shared_deq=None, routing=None, bias_selection_only=False,
              shared_gate_w=None):
    """Steps 1-7 for one token, computed directly (no dispatch): used to check
    sampled tokens of large workloads. Returns (idx, w, out[H])."""
    x_bits_row = np.asarray(x_bits_row).reshape(1, -1)
    logits, idx, w = route(x_bits_row, w_router, np.asarray(bias_row).reshape(1, -1), k, bias_selection_only)
    if routing is not None:
        idx, w = routing
        idx = np.asarray(idx).reshape(1, -1)
        w = np.asarray(w).reshape(1, -1)
    x = bf16_bits_to_f64(x_bits_row)
    out = np.zeros(x.shape[1])
    for j in range(k):
        wg, wu, wd = cache.get(int(idx[0, j]))
        out += w[0, j] * expert_forward(wg, wu, wd, x)[1][0]
    if shared_deq is not None:
        g = shared_gate(x_bits_row, shared_gate_w)[0] if shared_gate_w is not None else 1.0
        out += g * expert_forward(*shared_deq, x)[1][0]
    return idx[0], w[0], out
