"""Seeded synthetic inputs for the routed-MoE FFN step.

This module only draws numbers. It holds none of the layer's arithmetic
(no routing, no dequantisation, no matmul), so both the CUDA path and the
fp64 oracle consume what it makes without sharing any computation.

Every array is addressable on its own: the Philox key of an array is derived
from (seed, workload, layer, expert, matrix, kind), so one expert of one layer
can be generated without generating the rest.

Value distributions (the pages give the structure, not the numbers):
  * activations x ~ N(0, 1) in fp32, rounded to bf16 (round-to-nearest-even);
  * router weights W_r ~ N(0, 0.02) fp32, shape [E, H];
  * packed codes: uniform random bytes (so int4 and int2 codes are uniform);
    int8 codes uniform over [-127, 127];
  * int4 scales ~ U(0.005, 0.02) -> fp16;
  * int2 scales ~ U(0.01, 0.04), mins = -scale * U(1, 2) -> fp16;
  * int8 per-channel scales ~ U(0.005, 0.02) / 16 -> fp16;
  * router bias from a Zipf expert-popularity prior b[e] = -s * ln(e + 1)
    (expert 0 most popular; the Zipf normaliser is a constant shift that
    softmax ignores).

Shapes follow the layer described on the telli.sh page "Strata 与
Qwen3.8-Flash-Next：如何在个人电脑上运行 180B 级模型", section
"稀疏架构创造了机会" (48 layers, 512 routed experts per layer, 10 routed plus
one shared expert active per token).
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, field

import numpy as np

# Quantisation type codes; the same integers appear in include/moe.h.
Q_INT4_SYM_G32 = 1
Q_INT2_ASYM_G16 = 2
Q_INT8_PER_CHANNEL = 3

QTYPE_NAMES = {
    Q_INT4_SYM_G32: "int4_sym_g32",
    Q_INT2_ASYM_G16: "int2_asym_g16",
    Q_INT8_PER_CHANNEL: "int8_per_channel",
}


def qtype_group(qtype: int) -> int:
    """Group length along K for a qtype (0 = one scale per output row)."""
    return {Q_INT4_SYM_G32: 32, Q_INT2_ASYM_G16: 16, Q_INT8_PER_CHANNEL: 0}[qtype]


def qtype_bits(qtype: int) -> int:
    return {Q_INT4_SYM_G32: 4, Q_INT2_ASYM_G16: 2, Q_INT8_PER_CHANNEL: 8}[qtype]


def qmatrix_nbytes(qtype: int, rows: int, cols: int) -> int:
    """Bytes of codes + scales (+ mins) of one packed matrix."""
    code_bytes = rows * cols * qtype_bits(qtype) // 8
    g = qtype_group(qtype)
    if qtype == Q_INT8_PER_CHANNEL:
        return code_bytes + 2 * rows
    n_groups = rows * (cols // g)
    return code_bytes + 2 * n_groups * (2 if qtype == Q_INT2_ASYM_G16 else 1)


@dataclass
class QMatrix:
    """One packed weight matrix W[rows = N out, cols = K in].

    codes  uint8 [rows, cols*bits/8], row-major.
    scales float16 [rows, cols/group] (int8: [rows]).
    mins   float16 [rows, cols/group] for int2, else None.
    """

    qtype: int
    rows: int
    cols: int
    codes: np.ndarray
    scales: np.ndarray
    mins: np.ndarray | None = None

    @property
    def group(self) -> int:
        return qtype_group(self.qtype)

    @property
    def nbytes(self) -> int:
        return qmatrix_nbytes(self.qtype, self.rows, self.cols)


@dataclass
class Expert:
    gate: QMatrix  # [I, H]
    up: QMatrix  # [I, H]
    down: QMatrix  # [H, I]

    @property
    def nbytes(self) -> int:
        return self.gate.nbytes + self.up.nbytes + self.down.nbytes


@dataclass(frozen=True)
class Workload:
    """A named synthetic MoE-layer workload."""

    name: str
    T: int  # tokens per step
    H: int  # hidden size
    I: int  # expert intermediate size
    E: int  # routed experts
    k: int  # routed experts per token
    layers: int = 1
    steps: int = 1
    zipf_s: float = 0.0  # Zipf prior exponent (0 = no bias)
    uniform_frac: float = 0.0  # fraction of rows routed with b = 0
    routed_qtypes: tuple = ((0, None, Q_INT4_SYM_G32),)  # (first, last_excl, qtype)
    shared_qtype: int = Q_INT4_SYM_G32
    seed: int = 0

    def expert_qtype(self, e: int) -> int:
        for lo, hi, q in self.routed_qtypes:
            if e >= lo and (hi is None or e < hi):
                return q
        raise ValueError(e)


WORKLOADS = {
    # Tiny case the oracle finishes instantly.
    "tiny": Workload("tiny", T=4, H=256, I=128, E=16, k=2, seed=0),
    # Decode, one layer, one token per step, 200 fresh tokens, Zipf(1.1) prior.
    "decode1": Workload("decode1", T=1, H=2048, I=768, E=512, k=10, steps=200, zipf_s=1.1),
    # Decode, 48 independent layers, 4 slots per step, int2 experts + int8 shared.
    "decode48": Workload(
        "decode48", T=4, H=2048, I=768, E=512, k=10, layers=48, steps=200, zipf_s=1.1,
        routed_qtypes=((0, None, Q_INT2_ASYM_G16),), shared_qtype=Q_INT8_PER_CHANNEL,
    ),
    # Verification batch of speculative decoding: one sequence's current token
    # plus 3 drafted ones checked in one pass (4 tokens of ONE slot), the
    # decode1 layer otherwise. The telli.sh page "Strata 与 Qwen3.8-Flash-Next：
    # 如何在个人电脑上运行 180B 级模型", section "推测解码只有在验证通过时才节省计算",
    # drafts up to 3 tokens that the target model verifies in one pass.
    "verify4": Workload("verify4", T=4, H=2048, I=768, E=512, k=10, steps=200, zipf_s=1.1),
    # Prefill 8K tokens, Zipf(1.0) skew.
    "prefill8k": Workload("prefill8k", T=8192, H=2048, I=768, E=512, k=10, zipf_s=1.0),
    # Long prefill 32K, mixed per-expert precision, Zipf(1.2) + 5% uniform rows.
    "prefill32k": Workload(
        "prefill32k", T=32768, H=2048, I=768, E=512, k=10, zipf_s=1.2, uniform_frac=0.05,
        routed_qtypes=((0, 256, Q_INT4_SYM_G32), (256, None, Q_INT2_ASYM_G16)),
        shared_qtype=Q_INT8_PER_CHANNEL,
    ),
}


def _rng(seed: int, *parts) -> np.random.Generator:
    tag = "/".join(str(p) for p in parts).encode()
    k1 = int.from_bytes(hashlib.blake2b(tag, digest_size=8).digest(), "little")
    return np.random.Generator(np.random.Philox(key=np.array([seed & (2**64 - 1), k1], dtype=np.uint64)))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest-even), returning the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def gen_x(wl: Workload, step: int = 0, layer: int = 0, T: int | None = None) -> np.ndarray:
    """Activations for one step of one layer: bf16 bit patterns [T, H]."""
    T = wl.T if T is None else T
    g = _rng(wl.seed, wl.name, "x", layer, step)
    return f32_to_bf16_bits(g.standard_normal((T, wl.H), dtype=np.float32))


def gen_router(wl: Workload, layer: int = 0) -> np.ndarray:
    g = _rng(wl.seed, wl.name, "router", layer)
    return (g.standard_normal((wl.E, wl.H), dtype=np.float32) * np.float32(0.02)).astype(np.float32)


def gen_bias(wl: Workload, step: int = 0, layer: int = 0, T: int | None = None):
    """Router bias. Returns (bias fp32, row_stride): [E] with stride 0, or [T, E]."""
    T = wl.T if T is None else T
    e = np.arange(wl.E, dtype=np.float64)
    prior = (-wl.zipf_s * np.log(e + 1.0)).astype(np.float32)
    if wl.uniform_frac <= 0.0:
        return prior, 0
    g = _rng(wl.seed, wl.name, "uniform_rows", layer, step)
    n_uniform = int(round(wl.uniform_frac * T))
    rows = g.choice(T, size=n_uniform, replace=False)
    b = np.broadcast_to(prior, (T, wl.E)).copy()
    b[rows, :] = 0.0
    return b, wl.E


def gen_qmatrix(wl: Workload, layer, expert, matrix: str, qtype: int, rows: int, cols: int) -> QMatrix:
    g = _rng(wl.seed, wl.name, "w", layer, expert, matrix)
    bits = qtype_bits(qtype)
    nb = rows * cols * bits // 8
    if qtype == Q_INT8_PER_CHANNEL:
        q = g.integers(-127, 128, size=nb, dtype=np.int16).astype(np.int8)
        codes = q.view(np.uint8).reshape(rows, cols)
        scales = (g.uniform(0.005, 0.02, size=rows) / 16.0).astype(np.float16)
        return QMatrix(qtype, rows, cols, codes, scales, None)
    codes = np.frombuffer(g.bytes(nb), dtype=np.uint8).reshape(rows, cols * bits // 8).copy()
    ng = cols // qtype_group(qtype)
    if qtype == Q_INT4_SYM_G32:
        scales = g.uniform(0.005, 0.02, size=(rows, ng)).astype(np.float16)
        return QMatrix(qtype, rows, cols, codes, scales, None)
    if qtype == Q_INT2_ASYM_G16:
        s = g.uniform(0.01, 0.04, size=(rows, ng))
        m = -s * g.uniform(1.0, 2.0, size=(rows, ng))
        return QMatrix(qtype, rows, cols, codes, s.astype(np.float16), m.astype(np.float16))
    raise ValueError(qtype)


def gen_expert(wl: Workload, layer: int, expert) -> Expert:
    """expert is an int in [0, E) or the string 'shared'."""
    q = wl.shared_qtype if expert == "shared" else wl.expert_qtype(int(expert))
    return Expert(
        gate=gen_qmatrix(wl, layer, expert, "gate", q, wl.I, wl.H),
        up=gen_qmatrix(wl, layer, expert, "up", q, wl.I, wl.H),
        down=gen_qmatrix(wl, layer, expert, "down", q, wl.H, wl.I),
    )


@dataclass
class LayerInputs:
    wl: Workload
    layer: int
    w_router: np.ndarray
    experts: list = field(default_factory=list)  # E routed experts
    shared: Expert | None = None


def gen_layer(wl: Workload, layer: int = 0, with_shared: bool = True) -> LayerInputs:
    return LayerInputs(
        wl=wl, layer=layer, w_router=gen_router(wl, layer),
        experts=[gen_expert(wl, layer, e) for e in range(wl.E)],
        shared=gen_expert(wl, layer, "shared") if with_shared else None,
    )


def per_token_layer_bytes(wl: Workload, unique_experts: float | None = None) -> float:
    """Algorithmic HBM bytes one decode layer-step must stream.

    Each distinct selected expert's packed gate/up/down matrices are read once
    per step (shared by all tokens of the step that select it), plus the shared
    expert and the fp32 router matrix.
    """
    u = wl.k if unique_experts is None else unique_experts
    routed = qmatrix_nbytes(wl.expert_qtype(0), wl.I, wl.H) * 2 + qmatrix_nbytes(wl.expert_qtype(0), wl.H, wl.I)
    shared = qmatrix_nbytes(wl.shared_qtype, wl.I, wl.H) * 2 + qmatrix_nbytes(wl.shared_qtype, wl.H, wl.I)
    return u * routed + shared + 4 * wl.E * wl.H


# ------------------------------------------------------------------ device draws
def _torch_seed(*parts) -> int:
    h = hashlib.sha256(repr(parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _draw_block(g, qtype: int, n: int, rows: int, cols: int, device):
    """n packed [rows, cols] matrices of one qtype: (codes, scales, mins) with
    the distributions of gen_qmatrix, drawn with torch generator g."""
    import torch
    bits = qtype_bits(qtype)
    if qtype == Q_INT8_PER_CHANNEL:
        q = torch.randint(-127, 128, (n, rows, cols), dtype=torch.int16, device=device, generator=g)
        codes = q.to(torch.int8).view(torch.uint8)
        scales = (torch.empty((n, rows), dtype=torch.float32, device=device).uniform_(0.005, 0.02, generator=g)
                  / 16.0).to(torch.float16)
        return codes, scales, None
    codes = torch.randint(0, 256, (n, rows, cols * bits // 8), dtype=torch.int16, device=device,
                          generator=g).to(torch.uint8)
    ng = cols // qtype_group(qtype)
    if qtype == Q_INT4_SYM_G32:
        s = torch.empty((n, rows, ng), dtype=torch.float32, device=device).uniform_(0.005, 0.02, generator=g)
        return codes, s.to(torch.float16), None
    s = torch.empty((n, rows, ng), dtype=torch.float32, device=device).uniform_(0.01, 0.04, generator=g)
    m = -s * torch.empty((n, rows, ng), dtype=torch.float32, device=device).uniform_(1.0, 2.0, generator=g)
    return codes, s.to(torch.float16), m.to(torch.float16)


def draw_layer_device(wl: Workload, layer: int, device="cuda") -> dict:
    """One layer of `wl` drawn directly in device memory with a seeded torch
    generator: the distributions of gen_layer, different numbers. For stacks
    too large to draw on the host (48 layers of 512 experts are 58 GB).

    All routed experts must share one qtype. Returns torch tensors:
      w_router [E, H] fp32;
      routed: gu = (codes [E, 2, I, .], scales, mins) for gate (index 0) and
              up (index 1), dn = (codes [E, H, .], scales, mins);
      shared: sgu, sdn (the same with a leading 1).
    """
    import torch
    qs = {q for _, _, q in wl.routed_qtypes}
    assert len(qs) == 1, "one routed qtype per drawn layer"
    q = qs.pop()
    g = torch.Generator(device=device)
    g.manual_seed(_torch_seed(wl.seed, wl.name, "device_layer", layer))
    out = {"qtype": q, "shared_qtype": wl.shared_qtype}
    out["w_router"] = torch.randn((wl.E, wl.H), dtype=torch.float32, device=device, generator=g) * 0.02
    c, s, m = _draw_block(g, q, 2 * wl.E, wl.I, wl.H, device)
    out["gu"] = tuple(None if t is None else t.view(wl.E, 2, *t.shape[1:]) for t in (c, s, m))
    out["dn"] = _draw_block(g, q, wl.E, wl.H, wl.I, device)
    c, s, m = _draw_block(g, wl.shared_qtype, 2, wl.I, wl.H, device)
    out["sgu"] = tuple(None if t is None else t.view(1, 2, *t.shape[1:]) for t in (c, s, m))
    out["sdn"] = _draw_block(g, wl.shared_qtype, 1, wl.H, wl.I, device)
    return out
