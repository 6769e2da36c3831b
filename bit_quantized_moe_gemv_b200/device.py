"""Upload packed expert weights to device memory and build the descriptor
tables the C ABI takes (a device array of moe_expert structs).

All codes of a layer live in one device buffer, laid out expert by expert
(gate, up, down; codes then scales then mins, each 256-byte aligned), so a
layer is one host-to-device copy. This is marshalling: nothing here computes.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import _lib
from .workload import Q_INT2_ASYM_G16, Q_INT4_SYM_G32, Expert, qtype_group


def _align(n, a=256):
    return (n + a - 1) // a * a


def _parts(qm):
    out = [np.ascontiguousarray(qm.codes).view(np.uint8).reshape(-1),
           np.ascontiguousarray(qm.scales, dtype=np.float16).view(np.uint8).reshape(-1)]
    if qm.mins is not None:
        out.append(np.ascontiguousarray(qm.mins, dtype=np.float16).view(np.uint8).reshape(-1))
    return out


class DeviceExperts:
    """A list of Expert objects resident on the device, with descriptor table.

    `table` is a uint8 device tensor holding len(experts) moe_expert structs;
    pass it as `experts_dev` / `shared_dev`. `buffer` owns the weight bytes.
    """

    def __init__(self, experts: list[Expert], device="cuda"):
        import torch
        self.n = len(experts)
        offs, total = [], 0
        for ex in experts:
            eo = []
            for qm in (ex.gate, ex.up, ex.down):
                po = []
                for part in _parts(qm):
                    po.append(total)
                    total = _align(total + part.size)
                eo.append(po)
            offs.append(eo)
        host = np.zeros(max(total, 256), dtype=np.uint8)
        for ex, eo in zip(experts, offs):
            for qm, po in zip((ex.gate, ex.up, ex.down), eo):
                for part, o in zip(_parts(qm), po):
                    host[o:o + part.size] = part
        self.buffer = torch.from_numpy(host).to(device)
        base = self.buffer.data_ptr()
        arr = (_lib.ExpertC * max(self.n, 1))()
        for i, (ex, eo) in enumerate(zip(experts, offs)):
            for name, qm, po in zip(("gate", "up", "down"), (ex.gate, ex.up, ex.down), eo):
                d = getattr(arr[i], name)
                d.qtype, d.rows, d.cols, d.group = qm.qtype, qm.rows, qm.cols, qtype_group(qm.qtype)
                d.codes = base + po[0]
                d.scales = base + po[1]
                d.mins = base + po[2] if len(po) > 2 else None
        raw = np.frombuffer(bytes(arr), dtype=np.uint8).copy()
        self.table = torch.from_numpy(raw).to(device)
        self.nbytes = total

    def descriptor(self, i):
        """Host copy of descriptor i (for tests)."""
        raw = self.table[i * ctypes.sizeof(_lib.ExpertC):(i + 1) * ctypes.sizeof(_lib.ExpertC)].cpu().numpy()
        return _lib.ExpertC.from_buffer_copy(raw.tobytes())


def bf16_tensor(bits: np.ndarray, device="cuda"):
    """uint16 bf16 bit patterns -> torch.bfloat16 device tensor (bitwise)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def bf16_bits(t) -> np.ndarray:
    """torch.bfloat16 tensor -> uint16 numpy bit patterns."""
    import torch
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


__all__ = ["DeviceExperts", "bf16_tensor", "bf16_bits", "Q_INT4_SYM_G32", "Q_INT2_ASYM_G16"]


class BlockExperts:
    """Descriptor table over experts whose matrices are slices of stacked
    device tensors (as drawn by workload.draw_layer_device): gu = (codes,
    scales, mins) shaped [n, 2, rows, ...] for gate/up, dn = [n, rows, ...]."""

    def __init__(self, qtype, gu, dn, I, H, device="cuda"):
        import torch
        n = gu[0].shape[0]
        arr = (_lib.ExpertC * n)()
        g = qtype_group(qtype)
        for i in range(n):
            for name, j in (("gate", 0), ("up", 1), ("down", None)):
                d = getattr(arr[i], name)
                src = [t if t is None else (t[i, j] if j is not None else t[i]) for t in (gu if j is not None else dn)]
                d.qtype, d.group = qtype, g
                d.rows, d.cols = (I, H) if j is not None else (H, I)
                d.codes = src[0].data_ptr()
                d.scales = src[1].data_ptr()
                d.mins = src[2].data_ptr() if src[2] is not None else None
        self.n = n
        self.keep = (gu, dn)
        raw = np.frombuffer(bytes(arr), dtype=np.uint8).copy()
        self.table = torch.from_numpy(raw).to(device)
