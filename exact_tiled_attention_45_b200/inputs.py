"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle runs.

This module only draws random numbers; it holds none of the attention
arithmetic.  Recipe: a CPU ``torch.Generator`` seeded with ``seed`` draws Q,
then K, then V with ``torch.randn(B, H, N, d, dtype=float32)``; each is rounded
to bf16 (round-to-nearest-even).  The "x4" variant multiplies Q and K by 4
after rounding (exact in bf16) to give large logits.
"""
from __future__ import annotations

import torch

__all__ = ["make_qkv", "Workload", "WORKLOADS"]


def make_qkv(B: int, H: int, N: int, d: int, seed: int = 0, qk_mult: float = 1.0):
    """Return bf16 CPU tensors (q, k, v), each [B, H, N, d] contiguous."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = torch.randn(B, H, N, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn(B, H, N, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
    if qk_mult != 1.0:
        q = q * qk_mult
        k = k * qk_mult
    return q, k, v


class Workload:
    """One attention problem shape: [B, H, N, d], causal flag, Q/K multiplier."""

    def __init__(self, name: str, B: int, H: int, N: int, d: int, causal: bool,
                 qk_mult: float = 1.0):
        self.name, self.B, self.H, self.N, self.d = name, B, H, N, d
        self.causal, self.qk_mult = bool(causal), float(qk_mult)

    @property
    def flops(self) -> float:
        """Benchmark FLOP convention: 4*B*H*N^2*d, halved when causal."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def as_dict(self) -> dict:
        return {"workload": self.name, "B": self.B, "H": self.H, "N": self.N,
                "d": self.d, "causal": self.causal, "qk_mult": self.qk_mult}

    def __repr__(self) -> str:  # pragma: no cover
        return f"Workload({self.as_dict()})"


def _grid():
    out = []
    for d in (64, 128):
        for causal in (False, True):
            for N in (512, 1024, 2048, 4096, 8192, 16384):
                H = 2048 // d
                B = 16384 // N
                tag = f"grid_N{N}_d{d}_{'causal' if causal else 'full'}"
                out.append(Workload(tag, B, H, N, d, causal))
    return out


#: The workloads of the benchmark sweep (16k total tokens, hidden 2048).
WORKLOADS = {
    "tiny_B1_H2_N128_d64": Workload("tiny_B1_H2_N128_d64", 1, 2, 128, 64, False),
    "B8_H16_N2048_d128_causal": Workload("B8_H16_N2048_d128_causal", 8, 16, 2048, 128, True),
    "B1_H16_N16384_d128_causal": Workload("B1_H16_N16384_d128_causal", 1, 16, 16384, 128, True),
}
for _N in (512, 1024, 2048, 4096, 8192, 16384):
    _w = Workload(f"sweep_N{_N}_d64_full", 16384 // _N, 32, _N, 64, False)
    WORKLOADS[_w.name] = _w
for _w in _grid():
    WORKLOADS.setdefault(_w.name, _w)
