"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle runs.

This module only draws random numbers; it holds none of the attention
arithmetic.  Recipe: a CPU ``torch.Generator`` seeded with ``seed`` draws Q,
then K, then V with ``torch.randn(B, H, N, d, dtype=float32)``; each is rounded
to bf16 (round-to-nearest-even).  The "x4" variant multiplies Q and K by 4
after rounding (exact in bf16) to give large logits.
"""
from __future__ import annotations

import torch

__all__ = ["make_qkv", "make_q_kv", "Workload", "DecodeWorkload", "WORKLOADS"]


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


def make_q_kv(B: int, H: int, Nq: int, Nk: int, d: int, seed: int = 0, qk_mult: float = 1.0):
    """Q [B, H, Nq, d] and K, V [B, H, Nk, d] (bf16, CPU), drawn in that order.

    Same recipe as :func:`make_qkv`, which it equals when Nq == Nk.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = torch.randn(B, H, Nq, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn(B, H, Nk, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn(B, H, Nk, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
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

    @property
    def exps(self) -> float:
        """Exponentials by the same convention: B*H*N^2, halved when causal."""
        e = float(self.B * self.H) * self.N * self.N
        return e / 2 if self.causal else e

    @property
    def io_bytes(self) -> float:
        """Algorithmic HBM bytes: Q, K, V read once, O written (bf16), LSE written (fp32)."""
        return float(self.B * self.H) * (8 * self.N * self.d + 4 * self.N)

    def as_dict(self) -> dict:
        return {"workload": self.name, "B": self.B, "H": self.H, "N": self.N,
                "d": self.d, "causal": self.causal, "qk_mult": self.qk_mult}

    def __repr__(self) -> str:  # pragma: no cover
        return f"Workload({self.as_dict()})"


class DecodeWorkload:
    """Nq queries (the last Nq positions) against Nk keys per (batch, head)."""

    def __init__(self, name: str, B: int, H: int, Nq: int, Nk: int, d: int, causal: bool, qk_mult: float = 1.0):
        self.name, self.B, self.H, self.Nq, self.Nk, self.d = name, B, H, Nq, Nk, d
        self.causal, self.qk_mult = bool(causal), float(qk_mult)

    @property
    def pairs(self) -> int:
        """Allowed (query, key) pairs per head."""
        if not self.causal:
            return self.Nq * self.Nk
        off = self.Nk - self.Nq
        return sum(off + i + 1 for i in range(self.Nq))

    @property
    def flops(self) -> float:
        """4 * d FLOP per allowed (query, key) pair (two dot products of length d)."""
        return 4.0 * self.B * self.H * self.pairs * self.d

    @property
    def bytes(self) -> float:
        """Algorithmic HBM bytes: read Q, K, V once (bf16), write O (bf16) and LSE (fp32)."""
        bh = self.B * self.H
        return bh * (2 * self.Nq * self.d * 2 + 2 * self.Nk * self.d * 2 + self.Nq * 4)

    def as_dict(self) -> dict:
        return {"workload": self.name, "B": self.B, "H": self.H, "Nq": self.Nq, "Nk": self.Nk,
                "d": self.d, "causal": self.causal, "qk_mult": self.qk_mult}

    def __repr__(self) -> str:  # pragma: no cover
        return f"DecodeWorkload({self.as_dict()})"


def _grid():
    out = []
    for d in (64, 128, 256):
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

#: Few queries against a long key sequence (split-K/V entry point).
for _w in (DecodeWorkload("decode_B8_H16_Nk16384_d128", 8, 16, 1, 16384, 128, True),
           DecodeWorkload("decode_B1_H16_Nk65536_d128", 1, 16, 1, 65536, 128, True),
           DecodeWorkload("decode_B32_H16_Nk4096_d64", 32, 16, 1, 4096, 64, True),
           DecodeWorkload("chunk_B1_H16_Nq512_Nk16384_d128", 1, 16, 512, 16384, 128, True)):
    WORKLOADS[_w.name] = _w
