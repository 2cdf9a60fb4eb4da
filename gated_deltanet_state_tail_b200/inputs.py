"""Seeded synthetic inputs for Gated DeltaNet tail replay and suffix prefill.

This module only draws random tensors and integer layouts.  It holds none of
the recurrence's arithmetic, so both the CUDA path's callers and the fp64
oracle's tests can use it without sharing method code.

Value recipe (stand-ins for the LongBench / RULER prefixes of 8K, 16K and 32K
tokens that the Tail-Replay pages evaluate on; neither dataset nor any model
is used):
  * q, k ~ N(0, 1), then L2-normalised per (token, head) in fp32, then cast
    to the storage dtype;
  * v ~ N(0, 1), cast to the storage dtype;
  * beta = sigmoid(N(0, 1)) in fp32;
  * alpha ~ U[lo, hi] in fp32 (the gate value, not its log).
Integer layouts (lengths, replay budgets) come from numpy's PCG64 so they are
identical on every machine.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

__all__ = [
    "SeqBatch", "draw_tensors", "ceil_budget", "replay_budget_bp",
    "tiny_workload", "single_layer_workload", "stack_workload", "varlen_workload",
    "sweep_workloads",
]


def ceil_budget(L: int, num: int, den: int) -> int:
    """ceil(L * num / den) in exact integer arithmetic."""
    return (L * num + den - 1) // den


def replay_budget_bp(L: int, basis_points: int) -> int:
    """Replay length for a budget given in basis points of L (10000 = 100%)."""
    return ceil_budget(L, basis_points, 10000)


@dataclass
class SeqBatch:
    """Integer layout of one packed varlen batch (host side)."""
    name: str
    H: int
    dk: int
    dv: int
    dtype: str                  # "f32" or "bf16"
    alpha_lo: float
    alpha_hi: float
    match_len: list             # L_b, matched prefix per sequence
    cached_len: list            # rows of the cache entry (>= L_b)
    R: list                     # replay budget per sequence (may exceed L_b; clamped)
    suffix_len: list            # N_b, new tokens per sequence
    seeds: list                 # one tensor seed per sequence group (layer)
    layers: int = 1             # sequences are grouped as layers x requests
    extra: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return len(self.match_len)

    def seq_offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.cached_len)]).astype(np.int32)

    def suffix_cu(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.suffix_len)]).astype(np.int32)

    def full_cu(self) -> np.ndarray:
        """Offsets of prefix ++ suffix sequences (the full-prefill comparator)."""
        full = [l + n for l, n in zip(self.match_len, self.suffix_len)]
        return np.concatenate([[0], np.cumsum(full)]).astype(np.int32)


def _torch_dtype(name: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def draw_tensors(rows: int, H: int, dk: int, dv: int, dtype: str, alpha_lo: float,
                 alpha_hi: float, seed: int, device="cpu", with_q: bool = True):
    """Draw q, k, v [rows, H, d] (storage dtype) and alpha, beta [rows, H] (fp32)."""
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed))
    td = _torch_dtype(dtype)
    out = {}
    names = ("q", "k") if with_q else ("k",)
    for name in names:
        x = torch.randn((rows, H, dk), generator=g, device=dev, dtype=torch.float32)
        x = x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)
        out[name] = x.to(td)
        del x
    if not with_q:
        out["q"] = None
    out["v"] = torch.randn((rows, H, dv), generator=g, device=dev, dtype=torch.float32).to(td)
    out["beta"] = torch.sigmoid(torch.randn((rows, H), generator=g, device=dev, dtype=torch.float32))
    a = torch.rand((rows, H), generator=g, device=dev, dtype=torch.float32)
    out["alpha"] = (alpha_lo + (alpha_hi - alpha_lo) * a).to(torch.float32)
    return out


def tiny_workload() -> SeqBatch:
    """1 layer, batch 1, 1 head, d_k = d_v = 64, fp32; L=256, R=32, N=32; alpha~U[0.90,0.999]."""
    return SeqBatch("tiny-d64-f32-L256-R32-N32", 1, 64, 64, "f32", 0.90, 0.999,
                    match_len=[256], cached_len=[256], R=[32], suffix_len=[32], seeds=[0])


def single_layer_workload() -> SeqBatch:
    """1 layer, batch 1, 16 heads, d=128, bf16; L=8192, R=410 (5%), N=512."""
    L = 8192
    return SeqBatch("layer-H16-d128-bf16-L8192-R410-N512", 16, 128, 128, "bf16", 0.90, 0.999,
                    match_len=[L], cached_len=[L], R=[ceil_budget(L, 5, 100)],
                    suffix_len=[512], seeds=[0])


def stack_workload(layers: int = 24) -> SeqBatch:
    """24 GDN layers (independent seeds 0..23), 32 heads, d=128, bf16; L=32768, R=3277 (10%), N=1024.

    Layers are stacked as a batch of `layers` sequences (one request per layer).
    """
    L = 32768
    return SeqBatch(f"stack{layers}-H32-d128-bf16-L32768-R3277-N1024", 32, 128, 128, "bf16",
                    0.90, 0.999, match_len=[L] * layers, cached_len=[L] * layers,
                    R=[ceil_budget(L, 10, 100)] * layers, suffix_len=[1024] * layers,
                    seeds=list(range(layers)), layers=layers)


def varlen_workload(batch: int = 64, seed: int = 0) -> SeqBatch:
    """Varlen batch: L_b ~ U{1024..32768} (redrawn while L_b % 64 == 0), R_b = ceil(f_b L_b)
    with f_b ~ U[0.05, 0.10] in basis points, N_b ~ U{64..2048}, cached = L_b + U{0..255}."""
    rng = np.random.Generator(np.random.PCG64(seed))
    L, R, N, C, bp = [], [], [], [], []
    for _ in range(batch):
        while True:
            l = int(rng.integers(1024, 32768, endpoint=True))
            if l % 64:
                break
        f = int(rng.integers(500, 1000, endpoint=True))
        L.append(l)
        bp.append(f)
        R.append(replay_budget_bp(l, f))
        N.append(int(rng.integers(64, 2048, endpoint=True)))
        C.append(l + int(rng.integers(0, 255, endpoint=True)))
    return SeqBatch(f"varlen{batch}-H16-d128-bf16", 16, 128, 128, "bf16", 0.90, 0.999,
                    match_len=L, cached_len=C, R=R, suffix_len=N, seeds=[seed],
                    extra={"budget_bp": bp})


def sweep_workloads():
    """Replay-budget sweep: 1 layer, 32 heads, d=128, bf16, alpha~U[0.97,0.9999];
    L in {8K, 16K, 32K}, R/L in {1, 2, 5, 10, 25, 100}%."""
    out = []
    for L in (8192, 16384, 32768):
        for pct in (1, 2, 5, 10, 25, 100):
            out.append(SeqBatch(f"sweep-L{L}-p{pct}", 32, 128, 128, "bf16", 0.97, 0.9999,
                                match_len=[L], cached_len=[L], R=[ceil_budget(L, pct, 100)],
                                suffix_len=[0], seeds=[0], extra={"pct": pct}))
    return out
