"""The seeded input recipe: integer budgets and layouts, and the value ranges of
the drawn tensors, against what the recipe states."""
from fractions import Fraction
import math

import numpy as np
import pytest
import torch

from gated_deltanet_state_tail_b200 import inputs


def test_ceil_budget_is_the_exact_ceiling():
    rng = np.random.default_rng(11)
    for _ in range(2000):
        L = int(rng.integers(0, 1 << 20))
        den = int(rng.integers(1, 20000))
        num = int(rng.integers(0, den + 1))
        assert inputs.ceil_budget(L, num, den) == math.ceil(Fraction(L * num, den))
    assert inputs.ceil_budget(8192, 5, 100) == 410          # 409.6 rounds up
    assert inputs.ceil_budget(32768, 10, 100) == 3277       # 3276.8 rounds up
    assert inputs.replay_budget_bp(10000, 733) == 733


def test_sweep_budgets():
    got = {(w.match_len[0], w.extra["pct"]): w.R[0] for w in inputs.sweep_workloads()}
    assert [got[(8192, p)] for p in (1, 2, 5, 10, 25, 100)] == [82, 164, 410, 820, 2048, 8192]
    assert [got[(32768, p)] for p in (1, 2, 5, 10, 25, 100)] == [328, 656, 1639, 3277, 8192, 32768]
    for w in inputs.sweep_workloads():
        assert (w.alpha_lo, w.alpha_hi, w.H, w.dtype) == (0.97, 0.9999, 32, "bf16")


def test_fixed_workloads():
    t = inputs.tiny_workload()
    assert (t.H, t.dk, t.dv, t.dtype, t.match_len, t.R, t.suffix_len) == (1, 64, 64, "f32", [256], [32], [32])
    s = inputs.single_layer_workload()
    assert (s.H, s.dk, s.match_len, s.R, s.suffix_len) == (16, 128, [8192], [410], [512])
    st = inputs.stack_workload()
    assert st.layers == 24 and st.batch == 24 and st.seeds == list(range(24))
    assert set(st.match_len) == {32768} and set(st.R) == {3277} and set(st.suffix_len) == {1024}


def test_varlen_workload_constraints_and_reproducibility():
    w = inputs.varlen_workload(64, seed=0)
    assert w.batch == 64 and w.H == 16
    for L, C, R, N, bp in zip(w.match_len, w.cached_len, w.R, w.suffix_len, w.extra["budget_bp"]):
        assert 1024 <= L <= 32768 and L % 64 != 0
        assert L <= C <= L + 255
        assert 500 <= bp <= 1000 and R == math.ceil(Fraction(L * bp, 10000))
        assert 64 <= N <= 2048
    w2 = inputs.varlen_workload(64, seed=0)
    assert (w.match_len, w.cached_len, w.R, w.suffix_len) == (w2.match_len, w2.cached_len, w2.R, w2.suffix_len)
    assert inputs.varlen_workload(64, seed=1).match_len != w.match_len


def test_batch_offsets():
    w = inputs.varlen_workload(5, seed=3)
    off, cu, full = w.seq_offsets(), w.suffix_cu(), w.full_cu()
    assert off.dtype == np.int32 and off[0] == 0 and list(np.diff(off)) == w.cached_len
    assert cu[0] == 0 and list(np.diff(cu)) == w.suffix_len
    assert list(np.diff(full)) == [l + n for l, n in zip(w.match_len, w.suffix_len)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_draw_tensors_recipe(dtype):
    t = inputs.draw_tensors(300, 3, 64, 32, dtype, 0.9, 0.999, seed=7)
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    assert t["q"].shape == (300, 3, 64) and t["k"].shape == (300, 3, 64) and t["v"].shape == (300, 3, 32)
    assert t["q"].dtype == td and t["k"].dtype == td and t["v"].dtype == td
    assert t["alpha"].dtype == torch.float32 and t["beta"].dtype == torch.float32
    # q and k are unit rows per (token, head), up to the storage rounding
    tol = 1e-5 if dtype == "f32" else 1e-2
    for name in ("q", "k"):
        n = t[name].float().norm(dim=-1)
        assert torch.all((n - 1).abs() <= tol)
    assert torch.all((t["beta"] > 0) & (t["beta"] < 1))
    assert torch.all((t["alpha"] >= 0.9) & (t["alpha"] <= 0.999))
    # the same seed gives the same bytes; q is optional
    t2 = inputs.draw_tensors(300, 3, 64, 32, dtype, 0.9, 0.999, seed=7)
    for name in ("q", "k", "v", "alpha", "beta"):
        assert torch.equal(t[name], t2[name])
    t3 = inputs.draw_tensors(300, 3, 64, 32, dtype, 0.9, 0.999, seed=7, with_q=False)
    assert t3["q"] is None
    t4 = inputs.draw_tensors(300, 3, 64, 32, dtype, 0.9, 0.999, seed=8)
    assert not torch.equal(t["k"], t4["k"])
