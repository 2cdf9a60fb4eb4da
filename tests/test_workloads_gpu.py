"""Full-size workloads on the GPU, checked on sampled units against the fp64
oracle and through properties that hold at any size.

* varlen batch: 64 requests, 16 heads, matched prefixes 1K..32K not aligned
  to any chunk, replay budgets ceil(5..10% of L), suffixes 64..2048;
* replay-budget sweep: 32 heads, slow decay alpha ~ U[0.97, 0.9999],
  prefixes 8K / 16K / 32K, R/L in {1, 2, 5, 10, 25, 100}%.
"""
import numpy as np
import pytest
import torch

import gated_deltanet_state_tail_b200 as gdn
from gated_deltanet_state_tail_b200 import inputs
import oracle
from helpers import TOL, oracle_view, rel_err

pytestmark = pytest.mark.gpu


def _sub(t, rows):
    """Rows of every tensor of a dict, copied to the host for the oracle."""
    return {k: (None if x is None else x[rows]) for k, x in t.items()}


def test_varlen_batch_full_size_sampled():
    wl = inputs.varlen_workload(64, seed=0)
    off = wl.seq_offsets()
    H = wl.H
    cache = inputs.draw_tensors(int(off[-1]), H, 128, 128, "bf16", wl.alpha_lo, wl.alpha_hi, 100,
                                device="cuda", with_q=False)
    plan = gdn.ReplayPlan(H, 128, 128, "bf16", off, wl.match_len, wl.R)
    assert plan.info["kernel"] == gdn.GDN_KERNEL_CHUNKED_TC
    state = torch.empty((wl.batch, H, 128, 128), device="cuda")
    plan.run(cache["k"], cache["v"], cache["alpha"], cache["beta"], state,
             seq_offsets=torch.tensor(off, device="cuda"),
             match_len=torch.tensor(np.asarray(wl.match_len, np.int32), device="cuda"),
             R=torch.tensor(np.asarray(wl.R, np.int32), device="cuda"))
    assert plan.status() == gdn.GDN_OK
    # windows are bit-exact with the oracle's
    for b in range(wl.batch):
        assert plan.window(b) == oracle.replay_window(off, wl.match_len, wl.R, b)

    cu = wl.suffix_cu()
    suf = inputs.draw_tensors(int(cu[-1]), H, 128, 128, "bf16", wl.alpha_lo, wl.alpha_hi, 101, device="cuda")
    pplan = gdn.PrefillPlan(H, 128, 128, "bf16", cu)
    o = torch.zeros((int(cu[-1]), H, 128), dtype=torch.bfloat16, device="cuda")
    st2 = torch.empty_like(state)
    pplan.run(suf["q"], suf["k"], suf["v"], suf["alpha"], suf["beta"], o, state_in=state, state_out=st2,
              cu_seqlens=torch.tensor(cu, device="cuda"))
    assert pplan.status() == gdn.GDN_OK

    # sampled requests: the longest and shortest windows and a few in between; two heads each
    order = np.argsort(wl.R)
    picks = sorted({int(order[0]), int(order[-1]), int(order[len(order) // 3]), int(order[2 * len(order) // 3])})
    for b in picks:
        r0, n = plan.window(b)
        heads = [0, H - 1]
        rows = slice(r0, r0 + n)
        sub = _sub(cache, rows)
        for hh in heads:
            ref = oracle.replay_state(oracle_view(sub["k"][:, hh:hh + 1]), oracle_view(sub["v"][:, hh:hh + 1]),
                                      oracle_view(sub["alpha"][:, hh:hh + 1]), oracle_view(sub["beta"][:, hh:hh + 1]),
                                      [0, n], [n], [n])[0, 0]
            assert rel_err(state[b, hh].cpu().numpy(), ref) <= TOL["bf16"], f"replay request {b} head {hh}"
            srows = slice(int(cu[b]), int(cu[b + 1]))
            ss = _sub(suf, srows)
            ref_o, ref_s = oracle.prefill(oracle_view(ss["q"][:, hh:hh + 1]), oracle_view(ss["k"][:, hh:hh + 1]),
                                          oracle_view(ss["v"][:, hh:hh + 1]), oracle_view(ss["alpha"][:, hh:hh + 1]),
                                          oracle_view(ss["beta"][:, hh:hh + 1]), [0, int(cu[b + 1] - cu[b])],
                                          state_in=state[b:b + 1, hh:hh + 1].double().cpu().numpy())
            assert rel_err(o[srows, hh].float().cpu().numpy(), ref_o[:, 0]) <= TOL["bf16"], f"suffix o {b} {hh}"
            assert rel_err(st2[b, hh].cpu().numpy(), ref_s[0, 0]) <= TOL["bf16"], f"suffix state {b} {hh}"
    plan.close()
    pplan.close()


@pytest.mark.parametrize("L", [8192, 32768])
def test_replay_budget_sweep_error_curve(L):
    """The replay-budget sweep (slow decay, alpha ~ U[0.97, 0.9999]) on sampled heads:

    * at every budget R/L in {1, 2, 5, 10, 25, 100}% the GPU's replayed state
      matches the fp64 oracle's replay of the same window element by element;
    * the truncation error ||S_R - S_L|| / ||S_L||, taken from the oracle alone
      (fp64, no kernel rounding in it), shrinks as R grows (gated updates
      attenuate older inputs), is exactly 0 at R = L, and falls below the
      kernel's own rounding error once the window is long enough."""
    H = 32
    t = inputs.draw_tensors(L, H, 128, 128, "bf16", 0.97, 0.9999, 7, device="cuda", with_q=False)
    heads = [0, 17]
    sub = {n: oracle_view(t[n][:, heads]) for n in ("k", "v", "alpha", "beta")}
    S_full = oracle.replay_state(sub["k"], sub["v"], sub["alpha"], sub["beta"], [0, L], [L], [L])[0]
    trunc, kern = [], []
    for pct in (1, 2, 5, 10, 25, 100):
        R = inputs.ceil_budget(L, pct, 100)
        plan = gdn.ReplayPlan(H, 128, 128, "bf16", [0, L], [L], [R])
        st = torch.empty((1, H, 128, 128), device="cuda")
        plan.run(t["k"], t["v"], t["alpha"], t["beta"], st)
        assert plan.status() == gdn.GDN_OK
        plan.close()
        S_rep = oracle.replay_state(sub["k"], sub["v"], sub["alpha"], sub["beta"], [0, L], [L], [R])[0]
        got = st[0, heads].cpu().numpy()
        for i, hh in enumerate(heads):
            e = rel_err(got[i], S_rep[i])
            assert e <= TOL["bf16"], f"L {L} R {R} head {hh}: {e}"
            kern.append(e)
        trunc.append([np.linalg.norm(S_rep[i] - S_full[i]) / np.linalg.norm(S_full[i]) for i in range(len(heads))])
    trunc = np.array(trunc)
    assert np.all(trunc[-1] == 0.0)                       # R = L replays the whole prefix
    assert np.all(np.diff(trunc, axis=0) <= 1e-12)        # non-increasing in R
    assert np.all(trunc[0] > 1e-4)                        # 1% of the prefix is a visible truncation
    floor = max(kern)
    assert np.all(trunc[4] < floor), f"25% budget: truncation {trunc[4]} vs kernel rounding {floor}"
