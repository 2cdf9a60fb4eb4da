"""GPU parity of the fused rebuild + suffix prefill against the fp64 oracle's
replay followed by its prefill, on ragged batches that include an empty window,
an empty suffix, R = 0 and R > L.  Tolerance: max|err|/max|ref| per request and
tensor.

The tensor-core kernel runs a fused call as one launch when no replay window is
longer than 320 tokens, or when the plan has at most one (sequence, head) unit per
SM and no window is longer than 1024 tokens, and otherwise (or with a replay kernel
pinned) as the state-only replay launch followed by the prefill launch; both
schedules are covered, and the two-launch one must equal separate replay and
prefill plans bit for bit."""
import numpy as np
import pytest
import torch

import gated_deltanet_state_tail_b200 as gdn
from gated_deltanet_state_tail_b200 import inputs
import oracle
from helpers import TOL, oracle_view, per_request_rows_err, per_request_state_err

pytestmark = pytest.mark.gpu

KERNELS = {"recurrent": gdn.GDN_KERNEL_RECURRENT, "chunked": gdn.GDN_KERNEL_CHUNKED_TC,
           "two_cta": gdn.GDN_KERNEL_CHUNKED_TC_TWO_CTA}
FAMILY = {"recurrent": gdn.GDN_KERNEL_RECURRENT, "chunked": gdn.GDN_KERNEL_CHUNKED_TC,
          "two_cta": gdn.GDN_KERNEL_CHUNKED_TC}
LAUNCHES = {"recurrent": 2, "chunked": 1, "two_cta": 2}


@pytest.mark.parametrize("kname", ["recurrent", "chunked", "two_cta"])
@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 64, 64), ("f32", 128, 128)])
@pytest.mark.parametrize("with_mid", [True, False])
def test_fused_matches_replay_then_prefill(kname, dtype, dk, dv, with_mid):
    if kname != "recurrent" and not (dtype == "bf16" and dk == 128 and dv == 128):
        pytest.skip("chunked kernel serves bf16 with d = 128")
    kernel = KERNELS[kname]
    cached = [300, 64, 129, 0, 77, 1000, 50]
    ml = [300, 64, 100, 0, 50, 997, 50]
    R = [190, 64, 0, 10, 80, 333, 50]
    slen = [65, 0, 130, 7, 64, 200, 0]
    off = np.concatenate([[0], np.cumsum(cached)]).astype(np.int32)
    so = np.concatenate([[0], np.cumsum(slen)]).astype(np.int32)
    H = 2
    cache = inputs.draw_tensors(int(off[-1]), H, dk, dv, dtype, 0.9, 0.999, 51, device="cpu", with_q=False)
    suf = inputs.draw_tensors(int(so[-1]), H, dk, dv, dtype, 0.9, 0.999, 52, device="cpu")
    c = {k: (None if x is None else x.cuda()) for k, x in cache.items()}
    s = {k: x.cuda() for k, x in suf.items()}
    plan = gdn.FusedPlan(H, dk, dv, dtype, off, ml, R, so, kernel)
    assert plan.info["kernel"] == FAMILY[kname]
    assert plan.launches == LAUNCHES[kname]
    sentinel = -5.0
    o = torch.full((int(so[-1]), H, dv), sentinel, dtype=s["v"].dtype, device="cuda")
    st = torch.full((len(ml), H, dk, dv), float("nan"), device="cuda")
    mid = torch.full_like(st, float("nan")) if with_mid else None
    plan.run(c["k"], c["v"], c["alpha"], c["beta"], s["q"], s["k"], s["v"], s["alpha"], s["beta"], o, st,
             state_mid=mid)
    assert plan.status() == gdn.GDN_OK
    for b in range(len(ml)):
        assert plan.window(b) == oracle.replay_window(off, ml, R, b)
    plan.close()
    ref_mid = oracle.replay_state(oracle_view(cache["k"]), oracle_view(cache["v"]), oracle_view(cache["alpha"]),
                                  oracle_view(cache["beta"]), off, ml, R)
    ref_o, ref_st = oracle.prefill(oracle_view(suf["q"]), oracle_view(suf["k"]), oracle_view(suf["v"]),
                                   oracle_view(suf["alpha"]), oracle_view(suf["beta"]), so, state_in=ref_mid)
    assert per_request_rows_err(o.float().cpu().numpy(), ref_o, so) <= TOL[dtype]
    assert per_request_state_err(st.cpu().numpy(), ref_st) <= TOL[dtype]
    if with_mid:
        got_mid = mid.cpu().numpy()
        assert per_request_state_err(got_mid, ref_mid) <= TOL[dtype]
        assert np.count_nonzero(got_mid[2]) == 0 and np.count_nonzero(got_mid[3]) == 0   # R = 0, L = 0
    # empty suffixes: the final state is the rebuilt state
    for b in (1, 6):
        assert per_request_state_err(st.cpu().numpy()[b:b + 1], ref_mid[b:b + 1]) <= TOL[dtype]


def _fused_vs_separate(H, cached, ml, R, slen, seed):
    """Runs the default fused plan and separate replay + prefill plans on the same rows;
    returns the fused plan's launch count, both results and the oracle's."""
    off = np.concatenate([[0], np.cumsum(cached)]).astype(np.int32)
    so = np.concatenate([[0], np.cumsum(slen)]).astype(np.int32)
    D = 128
    cache = inputs.draw_tensors(int(off[-1]), H, D, D, "bf16", 0.9, 0.999, seed, device="cpu", with_q=False)
    suf = inputs.draw_tensors(int(so[-1]), H, D, D, "bf16", 0.9, 0.999, seed + 1, device="cpu")
    c = {k: (None if x is None else x.cuda()) for k, x in cache.items()}
    s = {k: x.cuda() for k, x in suf.items()}
    B = len(ml)
    fp = gdn.FusedPlan(H, D, D, "bf16", off, ml, R, so)
    o = torch.full((int(so[-1]), H, D), -5.0, dtype=torch.bfloat16, device="cuda")
    st = torch.full((B, H, D, D), float("nan"), device="cuda")
    mid = torch.full_like(st, float("nan"))
    fp.run(c["k"], c["v"], c["alpha"], c["beta"], s["q"], s["k"], s["v"], s["alpha"], s["beta"], o, st,
           state_mid=mid)
    fp.check()
    rp = gdn.ReplayPlan(H, D, D, "bf16", off, ml, R)
    pp = gdn.PrefillPlan(H, D, D, "bf16", so)
    o2 = torch.full_like(o, -5.0)
    mid2 = torch.full_like(st, float("nan"))
    st2 = torch.full_like(st, float("nan"))
    rp.run(c["k"], c["v"], c["alpha"], c["beta"], mid2)
    pp.run(s["q"], s["k"], s["v"], s["alpha"], s["beta"], o2, state_in=mid2, state_out=st2)
    rp.check()
    pp.check()
    launches = fp.launches
    for p in (fp, rp, pp):
        p.close()
    ref_mid = oracle.replay_state(oracle_view(cache["k"]), oracle_view(cache["v"]), oracle_view(cache["alpha"]),
                                  oracle_view(cache["beta"]), off, ml, R)
    ref_o, ref_st = oracle.prefill(oracle_view(suf["q"]), oracle_view(suf["k"]), oracle_view(suf["v"]),
                                   oracle_view(suf["alpha"]), oracle_view(suf["beta"]), so, state_in=ref_mid)
    got = (o.float().cpu().numpy(), mid.cpu().numpy(), st.cpu().numpy())
    sep = (o2.float().cpu().numpy(), mid2.cpu().numpy(), st2.cpu().numpy())
    ref = (ref_o, ref_mid, ref_st)
    for g, r in zip(got, ref):
        if g.ndim == 3:
            assert per_request_rows_err(g, r, so) <= TOL["bf16"]
        else:
            assert per_request_state_err(g, r) <= TOL["bf16"]
    return launches, got, sep


def test_fused_long_window_runs_as_replay_then_prefill():
    # one window of 1200 tokens (19 chunks, above 1024): two launches, the same kernels as
    # separate plans, so the same bits
    launches, got, sep = _fused_vs_separate(4, [1500, 400, 64], [1400, 380, 64], [1200, 300, 64],
                                            [100, 64, 0], 61)
    assert launches == 2
    for g, e in zip(got, sep):
        assert np.array_equal(g, e)


def test_fused_more_units_than_sms_runs_as_replay_then_prefill():
    # more units than SMs and one window over 320 tokens: two launches
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    H = 4
    B = sms // H + 2                  # H * B > SMs
    rng = np.random.default_rng(9)
    cached = rng.integers(40, 200, size=B)
    ml = np.minimum(cached, rng.integers(30, 200, size=B)).astype(np.int32)
    R = rng.integers(0, 160, size=B).astype(np.int32)
    cached[0] = ml[0] = R[0] = 330
    slen = rng.integers(0, 90, size=B)
    launches, got, sep = _fused_vs_separate(H, cached, ml, R, slen, 71)
    assert launches == 2
    for g, e in zip(got, sep):
        assert np.array_equal(g, e)


def test_fused_more_units_than_sms_short_windows_run_as_one_launch():
    # more units than SMs, every window <= 320 tokens (one of exactly 320): one launch,
    # checked against the oracle
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    H = 4
    B = sms // H + 2
    rng = np.random.default_rng(12)
    cached = rng.integers(40, 400, size=B)
    ml = np.minimum(cached, rng.integers(30, 400, size=B)).astype(np.int32)
    R = np.minimum(rng.integers(0, 321, size=B), 320).astype(np.int32)
    cached[0] = ml[0] = R[0] = 320
    slen = rng.integers(0, 90, size=B)
    launches, _, _ = _fused_vs_separate(H, cached, ml, R, slen, 91)
    assert launches == 1


def test_fused_short_windows_run_as_one_launch():
    # at most one unit per SM and every window <= 1024 tokens (one of exactly 1024): one
    # launch, checked against the oracle (its rounding differs from the separate plans')
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    H = 4
    B = sms // H
    rng = np.random.default_rng(10)
    cached = rng.integers(40, 1100, size=B)
    ml = np.minimum(cached, rng.integers(30, 1100, size=B)).astype(np.int32)
    R = np.minimum(rng.integers(0, 1025, size=B), 1024).astype(np.int32)
    R[0] = 1024
    ml[0] = cached[0] = 1100
    slen = rng.integers(0, 90, size=B)
    launches, _, _ = _fused_vs_separate(H, cached, ml, R, slen, 81)
    assert launches == 1
