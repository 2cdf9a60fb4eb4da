"""The allocation-free replay entry point, for callers that cannot call
cudaMalloc (a memory pool that owns the whole device heap, or a runtime that
only hands out its own buffers): on two calls in a row its output must equal
the plan-based entry point's bit for bit (both run the same kernel on the same
schedule), and match the fp64 oracle within the parity tolerance.  This file
is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import gated_deltanet_state_tail_b200 as gdn
from gated_deltanet_state_tail_b200 import inputs
import oracle
from helpers import TOL, oracle_view, rel_err

pytestmark = pytest.mark.gpu


def _case(seed, dtype, dk, dv, H=3):
    cached = [300, 64, 129, 0, 77, 1000]
    ml = [300, 64, 100, 0, 50, 997]
    R = [190, 64, 0, 10, 80, 333]
    off = np.concatenate([[0], np.cumsum(cached)]).astype(np.int32)
    t = inputs.draw_tensors(int(off[-1]), H, dk, dv, dtype, 0.9, 0.999, seed, device="cpu")
    t = {k: (None if x is None else x.cuda()) for k, x in t.items()}
    return t, off, ml, R


def _plan_replay(t, off, ml, R, dtype, dk, dv, H):
    plan = gdn.ReplayPlan(H, dk, dv, dtype, off, ml, R)
    out = torch.empty((len(ml), H, dk, dv), device="cuda")
    plan.run(t["k"], t["v"], t["alpha"], t["beta"], out)
    assert plan.status() == gdn.GDN_OK
    plan.close()
    return out


@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 64, 64)])
def test_noalloc_matches_plan_entry_point_twice(dtype, dk, dv):
    H = 3
    for call, seed in enumerate((21, 22)):
        t, off, ml, R = _case(seed, dtype, dk, dv, H)
        ref = _plan_replay(t, off, ml, R, dtype, dk, dv, H)
        out = torch.full((len(ml), H, dk, dv), float("nan"), device="cuda")
        status = gdn.gdn_tail_replay_state_noalloc(H, dk, dv, dtype, off, ml, R, t["k"], t["v"],
                                                   t["alpha"], t["beta"], out)
        assert status == 0, f"call {call}: device status {status}"
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"call {call}: differs from the plan entry point"
        want = oracle.replay_state(oracle_view(t["k"]), oracle_view(t["v"]), oracle_view(t["alpha"]),
                                   oracle_view(t["beta"]), off, ml, R)
        got = out.cpu().numpy()
        for b in range(len(ml)):
            assert rel_err(got[b], want[b]) <= TOL[dtype], f"call {call} request {b}"


def test_noalloc_rejects_batches_beyond_its_scratch():
    # 256 + 32 * 300 + 8 * 300 * 64 bytes > 64 KB
    B, H = 300, 64
    off = np.arange(B + 1, dtype=np.int32) * 10
    with pytest.raises(gdn.GdnError) as e:
        gdn.gdn_tail_replay_state_noalloc(H, 64, 64, "f32", off, [10] * B, [5] * B, None, None, None,
                                          None, None)
    assert e.value.status == gdn.GDN_ERR_UNSUPPORTED
