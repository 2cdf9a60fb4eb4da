"""The state-only replay's two tensor-core kernels, each pinned through the
descriptor, on launches on both sides of one unit per SM.

The chunked path runs the replay on a kernel with two CTAs per SM (the default)
or, when the descriptor pins it, on a warp-specialised kernel with one CTA per
SM (the front of a unit's chunks runs ahead of its state chain).  Each kernel
replays the same ragged windows (several 64-token chunks and a partial last
chunk) on a launch with at most one (request, head) unit per SM and on one with
more; every unit is checked element by element against the fp64 oracle, the
default must be the two-CTA kernel bit for bit, and the two kernels must agree
within the same bound.
"""
import numpy as np
import pytest
import torch

import gated_deltanet_state_tail_b200 as gdn
from gated_deltanet_state_tail_b200 import inputs
import oracle
from helpers import TOL, oracle_view, rel_err

pytestmark = pytest.mark.gpu

H, D = 4, 128


def _replay(t, off, ml, R, kernel):
    plan = gdn.ReplayPlan(H, D, D, "bf16", off, ml, R, kernel)
    out = torch.full((len(ml), H, D, D), float("nan"), device="cuda")
    plan.run(t["k"], t["v"], t["alpha"], t["beta"], out)
    plan.check()
    plan.close()
    return out.cpu().numpy()


def test_both_replay_kernels_around_one_unit_per_sm():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    b_small = sms // H                  # units = H * b_small <= SMs
    b_large = b_small + 2               # units > SMs
    rng = np.random.default_rng(5)
    ml = rng.integers(70, 330, size=b_large).astype(np.int32)
    cached = ml + rng.integers(0, 40, size=b_large)
    R = np.minimum(ml, rng.integers(60, 300, size=b_large)).astype(np.int32)
    off = np.concatenate([[0], np.cumsum(cached)]).astype(np.int32)
    t = inputs.draw_tensors(int(off[-1]), H, D, D, "bf16", 0.9, 0.999, 21, device="cuda", with_q=False)
    ref = oracle.replay_state(oracle_view(t["k"]), oracle_view(t["v"]), oracle_view(t["alpha"]),
                              oracle_view(t["beta"]), off, ml, R)
    assert H * b_small <= sms < H * b_large
    for nb in (b_small, b_large):
        o, m, r = off[:nb + 1], ml[:nb], R[:nb]
        two = _replay(t, o, m, r, gdn.GDN_KERNEL_CHUNKED_TC_TWO_CTA)
        ws = _replay(t, o, m, r, gdn.GDN_KERNEL_CHUNKED_TC_WARP_SPEC)
        auto = _replay(t, o, m, r, gdn.GDN_KERNEL_AUTO)
        assert np.array_equal(auto, two), f"{nb} requests: the default is not the two-CTA kernel"
        for b in range(nb):
            assert rel_err(two[b], ref[b]) <= TOL["bf16"], f"{nb} requests, request {b} (two-CTA kernel)"
            assert rel_err(ws[b], ref[b]) <= TOL["bf16"], f"{nb} requests, request {b} (warp-specialised kernel)"
            assert rel_err(ws[b], two[b]) <= TOL["bf16"], f"{nb} requests, request {b}: the kernels disagree"
