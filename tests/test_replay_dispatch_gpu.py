"""The state-only replay's three tensor-core kernels, each pinned through the
descriptor, on launches of three sizes.

The chunked path runs the replay on a kernel with two CTAs per SM by default, on a
warp-specialised kernel with one CTA per SM or on a cluster-pair kernel (each unit
on two CTAs on two SMs) when the descriptor pins one.  Each kernel replays the same
ragged windows (several 64-token chunks and a partial last chunk) on a launch with
at most one (request, head) unit per two SMs, one with at most one per SM and one
with more; every unit is checked element by element against the fp64 oracle, the
default must equal the two-CTA kernel bit for bit, and so must the pair kernel (the
same operations in the same order); the warp-specialised kernel must agree within
the oracle's bound.
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


def test_replay_kernels_across_launch_sizes():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    b_pair = sms // (2 * H)             # units = H * b_pair <= SMs / 2
    b_small = sms // H                  # units <= SMs
    b_large = b_small + 2               # units > SMs
    rng = np.random.default_rng(5)
    ml = rng.integers(70, 330, size=b_large).astype(np.int32)
    cached = ml + rng.integers(0, 40, size=b_large)
    R = np.minimum(ml, rng.integers(60, 300, size=b_large)).astype(np.int32)
    off = np.concatenate([[0], np.cumsum(cached)]).astype(np.int32)
    t = inputs.draw_tensors(int(off[-1]), H, D, D, "bf16", 0.9, 0.999, 21, device="cuda", with_q=False)
    ref = oracle.replay_state(oracle_view(t["k"]), oracle_view(t["v"]), oracle_view(t["alpha"]),
                              oracle_view(t["beta"]), off, ml, R)
    assert 2 * H * b_pair <= sms < 2 * H * (b_pair + 1) and H * b_small <= sms < H * b_large
    names = {"two_cta": gdn.GDN_KERNEL_CHUNKED_TC_TWO_CTA, "warp_spec": gdn.GDN_KERNEL_CHUNKED_TC_WARP_SPEC,
             "pair": gdn.GDN_KERNEL_CHUNKED_TC_PAIR}
    for nb in (b_pair, b_small, b_large):
        o, m, r = off[:nb + 1], ml[:nb], R[:nb]
        got = {k: _replay(t, o, m, r, v) for k, v in names.items()}
        auto = _replay(t, o, m, r, gdn.GDN_KERNEL_AUTO)
        assert np.array_equal(auto, got["two_cta"]), f"{nb} requests: the default is not the two-CTA kernel"
        assert np.array_equal(got["pair"], got["two_cta"]), f"{nb} requests: the pair kernel's bits differ"
        for b in range(nb):
            for k, g in got.items():
                assert rel_err(g[b], ref[b]) <= TOL["bf16"], f"{nb} requests, request {b} ({k} kernel)"
                assert rel_err(g[b], got["two_cta"][b]) <= TOL["bf16"], f"{nb} requests, request {b}: {k} vs two_cta"
