"""The state-only replay's two tensor-core kernels, on each side of the launch
size that picks between them.

A replay launch with at most one (request, head) unit per SM runs the
warp-specialised kernel (one CTA per SM; the state-independent work of a unit's
chunks runs ahead of its state chain); a larger launch runs the two-chunk kernel
(two CTAs per SM).  Both launches here replay ragged windows (several 64-token
chunks and a partial last chunk) and are checked element by element against the
fp64 oracle on every unit; the units the two launches share must agree within
the same bound.
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


def _replay(t, off, ml, R):
    plan = gdn.ReplayPlan(H, D, D, "bf16", off, ml, R)
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
    small = _replay(t, off[:b_small + 1], ml[:b_small], R[:b_small])
    large = _replay(t, off, ml, R)
    for b in range(b_large):
        assert rel_err(large[b], ref[b]) <= TOL["bf16"], f"request {b} (two-chunk kernel)"
    for b in range(b_small):
        assert rel_err(small[b], ref[b]) <= TOL["bf16"], f"request {b} (warp-specialised kernel)"
        assert rel_err(small[b], large[b]) <= TOL["bf16"], f"request {b}: the kernels disagree"
