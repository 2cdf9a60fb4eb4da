"""GPU parity of the two entry points that widen the hot path: the replay that
also emits the window's outputs (layer chaining inside a replay group) and
the single-token decode step after the prefill.  Both go through the C ABI
and are compared with the fp64 oracle on the same seeded inputs (tolerance
max|err|/max|ref| per request and tensor: 1e-4 fp32, 2e-2 bf16)."""
import numpy as np
import pytest
import torch

import gated_deltanet_state_tail_b200 as gdn
from gated_deltanet_state_tail_b200 import inputs
import oracle
from helpers import TOL, oracle_view, per_request_rows_err, per_request_state_err, rel_err

pytestmark = pytest.mark.gpu

KERNELS = {"recurrent": gdn.GDN_KERNEL_RECURRENT, "chunked": gdn.GDN_KERNEL_CHUNKED_TC}


def kernel_or_skip(name, dtype, dk, dv):
    if name == "chunked" and not (dtype == "bf16" and dk == 128 and dv == 128):
        pytest.skip("chunked kernel serves bf16 with d = 128")
    return KERNELS[name]


@pytest.mark.parametrize("kname", ["recurrent", "chunked"])
@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 128, 64), ("bf16", 64, 64)])
def test_replay_outputs_varlen(kname, dtype, dk, dv):
    """Window outputs and states of a ragged replay (R = 0, R > L, L = 0,
    cache longer than the match); rows outside the windows stay untouched."""
    kernel = kernel_or_skip(kname, dtype, dk, dv)
    cached = [300, 64, 129, 0, 77, 1000]
    ml = [300, 64, 100, 0, 50, 997]
    R = [190, 64, 0, 10, 80, 333]
    off = np.concatenate([[0], np.cumsum(cached)]).astype(np.int32)
    H = 3
    t = inputs.draw_tensors(int(off[-1]), H, dk, dv, dtype, 0.9, 0.999, 21, device="cpu")
    td = {k: x.cuda() for k, x in t.items()}
    plan = gdn.ReplayPlan(H, dk, dv, dtype, off, ml, R, kernel)
    sentinel = -7.0
    o = torch.full((int(off[-1]), H, dv), sentinel, dtype=td["v"].dtype, device="cuda")
    st = torch.full((len(ml), H, dk, dv), float("nan"), device="cuda")
    dev = lambda a: torch.tensor(np.asarray(a, np.int32), device="cuda")
    plan.run_outputs(td["q"], td["k"], td["v"], td["alpha"], td["beta"], o, state_out=st,
                     seq_offsets=dev(off), match_len=dev(ml), R=dev(R))
    assert plan.status() == gdn.GDN_OK
    wins = [plan.window(b) for b in range(len(ml))]
    plan.close()
    for b, w in enumerate(wins):
        assert w == oracle.replay_window(off, ml, R, b)
    # oracle: a prefill from zero over the concatenated windows
    rows = np.concatenate([np.arange(r0, r0 + n) for r0, n in wins]).astype(np.int64)
    cu = np.concatenate([[0], np.cumsum([n for _, n in wins])]).astype(np.int32)
    sub = {k: x[torch.as_tensor(rows)] for k, x in t.items()}
    ref_o, ref_st = oracle.prefill(oracle_view(sub["q"]), oracle_view(sub["k"]), oracle_view(sub["v"]),
                                   oracle_view(sub["alpha"]), oracle_view(sub["beta"]), cu)
    got = o.float().cpu().numpy()
    assert per_request_rows_err(got[rows], ref_o, cu) <= TOL[dtype]
    assert per_request_state_err(st.cpu().numpy(), ref_st) <= TOL[dtype]
    # states agree with the state-only replay's oracle; other rows are untouched
    ref_replay = oracle.replay_state(oracle_view(t["k"]), oracle_view(t["v"]), oracle_view(t["alpha"]),
                                     oracle_view(t["beta"]), off, ml, R)
    assert per_request_state_err(st.cpu().numpy(), ref_replay) <= TOL[dtype]
    mask = np.ones(int(off[-1]), bool)
    mask[rows] = False
    assert np.all(got[mask] == sentinel)


@pytest.mark.parametrize("dtype,dk,dv", [("f32", 64, 64), ("f32", 128, 128), ("bf16", 128, 128),
                                         ("bf16", 64, 128), ("f32", 128, 64)])
@pytest.mark.parametrize("mode", ["zero_state", "separate_out", "in_place"])
def test_decode_step_matches_oracle(dtype, dk, dv, mode):
    B, H = 37, 5
    t = inputs.draw_tensors(B, H, dk, dv, dtype, 0.5, 1.0, 31, device="cpu")
    g = torch.Generator(device="cpu").manual_seed(3)
    s0 = None if mode == "zero_state" else torch.randn((B, H, dk, dv), generator=g) * 0.3
    td = {k: x.cuda() for k, x in t.items()}
    o = torch.empty((B, H, dv), dtype=td["v"].dtype, device="cuda")
    if mode == "in_place":
        st = s0.cuda()
        gdn.gdn_decode_step(td["q"], td["k"], td["v"], td["alpha"], td["beta"], st, st, o)
    else:
        st = torch.full((B, H, dk, dv), float("nan"), device="cuda")
        gdn.gdn_decode_step(td["q"], td["k"], td["v"], td["alpha"], td["beta"],
                            None if s0 is None else s0.cuda(), st, o)
    torch.cuda.synchronize()
    cu = np.arange(B + 1, dtype=np.int32)       # one token per request
    ref_o, ref_st = oracle.prefill(oracle_view(t["q"]), oracle_view(t["k"]), oracle_view(t["v"]),
                                   oracle_view(t["alpha"]), oracle_view(t["beta"]), cu,
                                   state_in=None if s0 is None else s0.double().numpy())
    assert per_request_rows_err(o.float().cpu().numpy(), ref_o, cu) <= TOL[dtype]
    assert per_request_state_err(st.cpu().numpy(), ref_st) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_prefill_then_decode_equals_longer_prefill(dtype):
    """Prefill of N tokens (chunked or recurrent by dtype) then one decode step
    gives the oracle's prefill over N + 1 tokens: output of the last token and
    the final state."""
    dk = dv = 128 if dtype == "bf16" else 64
    lens = [65, 1, 200, 130]
    H = 2
    cu1 = np.concatenate([[0], np.cumsum([n + 1 for n in lens])]).astype(np.int32)
    t = inputs.draw_tensors(int(cu1[-1]), H, dk, dv, dtype, 0.9, 0.999, 41, device="cpu")
    head_rows = np.concatenate([np.arange(cu1[b], cu1[b] + lens[b]) for b in range(len(lens))])
    last_rows = np.array([cu1[b] + lens[b] for b in range(len(lens))])
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    head = {k: x[torch.as_tensor(head_rows)].cuda() for k, x in t.items()}
    last = {k: x[torch.as_tensor(last_rows)].cuda() for k, x in t.items()}
    _, st = gdn.chunk_prefill(head["q"], head["k"], head["v"], head["alpha"], head["beta"], cu)
    o, st = gdn.decode_step(last["q"], last["k"], last["v"], last["alpha"], last["beta"], st)
    torch.cuda.synchronize()
    ref_o, ref_st = oracle.prefill(oracle_view(t["q"]), oracle_view(t["k"]), oracle_view(t["v"]),
                                   oracle_view(t["alpha"]), oracle_view(t["beta"]), cu1)
    assert rel_err(o.float().cpu().numpy(), ref_o[last_rows]) <= TOL[dtype]
    assert per_request_state_err(st.cpu().numpy(), ref_st) <= TOL[dtype]


def test_decode_step_empty_batch_and_validation():
    lib = gdn.library()
    assert lib.gdn_decode_step(0, 4, 128, 128, gdn.GDN_BF16, *([None] * 8), None) == gdn.GDN_OK
    x = torch.zeros((2, 2, 128), dtype=torch.bfloat16, device="cuda")
    a = torch.ones((2, 2), device="cuda")
    s = torch.zeros((2, 2, 128, 128), device="cuda")
    # misaligned state pointer: rejected before launch
    assert lib.gdn_decode_step(2, 2, 128, 128, gdn.GDN_BF16, x.data_ptr(), x.data_ptr(), x.data_ptr(),
                               a.data_ptr(), a.data_ptr(), s.data_ptr() + 4, s.data_ptr(), x.data_ptr(),
                               None) == gdn.GDN_ERR_INVALID_ARG
