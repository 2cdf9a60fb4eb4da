"""GPU parity: the CUDA kernels, called through the C ABI, against the fp64
oracle on the same seeded inputs.  Tolerance: max|err|/max|ref| per request
and tensor, 1e-4 for fp32 inputs and 2e-2 for bf16 inputs."""
import numpy as np
import pytest
import torch

import gated_deltanet_state_tail_b200 as gdn
from gated_deltanet_state_tail_b200 import inputs
import oracle
from helpers import TOL, oracle_view, per_request_rows_err, per_request_state_err, rel_err

pytestmark = pytest.mark.gpu

# "two_cta", "warp_spec" and "pair" run the chunked path with the state-only replay
# pinned to one of its three kernels (the default, "chunked", is the two-CTA kernel);
# every other entry point runs the chunked prefill kernel under all four
KERNELS = {"recurrent": gdn.GDN_KERNEL_RECURRENT, "chunked": gdn.GDN_KERNEL_CHUNKED_TC,
           "two_cta": gdn.GDN_KERNEL_CHUNKED_TC_TWO_CTA, "warp_spec": gdn.GDN_KERNEL_CHUNKED_TC_WARP_SPEC,
           "pair": gdn.GDN_KERNEL_CHUNKED_TC_PAIR}
CHUNKED = ("chunked", "two_cta", "warp_spec", "pair")
REPLAY_KERNELS = ["recurrent", "two_cta", "warp_spec", "pair"]


def kernel_or_skip(name, dtype, dk, dv):
    if name in CHUNKED and not (dtype == "bf16" and dk == 128 and dv == 128):
        pytest.skip("chunked kernel serves bf16 with d = 128")
    if name in CHUNKED:
        try:
            gdn.ReplayPlan(1, 128, 128, "bf16", [0, 64], [64], [64], KERNELS[name]).close()
        except gdn.GdnError as e:
            if e.status == gdn.GDN_ERR_UNSUPPORTED:
                pytest.skip("chunked tensor-core kernel not in this build")
            raise
    return KERNELS[name]


def make_cache(cached, H, dk, dv, dtype, seed, a_lo=0.9, a_hi=0.999):
    rows = int(sum(cached))
    t = inputs.draw_tensors(rows, H, dk, dv, dtype, a_lo, a_hi, seed, device="cpu")
    return {k: (None if x is None else x.cuda()) for k, x in t.items()}


def run_replay(t, off, ml, R, kernel, dtype, check_arrays=True):
    H, dk = t["k"].shape[1], t["k"].shape[2]
    dv = t["v"].shape[2]
    plan = gdn.ReplayPlan(H, dk, dv, dtype, off, ml, R, kernel)
    out = torch.full((len(ml), H, dk, dv), float("nan"), device="cuda")
    dev = (lambda a: torch.tensor(np.asarray(a, np.int32), device="cuda")) if check_arrays else (lambda a: None)
    plan.run(t["k"], t["v"], t["alpha"], t["beta"], out, seq_offsets=dev(off), match_len=dev(ml), R=dev(R))
    assert plan.status() == gdn.GDN_OK
    plan.close()
    return out


def run_prefill(t, cu, state_in, kernel, dtype):
    H, dk = t["k"].shape[1], t["k"].shape[2]
    dv = t["v"].shape[2]
    plan = gdn.PrefillPlan(H, dk, dv, dtype, cu, kernel)
    o = torch.zeros((t["k"].shape[0], H, dv), dtype=t["k"].dtype, device="cuda")
    st = torch.full((len(cu) - 1, H, dk, dv), float("nan"), device="cuda")
    plan.run(t["q"], t["k"], t["v"], t["alpha"], t["beta"], o, state_in=state_in, state_out=st,
             cu_seqlens=torch.tensor(np.asarray(cu, np.int32), device="cuda"))
    assert plan.status() == gdn.GDN_OK
    plan.close()
    return o, st


def oracle_replay(t, off, ml, R):
    return oracle.replay_state(oracle_view(t["k"]), oracle_view(t["v"]), oracle_view(t["alpha"]),
                               oracle_view(t["beta"]), off, ml, R)


def oracle_prefill(t, cu, state_in):
    si = None if state_in is None else state_in.detach().cpu().double().numpy()
    return oracle.prefill(oracle_view(t["q"]), oracle_view(t["k"]), oracle_view(t["v"]),
                          oracle_view(t["alpha"]), oracle_view(t["beta"]), cu, state_in=si)


@pytest.mark.parametrize("kname", ["recurrent"])
def test_tiny_f32_replay_then_suffix(kname):
    """1 head, d = 64, fp32: L = 256, R = 32, then a 32-token suffix from the rebuilt state."""
    wl = inputs.tiny_workload()
    kernel = kernel_or_skip(kname, wl.dtype, wl.dk, wl.dv)
    L, R, N = wl.match_len[0], wl.R[0], wl.suffix_len[0]
    t = make_cache([L + N], wl.H, wl.dk, wl.dv, wl.dtype, seed=0)
    off = [0, L + N]
    st = run_replay(t, off, [L], [R], kernel, wl.dtype)
    ref_st = oracle_replay(t, off, [L], [R])
    assert per_request_state_err(st.cpu().numpy(), ref_st) <= TOL["f32"]
    suf = {k: x[L:] for k, x in t.items()}
    o, st2 = run_prefill(suf, [0, N], st, kernel, wl.dtype)
    ref_o, ref_st2 = oracle_prefill(suf, [0, N], st)
    assert rel_err(o.cpu().numpy(), ref_o) <= TOL["f32"]
    assert per_request_state_err(st2.cpu().numpy(), ref_st2) <= TOL["f32"]


@pytest.mark.parametrize("kname", REPLAY_KERNELS)
@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 128, 128), ("bf16", 64, 128),
                                         ("f32", 128, 64)])
def test_varlen_replay_edges(kname, dtype, dk, dv):
    """Ragged windows spanning several 64-token chunks plus a ragged tail, R = 0,
    R > L (clamped), L = 0, and cache entries longer than the match."""
    kernel = kernel_or_skip(kname, dtype, dk, dv)
    cached = [300, 64, 129, 0, 77, 1000]
    ml = [300, 64, 100, 0, 50, 997]
    R = [190, 64, 0, 10, 80, 333]
    off = np.concatenate([[0], np.cumsum(cached)]).astype(np.int32)
    t = make_cache(cached, 3, dk, dv, dtype, seed=11)
    st = run_replay(t, off, ml, R, kernel, dtype)
    ref = oracle_replay(t, off, ml, R)
    assert per_request_state_err(st.cpu().numpy(), ref) <= TOL[dtype]
    # Zero-Only rows are exactly zero
    assert torch.count_nonzero(st[2]) == 0 and torch.count_nonzero(st[3]) == 0


@pytest.mark.parametrize("kname", ["recurrent", "chunked"])
@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 64, 64)])
@pytest.mark.parametrize("with_state", [False, True])
def test_varlen_prefill(kname, dtype, dk, dv, with_state):
    kernel = kernel_or_skip(kname, dtype, dk, dv)
    lens = [1, 63, 64, 65, 200, 0, 130]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    t = make_cache(lens, 2, dk, dv, dtype, seed=12)
    si = None
    if with_state:
        g = torch.Generator(device="cpu").manual_seed(5)
        si = (torch.randn((len(lens), 2, dk, dv), generator=g) * 0.5).cuda()
    o, st = run_prefill(t, cu, si, kernel, dtype)
    ref_o, ref_st = oracle_prefill(t, cu, si)
    assert per_request_rows_err(o.float().cpu().numpy(), ref_o, cu) <= TOL[dtype]
    assert per_request_state_err(st.cpu().numpy(), ref_st) <= TOL[dtype]


@pytest.mark.parametrize("kname", REPLAY_KERNELS)
def test_window_indexing_bit_exact(kname):
    """Orthonormal cycling keys, alpha = beta = 1, v_t carrying its row index:
    the state records exactly which rows were replayed (bf16 digits are exact)."""
    kernel = kernel_or_skip(kname, "bf16", 128, 128)
    H, dk, dv = 2, 128, 128
    cached = [500, 130, 2000, 7]
    rows = sum(cached)
    k = torch.zeros((rows, H, dk))
    idx = torch.arange(rows)
    k[idx, :, idx % dk] = 1.0
    v = torch.zeros((rows, H, dv))
    v[:, :, 0] = (idx % 256).float()[:, None]
    v[:, :, 1] = (idx // 256).float()[:, None]
    v[:, :, 2] = 1.0
    t = {"k": k.to(torch.bfloat16).cuda(), "v": v.to(torch.bfloat16).cuda(),
         "alpha": torch.ones((rows, H)).cuda(), "beta": torch.ones((rows, H)).cuda()}
    off = np.concatenate([[0], np.cumsum(cached)]).astype(np.int32)
    ml = [480, 130, 1999, 7]
    R = [100, 128, 77, 20]
    st = run_replay(t, off, ml, R, kernel, "bf16").cpu()
    for b in range(4):
        reff = min(R[b], ml[b])
        want = torch.zeros((dk, dv))
        for r in range(off[b] + ml[b] - reff, off[b] + ml[b]):
            want[r % dk, 0] = r % 256
            want[r % dk, 1] = r // 256
            want[r % dk, 2] = 1.0
        for h in range(H):
            assert torch.equal(st[b, h], want), f"request {b} head {h}"


def test_descriptor_mismatch_is_reported():
    t = make_cache([100, 100], 2, 64, 64, "f32", seed=13)
    off, ml, R = [0, 100, 200], [90, 100], [30, 40]
    plan = gdn.ReplayPlan(2, 64, 64, "f32", off, ml, R)
    out = torch.zeros((2, 2, 64, 64), device="cuda")
    bad = torch.tensor([90, 99], dtype=torch.int32, device="cuda")
    plan.run(t["k"], t["v"], t["alpha"], t["beta"], out, match_len=bad)
    assert plan.status() == gdn.GDN_ERR_MISMATCH
    good = torch.tensor(ml, dtype=torch.int32, device="cuda")
    plan.run(t["k"], t["v"], t["alpha"], t["beta"], out, match_len=good)
    assert plan.status() == gdn.GDN_OK
    plan.close()


def test_status_belongs_to_the_last_call_without_a_reset():
    """No call clears the workspace: each tags its reports with its own call number.  A
    workspace of arbitrary bytes reads GDN_OK after a good call, and neither a timeout nor
    a mismatch outlives the call that reported it."""
    t = make_cache([100, 100], 2, 128, 128, "bf16", seed=16)
    off, ml, R = [0, 100, 200], [90, 100], [30, 40]
    plan = gdn.ReplayPlan(2, 128, 128, "bf16", off, ml, R)
    out = torch.zeros((2, 2, 128, 128), device="cuda")
    ref = oracle_replay(t, np.array(off, np.int32), ml, R)
    ws = torch.full((256,), 0xFF, dtype=torch.uint8, device="cuda")
    ws[:8].fill_(0x07)                                       # every status bit set, under a stale tag
    plan.run(t["k"], t["v"], t["alpha"], t["beta"], out, workspace=ws)
    assert gdn.gdn_workspace_status(ws) == gdn.GDN_OK
    assert per_request_state_err(out.cpu().numpy(), ref) <= TOL["bf16"]
    gdn.gdn_selftest_bounded_wait(1_000_000, ws)
    assert gdn.gdn_workspace_status(ws) == gdn.GDN_ERR_TIMEOUT
    plan.run(t["k"], t["v"], t["alpha"], t["beta"], out, workspace=ws)
    assert gdn.gdn_workspace_status(ws) == gdn.GDN_OK
    bad = torch.tensor([90, 99], dtype=torch.int32, device="cuda")
    plan.run(t["k"], t["v"], t["alpha"], t["beta"], out, match_len=bad, workspace=ws)
    assert gdn.gdn_workspace_status(ws) == gdn.GDN_ERR_MISMATCH
    plan.run(t["k"], t["v"], t["alpha"], t["beta"], out, workspace=ws)
    assert gdn.gdn_workspace_status(ws) == gdn.GDN_OK
    assert per_request_state_err(out.cpu().numpy(), ref) <= TOL["bf16"]
    plan.close()


def test_call_validation_on_device():
    t = make_cache([64], 1, 64, 64, "f32", seed=14)
    plan = gdn.ReplayPlan(1, 64, 64, "f32", [0, 64], [64], [10])
    out = torch.zeros((1, 1, 64, 64), device="cuda")
    with pytest.raises(gdn.GdnError) as e:
        plan.run(t["k"], None, t["alpha"], t["beta"], out)
    assert e.value.status == gdn.GDN_ERR_INVALID_ARG
    buf = torch.zeros(64 * 64 + 1, device="cuda")
    with pytest.raises(gdn.GdnError):
        plan.run(t["k"], t["v"], t["alpha"], t["beta"], buf[1:])     # misaligned state_out
    with pytest.raises(gdn.GdnError):   # a replay plan cannot prefill
        gdn.gdn_chunk_prefill(plan.handle, t["q"], t["k"], t["v"], t["alpha"], t["beta"], None, None,
                              out, None, plan.workspace)
    plan.close()


@pytest.mark.parametrize("kname", REPLAY_KERNELS)
def test_rerun_bit_identical(kname):
    kernel = kernel_or_skip(kname, "bf16", 128, 128)
    t = make_cache([700], 4, 128, 128, "bf16", seed=15)
    a = run_replay(t, [0, 700], [650], [300], kernel, "bf16")
    b = run_replay(t, [0, 700], [650], [300], kernel, "bf16")
    assert torch.equal(a, b)


@pytest.mark.parametrize("kname", REPLAY_KERNELS)
def test_replay_then_suffix_equals_one_prefill(kname):
    """Replay(R) then prefill(suffix) matches one prefill from zero over tail ++ suffix."""
    kernel = kernel_or_skip(kname, "bf16", 128, 128)
    L, R, N = 900, 200, 150
    t = make_cache([L + N], 2, 128, 128, "bf16", seed=16)
    st = run_replay(t, [0, L + N], [L], [R], kernel, "bf16")
    suf = {k: x[L:] for k, x in t.items()}
    o1, s1 = run_prefill(suf, [0, N], st, kernel, "bf16")
    both = {k: x[L - R:] for k, x in t.items()}
    o2, s2 = run_prefill(both, [0, R + N], None, kernel, "bf16")
    assert rel_err(s1.cpu().numpy(), s2.cpu().numpy()) <= TOL["bf16"]
    assert rel_err(o1.float().cpu().numpy(), o2[R:].float().cpu().numpy()) <= TOL["bf16"]


@pytest.mark.parametrize("kname", REPLAY_KERNELS)
def test_full_window_replay_equals_prefill_state(kname):
    """R = L: the replay kernel reproduces the state of a prefill from zero over the same
    L tokens (the prefill kernel), and both match the oracle."""
    kernel = kernel_or_skip(kname, "bf16", 128, 128)
    L = 2000   # 31 full chunks and a ragged tail
    t = make_cache([L], 4, 128, 128, "bf16", seed=23)
    st = run_replay(t, [0, L], [L], [L], kernel, "bf16")
    _, sp = run_prefill(t, [0, L], None, kernel, "bf16")
    assert rel_err(st.cpu().numpy(), sp.cpu().numpy()) <= TOL["bf16"]
    ref = oracle_replay(t, [0, L], [L], [L])
    assert per_request_state_err(st.cpu().numpy(), ref) <= TOL["bf16"]
    assert per_request_state_err(sp.cpu().numpy(), ref) <= TOL["bf16"]


def _gates(case, rows, H, seed, last_window_row):
    """alpha, beta [rows, H] (fp32) for one gate regime."""
    g = np.random.default_rng(seed)
    a = g.uniform(0.9, 0.999, (rows, H))
    b = 1.0 / (1.0 + np.exp(-g.standard_normal((rows, H))))
    if case == "strong_decay":      # chunk decays far below 2^-100: the per-element exponent path
        a = g.uniform(0.0, 0.3, (rows, H))
    elif case == "zero_gates":      # alpha = 0 now and then, and on the window's last token
        a[::37] = 0.0
        a[last_window_row] = 0.0
    elif case == "no_write":        # beta = 0: nothing is written, the state only decays
        b[:] = 0.0
    elif case == "identity":        # alpha = 1, beta = 0: every token is an identity transition
        a[:] = 1.0
        b[:] = 0.0
    elif case == "mixed_heads":     # one launch, one head in each regime
        a[:, 0] = g.uniform(0.0, 0.3, rows)
    return torch.tensor(a, dtype=torch.float32), torch.tensor(b, dtype=torch.float32)


@pytest.mark.parametrize("kname", REPLAY_KERNELS)
@pytest.mark.parametrize("case", ["strong_decay", "zero_gates", "no_write", "identity", "mixed_heads"])
def test_gate_extremes(kname, case):
    """Degenerate and extreme gates: the replay of a 500-token window and the suffix prefill
    from a nonzero state, against the oracle.  Strong decay takes the kernels' per-element
    exponent path and folds the running scale into the state every chunk; alpha = 0 at the
    window's last token leaves beta k v^T; beta = 0 leaves a zero replay and a decayed
    state_in; alpha = 1, beta = 0 carries state_in through unchanged."""
    dtype, dk, dv = ("bf16", 128, 128) if kname in CHUNKED else ("f32", 64, 128)
    kernel = kernel_or_skip(kname, dtype, dk, dv)
    L, R, N, H = 700, 500, 300, 2   # window of 7 chunks and a ragged tail; suffix of 4 and a tail
    t = make_cache([L + N], H, dk, dv, dtype, seed=31)
    a, b = _gates(case, L + N, H, 41, L - 1)
    t["alpha"], t["beta"] = a.cuda(), b.cuda()
    st = run_replay(t, [0, L + N], [L], [R], kernel, dtype)
    ref = oracle_replay(t, [0, L + N], [L], [R])
    assert per_request_state_err(st.cpu().numpy(), ref) <= TOL[dtype], "replay"
    s = {k: x[L:] for k, x in t.items()}
    gen = torch.Generator(device="cuda").manual_seed(5)
    s0 = torch.randn((1, H, dk, dv), generator=gen, device="cuda") * 0.1
    o, st2 = run_prefill(s, [0, N], s0, kernel, dtype)
    ref_o, ref_st2 = oracle_prefill(s, [0, N], s0)
    assert rel_err(o.float().cpu().numpy(), ref_o) <= TOL[dtype], "suffix outputs"
    assert per_request_state_err(st2.cpu().numpy(), ref_st2) <= TOL[dtype], "suffix state"


@pytest.mark.parametrize("kname", ["recurrent", "chunked"])
def test_single_layer_full_size(kname):
    """One layer, 16 heads, d = 128, bf16: L = 8192, R = 410 (5%), N = 512, checked in full."""
    wl = inputs.single_layer_workload()
    kernel = kernel_or_skip(kname, wl.dtype, wl.dk, wl.dv)
    L, R, N = wl.match_len[0], wl.R[0], wl.suffix_len[0]
    t = inputs.draw_tensors(L + N, wl.H, wl.dk, wl.dv, wl.dtype, wl.alpha_lo, wl.alpha_hi, 0, device="cuda")
    st = run_replay(t, [0, L + N], [L], [R], kernel, wl.dtype)
    tail = {k: x[L - R:L] for k, x in t.items()}
    ref_st = oracle_replay(tail, [0, R], [R], [R])
    assert per_request_state_err(st.cpu().numpy(), ref_st) <= TOL["bf16"]
    suf = {k: x[L:] for k, x in t.items()}
    o, st2 = run_prefill(suf, [0, N], st, kernel, wl.dtype)
    ref_o, ref_st2 = oracle_prefill(suf, [0, N], st)
    assert rel_err(o.float().cpu().numpy(), ref_o) <= TOL["bf16"]
    assert per_request_state_err(st2.cpu().numpy(), ref_st2) <= TOL["bf16"]


def test_bounded_wait_timeout_is_reported_and_context_survives():
    """The failure path every kernel's waits use: a wait on an mbarrier that nothing
    arrives on runs out after 1 ms, the status word says GDN_ERR_TIMEOUT, and the
    next call on the same context works."""
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    gdn.gdn_selftest_bounded_wait(1_000_000, ws)
    assert gdn.gdn_workspace_status(ws) == gdn.GDN_ERR_TIMEOUT
    # header words: status (bits, call number), wait site (code, call number), recorded call number
    header = ws.view(torch.int32).cpu().numpy()
    assert header[2] == 99                                   # the wait site the self-test reports
    assert header[1] == header[3] == header[4] != 0          # both tagged with the recorded call
    # the context is still usable: a small replay runs and matches the oracle
    t = make_cache([200], 2, 128, 128, "bf16", seed=3)
    st = run_replay(t, np.array([0, 200], np.int32), [200], [150], gdn.GDN_KERNEL_AUTO, "bf16")
    ref = oracle_replay(t, np.array([0, 200], np.int32), [200], [150])
    assert per_request_state_err(st.cpu().numpy(), ref) <= TOL["bf16"]


@pytest.mark.parametrize("kname", REPLAY_KERNELS)
def test_random_varlen_batches(kname):
    """Seeded random batches: request count, heads, cached length, match, budget and suffix
    length drawn per batch (R = 0, R > L, L = 0 and partial chunks all occur); replay states,
    suffix outputs and final states against the oracle."""
    dtype, dk, dv = ("bf16", 128, 128) if kname in CHUNKED else ("f32", 64, 128)
    kernel = kernel_or_skip(kname, dtype, dk, dv)
    rng = np.random.default_rng(2024)
    for trial in range(12):
        B = int(rng.integers(1, 6))
        H = int(rng.integers(1, 4))
        cached = rng.integers(0, 400, B)
        ml = np.array([int(rng.integers(0, c + 1)) for c in cached])
        R = np.array([int(rng.integers(0, m + 80)) for m in ml])           # R > L happens
        slen = rng.integers(0, 200, B)
        off = np.concatenate([[0], np.cumsum(cached)]).astype(np.int32)
        cu = np.concatenate([[0], np.cumsum(slen)]).astype(np.int32)
        seed = 1000 + trial
        t = make_cache(list(cached) if off[-1] > 0 else [1], H, dk, dv, dtype, seed)
        st = run_replay(t, off, ml, R, kernel, dtype)
        ref = oracle_replay(t, off, ml, R)
        assert per_request_state_err(st.cpu().numpy(), ref) <= TOL[dtype], f"trial {trial} replay"
        if cu[-1] == 0:
            continue
        s = make_cache(list(slen), H, dk, dv, dtype, seed + 500)
        o, st2 = run_prefill(s, cu, st, kernel, dtype)
        ref_o, ref_st2 = oracle_prefill(s, cu, st)
        assert per_request_rows_err(o.float().cpu().numpy(), ref_o, cu) <= TOL[dtype], f"trial {trial} outputs"
        assert per_request_state_err(st2.cpu().numpy(), ref_st2) <= TOL[dtype], f"trial {trial} state"


def test_longest_windows_against_oracle():
    """The longest windows the workloads use, one head each: a full 32768-token replay (512
    chunks through the tensor-core replay) and a 33792-token prefill from zero (the
    full-prefill comparator's length), both against the fp64 oracle."""
    kernel_or_skip("chunked", "bf16", 128, 128)
    L = 32768
    t = make_cache([L], 1, 128, 128, "bf16", seed=77, a_lo=0.97, a_hi=0.9999)
    st = run_replay(t, np.array([0, L], np.int32), [L], [L], gdn.GDN_KERNEL_CHUNKED_TC, "bf16")
    ref = oracle_replay(t, np.array([0, L], np.int32), [L], [L])
    assert per_request_state_err(st.cpu().numpy(), ref) <= TOL["bf16"]
    N = 33792
    s = make_cache([N], 1, 128, 128, "bf16", seed=78, a_lo=0.97, a_hi=0.9999)
    o, st2 = run_prefill(s, np.array([0, N], np.int32), None, gdn.GDN_KERNEL_CHUNKED_TC, "bf16")
    ref_o, ref_st2 = oracle_prefill(s, np.array([0, N], np.int32), None)
    assert rel_err(o.float().cpu().numpy(), ref_o) <= TOL["bf16"]
    assert per_request_state_err(st2.cpu().numpy(), ref_st2) <= TOL["bf16"]


@pytest.mark.parametrize("kname", REPLAY_KERNELS)
def test_chunk_boundary_window_lengths(kname):
    """Windows of 1, 63, 64, 65, 127, 128, 129, 191, 192 and 193 rows in one launch: one to
    four chunks, with and without a partial last chunk (whose key and value rows past the
    window are zeroed in shared memory), so every iteration shape of the two-chunk
    schedule runs.  The cached entries are longer than their windows, so the rows past
    a window hold real data that must not leak in.  Replay, then a prefill of suffixes
    of the same lengths from the replayed states."""
    kernel = kernel_or_skip(kname, "bf16", 128, 128)
    lens = [1, 63, 64, 65, 127, 128, 129, 191, 192, 193]
    H = 2
    cached = [n + 37 for n in lens]
    ml = [n + 5 for n in lens]
    off = np.concatenate([[0], np.cumsum(cached)]).astype(np.int32)
    t = make_cache(cached, H, 128, 128, "bf16", seed=91)
    st = run_replay(t, off, ml, lens, kernel, "bf16")
    ref = oracle_replay(t, off, ml, lens)
    assert per_request_state_err(st.cpu().numpy(), ref) <= TOL["bf16"]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    s = make_cache(lens, H, 128, 128, "bf16", seed=92)
    o, st2 = run_prefill(s, cu, st, kernel, "bf16")
    ref_o, ref_st2 = oracle_prefill(s, cu, st)
    assert per_request_rows_err(o.float().cpu().numpy(), ref_o, cu) <= TOL["bf16"]
    assert per_request_state_err(st2.cpu().numpy(), ref_st2) <= TOL["bf16"]
