"""Row-strided inputs and output guard regions, on the GPU.

A serving stack holds q, k and v as slices of one fused projection buffer
[rows, 3, H, d], so their rows are 3*H*d elements apart.  The descriptor's
row_stride_elems lets every entry point read such views in place.  The
results must equal the packed-input results bit for bit (the arithmetic does
not depend on where the rows sit) and match the fp64 oracle.

Every output buffer here is a view into a larger allocation whose guard
regions (before and after) hold a sentinel; a write outside the output's
extent would change them.
"""
import numpy as np
import pytest
import torch

import gated_deltanet_state_tail_b200 as gdn
from gated_deltanet_state_tail_b200 import inputs
import oracle
from helpers import TOL, oracle_view, per_request_rows_err, per_request_state_err

pytestmark = pytest.mark.gpu

KERNELS = {"recurrent": gdn.GDN_KERNEL_RECURRENT, "chunked": gdn.GDN_KERNEL_CHUNKED_TC}
GUARD = 4096          # guard elements on each side (16 KB of fp32)


class Guarded:
    """An output tensor of `shape` inside a buffer with sentinel-filled guards."""

    def __init__(self, shape, dtype, fill=float("nan"), sentinel=-7.25):
        n = int(np.prod(shape))
        self.buf = torch.empty(n + 2 * GUARD, dtype=dtype, device="cuda")
        self.sentinel = sentinel
        self.buf[:GUARD] = sentinel
        self.buf[GUARD + n:] = sentinel
        self.t = self.buf[GUARD:GUARD + n].view(shape)
        self.t.fill_(fill)
        self.n = n

    def guards_intact(self):
        s = self.sentinel
        return bool((self.buf[:GUARD] == s).all()) and bool((self.buf[GUARD + self.n:] == s).all())


def fused_qkv(rows, H, d, dtype, seed):
    """q, k, v as slices of one [rows, 3, H, d] buffer, plus packed copies and gates."""
    t = inputs.draw_tensors(rows, H, d, d, dtype, 0.9, 0.999, seed, device="cpu")
    x = torch.stack([t["q"], t["k"], t["v"]], dim=1).cuda()
    views = {"q": x[:, 0], "k": x[:, 1], "v": x[:, 2]}
    packed = {n: views[n].contiguous() for n in ("q", "k", "v")}
    gates = {"alpha": t["alpha"].cuda(), "beta": t["beta"].cuda()}
    return x, views, packed, gates


@pytest.mark.parametrize("kname,dtype,d", [("chunked", "bf16", 128), ("recurrent", "bf16", 128),
                                           ("recurrent", "f32", 64)])
def test_row_strided_replay_and_prefill(kname, dtype, d):
    kernel = KERNELS[kname]
    H = 3
    cached = [300, 64, 129, 0, 77, 1000]
    ml = [300, 64, 100, 0, 50, 997]
    R = [190, 64, 0, 10, 80, 333]
    off = np.concatenate([[0], np.cumsum(cached)]).astype(np.int32)
    rows = int(off[-1])
    x, views, packed, g = fused_qkv(rows, H, d, dtype, seed=61)
    stride = 3 * H * d
    assert gdn.row_stride_of(views["q"], views["k"], views["v"]) == stride

    # replay: strided views and packed copies give identical states
    st_s = Guarded((len(ml), H, d, d), torch.float32)
    plan = gdn.ReplayPlan(H, d, d, dtype, off, ml, R, kernel, row_stride=stride)
    plan.run(views["k"], views["v"], g["alpha"], g["beta"], st_s.t)
    assert plan.status() == gdn.GDN_OK
    plan.close()
    st_p = torch.full((len(ml), H, d, d), float("nan"), device="cuda")
    plan = gdn.ReplayPlan(H, d, d, dtype, off, ml, R, kernel)
    plan.run(packed["k"], packed["v"], g["alpha"], g["beta"], st_p)
    assert plan.status() == gdn.GDN_OK
    plan.close()
    assert torch.equal(st_s.t, st_p)
    assert st_s.guards_intact()
    ref = oracle.replay_state(oracle_view(packed["k"]), oracle_view(packed["v"]), oracle_view(g["alpha"]),
                              oracle_view(g["beta"]), off, ml, R)
    assert per_request_state_err(st_s.t.cpu().numpy(), ref) <= TOL[dtype]

    # the allocation-free entry point takes the same stride
    st_n = Guarded((len(ml), H, d, d), torch.float32)
    status = gdn.gdn_tail_replay_state_noalloc(H, d, d, dtype, off, ml, R, views["k"], views["v"], g["alpha"],
                                               g["beta"], st_n.t, kernel=kernel, row_stride=stride)
    assert status == 0
    assert torch.equal(st_n.t, st_p) and st_n.guards_intact()

    # prefill over whole sequences from the replayed states, strided q/k/v, packed o
    o_s = Guarded((rows, H, d), x.dtype, fill=0.0, sentinel=-3.0)
    fin_s = Guarded((len(ml), H, d, d), torch.float32)
    pplan = gdn.PrefillPlan(H, d, d, dtype, off, kernel, row_stride=stride)
    pplan.run(views["q"], views["k"], views["v"], g["alpha"], g["beta"], o_s.t, state_in=st_p,
              state_out=fin_s.t)
    assert pplan.status() == gdn.GDN_OK
    pplan.close()
    o_p = torch.zeros((rows, H, d), dtype=x.dtype, device="cuda")
    fin_p = torch.full_like(st_p, float("nan"))
    pplan = gdn.PrefillPlan(H, d, d, dtype, off, kernel)
    pplan.run(packed["q"], packed["k"], packed["v"], g["alpha"], g["beta"], o_p, state_in=st_p, state_out=fin_p)
    assert pplan.status() == gdn.GDN_OK
    pplan.close()
    assert torch.equal(o_s.t, o_p) and torch.equal(fin_s.t, fin_p)
    assert o_s.guards_intact() and fin_s.guards_intact()
    ref_o, ref_fin = oracle.prefill(oracle_view(packed["q"]), oracle_view(packed["k"]), oracle_view(packed["v"]),
                                    oracle_view(g["alpha"]), oracle_view(g["beta"]), off,
                                    state_in=st_p.double().cpu().numpy())
    assert per_request_rows_err(o_s.t.float().cpu().numpy(), ref_o, off) <= TOL[dtype]
    assert per_request_state_err(fin_s.t.cpu().numpy(), ref_fin) <= TOL[dtype]


@pytest.mark.parametrize("kname,dtype,d", [("chunked", "bf16", 128), ("recurrent", "f32", 64)])
def test_row_strided_fused_replay_prefill(kname, dtype, d):
    """The fused rebuild + suffix reads strided cache rows and strided suffix rows."""
    kernel = KERNELS[kname]
    H = 2
    cached = [300, 129, 0, 1000]
    ml = [300, 100, 0, 997]
    R = [190, 0, 10, 333]
    slen = [65, 130, 7, 0]
    off = np.concatenate([[0], np.cumsum(cached)]).astype(np.int32)
    so = np.concatenate([[0], np.cumsum(slen)]).astype(np.int32)
    xc, cv, cp, cg = fused_qkv(int(off[-1]), H, d, dtype, seed=71)
    xs, sv, sp, sg = fused_qkv(int(so[-1]), H, d, dtype, seed=72)
    stride = 3 * H * d

    def run(c, s, rs):
        plan = gdn.FusedPlan(H, d, d, dtype, off, ml, R, so, kernel, row_stride=rs)
        o = Guarded((int(so[-1]), H, d), xs.dtype, fill=0.0, sentinel=-3.0)
        st = Guarded((len(ml), H, d, d), torch.float32)
        mid = Guarded((len(ml), H, d, d), torch.float32)
        plan.run(c["k"], c["v"], cg["alpha"], cg["beta"], s["q"], s["k"], s["v"], sg["alpha"], sg["beta"],
                 o.t, st.t, state_mid=mid.t)
        assert plan.status() == gdn.GDN_OK
        plan.close()
        assert o.guards_intact() and st.guards_intact() and mid.guards_intact()
        return o.t, st.t, mid.t

    o_s, st_s, mid_s = run(cv, sv, stride)
    o_p, st_p, mid_p = run(cp, sp, 0)
    assert torch.equal(o_s, o_p) and torch.equal(st_s, st_p) and torch.equal(mid_s, mid_p)
    ref_mid = oracle.replay_state(oracle_view(cp["k"]), oracle_view(cp["v"]), oracle_view(cg["alpha"]),
                                  oracle_view(cg["beta"]), off, ml, R)
    ref_o, ref_st = oracle.prefill(oracle_view(sp["q"]), oracle_view(sp["k"]), oracle_view(sp["v"]),
                                   oracle_view(sg["alpha"]), oracle_view(sg["beta"]), so, state_in=ref_mid)
    assert per_request_state_err(mid_s.cpu().numpy(), ref_mid) <= TOL[dtype]
    assert per_request_rows_err(o_s.float().cpu().numpy(), ref_o, so) <= TOL[dtype]
    assert per_request_state_err(st_s.cpu().numpy(), ref_st) <= TOL[dtype]


def test_one_shot_helpers_take_strided_views():
    """tail_replay_state / chunk_prefill read the stride from the views themselves."""
    H, d = 4, 128
    L, N = 700, 130
    x, views, packed, g = fused_qkv(L + N, H, d, "bf16", seed=81)
    st = gdn.tail_replay_state(views["k"][:L], views["v"][:L], g["alpha"][:L], g["beta"][:L], [0, L], [L], [200])
    st_p = gdn.tail_replay_state(packed["k"][:L], packed["v"][:L], g["alpha"][:L], g["beta"][:L], [0, L], [L],
                                 [200])
    assert torch.equal(st, st_p)
    o, st2 = gdn.chunk_prefill(views["q"][L:], views["k"][L:], views["v"][L:], g["alpha"][L:], g["beta"][L:],
                               [0, N], state_in=st)
    o_p, st2_p = gdn.chunk_prefill(packed["q"][L:], packed["k"][L:], packed["v"][L:], g["alpha"][L:],
                                   g["beta"][L:], [0, N], state_in=st)
    assert torch.equal(o, o_p) and torch.equal(st2, st2_p)
