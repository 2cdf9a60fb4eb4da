"""The 24-layer stack's own replay launch, and the replay under a concurrent
host-to-device copy, on the GPU.

* One replay launch of the cache-hit step: 8 GDN layers x 32 heads, each layer
  a 32768-row resident prefix whose last R = 3277 rows (10%) are replayed,
  then the 1024-row suffix prefilled from the rebuilt states.  Sampled
  (layer, head) units are checked element by element against the fp64 oracle.
* Transfer/replay overlap (the gist.science summary, "Mecanismos Principais":
  the full-attention layers' KV cache crosses to the GPU while the GDN state is
  replayed): a pinned host-to-device copy runs on a second stream while the
  same replay launch runs on the first.  The replay must finish inside the
  copy's span, its states must equal those of a replay run alone bit for bit,
  and the copied bytes must arrive intact.
"""
import numpy as np
import pytest
import torch

import gated_deltanet_state_tail_b200 as gdn
from gated_deltanet_state_tail_b200 import inputs
import oracle
from helpers import TOL, oracle_view, rel_err

pytestmark = pytest.mark.gpu

LAYERS, H, D = 8, 32, 128
L, N = 32768, 1024
R = inputs.ceil_budget(L, 10, 100)          # 3277
SAMPLES = [(0, 0), (7, 31), (3, 17), (5, 5), (1, 30), (6, 12), (2, 8), (4, 23)]
GUARD = 4096


@pytest.fixture(scope="module")
def stack():
    """Per-layer caches (seed = layer) of L rows and suffixes of N rows, packed by layer."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cache = {n: [] for n in ("k", "v", "alpha", "beta")}
    suf = {n: [] for n in ("q", "k", "v", "alpha", "beta")}
    for layer in range(LAYERS):
        c = inputs.draw_tensors(L, H, D, D, "bf16", 0.90, 0.999, seed=layer, device="cuda", with_q=False)
        s = inputs.draw_tensors(N, H, D, D, "bf16", 0.90, 0.999, seed=100 + layer, device="cuda")
        for n in cache:
            cache[n].append(c[n])
        for n in suf:
            suf[n].append(s[n])
    cache = {n: torch.cat(x) for n, x in cache.items()}
    suf = {n: torch.cat(x) for n, x in suf.items()}
    off = np.arange(LAYERS + 1, dtype=np.int32) * L
    cu = np.arange(LAYERS + 1, dtype=np.int32) * N
    yield cache, suf, off, cu
    del cache, suf
    torch.cuda.empty_cache()


def guarded(shape, dtype, sentinel):
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * GUARD,), sentinel, dtype=dtype, device="cuda")
    return buf, buf[GUARD:GUARD + n].view(shape)


def guards_intact(buf, n, sentinel):
    return bool((buf[:GUARD] == sentinel).all()) and bool((buf[GUARD + n:] == sentinel).all())


def replay(cache, off, state, stream=None):
    plan = gdn.ReplayPlan(H, D, D, "bf16", off, [L] * LAYERS, [R] * LAYERS)
    assert plan.info["kernel"] == gdn.GDN_KERNEL_CHUNKED_TC and plan.info["units"] == LAYERS * H
    plan.run(cache["k"], cache["v"], cache["alpha"], cache["beta"], state, stream=stream)
    return plan


def test_stack_launch_sampled_units_match_oracle(stack):
    cache, suf, off, cu = stack
    sbuf, state = guarded((LAYERS, H, D, D), torch.float32, -9.5)
    plan = replay(cache, off, state)
    assert plan.status() == gdn.GDN_OK
    for b in range(LAYERS):
        assert plan.window(b) == (int(off[b]) + L - R, R)
    plan.close()
    obuf, o = guarded((LAYERS * N, H, D), torch.bfloat16, -3.0)
    fbuf, fin = guarded((LAYERS, H, D, D), torch.float32, -9.5)
    pplan = gdn.PrefillPlan(H, D, D, "bf16", cu)
    pplan.run(suf["q"], suf["k"], suf["v"], suf["alpha"], suf["beta"], o, state_in=state, state_out=fin)
    assert pplan.status() == gdn.GDN_OK
    pplan.close()
    torch.cuda.synchronize()
    assert guards_intact(sbuf, state.numel(), -9.5)
    assert guards_intact(obuf, o.numel(), -3.0)
    assert guards_intact(fbuf, fin.numel(), -9.5)

    for layer, hh in SAMPLES:
        rows = slice(int(off[layer]) + L - R, int(off[layer]) + L)
        sub = {n: oracle_view(cache[n][rows, hh:hh + 1]) for n in cache}
        ref = oracle.replay_state(sub["k"], sub["v"], sub["alpha"], sub["beta"], [0, R], [R], [R])[0, 0]
        assert rel_err(state[layer, hh].cpu().numpy(), ref) <= TOL["bf16"], f"replay layer {layer} head {hh}"
        srows = slice(int(cu[layer]), int(cu[layer + 1]))
        ss = {n: oracle_view(suf[n][srows, hh:hh + 1]) for n in suf}
        ref_o, ref_s = oracle.prefill(ss["q"], ss["k"], ss["v"], ss["alpha"], ss["beta"], [0, N],
                                      state_in=state[layer:layer + 1, hh:hh + 1].double().cpu().numpy())
        assert rel_err(o[srows, hh].float().cpu().numpy(), ref_o[:, 0]) <= TOL["bf16"], f"suffix o {layer} {hh}"
        assert rel_err(fin[layer, hh].cpu().numpy(), ref_s[0, 0]) <= TOL["bf16"], f"suffix state {layer} {hh}"


def test_replay_runs_inside_a_concurrent_h2d_copy(stack):
    cache, suf, off, cu = stack
    n64 = (512 << 20) // 8                      # a 512 MiB pinned copy (about 10 ms over PCIe)
    host = torch.empty(n64, dtype=torch.int64, pin_memory=True)
    host.copy_(torch.arange(n64, dtype=torch.int64) * 2654435761)
    dev = torch.zeros(n64, dtype=torch.int64, device="cuda")

    alone = torch.empty((LAYERS, H, D, D), device="cuda")
    replay(cache, off, alone).close()
    torch.cuda.synchronize()

    s_main = torch.cuda.current_stream()
    s_copy = torch.cuda.Stream()
    ev = {k: torch.cuda.Event(enable_timing=True) for k in ("c0", "c1", "r0", "r1")}
    under = torch.full((LAYERS, H, D, D), float("nan"), device="cuda")
    torch.cuda.synchronize()
    ev["c0"].record(s_copy)
    with torch.cuda.stream(s_copy):
        dev.copy_(host, non_blocking=True)
    ev["c1"].record(s_copy)
    s_main.wait_event(ev["c0"])                  # the replay starts once the copy has been issued
    ev["r0"].record(s_main)
    plan = replay(cache, off, under, stream=s_main)
    ev["r1"].record(s_main)
    torch.cuda.synchronize()
    assert plan.status() == gdn.GDN_OK
    plan.close()

    copy_ms = ev["c0"].elapsed_time(ev["c1"])
    replay_ms = ev["r0"].elapsed_time(ev["r1"])
    # the replay started after the copy and finished before it: the two ran at once
    assert ev["c0"].elapsed_time(ev["r0"]) >= 0.0
    assert ev["r1"].elapsed_time(ev["c1"]) > 0.0, f"replay {replay_ms:.3f} ms, copy {copy_ms:.3f} ms"
    assert torch.equal(under, alone)
    want = torch.arange(n64, dtype=torch.int64, device="cuda") * 2654435761
    assert torch.equal(dev, want)
    for layer, hh in SAMPLES[:2]:
        rows = slice(int(off[layer]) + L - R, int(off[layer]) + L)
        sub = {n: oracle_view(cache[n][rows, hh:hh + 1]) for n in cache}
        ref = oracle.replay_state(sub["k"], sub["v"], sub["alpha"], sub["beta"], [0, R], [R], [R])[0, 0]
        assert rel_err(under[layer, hh].cpu().numpy(), ref) <= TOL["bf16"]
