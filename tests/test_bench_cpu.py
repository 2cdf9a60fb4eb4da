"""Host-side pieces of bench.py that need no GPU: the bounded fp64-oracle baselines
(their extrapolation and the varlen tail-window compaction)."""
import types

import numpy as np
import pytest
import torch

import bench
import oracle
from gated_deltanet_state_tail_b200 import inputs


def _bits(x):
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def test_oracle_throughput_both_kinds():
    for kind in ("replay", "prefill"):
        tps, dt = bench.oracle_throughput(kind, "bf16", 2, 64, 64, 64, 0.9, 0.999, min_seconds=0.0)
        assert tps > 0 and dt > 0


def test_cpu_full_prefill_sample_is_labelled_extrapolated():
    wl = types.SimpleNamespace(dtype="bf16", dk=64, dv=64, alpha_lo=0.9, alpha_hi=0.999,
                               match_len=[256], suffix_len=[32], H=4, layers=3)
    secs, text = bench.cpu_full_prefill_sample(wl, sample_tokens=64)
    assert secs > 0
    assert "extrapolated" in text and "3 layers x 4 heads x 288 tokens" in text


def _small_varlen():
    H, d = 2, 64
    cached = [300, 90, 200]          # cached rows per request
    match = [280, 90, 150]           # matched prefix (<= cached)
    R = [64, 200, 0]                 # replay budgets: one clamped to the prefix, one empty
    suffix = [40, 70, 5]
    off = np.concatenate([[0], np.cumsum(cached)]).astype(np.int32)
    cu = np.concatenate([[0], np.cumsum(suffix)]).astype(np.int32)
    wl = types.SimpleNamespace(match_len=match, R=R, suffix_len=suffix, batch=3, H=H)
    cache = inputs.draw_tensors(int(off[-1]), H, d, d, "bf16", 0.9, 0.999, 5, device="cpu", with_q=False)
    suf = inputs.draw_tensors(int(cu[-1]), H, d, d, "bf16", 0.9, 0.999, 6, device="cpu")
    return wl, off, cu, cache, suf


def test_varlen_tail_windows_replay_equals_packed_replay():
    """Replaying the compacted windows gives the oracle's replay of the packed batch."""
    wl, off, cu, cache, suf = _small_varlen()
    k, v, a, b, woff, rr = bench.varlen_tail_windows(wl, off, cache, 3)
    assert rr == [64, 90, 0]
    got = oracle.replay_state(_bits(k), _bits(v), a, b, woff, rr, rr)
    ref = oracle.replay_state(_bits(cache["k"]), _bits(cache["v"]), cache["alpha"].numpy(),
                              cache["beta"].numpy(), off, np.array(wl.match_len, np.int32),
                              np.array(wl.R, np.int32))
    np.testing.assert_array_equal(got, ref)


def test_cpu_varlen_sample_reports_rates():
    wl, off, cu, cache, suf = _small_varlen()
    r = bench.cpu_varlen_sample(wl, off, cu, cache, suf, nreq=2)
    assert r["kind"] == "oracle" and r["cores"] >= 1
    assert r["replayed_tokens_per_s"] > 0 and r["suffix_tokens_per_s"] > 0
    assert "requests 0-1 of 3" in r["sample"]


def test_reference_arm_line():
    """Rank 0 of `bench.py --impl reference` times the oracle on the host cores and
    prints the same metric and config as our arm, with the fields the driver reads."""
    class A:
        warmup, steps = 3, 1
    r = bench.bench_reference(A, 0, 1)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in r, key
    assert r["impl"] == "reference" and r["metric"] == bench.BENCH_METRIC
    assert r["value"] > 0 and r["unit"] == "replayed tokens/s" and r["higher_is_better"] is True
    assert r["config"]["workload"] == inputs.stack_workload(24).name
    assert r["cpu_baseline"]["kind"] == "oracle" and r["cpu_baseline"]["value"] == r["value"]
    assert r["cpu_baseline"]["cores"] >= 1
    assert r["e2e"]["h2d_bytes_per_step"] == 0 and r["e2e"]["d2h_bytes_per_step"] == 0
    assert bench.bench_reference(A, 1, 2) is None      # other ranks do no work


def test_profiled_traffic_matches_the_committed_record(monkeypatch):
    """roofline.traffic: the committed ncu record applies to the current replay sources,
    scales by work units, and is dropped for another kernel or changed sources."""
    rec = {}
    with open(bench.os.path.join(bench.ROOT, "profiles", "traffic.txt")) as f:
        for line in f:
            if ":" in line and not line.lstrip().startswith("#"):
                k, v = line.split(":", 1)
                rec[k.strip()] = v.strip()
    units = int(rec["units"])
    if rec["source_sha"] != bench.kernel_source_sha():     # the kernel changed since the capture
        assert bench.profiled_traffic(rec["kernel"], units) is None
        return
    full = bench.profiled_traffic(rec["kernel"], units)
    assert full == float(rec["dram_bytes"])
    assert bench.profiled_traffic(rec["kernel"], units // 2) == pytest.approx(full / 2)
    # the bench launch's algorithmic bytes: the measured traffic is within a few percent
    R, d, H, layers = 3277, 128, 32, 8
    alg = layers * H * (R * (2 * d * 2 + 8) + d * d * 4)
    assert units == layers * H and 0.95 <= full / alg <= 1.05
    assert bench.profiled_traffic("recurrent", units) is None
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: "0" * 16)
    assert bench.profiled_traffic(rec["kernel"], units) is None
