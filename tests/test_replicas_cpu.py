"""The multi-GPU path is replicas only (every (layer, request, head) unit is
independent; there is no exchange step).  Its host logic -- rendezvous, the
barrier, the max/sum over ranks of the device times, the whole-job
aggregate, and the reference arm that only rank 0 runs -- is exercised here
with two gloo ranks on CPU."""
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import bench
    r, w, local = bench.dist_init(world, backend="gloo")
    t_local = [0.50, 0.80][r]                      # this rank's rebuild time (s)
    t_max = bench.max_over_ranks(t_local, w)
    t_sum = bench.sum_over_ranks(t_local, w)
    bench.barrier(w)
    value = bench.replica_throughput(3277 * 10, w, t_max)

    class A:
        warmup, steps = 3, 1
    ref = bench.bench_reference(A, r, w) if r != 0 else "skipped"   # rank 0 would time the oracle
    out.put((r, w, t_max, t_sum, value, ref))
    torch.distributed.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, w, t_max, t_sum, value, ref in res:
        assert w == 2
        assert t_max == pytest.approx(0.80)            # the job lasts as long as its slowest rank
        assert t_sum == pytest.approx(1.30)
        assert value == pytest.approx(3277 * 10 * 2 / 0.80)   # whole-job tokens/s over both replicas
    assert res[1][5] is None                           # non-zero ranks of the reference arm do no work


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1.5, 1) == 1.5
    assert bench.sum_over_ranks(1.5, 1) == 1.5
    assert bench.replica_throughput(100, 1, 0.5) == 200
