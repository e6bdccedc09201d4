"""The replica harness on CPU with two gloo ranks: barriers, max-over-ranks
timing and whole-job throughput, the way bench.py uses them for N > 1."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    from cross_loop_sparsity_b200 import replicas
    w, r, _ = replicas.init(backend="gloo", timeout_s=60)
    replicas.barrier(w)
    ms = 10.0 + 5.0 * r                      # rank 1 is the slow one
    m = replicas.max_over_ranks(w, ms)
    out.put((r, m, replicas.job_throughput(w, 8, m)))
    replicas.barrier(w)
    replicas.finish(w)


def test_two_gloo_replicas_take_the_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for r, m, tps in res:
        assert m == 15.0
        assert tps == pytest.approx(2 * 8 / 0.015)


def test_single_process_needs_no_group():
    from cross_loop_sparsity_b200 import replicas
    assert replicas.max_over_ranks(1, 3.5) == 3.5
    assert replicas.job_throughput(1, 8, 2.0) == pytest.approx(4000.0)
