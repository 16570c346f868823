"""The N > 1 path of bench.py on CPU: two gloo ranks, as torchrun would start
them (one process per rank, rendezvous on 127.0.0.1). The GEMM has no exchange
step, so the only cross-rank work is the barrier, the max over ranks of the
step time, and the whole-job throughput computed from it."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, _ = bench.dist_setup(world, backend="gloo")
    bench.barrier(w)
    local_ms = [2.0, 3.5][r]                       # rank 1 is the slow replica
    ms_max = bench.max_over_ranks(local_ms, w, device="cpu")
    q.put((r, w, ms_max, bench.job_tflops(10 ** 12, w, ms_max)))
    bench._finish(w)


def test_two_gloo_ranks_agree_on_the_slowest_step_and_the_job_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[0] for g in got] == [0, 1] and all(g[1] == 2 for g in got)
    assert all(g[2] == 3.5 for g in got)                       # max over ranks, on every rank
    assert all(g[3] == pytest.approx(2 * 1e12 / 3.5e-3 / 1e12) for g in got)


def test_single_process_is_world_one():
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        os.environ.pop(k, None)
    r, w, _ = bench.dist_setup(1, backend="gloo")
    assert (r, w) == (0, 1)
    assert bench.max_over_ranks(4.0, 1) == 4.0
    assert bench.job_tflops(2 * 10 ** 12, 1, 1.0) == pytest.approx(2000.0)
