"""Host logic of the multi-rank bench path, on two gloo ranks (CPU only).

bench.py under torchrun gives every rank its own chunk of the same shape
(weak scaling, no data-path collective), times the steps on each rank and
reports the whole-job rate for the max step time over ranks; the reference
arm runs on rank 0 only.
"""
import argparse
import contextlib
import datetime
import io
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench

        w, r, lr = bench.dist_env()
        step_ms = 4.0 + rank  # rank 1 is the slow one
        worst = bench.max_over_ranks(step_ms, w)
        bench.barrier(w)
        rate = bench.whole_job_rate(w, 8192, worst)
        seed = bench.rank_seed(2, r)
        out = io.StringIO()
        if r != 0:  # the reference arm: ranks other than 0 leave without work
            args = argparse.Namespace(workload="tiny_256q", steps=1, warmup=1, cpu_rows=1)
            with contextlib.redirect_stdout(out):
                bench.run_reference(args)
        q.put((rank, w, r, lr, worst, rate, seed, out.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_bench_host_logic():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in procs:
            item = q.get(timeout=120)
            results[item[0]] = item
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert sorted(results) == [0, 1]
    for rank, (_, w, r, lr, worst, rate, seed, out) in results.items():
        assert (w, r, lr) == (2, rank, rank)
        assert worst == pytest.approx(5.0)          # max over ranks, not this rank's time
        assert rate == pytest.approx(2 * 8192 / 5e-3)  # whole-job queries/s
    assert results[0][6] != results[1][6]           # each rank draws its own chunk
    assert results[1][7] == ""                      # reference arm: rank 1 prints nothing
    assert all(p.exitcode == 0 for p in procs)
