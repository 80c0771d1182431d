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


# ------------------------------------------------ one chunk split by queries


def test_partition_covers_every_query_once_and_balances_work():
    """dsa_partition_queries (host arithmetic in the C library, no device):
    contiguous ranges covering [0, n_q) once, 4-row aligned boundaries, and
    useful work per rank within 1 % of an equal share."""
    sys.path.insert(0, ROOT)
    import numpy as np

    import sparse_attention_prefill_dsa_b200 as dsa
    import workloads
    from sparse_attention_prefill_dsa_b200 import build

    build.build()
    for name in ("chunk2k_ctx8k", "chunk8k_ctx17k", "chunk16k_ctx48k", "ties_4k_ctx8k"):
        d = workloads.BY_NAME[name].dims
        t = d.q_pos0 + np.arange(d.n_q, dtype=np.float64)
        work = (t + 1) * 2 * d.n_idx_heads * d.d_idx + \
            np.minimum(t + 1, d.top_k) * 2 * d.n_heads * (2 * d.d_latent + d.d_rope)
        for world in (2, 3, 4, 8):
            st, starts = dsa.dsa_partition_queries(d, world)
            assert st == dsa.DSA_OK
            assert starts[0] == 0 and starts[-1] == d.n_q
            assert all(a <= b for a, b in zip(starts, starts[1:]))
            shares = np.array([work[a:b].sum() for a, b in zip(starts, starts[1:])])
            assert np.abs(shares / (work.sum() / world) - 1).max() < 0.01, (name, world)
    d = workloads.BY_NAME["tiny_256q"].dims
    assert dsa.dsa_partition_queries(d, 0)[0] == dsa.DSA_ERR_DIMS
    st, starts = dsa.dsa_partition_queries(workloads.make_dims(6, 0, 6, 4, 64, 16, 2, 32, 4), 4)
    assert st == dsa.DSA_OK and starts[0] == 0 and starts[-1] == 6  # some ranks get no rows
    # 2 indexer heads: 8-byte w_idx rows, so boundaries fall on even rows
    st, starts = dsa.dsa_partition_queries(d, 8)
    assert all(s % 2 == 0 for s in starts) and starts[-1] == d.n_q
    # top_k = 1: 4-byte idx rows, so boundaries fall on multiples of 4 rows
    d1 = workloads.make_dims(200, 0, 200, 32, 512, 64, 32, 128, 1)
    st, starts = dsa.dsa_partition_queries(d1, 7)
    assert all(s % 4 == 0 for s in starts[:-1])


def _sharded_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    import torch.distributed as dist

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import workloads
        from sparse_attention_prefill_dsa_b200 import multi_gpu

        d0 = workloads.BY_NAME["tiny_256q"].dims
        d = workloads.make_dims(150, 106, 256, d0.n_heads, d0.d_latent, d0.d_rope,
                                d0.n_idx_heads, d0.d_idx, d0.top_k, d0.softmax_scale)
        x = workloads.generate(d, 9, "normal", "uniform")
        ranges = multi_gpu.query_ranges(d, world)
        s, e = ranges[rank]
        # this rank's cache: the prefix plus its own chunk rows; the other
        # ranks' chunk rows are garbage until the exchange
        cache = {}
        for key in ("latent", "rope", "k_idx"):
            c = torch.from_numpy(x[key].astype(np.int32)).clone()
            garbage = torch.full_like(c[d.q_pos0:], -77)
            garbage[s:e] = c[d.q_pos0 + s: d.q_pos0 + e]
            c[d.q_pos0:] = garbage
            cache[key] = c
        chunk = {k: torch.from_numpy(x[k].astype(np.int32) if x[k].dtype == np.uint16 else x[k])
                 for k in ("q", "q_idx", "w_idx")}
        outputs = {"out": torch.full((d.n_q, d.n_heads, d.d_latent), np.nan, dtype=torch.float64),
                   "lse": torch.full((d.n_q, d.n_heads), np.nan, dtype=torch.float64),
                   "idx": torch.full((d.n_q, d.top_k), -5, dtype=torch.int32)}

        def stand_in(sd, q_, latent, rope, q_idx, k_idx, w_idx, out, lse, idx):
            # the float64 oracle on this range (CPU stand-in for the CUDA layer)
            u16 = lambda t: t.numpy().astype(np.uint16)  # noqa: E731
            o, l, ix = oracle.prefill_layer(sd, u16(q_), u16(latent), u16(rope), u16(q_idx),
                                            u16(k_idx), w_idx.numpy(), n_threads=2)
            out.copy_(torch.from_numpy(o))
            lse.copy_(torch.from_numpy(l))
            idx.copy_(torch.from_numpy(ix))

        multi_gpu.prefill_layer_sharded(d, rank, world, cache, chunk, outputs, stand_in)
        cache_ok = all(np.array_equal(cache[k].numpy().astype(np.uint16), x[k])
                       for k in ("latent", "rope", "k_idx"))
        q.put((rank, (s, e), cache_ok, outputs["out"].numpy(), outputs["lse"].numpy(),
               outputs["idx"].numpy()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_one_chunk_by_queries():
    """Two gloo ranks each run the layer (the float64 oracle as the CPU stand-in)
    on their own query range: after the two exchanges every rank holds the whole
    chunk's cache rows and outputs, equal to one call on the whole chunk."""
    import numpy as np
    import torch.multiprocessing as mp

    sys.path.insert(0, ROOT)
    import oracle
    import workloads

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sharded_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in procs:
            item = q.get(timeout=180)
            results[item[0]] = item
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert sorted(results) == [0, 1]
    d0 = workloads.BY_NAME["tiny_256q"].dims
    d = workloads.make_dims(150, 106, 256, d0.n_heads, d0.d_latent, d0.d_rope, d0.n_idx_heads,
                            d0.d_idx, d0.top_k, d0.softmax_scale)
    x = workloads.generate(d, 9, "normal", "uniform")
    ref_out, ref_lse, ref_idx = oracle.prefill_layer(d, **x)
    (s0, e0), (s1, e1) = results[0][1], results[1][1]
    assert s0 == 0 and e0 == s1 and e1 == d.n_q and 0 < e0 < d.n_q
    for rank in (0, 1):
        _, _, cache_ok, out, lse, idx = results[rank]
        assert cache_ok, rank
        assert np.array_equal(out, ref_out) and np.array_equal(lse, ref_lse)
        assert np.array_equal(idx, ref_idx)
    assert all(p.exitcode == 0 for p in procs)
