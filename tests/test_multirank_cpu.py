"""Multi-rank host logic of the benchmark on CPU: two gloo ranks, each with its own batch
(distinct seeds), the maximum over ranks of a per-rank time, and the whole-job
throughput.  No GPU; the data path has no collective to test."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import bench
    import workloads
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = workloads.WORKLOADS["causal_b8_h32_n4k_d128"].with_(B=1, Hq=2, Hkv=2, N=64, d=64)
        seeds = bench.rank_seeds(w, rank)
        q, _, _ = workloads.make_inputs(w, seeds=seeds)
        digest = float(q.float().sum())
        elapsed = 10.0 + 5.0 * rank          # a per-rank "time"
        m = bench.max_over_ranks(elapsed)
        gathered = [None] * world
        dist.all_gather_object(gathered, (seeds, digest))
        if rank == 0:
            out.put((m, gathered, bench.job_tflops(world, 1e12, 10, m)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    m, gathered, tflops = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert m == 15.0                      # slowest rank's time
    (s0, d0), (s1, d1) = gathered
    assert s0 != s1 and d0 != d1          # each rank has its own batch
    assert tflops == pytest.approx(2 * 1e12 * 10 / 0.015 / 1e12)


def test_single_process_reduction_is_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_tflops(1, 2e12, 4, 8.0) == pytest.approx(1000.0)
