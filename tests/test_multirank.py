"""Multi-rank host logic of bench.py on CPU with the gloo backend (world size 2): every rank
gets its own batch, timings are reduced with a max over ranks, and the job throughput counts
every rank's work against the slowest rank's time.  No GPU and no data-path collective."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import torch.distributed as dist
    import bench
    from attention_kl_divergence_02_b200 import inputs
    try:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        assert bench.dist_env() == (world, rank, rank)
        w = bench.rank_workload(inputs.WORKLOADS["headline"], rank)
        # per-rank timings: rank r is slower on some calls, faster on others
        local = [10.0 + rank, 3.0 - rank, 4.0 + 2 * rank, 4.5]
        got = bench.max_over_ranks(local)
        q.put((rank, w.seed, got, bench.job_tflops(world, 1e12, got[0])))
        dist.barrier()
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_rank_reduction_and_sharding():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    seeds = [r[1] for r in res]
    assert len(set(seeds)) == world                       # independent batch per rank
    for _, _, got, value in res:
        assert got == [11.0, 3.0, 6.0, 4.5]               # max over ranks, element-wise
        assert value == pytest.approx(world * 1e12 / 11e-3 / 1e12)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks([1.0, 2.0]) == [1.0, 2.0]
    assert bench.job_tflops(1, 2e12, 1000.0) == pytest.approx(2.0)
