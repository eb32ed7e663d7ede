"""Host-side multi-rank logic of bench.py on CPU with gloo, world size 2.

The convolution shards as independent replicas (each rank its own batch
sample), so the only cross-rank steps are the timing barrier, the MAX
reduction of per-rank times and the SUM of the ranks' kernel-launch counts;
these run here without a GPU.
"""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from seeded_inputs.workloads import WORKLOADS
        wl = WORKLOADS["cfg2"]
        my_ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        mx = bench.max_over_ranks(my_ms, torch.device("cpu"))
        launches = bench.sum_over_ranks(20 + rank, torch.device("cpu"))   # per-rank kernel counts
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed(wl, rank))
        dist.barrier()
        out.put((rank, mx, launches, seeds))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_sharding():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, launches, seeds in res:
        assert mx == 15.0                              # max over ranks, on every rank
        assert launches == 41                          # the job's launches: summed over ranks
        assert len(set(seeds)) == 2                    # distinct samples per rank


def test_whole_job_throughput_counts_all_ranks():
    import bench
    one = bench.whole_job_tflops(1e12, 1, 10, 1000.0)
    two = bench.whole_job_tflops(1e12, 2, 10, 1000.0)
    assert one == pytest.approx(10.0)
    assert two == pytest.approx(20.0)
