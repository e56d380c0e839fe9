"""The multi-rank path of bench.py on CPU: world size 2 over gloo (127.0.0.1). Replicas only: the
one cross-rank step is the timing reduction (max over ranks) and the edge count (sum)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        times, edges = bench.combine_ranks([1.0 + rank, 5.0 - rank, 0.25 * (rank + 1)], 1000 + rank, world, "cpu")
        dist.barrier()
        out[rank] = (times, edges)
    finally:
        dist.destroy_process_group()


def test_combine_ranks_max_times_sum_edges():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        times, edges = res[rank]
        assert times == [2.0, 5.0, 0.5]
        assert edges == 2001.0


def test_combine_ranks_single_rank_is_identity():
    import bench
    times, edges = bench.combine_ranks([3.0, 4.0], 17, 1, "cpu")
    assert times == [3.0, 4.0] and edges == 17.0


def test_reference_arm_runs_on_rank_zero_only():
    import bench

    class Args:
        workload = "tiny"
        warmup = 3
        steps = 1
        cpu_budget = 5.0

    assert bench.run_reference(Args, rank=1, world=2) is None
    line = bench.run_reference(Args, rank=0, world=2)
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
