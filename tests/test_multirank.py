"""The multi-GPU plumbing of bench.py on CPU: two gloo ranks, as torchrun
would start them. Each rank draws its own stack (different seeds); the
timing reduction takes the maximum over ranks; whole-job throughput counts
every rank's bytes over the slowest rank's time; the reference arm runs on
rank 0 only."""
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


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, _ = bench.dist_env()
    d = bench.init_dist(w, "gloo")
    cpu = torch.device("cpu")
    slow = bench.max_over_ranks(1.0 + rank, d, cpu)          # rank 1 is the slowest
    bench.barrier(d, cpu)
    seed = bench.rank_seed_base(r)
    gathered = [None] * w
    dist.all_gather_object(gathered, seed)
    rc_ref = bench.run_reference(type("A", (), {"warmup": 0, "steps": 1, "gpus": w})) if r else 0
    results[rank] = (w, r, slow, tuple(gathered), rc_ref)
    dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    manager = mp.get_context("spawn").Manager()
    results = manager.dict()
    mp.start_processes(_worker, args=(world, port, results), nprocs=world, start_method="spawn",
                       join=True)
    assert sorted(results.keys()) == [0, 1]
    for rank in (0, 1):
        w, r, slow, seeds, rc_ref = results[rank]
        assert (w, r) == (2, rank)
        assert slow == 2.0
        assert len(set(seeds)) == 2      # every rank draws a different stack
        assert rc_ref == 0               # non-zero ranks leave the reference arm without work


def test_whole_job_throughput():
    import bench
    # two ranks, 1 GB each per step, 4 steps, slowest rank 2 s -> 4 GB/s
    assert bench.whole_job_gbs(2, 1e9, 4, 2.0) == pytest.approx(4.0)
    assert bench.whole_job_gbs(1, 16.06e9, 10, 0.05) == pytest.approx(3212.0)
