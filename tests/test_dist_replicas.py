"""Multi-GPU logic of the benchmark, exercised as world-size-2 gloo ranks on the CPU.

The decode path has no exchange step (each request's attention is independent), so N GPUs
run N independent replicas.  What the ranks share is host logic: distinct seeded
workloads per rank, the barrier, the max-over-ranks reduction of the timings, the whole-job
value, and the reference arm that only rank 0 runs.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        from paged_kv_mla_create_b200 import workloads as W
        r, w, local = bench.dist_env()
        assert (r, w, local) == (rank, world, rank)
        # distinct replicas: each rank's pool and batch come from its own seed
        wl = W.make_workload(1, seed=bench.replica_seed(1, rank))
        digest = float(wl.kv_cache.float().abs().sum()) + float(wl.cache_seqlens.sum())
        digests = [None] * world
        dist.all_gather_object(digests, digest)
        # timings: rank k reports (k + 1) ms per step; the job takes the slowest
        times = bench.reduce_max_over_ranks([1.0 + rank, 10.0 - rank, 0.5], "cpu", world)
        dist.barrier()
        # the reference arm: ranks other than 0 return at once without work
        ref_rc = bench.run_reference(bench.parse_args(["--impl", "reference", "--steps", "1",
                                                       "--warmup", "0", "--config", "1"])) \
            if rank != 0 else 0
        out[rank] = {"digests": digests, "times": times, "ref_rc": ref_rc}
    finally:
        dist.destroy_process_group()


def test_replicas_world2_gloo():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    assert set(out.keys()) == {0, 1}
    for rank in range(world):
        res = out[rank]
        assert res["times"] == [2.0, 10.0, 0.5]
        assert res["ref_rc"] == 0
        d = res["digests"]
        assert len(d) == 2 and d[0] != d[1], "replicas must not share a workload"
    assert out[0]["digests"] == out[1]["digests"]


def test_job_value_counts_every_replica():
    import bench
    kv = 198.2e6
    one = bench.job_value(1, kv, 0.1)
    assert one == pytest.approx(kv / 1e-4 / 1e9)
    assert bench.job_value(4, kv, 0.1) == pytest.approx(4 * one)
    # single rank: the reduction is the identity
    assert bench.reduce_max_over_ranks([3.0, 1.5], "cpu", 1) == [3.0, 1.5]
