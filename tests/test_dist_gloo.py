"""Multi-rank host logic of bench.py on CPU: world size 2 over gloo.  Each
rank is an independent replica (its own seed); the only cross-rank steps are
the barrier and the max-over-ranks timing reduction."""
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import bench
    try:
        ws, r = bench.init_dist("gloo")
        assert (ws, r) == (world, rank)
        bench.barrier()
        local_ms = 10.0 + 5.0 * rank                     # rank 1 is the slow one
        m = bench.max_over_ranks(local_ms, torch.device("cpu"))
        # each replica draws its own batch: seeds differ per rank
        from quantization_nvfp4_quantize_b200 import workloads as wl
        cfg = wl.CONFIGS["dense_64x256"]
        x = wl.activations(cfg, 0 + rank)
        digest = float(x.float().sum())
        digests = [None] * world
        dist.all_gather_object(digests, digest)
        q.put((rank, m, digests))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_rank_max_timing_and_independent_replicas():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, digests in results:
        assert m == 15.0, "time must be the max over ranks"
        assert digests[0] != digests[1], "replicas must draw different batches"


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5


def _ref_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import argparse
    import bench
    try:
        args = argparse.Namespace(workload="moe_t512_e8", steps=1, warmup=0, seed=0, gpus=world)
        out = bench.run_reference(args)
        q.put((rank, None if out is None else (out["impl"], out["n_gpus"], out["cpu_baseline"]["kind"])))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun the oracle arm runs on rank 0 alone; other ranks exit
    without work."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ref_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results[1] is None
    assert results[0] == ("reference", world, "oracle")
