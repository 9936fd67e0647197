"""The multi-GPU plumbing of bench.py on CPU ranks (gloo, world size 2): the
timing reduction is a max over ranks, the barrier joins every rank, each
rank draws its own instance (seed offset by rank), and the reference arm
runs on rank 0 only.  The data path itself has no collective: every rank
processes an independent layer instance."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, lr = bench.dist_env()
        assert (r, w, lr) == (rank, world, rank)
        bench.barrier(world)
        # per-rank timings: the reported one is the slowest rank's
        t = bench.max_over_ranks(10.0 + 5.0 * rank, world, torch.device("cpu"))
        out[rank] = t
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_timing_is_max_over_ranks_gloo():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert dict(out) == {0: 15.0, 1: 15.0}


def test_reference_arm_is_rank0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0
    assert res.stdout.strip() == ""


def test_rank_instances_differ_by_seed():
    """Each rank draws its own instance: the bench seeds rank k with
    seed + 1000 k, and the generator gives different inputs for them."""
    from hierarchical_latent_key_gemm_b200.workloads import WORKLOADS, make_inputs
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=512, level_sizes=(2, 8), needles=0, components=16)
    a = make_inputs(w, seed=0)
    b = make_inputs(w, seed=1000)
    c = make_inputs(w, seed=0)
    assert not torch.equal(a["K"], b["K"]) and torch.equal(a["K"], c["K"])
