"""Context parallelism on CPU ranks (gloo, world size 2): the shard ranges,
and the two exchanges of the sharded path (the shards' scored picks, then
the attention parts) through the package's all_gather, with the oracle
standing in for the per-shard kernels.  After the exchange every rank merges
and must hold exactly the unsharded result: with a beam that keeps every
node, the global full scan's selection; and attention over the whole
selection."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402
from hierarchical_latent_key_gemm_b200 import context_parallel as CP  # noqa: E402


def test_shard_range_matches_the_oracle():
    for n, world, pool in ((10, 3, 2), (11, 2, 4), (7, 1, 4), (1000, 4, 4), (1003, 3, 2), (64, 8, 8),
                           (10_000_000, 8, 4)):
        want = O.shard_ranges(n, world, pool)
        got = [CP.shard_range(n, world, r, pool) for r in range(world)]
        assert got == want


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


N, POOL, SINK, WINDOW, TOPK, R, D = 600, 2, 6, 10, 40, 4, 8
SIZES = (2, 8)


def _data():
    rng = np.random.default_rng(11)
    Kl = rng.standard_normal((N // POOL, R))
    K = rng.standard_normal((N, D))
    V = rng.standard_normal((N, D))
    qpos = np.array([5, 30, 101, 299, 300, 301, 450, N - 1])
    qbar = rng.standard_normal((qpos.size, R))
    q = rng.standard_normal((qpos.size, 2, D))
    return Kl, K, V, qpos, qbar, q


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        Kl, K, V, qpos, qbar, q = _data()
        shard = CP.ContextShard(rank, world, N, POOL, SINK)
        t0, t1 = shard.t0, shard.t1
        b0, b1 = t0 // POOL, t1 // POOL
        tree = O.build_tree(Kl[b0:b1], SIZES, 3, 0, shard.local_sink, POOL)
        kb = O.blocks_per_topk(TOPK, POOL)
        nq = qpos.size
        # this shard's picks (oracle), in the layout of lsa_select_blocks
        sc = torch.full((1, nq, 1, kb), -float("inf"), dtype=torch.float32)
        bl = torch.full((1, nq, 1, kb), -1, dtype=torch.int32)
        ct = torch.zeros((1, nq, 1), dtype=torch.int32)
        for k, i in enumerate(qpos):
            b, s = O.scored_blocks(tree, Kl[b0:b1], qbar[k], int(i) - t0, 1000, TOPK, WINDOW)
            sc[0, k, 0, : b.size] = torch.from_numpy(s.astype(np.float32))
            bl[0, k, 0, : b.size] = torch.from_numpy((b + b0).astype(np.int32))
            ct[0, k, 0] = b.size
        S, B, C = shard.gather(sc), shard.gather(bl), shard.gather(ct)
        assert S.shape == (world, 1, nq, 1, kb) and B.dtype == torch.int32 and C.shape == (world, 1, nq, 1)
        sels = []
        for k, i in enumerate(qpos):
            ids = np.concatenate([B[s, 0, k, 0, : C[s, 0, k, 0]].numpy() for s in range(world)]).astype(np.int64)
            scs = np.concatenate([S[s, 0, k, 0, : C[s, 0, k, 0]].numpy() for s in range(world)]).astype(np.float64)
            chosen = np.sort(O.top_by_score(ids, scs, kb))
            sels.append(O.selection_tokens(chosen, int(i), SINK, WINDOW, POOL))
        # attention parts over this shard's rows, exchanged and merged
        ok, lk = [], []
        for k, sel in enumerate(sels):
            mine = sel[(sel >= t0) & (sel < t1)]
            if mine.size:
                o, l = O.sparse_attention(q[k], K, V, mine)
            else:
                o, l = np.zeros((2, D)), np.full(2, -np.inf)
            ok.append(o)
            lk.append(l)
        Op = shard.gather(torch.tensor(np.stack(ok)))
        Lp = shard.gather(torch.tensor(np.stack(lk)))
        res = []
        for k in range(nq):
            o, l = O.merge_attention([Op[s, k].numpy() for s in range(world)], [Lp[s, k].numpy() for s in range(world)])
            res.append((sels[k], o, l))
        out[rank] = res
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_context_parallel_exchange_gloo(world):
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    Kl, K, V, qpos, qbar, q = _data()
    for rank in range(world):
        for k, i in enumerate(qpos):
            sel, o, l = out[rank][k]
            # full beam: the sharded search is the global full scan
            want_blocks = O.fullscan_blocks(Kl, qbar[k], int(i), TOPK, SINK, WINDOW, POOL)
            want = O.selection_tokens(want_blocks, int(i), SINK, WINDOW, POOL)
            np.testing.assert_array_equal(sel, want)
            wo, wl = O.sparse_attention(q[k], K, V, want)
            np.testing.assert_allclose(o, wo, atol=1e-12, rtol=0)
            np.testing.assert_allclose(l, wl, atol=1e-12, rtol=0)
