"""Context parallelism on one GPU: the shards of one sequence run one after
another on the same device (no process group: the exchange is a stack of the
shards' outputs, which is what the all-gather of the multi-GPU path
returns), through the C ABI, against the oracle's sharded reading
(oracle.cp_select_blocks, oracle.merge_attention) and against the unsharded
path.  Integer workload: selections bit-exact.  Float workload, beam over
every node: the sharded selection equals the unsharded full scan bit for bit
(the shards compute the same fp32 scores)."""
import numpy as np
import pytest
import torch

import oracle as O
from hierarchical_latent_key_gemm_b200 import lsa
from hierarchical_latent_key_gemm_b200.context_parallel import ContextShard
from hierarchical_latent_key_gemm_b200.workloads import WORKLOADS, make_inputs

import lsa_testutil as TU

pytestmark = pytest.mark.gpu

BF16_MAX_ABS, BF16_MEAN_ABS = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lsa.lib()
    yield
    torch.cuda.synchronize()


def _shards(w, world, N):
    return [ContextShard(s, world, N, w.pool, w.sink) for s in range(world)]


def _build(w, shards, K, W, append=0):
    out = []
    for sh in shards:
        n_loc = sh.t1 - sh.t0 + (append if sh.last else 0)
        Kloc = K[:, sh.t0:sh.t0 + n_loc].contiguous()
        bp = sh.build_params(w.batch, n_loc, w.hkv, w.d, w.r,
                             lsa.LSA_F32 if w.dtype == "f32" else lsa.LSA_BF16, w.level_sizes, w.lloyd_iters,
                             w.grid_log2, append_capacity=append)
        out.append((lsa.lsa_build_index(bp, Kloc, W), Kloc))
    return out


def _cp_select(shards, built, sp, Q, q_pos=None, q_pos0=0):
    picks = [sh.local_picks(ix, sp, Q, q_pos=q_pos, q_pos0=q_pos0) for sh, (ix, _) in zip(shards, built)]
    S = torch.stack([p[0] for p in picks])
    B = torch.stack([p[1] for p in picks])
    C = torch.stack([p[2] for p in picks])
    return shards[0].merge_picks(S, B, C, sp, q_pos=q_pos, q_pos0=q_pos0)


def _cp_attend(shards, built, Q, V, idx, cnt, hkv):
    parts = []
    for sh, (ix, Kloc) in zip(shards, built):
        n_loc = Kloc.shape[1]
        Vloc = V[:, sh.t0:sh.t0 + n_loc].contiguous()
        parts.append(sh.local_attend(Q, Kloc, Vloc, idx, cnt, hkv))
    return ContextShard.merge_parts(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_integer_workload_is_bit_exact(world):
    w = WORKLOADS["int_exact_16k"].scaled(n_tokens=4096 + 5, level_sizes=(8, 64))
    inp = make_inputs(w, seed=21)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    N = w.n_tokens
    shards = _shards(w, world, N)
    built = _build(w, shards, d["K"], d["W"])
    sp = TU.select_params(w)
    idx, cnt = _cp_select(shards, built, sp, d["Q"])
    assert lsa.lsa_check(None) == lsa.LSA_OK
    for ix, _ in built:
        assert lsa.lsa_check(ix) == lsa.LSA_OK
    # the oracle's sharded reading: per-shard trees on the grid, merged picks
    Wm = inp["W"].double().numpy()
    Kn = inp["K"][0, :, 0].float().double().numpy()
    Vn = inp["V"][0, :, 0].float().double().numpy()
    oshards = []
    for sh in shards:
        Kl_s = O.project_pool(Kn[sh.t0:sh.t1], Wm, w.pool)
        oshards.append((sh.t0, O.build_tree(Kl_s, w.level_sizes, w.lloyd_iters, w.grid_log2, sh.local_sink,
                                            w.pool), Kl_s))
    q = O.query_latent(TU.unit_queries(inp["Q"], 0, 0, w.group), Wm)
    rows = list(range(0, N, 7)) + [N - 1]
    sels = []
    for i in rows:
        blk = O.cp_select_blocks(oshards, q[i], i, w.beam, w.topk, w.window, w.pool)
        want = O.selection_tokens(blk, i, w.sink, w.window, w.pool)
        got = idx[0, i, 0, : cnt[0, i, 0]].cpu().numpy()
        np.testing.assert_array_equal(got, want, err_msg=f"query {i}")
        sels.append(want)
    # attention: shards' parts merged, against the oracle on the whole row
    O_, lse = _cp_attend(shards, built, d["Q"], d["V"], idx, cnt, w.hkv)
    assert lsa.lsa_check(None) == lsa.LSA_OK
    # (|O| reaches 4 here and the path rounds to bf16 twice, the shards' parts
    # and the merged output: two half-ulps of 4 plus fp32 accumulation)
    tol = 2 * 2.0 ** -8 * 4 + 1e-3
    errs = []
    for k, i in enumerate(rows):
        o, l = O.sparse_attention(TU.unit_queries(inp["Q"], 0, 0, w.group, [i])[0], Kn, Vn, sels[k])
        got = O_[0, i].double().cpu().numpy()
        assert np.all(np.abs(got - o) <= tol), f"query {i}"
        errs.append(np.abs(lse[0, i].double().cpu().numpy() - l).max())
    assert max(errs) <= 1e-3
    for ix, _ in built:
        ix.free()


def test_sharded_full_beam_equals_unsharded_fullscan():
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=8192 + 6, level_sizes=(4, 32), needles=0, components=128)
    inp = make_inputs(w, seed=22, device="cuda")
    N, world = w.n_tokens, 3
    shards = _shards(w, world, N)
    built = _build(w, shards, inp["K"], inp["W"])
    sp = TU.select_params(w, beam=1024)
    idx, cnt = _cp_select(shards, built, sp, inp["Q"])
    ix = lsa.lsa_build_index(TU.build_params(w), inp["K"], inp["W"])
    fidx, fcnt = lsa.lsa_fullscan_select(ix, sp, inp["Q"])
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    assert torch.equal(cnt, fcnt)
    assert torch.equal(idx, fidx)
    # attention over the same rows: sharded parts merged vs one pass
    O_, lse = _cp_attend(shards, built, inp["Q"], inp["V"], idx, cnt, w.hkv)
    O1, lse1 = lsa.lsa_sparse_attn(inp["Q"], inp["K"], inp["V"], idx, cnt, w.hkv)
    assert lsa.lsa_check(None) == lsa.LSA_OK
    e = (O_.float() - O1.float()).abs()
    assert e.max().item() <= BF16_MAX_ABS and e.mean().item() <= BF16_MEAN_ABS
    assert (lse - lse1).abs().max().item() <= 1e-4
    ix.free()
    for b, _ in built:
        b.free()


def test_sharded_decode_appends_to_the_last_shard():
    """Decode over two shards: tokens appended after the build go to the last
    shard's index; every step's selection equals the oracle's sharded reading
    (integer workload, bit-exact) and its attention the oracle's."""
    w = WORKLOADS["int_exact_16k"].scaled(n_tokens=2048 + 3, level_sizes=(8, 32), decode_steps=12, window=16,
                                          topk=128)
    inp = make_inputs(w, seed=23)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    N, steps = w.n_tokens, w.decode_steps
    shards = _shards(w, 2, N)
    built = _build(w, shards, d["K"], d["W"], append=steps)
    sp = TU.select_params(w)
    Wm = inp["W"].double().numpy()
    Kn = inp["K"][0, :, 0].float().double().numpy()
    Vn = inp["V"][0, :, 0].float().double().numpy()
    oshards = []
    for sh in shards:
        Kl_s = O.project_pool(Kn[sh.t0:sh.t1], Wm, w.pool)
        oshards.append([sh.t0, O.build_tree(Kl_s, w.level_sizes, w.lloyd_iters, w.grid_log2, sh.local_sink,
                                            w.pool), list(Kl_s)])
    last_ix = built[-1][0]
    for s in range(steps):
        t = N + s
        shards[-1].append(last_ix, built[-1][1], 1)
        # the oracle's last shard: every completed block joins its nearest leaf
        t0, tree, rows = oshards[-1]
        if (t + 1 - t0) % w.pool == 0:
            x = O.project_pool(Kn[t + 1 - w.pool:t + 1], Wm, w.pool)[0]
            O.append_block(tree, rows, x)
        q = d["Q"][:, s:s + 1].contiguous()
        idx, cnt = _cp_select(shards, built, sp, q, q_pos0=t)
        qb = O.query_latent(TU.unit_queries(inp["Q"], 0, 0, w.group, [s]), Wm)[0]
        blk = O.cp_select_blocks([(a, b, np.array(c)) for a, b, c in oshards], qb, t, w.beam, w.topk, w.window,
                                 w.pool)
        want = O.selection_tokens(blk, t, w.sink, w.window, w.pool)
        np.testing.assert_array_equal(idx[0, 0, 0, : cnt[0, 0, 0]].cpu().numpy(), want, err_msg=f"step {s}")
        O_, _ = _cp_attend(shards, built, q, d["V"], idx, cnt, w.hkv)
        o, _ = O.sparse_attention(TU.unit_queries(inp["Q"], 0, 0, w.group, [s])[0], Kn, Vn, want)
        got = O_[0, 0].double().cpu().numpy()
        assert np.all(np.abs(got - o) <= 2 * 2.0 ** -8 * 4 + 1e-3), f"step {s}"
    for ix, _ in built:
        assert lsa.lsa_check(ix) == lsa.LSA_OK
        ix.free()


def test_merge_and_localize_edges():
    """Rows with no entries in a shard, and parts that are all empty."""
    idx = torch.tensor([[[[0, 5, 9, 12, -1, -1]], [[3, 4, -1, -1, -1, -1]], [[-1] * 6]]], dtype=torch.int32,
                       device="cuda")
    cnt = torch.tensor([[[4], [2], [0]]], dtype=torch.int32, device="cuda")
    li, lc = lsa.lsa_localize_rows(idx, cnt, 5, 12)
    assert lc.flatten().tolist() == [2, 0, 0]
    assert li[0, 0, 0].tolist() == [0, 4, -1, -1, -1, -1]
    # in place
    idx2, cnt2 = idx.clone(), cnt.clone()
    lsa.lsa_localize_rows(idx2, cnt2, 0, 5, idx_out=idx2, cnt_out=cnt2)
    assert cnt2.flatten().tolist() == [1, 2, 0] and idx2[0, 1, 0, :3].tolist() == [3, 4, -1]
    Op = torch.zeros((2, 1, 3, 2, 64), dtype=torch.bfloat16, device="cuda")
    Lp = torch.full((2, 1, 3, 2), -float("inf"), device="cuda")
    Op[1, 0, 1] = 1.0
    Lp[1, 0, 1] = 0.5
    O_, lse = lsa.lsa_merge_attn(Op, Lp)
    assert torch.all(O_[0, 0] == 0) and torch.all(lse[0, 0] == -float("inf"))
    assert torch.all(O_[0, 1] == 1) and torch.allclose(lse[0, 1], torch.tensor(0.5, device="cuda"))
    assert lsa.lsa_check(None) == lsa.LSA_OK
