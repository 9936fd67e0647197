"""Full-size parity: the workloads bench.py times, in the same launch
configuration (select and attention over every query), checked against the
oracle on sampled outputs and by properties that hold at any size.

The oracle never consumes a GPU result here: either it builds the tree that
the GPU index imports (lsa_build_index_from_tree), or the test checks
properties of the GPU's own output in plain numpy.
"""
import numpy as np
import pytest
import torch

import oracle as O
from hierarchical_latent_key_gemm_b200 import lsa
from hierarchical_latent_key_gemm_b200.workloads import WORKLOADS, make_inputs

import lsa_testutil as TU

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

BF16_MAX_ABS, BF16_MEAN_ABS = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lsa.lib()
    yield
    torch.cuda.synchronize()


def _oracle_rows(tree, Kl, inp, w, b, h, rows, Wm):
    q = O.query_latent(TU.unit_queries(inp["Q"], b, h, w.group, rows), Wm)
    out = []
    for k, i in enumerate(rows):
        blk = O.select_blocks(tree, Kl, q[k], int(i), w.beam, w.topk, w.window)
        out.append(O.selection_tokens(blk, int(i), w.sink, w.window, w.pool))
    return out, q


def _sample_rows(w, inp, rng, count):
    rows = set(rng.integers(0, w.n_tokens, count).tolist())
    rows |= {0, 1, w.sink + w.window + w.pool, w.n_tokens - 1}
    rows |= {qp for (_, _, _, qp) in inp["needles"][:32]}
    return np.array(sorted(rows))


def _check_selection_and_attention(w, inp, trees, Kls, sample, seed):
    """Import the oracle's trees, run select + banded attention over every query
    (the bench's launches), compare sampled rows with the oracle."""
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    leaf, par, cen = TU.trees_to_device(trees, w)
    ix = lsa.lsa_build_index_from_tree(TU.build_params(w), d["K"], d["W"], leaf, par, cen)
    sp = TU.select_params(w)
    idx, cnt = lsa.lsa_select(ix, sp, d["Q"])
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    Wm = inp["W"].double().cpu().numpy()
    rng = np.random.default_rng(seed)
    rows = _sample_rows(w, inp, rng, sample)
    oracle_sel = {}
    for h in range(w.hkv):
        u = h
        want, q = _oracle_rows(trees[u], Kls[u], inp, w, 0, h, rows, Wm)
        got = TU.gpu_rows(idx, cnt, 0, rows, h)
        assert TU.recall(got, want) >= 0.999
        for k, i in enumerate(rows):
            assert TU.selection_mismatch_ok(trees[u], Kls[u], q[k], int(i), w.beam, w.topk, w.window, got[k],
                                            want[k]), f"head {h} query {i}"
        oracle_sel[h] = want
        # the oracle's rows go into the index list the attention reads
        ii, cc = TU.rows_to_idx(want, w.max_sel)
        idx[0, torch.as_tensor(rows, device="cuda"), h] = ii
        cnt[0, torch.as_tensor(rows, device="cuda"), h] = cc
    # the bench's attention path: banded (dense sink/window tiles + ordered
    # long-range gather) over every query
    O_, lse = lsa.lsa_sparse_attn_banded(d["Q"], d["K"], d["V"], idx, cnt, w.hkv, w.sink, w.window)
    assert lsa.lsa_check(None) == lsa.LSA_OK
    errs = []
    G = w.group
    for h in range(w.hkv):
        Kh = inp["K"][0, :, h].float().cpu().double().numpy()
        Vh = inp["V"][0, :, h].float().cpu().double().numpy()
        for k, i in enumerate(rows):
            q = TU.unit_queries(inp["Q"], 0, h, G, [int(i)])[0]
            o, _ = O.sparse_attention(q, Kh, Vh, oracle_sel[h][k])
            errs.append(np.abs(O_[0, int(i), h * G:(h + 1) * G].double().cpu().numpy() - o).ravel())
    e = np.concatenate(errs)
    assert e.max() <= BF16_MAX_ABS and e.mean() <= BF16_MEAN_ABS
    ix.free()
    return idx, cnt


def test_gqa_128k_full_size():
    w = WORKLOADS["gqa_128k"]
    inp = make_inputs(w, seed=0, device="cuda")
    inp = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in inp.items()}
    Kls = TU.oracle_latents(inp, w)
    trees = TU.oracle_trees(Kls, w)
    # the GPU's own build against the oracle's (same inputs, same init)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    ix = lsa.lsa_build_index(TU.build_params(w), d["K"], d["W"])
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    leaf = ix.get(lsa.LSA_GET_LEAF_OF_BLOCK).cpu().numpy()
    obj = ix.get(lsa.LSA_GET_OBJECTIVE, 1).cpu().numpy()
    for u in range(w.hkv):
        assert (leaf[u] == trees[u].leaf_of_block).mean() >= 0.99
        assert abs(obj[0, u] - trees[u].objectives[1][0]) <= 1e-6 * trees[u].objectives[1][0]
        assert abs(obj[-1, u] - trees[u].objectives[1][-1]) <= 1e-3 * trees[u].objectives[1][-1]
    ix.free()
    _check_selection_and_attention(w, inp, trees, Kls, 160, 1)


def test_prefill_1m_full_size():
    w = WORKLOADS["prefill_1m"]
    inp = make_inputs(w, seed=0, device="cuda")
    d = inp
    inp = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in inp.items()}
    Kls = TU.oracle_latents(inp, w)
    # first Lloyd round at full size: GPU (tensor cores) vs fp64 argmin on sampled points
    Kl_gpu = lsa.lsa_project_pool(d["K"], d["W"], w.n_tokens, w.pool)
    labels, C1, _ = lsa.lsa_kmeans(Kl_gpu, w.level_sizes[-1], 1)
    rng = np.random.default_rng(3)
    for u in range(w.hkv):
        X = Kls[u]
        C0 = O.kmeans_init(X, w.level_sizes[-1])
        pts = rng.integers(0, X.shape[0], 2048)
        d2 = O.squared_distances(X[pts], C0)
        want = np.argmin(d2, axis=1)
        srt = np.sort(d2, axis=1)
        gap = (srt[:, 1] - srt[:, 0]) / np.maximum(1.0, (X[pts] ** 2).sum(1) + srt[:, 0])
        got = labels[u].cpu().numpy()[pts]
        assert not ((got != want) & (gap > 1e-5)).any()
    # one-round oracle trees, imported; select + attention over every query
    trees = [O.build_tree(Kl, w.level_sizes, 1, 0, w.sink, w.pool) for Kl in Kls]
    _check_selection_and_attention(w, inp, trees, Kls, 96, 2)


def test_decode_10m_x4_properties():
    """Build over 4 x 10M tokens and run decode steps; every selection row is
    valid (sorted, unique, causal, sink and window present, chosen blocks of
    the leaves the index reports) and every appended block sits in its nearest
    leaf of the frozen centroids (checked in plain numpy)."""
    w = WORKLOADS["decode_10m_x4"]
    free = torch.cuda.mem_get_info()[0]
    if free < 60 << 30:
        pytest.skip("needs about 60 GB of free device memory")
    inp = make_inputs(w, seed=0, device="cuda")
    steps = 32
    ix = lsa.lsa_build_index(TU.build_params(w, append_capacity=w.decode_steps), inp["K"], inp["W"])
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    sp = TU.select_params(w)
    n0 = w.n_tokens
    for s in range(steps):
        lsa.lsa_append(ix, inp["K"], 1)
        t = n0 + s
        q = inp["Q"][:, s:s + 1].contiguous()
        idx, cnt = lsa.lsa_select(ix, sp, q, q_pos0=t)
        O_, lse = lsa.lsa_sparse_attn(q, inp["K"], inp["V"], idx, cnt, w.hkv)
        assert lsa.lsa_check(ix) == lsa.LSA_OK
        for b in range(w.batch):
            row = idx[b, 0, 0, : cnt[b, 0, 0]].cpu().numpy()
            assert np.all(np.diff(row) > 0) and row[-1] == t and row[0] == 0
            assert set(range(w.sink)) <= set(row.tolist())
            assert set(range(t - w.window + 1, t + 1)) <= set(row.tolist())
            # sink + window + whole blocks of the budget; every long-range token is a
            # candidate (at or after the sink, before the window, in a complete block)
            n_long = int(cnt[b, 0, 0]) - w.sink - w.window
            assert 0 <= n_long <= w.topk and n_long % w.pool == 0
            longr = row[(row >= w.sink) & (row < t - w.window + 1)]
            assert longr.size == n_long
            assert np.all(longr // w.pool * w.pool + w.pool - 1 <= t - w.window)
        assert torch.isfinite(O_.float()).all()
    # appended blocks: nearest leaf of the frozen leaf centroids
    nb0 = n0 // w.pool
    nb1 = (n0 + steps) // w.pool
    leaf = ix.get(lsa.LSA_GET_LEAF_OF_BLOCK)[:, nb0:nb1].cpu().numpy()
    lat = ix.get(lsa.LSA_GET_LATENT)[:, nb0:nb1].double().cpu().numpy()
    cent = ix.get(lsa.LSA_GET_CENTROIDS, len(w.level_sizes) - 1).double().cpu().numpy()
    for b in range(w.batch):
        d2 = ((lat[b][:, None, :] - cent[b][None, :, :]) ** 2).sum(-1)
        best = d2.min(axis=1)
        chosen = d2[np.arange(d2.shape[0]), leaf[b]]
        assert np.all(chosen <= best * (1 + 1e-5) + 1e-6)
    ix.free()
