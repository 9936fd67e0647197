"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Index sets: bit-exact on the integer workload; float
workloads: recall >= 0.999 with every mismatch within 1e-3 relative of the
K-th (or a level's B-th) threshold.  Attention on the oracle's index sets:
max-abs 2e-2 / mean-abs 2e-3 for bf16 I/O (fp32 accumulate), 1e-4 for fp32.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from hierarchical_latent_key_gemm_b200 import lsa
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


def _dev(inp):
    return {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}


def _assert_clean(index=None):
    assert lsa.lsa_check(index) == lsa.LSA_OK


# ------------------------------------------------------------------ latents
@pytest.mark.parametrize("name,n", [("flat_4k_f32", 1000), ("int_exact_16k", 777), ("gqa_128k", 1031)])
def test_project_pool_and_query_latent(name, n):
    w = WORKLOADS[name].scaled(n_tokens=n, needles=0)
    inp = make_inputs(w, seed=3)
    d = _dev(inp)
    Kl = lsa.lsa_project_pool(d["K"], d["W"], n, w.pool)
    qb = lsa.lsa_query_latent(d["Q"], d["W"], w.hkv)
    _assert_clean()
    Wm = inp["W"].double().numpy()
    exact = w.kind == "int"
    for h in range(w.hkv):
        want = O.project_pool(TU.unit_keys(inp["K"], 0, h, n), Wm, w.pool)
        got = Kl[h].double().cpu().numpy()
        assert got.shape == want.shape
        if exact:
            np.testing.assert_array_equal(got, want)
        else:
            np.testing.assert_allclose(got, want, rtol=1e-5, atol=2e-5)
        wq = O.query_latent(TU.unit_queries(inp["Q"], 0, h, w.group), Wm)
        gq = qb[0, :, h].double().cpu().numpy()
        if exact:
            np.testing.assert_array_equal(gq, wq)
        else:
            np.testing.assert_allclose(gq, wq, rtol=1e-5, atol=2e-5)


# ------------------------------------------------------------------ k-means
def test_kmeans_integer_grid_bit_exact():
    g = torch.Generator().manual_seed(11)
    X = torch.randint(-40, 41, (2, 1001, 16), generator=g).float()
    labels, C, obj = lsa.lsa_kmeans(X.cuda(), 37, 5, grid_log2=4)
    _assert_clean()
    for u in range(2):
        res = O.kmeans(X[u].double().numpy(), 37, 5, grid_log2=4)
        np.testing.assert_array_equal(labels[u].cpu().numpy(), res.labels)
        np.testing.assert_array_equal(C[u].double().cpu().numpy(), res.centroids)
        np.testing.assert_array_equal(obj[:, u].cpu().numpy(), np.array(res.objectives))


def _mixture_points(U, n, r, comps, seed):
    g = torch.Generator().manual_seed(seed)
    mu = torch.randn(comps, r, generator=g) * 2
    lab = torch.randint(0, comps, (U, n), generator=g)
    return mu[lab] + 0.3 * torch.randn(U, n, r, generator=g)


@pytest.mark.parametrize("r", [16, 32, 64])
def test_kmeans_float_single_round(r):
    X = _mixture_points(2, 3001, r, 50, 12 + r)
    labels, C, obj = lsa.lsa_kmeans(X.cuda(), 64, 1)
    _assert_clean()
    for u in range(2):
        Xu = X[u].double().numpy()
        C0 = O.kmeans_init(Xu, 64)
        d2 = O.squared_distances(Xu, C0)
        want = np.argmin(d2, axis=1)
        got = labels[u].cpu().numpy()
        srt = np.sort(d2, axis=1)
        gap = (srt[:, 1] - srt[:, 0]) / np.maximum(1.0, np.abs(srt[:, 0]) + (Xu ** 2).sum(1))
        bad = (got != want) & (gap > 1e-5)
        assert not bad.any(), f"{bad.sum()} labels differ away from ties"
        res = O.kmeans(Xu, 64, 1)
        if (got == want).all():
            np.testing.assert_allclose(C[u].double().cpu().numpy(), res.centroids, rtol=1e-6, atol=1e-6)
            assert abs(obj[0, u].item() - res.objectives[0]) <= 1e-9 * res.objectives[0]


def test_kmeans_float_many_rounds():
    X = _mixture_points(2, 4096, 32, 64, 21)
    labels, C, obj = lsa.lsa_kmeans(X.cuda(), 64, 10)
    _assert_clean()
    for u in range(2):
        res = O.kmeans(X[u].double().numpy(), 64, 10)
        agree = (labels[u].cpu().numpy() == res.labels).mean()
        assert agree >= 0.999
        o = obj[:, u].cpu().numpy()
        assert np.all(np.diff(o) <= 1e-6 * o[0])
        assert abs(o[-1] - res.objectives[-1]) <= 1e-4 * res.objectives[-1]


# ------------------------------------------------------------------ build
def _check_tree_invariants(ix, w, Kl_host_units, exact):
    U = w.batch * w.hkv
    leaf = ix.get(lsa.LSA_GET_LEAF_OF_BLOCK).cpu().numpy()
    cnts = ix.get(lsa.LSA_GET_LEAF_COUNT).cpu().numpy()
    cents = [ix.get(lsa.LSA_GET_CENTROIDS, l).double().cpu().numpy() for l in range(len(w.level_sizes))]
    mps = [ix.get(lsa.LSA_GET_MINPOS, l).cpu().numpy() for l in range(len(w.level_sizes))]
    L = w.level_sizes[-1]
    for u in range(U):
        assert leaf[u].min() >= 0 and leaf[u].max() < L            # every block in exactly one leaf
        np.testing.assert_array_equal(np.bincount(leaf[u], minlength=L), cnts[u])
        Kl = Kl_host_units[u]
        for j in np.unique(leaf[u]):
            mem = np.flatnonzero(leaf[u] == j)
            if exact:
                want = O.kmeans_update(Kl, leaf[u].astype(np.int64), cents[-1][u], w.grid_log2)[j]
                np.testing.assert_array_equal(cents[-1][u][j], want)
            else:
                np.testing.assert_allclose(cents[-1][u][j], Kl[mem].mean(axis=0), rtol=1e-5, atol=1e-5)
            starts = mem * w.pool
            starts = starts[starts >= w.sink]
            assert mps[-1][u][j] == (starts.min() if starts.size else np.iinfo(np.int64).max)
        for l in range(len(w.level_sizes) - 1):
            par = ix.get(lsa.LSA_GET_PARENT, l + 1).cpu().numpy()[u]
            assert par.min() >= 0 and par.max() < w.level_sizes[l]
            for j in range(w.level_sizes[l]):
                kids = np.flatnonzero(par == j)
                want = min([mps[l + 1][u][c] for c in kids], default=np.iinfo(np.int64).max)
                assert mps[l][u][j] == want
        for l in range(len(w.level_sizes)):
            o = ix.get(lsa.LSA_GET_OBJECTIVE, l).cpu().numpy()[:, u]
            assert np.all(np.diff(o) <= (0 if exact else 1e-6 * o[0]))


def test_build_integer_workload_matches_oracle_exactly():
    w = WORKLOADS["int_exact_16k"]
    inp = make_inputs(w, seed=0)
    d = _dev(inp)
    ix = lsa.lsa_build_index(TU.build_params(w), d["K"], d["W"])
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    Kls = TU.oracle_latents(inp, w)
    trees = TU.oracle_trees(Kls, w)
    t = trees[0]
    np.testing.assert_array_equal(ix.get(lsa.LSA_GET_LATENT).double().cpu().numpy()[0], Kls[0])
    np.testing.assert_array_equal(ix.get(lsa.LSA_GET_LEAF_OF_BLOCK).cpu().numpy()[0], t.leaf_of_block)
    for l in range(t.levels):
        np.testing.assert_array_equal(ix.get(lsa.LSA_GET_CENTROIDS, l).double().cpu().numpy()[0], t.centroids[l])
        mp = ix.get(lsa.LSA_GET_MINPOS, l).cpu().numpy()[0]
        np.testing.assert_array_equal(np.where(mp == np.iinfo(np.int64).max, np.inf, mp.astype(float)), t.minpos[l])
        np.testing.assert_array_equal(ix.get(lsa.LSA_GET_OBJECTIVE, l).cpu().numpy()[:, 0], t.objectives[l])
    np.testing.assert_array_equal(ix.get(lsa.LSA_GET_PARENT, 1).cpu().numpy()[0], t.parent[1])
    _check_tree_invariants(ix, w, Kls, exact=True)
    ix.free()


def test_build_flat_float_invariants_and_objective():
    w = WORKLOADS["flat_4k_f32"]
    inp = make_inputs(w, seed=0)
    d = _dev(inp)
    ix = lsa.lsa_build_index(TU.build_params(w), d["K"], d["W"])
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    Kls = TU.oracle_latents(inp, w)
    _check_tree_invariants(ix, w, [ix.get(lsa.LSA_GET_LATENT).double().cpu().numpy()[0]], exact=False)
    t = TU.oracle_trees(Kls, w)[0]
    agree = (ix.get(lsa.LSA_GET_LEAF_OF_BLOCK).cpu().numpy()[0] == t.leaf_of_block).mean()
    assert agree >= 0.999
    o = ix.get(lsa.LSA_GET_OBJECTIVE, 0).cpu().numpy()[:, 0]
    assert abs(o[-1] - t.objectives[0][-1]) <= 1e-4 * t.objectives[0][-1]


# ------------------------------------------------------------------ select
def _oracle_select_rows(trees, Kls, inp, w, b, h, rows, full=False, beam=None, topk=None):
    Wm = inp["W"].double().numpy()
    q = O.query_latent(TU.unit_queries(inp["Q"], b, h, w.group, rows), Wm)
    u = b * w.hkv + h
    out = []
    for k, i in enumerate(rows):
        if full:
            blk = O.fullscan_blocks(Kls[u], q[k], int(i), w.topk if topk is None else topk, w.sink, w.window, w.pool)
        else:
            blk = O.select_blocks(trees[u], Kls[u], q[k], int(i), beam or w.beam,
                                  w.topk if topk is None else topk, w.window)
        out.append(O.selection_tokens(blk, int(i), w.sink, w.window, w.pool))
    return out, q


def test_select_integer_workload_bit_exact_end_to_end():
    w = WORKLOADS["int_exact_16k"]
    inp = make_inputs(w, seed=0)
    d = _dev(inp)
    ix = lsa.lsa_build_index(TU.build_params(w), d["K"], d["W"])
    sp = TU.select_params(w)
    idx, cnt = lsa.lsa_select(ix, sp, d["Q"])
    fidx, fcnt = lsa.lsa_fullscan_select(ix, sp, d["Q"])
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    Kls = TU.oracle_latents(inp, w)
    trees = TU.oracle_trees(Kls, w)
    rows = np.arange(w.n_tokens)
    want, _ = _oracle_select_rows(trees, Kls, inp, w, 0, 0, rows)
    got = TU.gpu_rows(idx, cnt, 0, rows, 0)
    bad = [i for i in rows if not np.array_equal(got[i], want[i])]
    assert not bad, f"{len(bad)} rows differ, first {bad[:5]}"
    assert (idx[0, :, 0][torch.arange(w.max_sel, device="cuda")[None, :] >= cnt[0, :, 0][:, None]] == -1).all()
    frows = np.arange(0, w.n_tokens, 7)
    fwant, _ = _oracle_select_rows(trees, Kls, inp, w, 0, 0, frows, full=True)
    fgot = TU.gpu_rows(fidx, fcnt, 0, frows, 0)
    assert all(np.array_equal(a, b) for a, b in zip(fgot, fwant))
    ix.free()


def _float_select_check(w, seed, sample, from_tree=True):
    inp = make_inputs(w, seed=seed)
    d = _dev(inp)
    Kls = TU.oracle_latents(inp, w)
    trees = TU.oracle_trees(Kls, w)
    if from_tree:
        leaf, par, cen = TU.trees_to_device(trees, w)
        ix = lsa.lsa_build_index_from_tree(TU.build_params(w), d["K"], d["W"], leaf, par, cen)
    else:
        ix = lsa.lsa_build_index(TU.build_params(w), d["K"], d["W"])
    sp = TU.select_params(w)
    idx, cnt = lsa.lsa_select(ix, sp, d["Q"])
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([np.arange(0, 40), np.arange(w.n_tokens - 40, w.n_tokens),
                                     rng.integers(0, w.n_tokens, sample)]))
    if not from_tree:
        trees = TU.oracle_trees(Kls, w)
    for b in range(w.batch):
        for h in range(w.hkv):
            u = b * w.hkv + h
            want, q = _oracle_select_rows(trees, Kls, inp, w, b, h, rows)
            got = TU.gpu_rows(idx, cnt, b, rows, h)
            assert TU.recall(got, want) >= 0.999
            for k, i in enumerate(rows):
                assert TU.selection_mismatch_ok(trees[u], Kls[u], q[k], int(i), w.beam, w.topk, w.window,
                                                got[k], want[k]), f"unit {u} query {i}"
    ix.free()
    return idx, cnt


def test_select_flat_4k_end_to_end():
    _float_select_check(WORKLOADS["flat_4k_f32"], seed=0, sample=600, from_tree=False)


def test_select_flat_4k_on_oracle_tree():
    _float_select_check(WORKLOADS["flat_4k_f32"], seed=1, sample=600, from_tree=True)


def test_select_gqa_two_levels_ragged_on_oracle_tree():
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=16384 + 13, level_sizes=(16, 256), needles=8, needle_gap=8000,
                                     components=512)
    _float_select_check(w, seed=2, sample=300)


def test_select_three_levels_ragged_on_oracle_tree():
    w = WORKLOADS["prefill_1m"].scaled(n_tokens=32768 + 5, level_sizes=(4, 32, 256), beam=16, topk=512,
                                       window=256, needles=8, needle_gap=16000, components=1024, drift_every=8192)
    _float_select_check(w, seed=3, sample=200)


def test_select_and_attention_are_deterministic():
    w = WORKLOADS["prefill_1m"].scaled(n_tokens=16384 + 9, level_sizes=(4, 32, 256), beam=16, topk=512,
                                       window=256, needles=0, components=256, drift_every=4096)
    inp = make_inputs(w, seed=21)
    d = _dev(inp)
    ix = lsa.lsa_build_index(TU.build_params(w), d["K"], d["W"])
    sp = TU.select_params(w)
    outs = []
    for _ in range(3):
        idx, cnt = lsa.lsa_select(ix, sp, d["Q"])
        O_, lse = lsa.lsa_sparse_attn(d["Q"], d["K"], d["V"], idx, cnt, w.hkv)
        outs.append((idx.clone(), cnt.clone(), O_.clone(), lse.clone()))
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    for o in outs[1:]:
        assert torch.equal(o[0], outs[0][0]) and torch.equal(o[1], outs[0][1])
        assert torch.equal(o[2], outs[0][2]) and torch.equal(o[3], outs[0][3])
    ix2 = lsa.lsa_build_index(TU.build_params(w), d["K"], d["W"])
    for what in (lsa.LSA_GET_LEAF_OF_BLOCK, lsa.LSA_GET_CENTROIDS):
        assert torch.equal(ix.get(what, 2), ix2.get(what, 2))
    ix.free()
    ix2.free()


def test_full_beam_equals_fullscan_on_gpu():
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=8192 + 3, level_sizes=(8, 64), needles=0, components=256)
    inp = make_inputs(w, seed=4)
    d = _dev(inp)
    ix = lsa.lsa_build_index(TU.build_params(w), d["K"], d["W"])
    sp_all = TU.select_params(w, beam=1024)
    a, ac = lsa.lsa_select(ix, sp_all, d["Q"])
    f, fc = lsa.lsa_fullscan_select(ix, sp_all, d["Q"])
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    assert torch.equal(ac, fc) and torch.equal(a, f)
    ix.free()


# ------------------------------------------------------------------ attention
def _attn_case(w, seed, rows):
    inp = make_inputs(w, seed=seed)
    d = _dev(inp)
    Kls = TU.oracle_latents(inp, w)
    trees = TU.oracle_trees(Kls, w)
    G = w.group
    sels_all = {}
    for h in range(w.hkv):
        sels_all[h], _ = _oracle_select_rows(trees, Kls, inp, w, 0, h, rows)
    idx = torch.full((1, len(rows), w.hkv, w.max_sel), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros((1, len(rows), w.hkv), dtype=torch.int32, device="cuda")
    for h in range(w.hkv):
        ii, cc = TU.rows_to_idx(sels_all[h], w.max_sel)
        idx[0, :, h] = ii
        cnt[0, :, h] = cc
    Qs = d["Q"][:, torch.as_tensor(rows, device="cuda")].contiguous()
    O_, lse = lsa.lsa_sparse_attn(Qs, d["K"], d["V"], idx, cnt, w.hkv)
    _assert_clean()
    Kn = inp["K"][0].float().numpy().astype(np.float64)
    Vn = inp["V"][0].float().numpy().astype(np.float64)
    errs, lerr, ulps = [], [], []
    for h in range(w.hkv):
        for k, i in enumerate(rows):
            q = TU.unit_queries(inp["Q"], 0, h, G, [i])[0]
            o, l = O.sparse_attention(q, Kn[:, h], Vn[:, h], sels_all[h][k])
            got = O_[0, k, h * G:(h + 1) * G].double().cpu().numpy()
            errs.append(np.abs(got - o))
            # one bf16 ulp of the oracle value: 2^(floor(log2|o|) - 7)
            ulps.append(np.exp2(np.floor(np.log2(np.maximum(np.abs(o), 1e-30))) - 7))
            lerr.append(np.abs(lse[0, k, h * G:(h + 1) * G].double().cpu().numpy() - l))
    e = np.concatenate([x.ravel() for x in errs])
    le = np.concatenate(lerr)
    return e, le, np.concatenate([x.ravel() for x in ulps])


@pytest.mark.parametrize("name,over", [
    ("flat_4k_f32", {}),
    ("int_exact_16k", {"n_tokens": 4096 + 3}),
    ("gqa_128k", {"n_tokens": 8192 + 1, "level_sizes": (8, 64), "needles": 0, "components": 256}),
    ("decode_10m_x4", {"n_tokens": 8192 + 2, "batch": 1, "level_sizes": (4, 16, 64), "needles": 0,
                       "components": 256, "decode_steps": 0}),
])
def test_attention_on_oracle_index_sets(name, over):
    w = WORKLOADS[name].scaled(**over)
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, 1, 2, w.sink + w.window + w.pool], rng.integers(0, w.n_tokens, 120),
                                     [w.n_tokens - 1]]))
    e, le, ulp = _attn_case(w, 5, rows)
    if w.dtype == "f32":
        assert e.max() <= 1e-4 and le.max() <= 1e-4
    elif w.kind == "int":
        # |O| reaches 4 here, so the bf16 output rounding alone exceeds the
        # float workloads' mean-abs bound: compare within one bf16 ulp of the
        # oracle value (plus fp32 accumulation slack) instead
        assert np.all(e <= ulp + 1e-3) and e.max() <= BF16_MAX_ABS
        assert le.max() <= 1e-2
    else:
        assert e.max() <= BF16_MAX_ABS and e.mean() <= BF16_MEAN_ABS
        assert le.max() <= 1e-2


def test_attention_select_everything_is_dense_causal():
    # pool 1 and K >= N: every earlier token is selected, so the result is
    # dense causal attention
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=300, pool=1, level_sizes=(2, 8), topk=4096, sink=4, window=8,
                                     needles=0, components=16)
    inp = make_inputs(w, seed=6)
    d = _dev(inp)
    ix = lsa.lsa_build_index(TU.build_params(w), d["K"], d["W"])
    idx, cnt = lsa.lsa_select(ix, TU.select_params(w, beam=1024), d["Q"])
    O_, lse = lsa.lsa_sparse_attn(d["Q"], d["K"], d["V"], idx, cnt, w.hkv)
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    Kn = inp["K"][0].float().double().numpy()
    Vn = inp["V"][0].float().double().numpy()
    for i in [0, 5, 50, 299]:
        for h in range(w.hkv):
            assert idx[0, i, h, : cnt[0, i, h]].tolist() == list(range(i + 1))
            q = TU.unit_queries(inp["Q"], 0, h, w.group, [i])[0]
            s = q @ Kn[: i + 1, h].T / math.sqrt(w.d)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            dense = (p @ Vn[: i + 1, h]) / p.sum(axis=1, keepdims=True)
            got = O_[0, i, h * w.group:(h + 1) * w.group].double().cpu().numpy()
            assert np.abs(got - dense).max() <= BF16_MAX_ABS
    ix.free()


# ------------------------------------------------------------------ decode
def test_append_matches_oracle_and_selects():
    w = WORKLOADS["decode_10m_x4"].scaled(n_tokens=8192, batch=2, level_sizes=(4, 16, 64), needles=0,
                                          components=256, decode_steps=40, window=8, topk=256, sink=8, beam=8)
    inp = make_inputs(w, seed=7)
    d = _dev(inp)
    Kls = TU.oracle_latents(inp, w)
    trees = TU.oracle_trees(Kls, w)
    leaf, par, cen = TU.trees_to_device(trees, w)
    ix = lsa.lsa_build_index_from_tree(TU.build_params(w, append_capacity=w.decode_steps), d["K"], d["W"],
                                       leaf, par, cen)
    Wm = inp["W"].double().numpy()
    rows = [list(k) for k in Kls]
    sp = TU.select_params(w)
    for step in range(w.decode_steps):
        lsa.lsa_append(ix, d["K"], 1)
        t = w.n_tokens + step
        if (t + 1) % w.pool == 0:
            for b in range(w.batch):
                x = O.project_pool(TU.unit_keys(inp["K"], b, 0, t + 1)[t + 1 - w.pool:], Wm, w.pool)[0]
                O.append_block(trees[b], rows[b], x)
        q = d["Q"][:, step:step + 1].contiguous()
        idx, cnt = lsa.lsa_select(ix, sp, q, q_pos0=t)
        for b in range(w.batch):
            qb = O.query_latent(TU.unit_queries(inp["Q"], b, 0, w.group, [step]), Wm)[0]
            Klb = np.array(rows[b])
            blk = O.select_blocks(trees[b], Klb, qb, t, w.beam, w.topk, w.window)
            want = O.selection_tokens(blk, t, w.sink, w.window, w.pool)
            got = idx[b, 0, 0, : cnt[b, 0, 0]].cpu().numpy()
            assert TU.selection_mismatch_ok(trees[b], Klb, qb, t, w.beam, w.topk, w.window, got, want)
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    # every appended block: the oracle's nearest leaf, or a near tie (fp64
    # distances on the oracle's values within 1e-4 relative of the nearest)
    got_leaf = ix.get(lsa.LSA_GET_LEAF_OF_BLOCK).cpu().numpy()
    for b in range(w.batch):
        want = trees[b].leaf_of_block
        assert got_leaf[b].shape == want.shape
        Cl = trees[b].centroids[-1]
        X = np.array(rows[b])
        for blk in np.flatnonzero(got_leaf[b] != want):
            dg = ((X[blk] - Cl[got_leaf[b][blk]]) ** 2).sum()
            dw = ((X[blk] - Cl[want[blk]]) ** 2).sum()
            assert dg - dw <= 1e-4 * dw, f"sequence {b} block {blk}"
    ix.free()


# ------------------------------------------------------------------ edges
def test_edge_cases_and_errors():
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=2048 + 3, level_sizes=(4, 32), needles=0, components=64)
    inp = make_inputs(w, seed=8)
    d = _dev(inp)
    ix = lsa.lsa_build_index(TU.build_params(w), d["K"], d["W"])
    sp = TU.select_params(w)
    # no queries
    e_idx, e_cnt = lsa.lsa_select(ix, sp, d["Q"][:, :0].contiguous())
    assert e_idx.numel() == 0
    # queries before any candidate exists: sink + window only
    idx, cnt = lsa.lsa_select(ix, sp, d["Q"][:, :16].contiguous())
    for i in range(16):
        assert idx[0, i, 0, : cnt[0, i, 0]].tolist() == list(range(i + 1))
    # topk = 0
    idx, cnt = lsa.lsa_select(ix, TU.select_params(w, topk=0), d["Q"])
    i = w.n_tokens - 1
    lo = i - w.window + 1
    assert idx[0, i, 1, : cnt[0, i, 1]].tolist() == list(range(w.sink)) + list(range(lo, i + 1))
    # bad arguments are refused before anything runs
    with pytest.raises(lsa.LsaError) as ei:
        lsa.lsa_select(ix, sp, d["Q"], max_sel=10)
    assert ei.value.status == lsa.LSA_ERR_INVALID_ARG
    with pytest.raises(lsa.LsaError):
        lsa.lsa_select(ix, lsa.make_select_params(w.hq, w.beam, w.topk, w.sink + 1, w.window), d["Q"])
    st = lsa.lib().lsa_sparse_attn(None, None, None, None, None, 1, 1, 1, 1, 128, 1, 8, 8, None, None, None)
    assert st == lsa.LSA_ERR_INVALID_ARG
    # out-of-range rows are skipped and reported
    idx2, cnt2 = lsa.lsa_select(ix, sp, d["Q"][:, :64].contiguous())
    idx2[0, 3, 0, 0] = 10 ** 8
    O_, _ = lsa.lsa_sparse_attn(d["Q"][:, :64].contiguous(), d["K"], d["V"], idx2, cnt2, w.hkv)
    assert lsa.lsa_check(None) == lsa.LSA_ERR_DEVICE
    assert torch.isfinite(O_.float()).all()
    assert lsa.lsa_check(None) == lsa.LSA_OK
    # allocation failure: reported, and nothing leaked (repeating the failing
    # builds does not lower free memory; freed blocks stay in the pool)
    frees = []
    for _ in range(3):
        for n in (1, 3, 9, 21, 30, 40, 46):
            lsa.lsa_debug_fail_alloc_after(n)
            with pytest.raises(lsa.LsaError) as ei:
                lsa.lsa_build_index(TU.build_params(w), d["K"], d["W"])
            assert ei.value.status == lsa.LSA_ERR_OOM
        lsa.lsa_debug_fail_alloc_after(0)
        torch.cuda.synchronize()
        frees.append(torch.cuda.mem_get_info()[0])
    assert abs(frees[2] - frees[1]) < (16 << 20)
    ok = lsa.lsa_build_index(TU.build_params(w), d["K"], d["W"])
    assert lsa.lsa_check(ok) == lsa.LSA_OK
    ok.free()
    # double free is harmless
    h = ix.handle
    ix.free()
    lsa.lib().lsa_free_index(h)


def test_append_capacity_error_is_latched():
    w = WORKLOADS["flat_4k_f32"].scaled(decode_steps=64)
    inp = make_inputs(w, seed=9)
    K = inp["K"].clone()
    K[0, w.n_tokens:] = K[0, 100]  # every appended key is the same: one leaf takes them all
    K = K.cuda()
    ix = lsa.lsa_build_index(TU.build_params(w, append_capacity=64), K, inp["W"].cuda())
    lsa.lsa_append(ix, K, 64)
    assert lsa.lsa_check(ix) == lsa.LSA_ERR_CAPACITY
    ix.free()


def test_select_work_counts_scored_rows():
    """lsa_select_work returns lsa_select's rows and counts the eligible nodes
    and blocks it scored.  With a beam wider than every level the tree search
    scores every eligible node of every level and every candidate block, so
    the count has a closed form from the index's minpos and the positions."""
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=4096 + 5, level_sizes=(8, 64), needles=0, components=64)
    inp = make_inputs(w, seed=12, device="cuda")
    ix = lsa.lsa_build_index(TU.build_params(w), inp["K"], inp["W"])
    sp = TU.select_params(w, beam=1024)
    i1, c1 = lsa.lsa_select(ix, sp, inp["Q"])
    i2, c2, nodes, blocks = lsa.lsa_select_work(ix, sp, inp["Q"])
    assert torch.equal(i1, i2) and torch.equal(c1, c2)
    pos = np.arange(w.n_tokens, dtype=np.int64)
    bound = pos - w.window - w.pool + 1
    want_nodes = 0
    for lvl in range(len(w.level_sizes)):
        mp = ix.get(lsa.LSA_GET_MINPOS, lvl).cpu().numpy()          # [units][n_l]
        for u in range(mp.shape[0]):
            srt = np.sort(mp[u])
            want_nodes += int(np.searchsorted(srt, bound, side="right").sum())
    b_lo = -(-w.sink // w.pool)
    b_hi = np.where(bound >= 0, bound // w.pool, -1)
    nblk = np.maximum(0, np.minimum(b_hi, w.n_tokens // w.pool - 1) - b_lo + 1)
    assert nodes == want_nodes
    assert blocks == int(nblk.sum()) * w.hkv
    # the narrow beam of the workload scores fewer rows of both kinds
    _, _, n2, b2 = lsa.lsa_select_work(ix, TU.select_params(w), inp["Q"])
    assert 0 < n2 <= nodes and 0 < b2 <= blocks
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    ix.free()

