"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: hand-worked
examples under tests/golden/ (derivations stored beside the values), closed
forms, invariants of the method, and brute force on tiny inputs.  CPU only.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- latent map
def test_project_pool_worked_example():
    g = gold("latent_small.json")
    Kl = O.project_pool(np.array(g["K"]), np.array(g["W"]), g["pool"])
    np.testing.assert_array_equal(Kl, np.array(g["Kl"], dtype=np.float64))
    qb = O.query_latent(np.array(g["Qg"]), np.array(g["W"]))
    np.testing.assert_array_equal(qb, np.array(g["qbar"], dtype=np.float64))


def test_project_identity_map_and_pooling_closed_form():
    rng = np.random.default_rng(1)
    K = rng.standard_normal((37, 8))
    # W = I with pool 1 leaves the keys unchanged.
    np.testing.assert_array_equal(O.project_pool(K, np.eye(8), 1), K)
    # pool 4 with W = I is the running mean of each complete run of 4 keys.
    Kl = O.project_pool(K, np.eye(8), 4)
    assert Kl.shape == (9, 8)
    for b in range(9):
        np.testing.assert_allclose(Kl[b], sum(K[4 * b + t] for t in range(4)) / 4, rtol=0, atol=1e-14)


def test_query_latent_single_head_and_permutation():
    rng = np.random.default_rng(2)
    Q = rng.standard_normal((5, 3, 6))
    W = rng.standard_normal((6, 2))
    # G = 1: the latent query is q W.
    np.testing.assert_allclose(O.query_latent(Q[:, :1], W), Q[:, 0] @ W, atol=1e-13)
    # the group mean does not depend on the order of the heads.
    np.testing.assert_allclose(O.query_latent(Q[:, ::-1], W), O.query_latent(Q, W), atol=1e-13)


# ---------------------------------------------------------------- k-means
@pytest.mark.parametrize("case", gold("kmeans_small.json")["cases"])
def test_kmeans_worked_examples(case):
    res = O.kmeans(np.array(case["points"], dtype=np.float64), case["k"], case["iters"])
    np.testing.assert_array_equal(res.labels, case["labels"])
    np.testing.assert_allclose(res.centroids, case["centroids"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(res.objectives, case["objectives"], rtol=0, atol=1e-12)


@pytest.mark.parametrize("case", gold("grid_rounding.json")["cases"])
def test_grid_rounding_worked_examples(case):
    g = gold("grid_rounding.json")["grid_log2"]
    res = O.kmeans(np.array(case["points"], dtype=np.float64), 1, 1, grid_log2=g)
    np.testing.assert_array_equal(res.centroids[0], np.array(case["centroid"]))


def test_kmeans_single_cluster_is_the_mean():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((50, 4)) * 3 + 1
    res = O.kmeans(X, 1, 2)
    np.testing.assert_allclose(res.centroids[0], X.mean(axis=0), atol=1e-13)
    assert np.all(res.labels == 0)
    # the first assign uses the init point x[0]; the second uses the mean
    np.testing.assert_allclose(res.objectives[0], ((X - X[0]) ** 2).sum(), rtol=1e-12)
    np.testing.assert_allclose(res.objectives[1], X.shape[0] * X.var(axis=0).sum(), rtol=1e-12)


def test_assign_matches_direct_difference_brute_force():
    rng = np.random.default_rng(4)
    X = rng.standard_normal((40, 5))
    C = rng.standard_normal((7, 5))
    lab, obj = O.kmeans_assign(X, C)
    tot = 0.0
    for i in range(40):
        best, bj = math.inf, -1
        for j in range(7):
            d = sum((X[i, t] - C[j, t]) ** 2 for t in range(5))
            if d < best:
                best, bj = d, j
        assert lab[i] == bj
        tot += best
    assert abs(obj - tot) < 1e-9


@pytest.mark.parametrize("grid", [0, 4])
def test_kmeans_objective_non_increasing_and_partition(grid):
    rng = np.random.default_rng(5 + grid)
    if grid:
        X = rng.integers(-20, 21, size=(300, 6)).astype(np.float64)
    else:
        X = rng.standard_normal((300, 6))
        X[:100] += 4
    res = O.kmeans(X, 9, 8, grid_log2=grid)
    obj = np.array(res.objectives)
    if grid:
        assert np.all(np.diff(obj) <= 0)  # exact arithmetic: strictly monotone or equal
        assert np.all(res.centroids * 16 == np.round(res.centroids * 16))
    else:
        assert np.all(np.diff(obj) <= 1e-9 * obj[0])
    assert res.labels.shape == (300,) and res.labels.min() >= 0 and res.labels.max() < 9


def test_kmeans_converged_fixed_point():
    rng = np.random.default_rng(6)
    X = np.concatenate([rng.standard_normal((40, 3)) + c for c in ([0, 0, 0], [6, 0, 0], [0, 6, 0])])
    res = O.kmeans(X, 3, 30)
    # at a Lloyd fixed point every point sits at its nearest centroid and
    # every non-empty centroid is the mean of its points
    lab2, _ = O.kmeans_assign(X, res.centroids)
    np.testing.assert_array_equal(lab2, res.labels)
    for j in range(3):
        np.testing.assert_allclose(res.centroids[j], X[res.labels == j].mean(axis=0), atol=1e-12)


def test_grid_mode_rejects_off_grid_points():
    with pytest.raises(ValueError):
        O.kmeans(np.array([[0.01], [1.0]]), 1, 1, grid_log2=4)


# ---------------------------------------------------------------- tree
def _random_tree(seed, nb=200, r=4, sizes=(3, 12), pool=2, sink=4, iters=4, grid=0):
    rng = np.random.default_rng(seed)
    Kl = rng.standard_normal((nb, r)) if not grid else rng.integers(-9, 10, size=(nb, r)).astype(float)
    return Kl, O.build_tree(Kl, sizes, iters, grid, sink, pool)


def test_tree_partition_and_minpos_brute_force():
    Kl, t = _random_tree(7)
    seen = np.concatenate(t.members)
    assert sorted(seen.tolist()) == list(range(Kl.shape[0]))  # each block in exactly one leaf
    for j, mem in enumerate(t.members):
        assert np.all(np.diff(mem) > 0)
        assert np.all(t.leaf_of_block[mem] == j)
    kids = np.concatenate(t.children[0])
    assert sorted(kids.tolist()) == list(range(t.level_sizes[1]))
    for j in range(t.level_sizes[1]):
        starts = [b * t.pool for b in t.members[j] if b * t.pool >= t.sink]
        assert t.minpos[1][j] == (min(starts) if starts else math.inf)
    for j in range(t.level_sizes[0]):
        vals = [t.minpos[1][c] for c in t.children[0][j]]
        assert t.minpos[0][j] == (min(vals) if vals else math.inf)
    # leaf centroids are the means of their buckets (last update of the last assign)
    for j, mem in enumerate(t.members):
        if mem.size:
            np.testing.assert_allclose(t.centroids[1][j], Kl[mem].mean(axis=0), atol=1e-12)


def _minpos_list(v):
    return np.array([math.inf if x == "inf" else float(x) for x in v])


@pytest.mark.parametrize("case", gold("tree_small.json")["builds"])
def test_build_tree_upper_levels_worked_examples(case):
    """Hand-worked two-level builds: the leaf clustering, then the clustering
    of the leaf centroids (unweighted, stride init over the leaf ids), the
    parents, the centroids and objectives of both levels, and minpos."""
    X = np.array(case["latents"], dtype=np.float64)[:, None]
    t = O.build_tree(X, case["level_sizes"], case["iters"], 0, case["sink"], case["pool"])
    np.testing.assert_array_equal(t.leaf_of_block, case["leaf_of_block"])
    np.testing.assert_array_equal(t.centroids[1][:, 0], case["leaf_centroids"])
    np.testing.assert_array_equal(t.objectives[1], case["leaf_objectives"])
    np.testing.assert_array_equal(t.parent[1], case["parent_of_leaf"])
    np.testing.assert_array_equal(t.centroids[0][:, 0], case["top_centroids"])
    np.testing.assert_array_equal(t.objectives[0], case["top_objectives"])
    np.testing.assert_array_equal(t.minpos[1], _minpos_list(case["minpos_leaf"]))
    np.testing.assert_array_equal(t.minpos[0], _minpos_list(case["minpos_top"]))


@pytest.mark.parametrize("case", gold("tree_small.json")["minpos_trees"])
def test_minpos_worked_examples(case):
    """minpos on given trees: blocks before the sink and empty leaves count as
    +inf, and each upper node takes the minimum over its children."""
    L = len(case["level_sizes"])
    parent = [None] * L
    parent[L - 1] = np.array(case["parent_of_leaf"])
    if L == 3:
        parent[1] = np.array(case["parent_of_mid"])
    cents = [np.zeros((n, 1)) for n in case["level_sizes"]]
    t = O.Tree(case["pool"], case["sink"], case["level_sizes"], cents, parent, np.array(case["leaf_of_block"]),
               [[]] * L).finish()
    np.testing.assert_array_equal(t.minpos[L - 1], _minpos_list(case["minpos_leaf"]))
    np.testing.assert_array_equal(t.minpos[0], _minpos_list(case["minpos_top"]))
    if L == 3:
        np.testing.assert_array_equal(t.minpos[1], _minpos_list(case["minpos_mid"]))


def _tree_from_gold(g):
    tr = g["tree"]
    return O.Tree(tr["pool"], tr["sink"], tr["level_sizes"],
                  [np.array(c, dtype=np.float64) for c in tr["centroids"]],
                  [None, np.array(tr["parent_of_leaf"])],
                  np.array(tr["leaf_of_block"]), [[], []]).finish()


@pytest.mark.parametrize("case", gold("select_small.json")["cases"])
def test_select_worked_examples(case):
    g = gold("select_small.json")
    t = _tree_from_gold(g)
    Kl = np.array(g["Kl"], dtype=np.float64)
    q = np.array(case["q"], dtype=np.float64)
    W = g["window"]
    if "tree_tokens" in case:
        b = O.select_blocks(t, Kl, q, case["i"], case["beam"], case["topk"], W)
        toks = O.selection_tokens(b, case["i"], t.sink, W, t.pool)
        assert toks.tolist() == case["tree_tokens"]
    if "fullscan_tokens" in case:
        b = O.fullscan_blocks(Kl, q, case["i"], case["topk"], t.sink, W, t.pool)
        toks = O.selection_tokens(b, case["i"], t.sink, W, t.pool)
        assert toks.tolist() == case["fullscan_tokens"]


@pytest.mark.parametrize("case", gold("latent_small.json")["fullscan_pool2"]["cases"])
def test_fullscan_pooled_worked_example(case):
    g = gold("latent_small.json")["fullscan_pool2"]
    b = O.fullscan_blocks(np.array(g["Kl"], float), np.array(g["q"], float), g["i"], case["topk"],
                          g["sink"], g["window"], g["pool"])
    assert O.selection_tokens(b, g["i"], g["sink"], g["window"], g["pool"]).tolist() == case["tokens"]


@pytest.mark.parametrize("seed,pool,sink,window", [(8, 1, 1, 4), (9, 2, 4, 6), (10, 4, 8, 8)])
def test_full_beam_equals_fullscan(seed, pool, sink, window):
    Kl, t = _random_tree(seed, pool=pool, sink=sink)
    rng = np.random.default_rng(seed + 100)
    N = Kl.shape[0] * pool
    for i in list(range(0, 40)) + list(rng.integers(0, N, 30)):
        q = rng.standard_normal(Kl.shape[1])
        for topk in (1, 5, 17):
            a = O.select_blocks(t, Kl, q, int(i), 10 ** 6, topk, window)
            b = O.fullscan_blocks(Kl, q, int(i), topk, sink, window, pool)
            assert a.tolist() == b.tolist()


def test_fullscan_identity_map_is_textbook_topk():
    rng = np.random.default_rng(11)
    N, d, S, Wn, K = 64, 8, 3, 5, 7
    Kx = rng.standard_normal((N, d))
    Kl = O.project_pool(Kx, np.eye(d), 1)
    for i in range(N):
        q = rng.standard_normal(d)
        got = O.fullscan_blocks(Kl, q, i, K, S, Wn, 1)
        elig = np.arange(S, max(S, i - Wn + 1))
        sc = Kx[elig] @ q
        want = np.sort(elig[np.argsort(-sc, kind="stable")[:K]])
        assert got.tolist() == want.tolist()


def test_selection_set_properties():
    Kl, t = _random_tree(12, pool=4, sink=8)
    rng = np.random.default_rng(13)
    N = Kl.shape[0] * 4
    S, Wn, K = 8, 12, 20
    for i in range(N):
        q = rng.standard_normal(Kl.shape[1])
        b = O.select_blocks(t, Kl, q, i, 3, K, Wn)
        s = O.selection_tokens(b, i, S, Wn, 4)
        assert np.all(np.diff(s) > 0) and s.max() == i and s.min() == 0
        assert set(range(min(S, i + 1))) <= set(s.tolist())
        assert set(range(max(0, i - Wn + 1), i + 1)) <= set(s.tolist())
        assert b.size <= O.blocks_per_topk(K, 4)
        # disjoint union: the count is known in closed form
        lo = max(0, i - Wn + 1)
        assert s.size == min(S, lo) + (i - lo + 1) + 4 * b.size


def test_beam_restricts_to_children_of_kept_nodes():
    Kl, t = _random_tree(14, nb=300, sizes=(4, 16))
    rng = np.random.default_rng(15)
    i = 300 * 2 - 1
    bound = O.candidate_bound(i, 6, t.pool)
    for _ in range(20):
        q = rng.standard_normal(Kl.shape[1])
        leaves = O.beam_search(t, q, i, 2, 6)
        top_scores = t.centroids[0] @ q
        elig_top = np.flatnonzero(t.minpos[0] <= bound)
        kept_top = elig_top[np.lexsort((elig_top, -top_scores[elig_top]))[:2]]
        allowed = np.concatenate([t.children[0][j] for j in kept_top])
        allowed = allowed[t.minpos[1][allowed] <= bound]
        assert set(leaves.tolist()) <= set(allowed.tolist())
        assert leaves.size == min(2, allowed.size)
        # the kept leaves outscore every other allowed leaf
        sc = t.centroids[1] @ q
        rest = np.setdiff1d(allowed, leaves)
        if rest.size and leaves.size:
            assert sc[leaves].min() >= sc[rest].max()


# ---------------------------------------------------------------- attention
@pytest.mark.parametrize("case", gold("attention_small.json")["cases"])
def test_attention_worked_example(case):
    g = gold("attention_small.json")
    o, lse = O.sparse_attention(np.array(g["q"], float), np.array(g["K"], float),
                                np.array(g["V"], float), np.array(case["sel"]))
    np.testing.assert_allclose(o, case["O"], atol=1e-12)
    np.testing.assert_allclose(lse, case["lse"], atol=1e-12)


def test_select_everything_equals_dense_causal_attention():
    rng = np.random.default_rng(16)
    N, d, G, r = 24, 4, 2, 3
    Q = rng.standard_normal((N, G, d))
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    Wm = rng.standard_normal((d, r))
    Kl = O.project_pool(K, Wm, 1)
    t = O.build_tree(Kl, [2, 4], 3, 0, 1, 1)
    qb = O.query_latent(Q, Wm)
    for i in range(N):
        b = O.select_blocks(t, Kl, qb[i], i, 4, N, 3)  # K >= N selects every candidate
        sel = O.selection_tokens(b, i, 1, 3, 1)
        assert sel.tolist() == list(range(i + 1))
        o, lse = O.sparse_attention(Q[i], K, V, sel)
        for h in range(G):
            w = [math.exp(sum(Q[i, h, t] * K[j, t] for t in range(d)) / math.sqrt(d)) for j in range(i + 1)]
            z = sum(w)
            ref = [sum(w[j] * V[j, t] for j in range(i + 1)) / z for t in range(d)]
            np.testing.assert_allclose(o[h], ref, rtol=1e-12, atol=1e-12)
            assert abs(lse[h] - math.log(z)) < 1e-12


def test_attention_single_key_and_uniform_scores():
    rng = np.random.default_rng(17)
    K = rng.standard_normal((10, 8))
    V = rng.standard_normal((10, 8))
    o, lse = O.sparse_attention(rng.standard_normal((3, 8)), K, V, np.array([4]))
    np.testing.assert_allclose(o, np.repeat(V[4:5], 3, axis=0), atol=1e-14)
    o, lse = O.sparse_attention(np.zeros((1, 8)), K, V, np.array([1, 3, 7]))
    np.testing.assert_allclose(o[0], V[[1, 3, 7]].mean(axis=0), atol=1e-14)
    assert abs(lse[0] - math.log(3)) < 1e-14


# ---------------------------------------------------------------- decode
def test_append_block_by_block_equals_one_assign_pass():
    rng = np.random.default_rng(18)
    Kl0 = rng.standard_normal((120, 4))
    t = O.build_tree(Kl0, [3, 9], 4, 0, 8, 2)
    new = rng.standard_normal((40, 4))
    rows = list(Kl0)
    labs = [O.append_block(t, rows, x) for x in new]
    want, _ = O.kmeans_assign(new, t.centroids[-1])
    assert labs == want.tolist()
    # the appended tree equals a tree made from the same labels directly
    full = O.Tree(t.pool, t.sink, t.level_sizes, t.centroids, t.parent,
                  np.concatenate([O.build_tree(Kl0, [3, 9], 4, 0, 8, 2).leaf_of_block, want]),
                  t.objectives).finish()
    for l in range(2):
        np.testing.assert_array_equal(full.minpos[l], t.minpos[l])
    for a, b in zip(full.members, t.members):
        assert a.tolist() == b.tolist()


def test_integer_workload_stays_exact():
    # integer keys, a {-1,0,1} map and the 1/16 grid: every latent, centroid
    # and score is a small multiple of a power of two, so float64 is exact.
    rng = np.random.default_rng(19)
    d, r, N = 16, 4, 400
    Kx = rng.integers(-4, 5, size=(N, d)).astype(float)
    Wm = np.zeros((d, r))
    for row in range(d):
        cols = rng.choice(r, 2, replace=False)
        Wm[row, cols] = rng.choice([-1.0, 1.0], 2)
    Kl = O.project_pool(Kx, Wm, 1)
    assert np.all(Kl == np.round(Kl))
    t = O.build_tree(Kl, [3, 8], 5, 4, 2, 1)
    for C in t.centroids:
        assert np.all(C * 16 == np.round(C * 16))
    Qx = rng.integers(-4, 5, size=(N, 4, d)).astype(float)
    qb = O.query_latent(Qx, Wm)
    assert np.all(qb * 4 == np.round(qb * 4))
    s = t.centroids[1] @ qb.T
    assert np.all(s * 64 == np.round(s * 64)) and np.abs(s).max() < 2 ** 20


# ---------------------------------------------------------------- PCA map (R17)
def test_pca_map_axes_closed_form():
    """Pooled keys +-a_k e_k (k = 0, 1, 2) plus two zero rows: mean 0, covariance
    diag(2 a_k^2 / n), so the map is the axes in order of a_k and the
    eigenvalues are those variances."""
    d, a = 6, [3.0, 1.0, 2.0]
    rows = [np.zeros(d), np.zeros(d)]
    for k, ak in enumerate(a):
        e = np.zeros(d)
        e[k] = ak
        rows += [e, -e]
    K = np.array(rows)
    n = K.shape[0]
    W, ev = O.pca_map([K], pool=1, r=3)
    assert np.allclose(ev, [2 * 9 / n, 2 * 4 / n, 2 * 1 / n])
    assert np.allclose(W[:, 0], np.eye(d)[0]) and np.allclose(W[:, 1], np.eye(d)[2])
    assert np.allclose(W[:, 2], np.eye(d)[1])


def test_pca_map_pools_before_the_covariance():
    """Keys alternate +v, -v inside every block of 2: pooling cancels v, so
    with pool 2 the map ignores v; with pool 1 v is the leading direction."""
    rng = np.random.default_rng(3)
    d, n = 5, 400
    v = np.zeros(d)
    v[4] = 10.0
    base = rng.normal(size=(n // 2, d)) * np.array([1.0, 0.5, 0.25, 0.1, 0.0])
    K = np.repeat(base, 2, axis=0)
    K[0::2] += v
    K[1::2] -= v
    W1, _ = O.pca_map([K], pool=1, r=1)
    W2, _ = O.pca_map([K], pool=2, r=2)
    assert abs(W1[4, 0]) > 0.99
    assert np.all(np.abs(W2[4, :]) < 1e-9)


def test_pca_map_invariants_and_sign():
    rng = np.random.default_rng(4)
    Ks = [rng.normal(size=(64, 8)) @ rng.normal(size=(8, 8)) for _ in range(3)]
    W, ev = O.pca_map(Ks, pool=4, r=5)
    assert np.allclose(W.T @ W, np.eye(5), atol=1e-12)
    assert np.all(np.diff(ev) <= 0)
    for c in range(5):
        j = int(np.argmax(np.abs(W[:, c])))
        assert W[j, c] > 0
    # the same sample in another order (units swapped) gives the same map
    W2, ev2 = O.pca_map(Ks[::-1], pool=4, r=5)
    assert np.allclose(W, W2) and np.allclose(ev, ev2)


def test_pca_map_is_centred():
    """Adding one large constant vector to every key moves the mean only: the
    centred covariance, and so the map, do not change (an uncentred second
    moment would put the constant direction first)."""
    rng = np.random.default_rng(5)
    K = rng.normal(size=(256, 6)) * np.array([3.0, 2.0, 1.5, 1.0, 0.5, 0.25])
    W0, ev0 = O.pca_map([K], pool=1, r=3)
    shift = np.array([0.0, 0.0, 0.0, 0.0, 0.0, 50.0])
    W1, ev1 = O.pca_map([K + shift], pool=1, r=3)
    assert np.allclose(W0, W1, atol=1e-9) and np.allclose(ev0, ev1)


# ---------------------------------------------------------------- decode upkeep
def _given_tree(case):
    """A tree written out by hand (pool 1, sink 0, levels [2, 3])."""
    t = O.Tree(pool=1, sink=0, level_sizes=[2, 3],
               centroids=[np.array(case["top_centroids"], dtype=np.float64)[:, None],
                          np.array(case["leaf_centroids"], dtype=np.float64)[:, None]],
               parent=[None, np.array([0, 1, 1])],
               leaf_of_block=np.array(case["leaf_of_block"]), objectives=[[], []])
    return t.finish()


@pytest.mark.parametrize("case", gold("refresh_small.json")["cases"])
def test_refresh_centroids_worked_examples(case):
    t = _given_tree(case)
    rows = [np.array([x]) for x in case["latents"]]
    for x, want_leaf in zip(case["append"], case["append_leaf"]):
        assert O.append_block(t, rows, np.array([x])) == want_leaf
    O.refresh_centroids(t, np.array(rows), case["grid_log2"])
    np.testing.assert_array_equal(t.centroids[1][:, 0], case["want_leaf_centroids"])
    np.testing.assert_array_equal(t.centroids[0][:, 0], case["want_top_centroids"])


@pytest.mark.parametrize("grid_log2", [0, 4])
def test_refresh_right_after_a_build_changes_nothing(grid_log2):
    """R10 makes every built centroid the last update of its level, i.e. the
    mean of its current members, so a refresh with no append is the identity."""
    rng = np.random.default_rng(40)
    X = rng.integers(-4, 5, size=(300, 3)).astype(np.float64) if grid_log2 else rng.standard_normal((300, 3))
    t = O.build_tree(X, [3, 9, 27], 4, grid_log2, sink=0, pool=1)
    before = [c.copy() for c in t.centroids]
    O.refresh_centroids(t, X, grid_log2)
    for a, b in zip(before, t.centroids):
        np.testing.assert_array_equal(a, b)


def test_refresh_makes_each_centroid_the_mean_of_its_members():
    """After appends, a refreshed leaf centroid has zero summed offset to its
    members (the stationarity condition of the squared loss), an upper node's
    to its children's centroids, and an empty node is unchanged."""
    rng = np.random.default_rng(41)
    X = rng.standard_normal((200, 4))
    t = O.build_tree(X, [2, 6, 40], 3, 0, sink=0, pool=1)
    rows = [x for x in X]
    for x in rng.standard_normal((60, 4)) * 2.0:
        O.append_block(t, rows, x)
    old = [c.copy() for c in t.centroids]
    O.refresh_centroids(t, np.array(rows), 0)
    Kl = np.array(rows)
    for j in range(t.level_sizes[-1]):
        mem = np.flatnonzero(t.leaf_of_block == j)
        if mem.size:
            assert np.abs((Kl[mem] - t.centroids[-1][j]).sum(axis=0)).max() <= 1e-12 * mem.size
        else:
            np.testing.assert_array_equal(t.centroids[-1][j], old[-1][j])
    for l in range(t.levels - 1):
        for j in range(t.level_sizes[l]):
            ch = np.flatnonzero(t.parent[l + 1] == j)
            if ch.size:
                assert np.abs((t.centroids[l + 1][ch] - t.centroids[l][j]).sum(axis=0)).max() <= 1e-12 * ch.size
            else:
                np.testing.assert_array_equal(t.centroids[l][j], old[l][j])
    # the appended blocks moved some leaf: the refresh did something
    assert any(not np.array_equal(a, b) for a, b in zip(old, t.centroids))


# ------------------------------------------------------- context parallelism
def test_shard_ranges_worked_examples():
    # 5 blocks of 2 over 3 shards: 2, 2, 1 blocks
    assert O.shard_ranges(10, 3, 2) == [(0, 4), (4, 8), (8, 10)]
    # 2 whole blocks of 4 over 2 shards; the last shard keeps the 3 trailing tokens
    assert O.shard_ranges(11, 2, 4) == [(0, 4), (4, 11)]
    assert O.shard_ranges(7, 1, 4) == [(0, 7)]
    for n, world, pool in ((1000, 4, 4), (1003, 3, 2), (64, 8, 8)):
        rs = O.shard_ranges(n, world, pool)
        assert rs[0][0] == 0 and rs[-1][1] == n
        assert all(a[1] == b[0] for a, b in zip(rs[:-1], rs[1:]))
        assert all(t0 % pool == 0 for t0, _ in rs)
        sizes = [(t1 - t0) // pool for t0, t1 in rs]
        assert max(sizes) - min(sizes) <= 1


def _shards(Kl_tokens_blocks, n_tokens, world, pool, sink, sizes, iters, seed_shift=0):
    """Per-shard trees over the shards' latent keys (block rows of Kl)."""
    out = []
    for t0, t1 in O.shard_ranges(n_tokens, world, pool):
        b0, b1 = t0 // pool, t1 // pool
        Kl_s = Kl_tokens_blocks[b0:b1]
        tree = O.build_tree(Kl_s, sizes, iters, 0, O.local_sink(sink, t0), pool)
        out.append((t0, tree, Kl_s))
    return out


def test_cp_one_shard_equals_tree_selection():
    Kl, t = _random_tree(21, nb=150, sizes=(3, 12), pool=2, sink=4)
    rng = np.random.default_rng(5)
    for i in (0, 9, 40, 150, 299):
        q = rng.standard_normal(Kl.shape[1])
        want = O.select_blocks(t, Kl, q, i, 4, 40, 8)
        got = O.cp_select_blocks([(0, t, Kl)], q, i, 4, 40, 8, 2)
        np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("world,pool,sink", [(2, 2, 6), (3, 1, 0), (4, 4, 9)])
def test_cp_full_beam_equals_global_fullscan(world, pool, sink):
    """With a beam that keeps every node, each shard returns its own exact
    top-K, and the merge is then the full scan over the whole sequence."""
    rng = np.random.default_rng(world * 10 + pool)
    n_tokens = 400 + pool - 1
    nb = n_tokens // pool
    Kl = rng.standard_normal((nb, 4))
    shards = _shards(Kl, n_tokens, world, pool, sink, (2, 6), 3)
    window, topk = 5, 24
    for i in list(range(0, n_tokens, 37)) + [n_tokens - 1]:
        q = rng.standard_normal(4)
        got = O.cp_select_blocks(shards, q, i, 1000, topk, window, pool)
        want = O.fullscan_blocks(Kl, q, i, topk, sink, window, pool)
        np.testing.assert_array_equal(got, want)


def test_merge_attention_equals_attention_over_the_union():
    rng = np.random.default_rng(3)
    N, d, G = 90, 8, 3
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    q = rng.standard_normal((G, d))
    sel = np.sort(rng.choice(N, 50, replace=False))
    want_o, want_l = O.sparse_attention(q, K, V, sel)
    # split into 4 disjoint parts, one of them empty
    cuts = [sel[sel < 20], sel[(sel >= 20) & (sel < 20)], sel[(sel >= 20) & (sel < 61)], sel[sel >= 61]]
    outs, lses = [], []
    for part in cuts:
        if part.size:
            o, l = O.sparse_attention(q, K, V, part)
        else:
            o, l = np.zeros((G, d)), np.full(G, -np.inf)
        outs.append(o)
        lses.append(l)
    got_o, got_l = O.merge_attention(outs, lses)
    np.testing.assert_allclose(got_o, want_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got_l, want_l, rtol=0, atol=1e-12)
    # every part empty: O = 0, lse = -inf
    o, l = O.merge_attention([np.zeros((G, d))] * 2, [np.full(G, -np.inf)] * 2)
    assert np.all(o == 0) and np.all(l == -np.inf)
