"""Plain CPU oracle for the Latent Sparse Attention (LSA) hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, constants or helpers with the CUDA path; both sides only consume the
same seeded inputs.

It restates, step by step and without any blocking, fusion or reordering, what
the method computes.  All floating point is numpy float64.  The integer-grid
mode (centroids rounded to multiples of 2**-g, see ``kmeans_update``) is exact:
every value it produces is an integer multiple of a power of two far below
2**52, so float64 holds it and every sum of such values exactly; the grid
rounding itself is done with integer division.

Sources, cited below by key and section:
  [p1] "The 10M-token attention layer spends 98% of its time finding tokens"
       (Wink Pings news post)
  [p2] "Latent Sparse Attention speeds up the search for useful tokens in very
       long contexts" (editorial), section "Reduce the cost of finding the
       tokens to attend to"
  [p3] "Latent Sparse Attention: tree search over keys for 10M-token context"
       (wiki note), TL;DR and flowchart
  [p4] "Researchers report 72.4x faster attention-layer prefill at 10 million
       tokens", sections "Search the clusters, not every key" and "Prompt
       processing is not response generation"
  [p5] "Latent Sparse Attention (LSA): The 72.4x and 22.7x Speedups, and What
       They Compare Against", section "How does LSA work?" (steps 1-3) and
       section "Prefill, decode and training"

What the pages fix: blocks of keys are averaged, mapped to a latent space and
grouped into buckets that form a tree [p5 step 1; p2; p4]; a query is compared with
the bucket centroids, goes on into a few of the best buckets only, and compares
itself with the keys in those [p1; p3 TL;DR; p5 step 2]; exact attention then
covers the chosen distant keys, the first S tokens and the last W tokens, the
attention itself being unchanged [p5 step 3; p3 flowchart, the sparse-attention
node].  The old
indexer scores every key [p3 flowchart, red path].  In decode, every generated
token looks at all earlier tokens [p5 "Prefill, decode and training"].

Readings where the pages are silent:
  R1  one latent map W (d x r) serves keys and queries.
  R2  scores are unscaled inner products in latent space; k-means uses squared
      Euclidean distance.
  R3  pooling = mean of ``pool`` consecutive keys, then the map (linear, so the
      order does not matter in exact arithmetic); only complete blocks exist.
  R4  the top-K budget counts tokens: ceil(K / pool) blocks are taken.
  R5  the tree is built once over the whole prompt; for the query at position
      i a block b is a candidate iff b*pool >= S and b*pool + pool - 1 <= i - W;
      a node is eligible iff it holds a candidate, i.e. minpos(node) <= i - W -
      pool + 1 where minpos ranges over blocks that start at or after S.
  R6  top-K is drawn only from outside sink and window; the union is disjoint.
  R7  every tie goes to the lower index (argmin label, node, block).
  R8  an empty cluster keeps its previous centroid and is never eligible.
  R9  Lloyd init: centroid j starts at point floor(j * n / k), at every level.
  R10 upper levels are k-means of the level-below centroids (all of them,
      unweighted); bucket membership is the last assignment and the centroids
      are the last update (the means of those buckets).
  R11 GQA: the query latent of a KV head is the mean over its query heads.
  R12 softmax scale 1/sqrt(d).
  R13 decode: centroids are frozen; a completed block goes to its nearest leaf
      over all leaves.
  R18 decode upkeep of the layout: the oracle's leaves are unbounded member
      lists, so a block always joins its nearest leaf; a device index whose
      leaf ran out of free slots must, once its leaves are laid out again,
      hold exactly these lists (nothing in the method changes).
  R19 centroid refresh during decode (the pages are silent; plainest upkeep
      consistent with R10): memberships held fixed, every centroid is
      recomputed bottom-up as the mean of its current members (a leaf from
      the latent keys of its blocks, appended ones included; an upper node
      from its children's refreshed centroids), by the rules of
      ``kmeans_update``.  Right after a build this changes nothing (R10).
  R17 the training-free map [p5 "How does LSA work?", the D-LSA options, one
      of which needs no training and takes a PCA map]: W = the r leading principal
      directions of the pooled keys of every (sequence, KV head), i.e. the
      eigenvectors of their covariance (centred, divided by the count) for the
      r largest eigenvalues, in descending order; each column's entry of
      largest magnitude (lowest index among equal magnitudes) is positive.

Parity pins live in tests/test_oracle_pins.py (closed forms, hand-worked
examples under tests/golden/, invariants, brute force on tiny inputs).  Parity
unpinned: needle hit-rate and tree-vs-full-scan recall are measurements only;
the pages print no value for either.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

INF = np.inf


# ---------------------------------------------------------------------------
# Latent map and pooling  [p5 "How does LSA work?" step 1; p2; p4 "Search the
# clusters, not every key": keys live in a learned latent space]
# ---------------------------------------------------------------------------
def project_pool(K: np.ndarray, W: np.ndarray, pool: int) -> np.ndarray:
    """Latent keys of one (sequence, KV head): mean of each run of ``pool``
    consecutive keys, mapped by W.  K: [N, d]; W: [d, r]; returns [N//pool, r].
    Only complete blocks are returned (reading R3)."""
    K = np.asarray(K, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    nb = K.shape[0] // pool
    pooled = K[: nb * pool].reshape(nb, pool, K.shape[1]).mean(axis=1)
    return pooled @ W


def pca_map(K_units, pool: int, r: int):
    """Training-free latent map (reading R17).  K_units: sequence of [N, d]
    key arrays, one per (sequence, KV head); every one is pooled as in
    ``project_pool`` (the map here is the identity) and all pooled keys are
    one sample.  Returns (W [d, r], the r largest covariance eigenvalues in
    descending order)."""
    X = np.concatenate([project_pool(Ku, np.eye(np.asarray(Ku).shape[1]), pool) for Ku in K_units], axis=0)
    mu = X.mean(axis=0)
    Xc = X - mu
    C = Xc.T @ Xc / X.shape[0]
    evals, evecs = np.linalg.eigh(C)              # ascending
    order = np.argsort(-evals, kind="stable")[:r]
    W = evecs[:, order].copy()
    for c in range(r):
        j = int(np.argmax(np.abs(W[:, c])))       # first index of the largest magnitude
        if W[j, c] < 0:
            W[:, c] = -W[:, c]
    return W, evals[order]


def query_latent(Qg: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Latent query shared by one GQA group (reading R11): the mean over the
    group's query heads of q_h mapped by W.  Qg: [Nq, G, d]; returns [Nq, r]."""
    Qg = np.asarray(Qg, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    return (Qg @ W).mean(axis=1)


# ---------------------------------------------------------------------------
# Lloyd k-means  [p1: keys are grouped into clusters first; p5 step 1: the
# clusters are the buckets]
# ---------------------------------------------------------------------------
def squared_distances(X: np.ndarray, C: np.ndarray) -> np.ndarray:
    """||x - c||^2 for every (point, centroid) pair, [n, k].  Uses the exact
    identity ||x-c||^2 = ||x||^2 - 2 x.c + ||c||^2 (float64; exact on the
    integer grid)."""
    X = np.asarray(X, dtype=np.float64)
    C = np.asarray(C, dtype=np.float64)
    xx = np.einsum("ij,ij->i", X, X)[:, None]
    cc = np.einsum("ij,ij->i", C, C)[None, :]
    return xx - 2.0 * (X @ C.T) + cc


def kmeans_assign(X: np.ndarray, C: np.ndarray, chunk: int = 0):
    """Nearest centroid of every point, ties to the lower centroid id (R7).
    Returns (labels int64 [n], objective = sum of the chosen squared distances).
    Points are taken ``chunk`` at a time only to bound the size of the
    distance matrix (default: about 4 M entries); each point's distances, its
    argmin and the final sum do not depend on the chunking."""
    n = X.shape[0]
    if chunk <= 0:
        chunk = max(1, (1 << 22) // max(1, C.shape[0]))
    labels = np.empty(n, dtype=np.int64)
    dmin = np.empty(n, dtype=np.float64)
    for s in range(0, n, chunk):
        d2 = squared_distances(X[s : s + chunk], C)
        lab = np.argmin(d2, axis=1)  # first minimum = lower id
        labels[s : s + chunk] = lab
        dmin[s : s + chunk] = d2[np.arange(d2.shape[0]), lab]
    return labels, float(dmin.sum())


def _round_half_even_div(s: np.ndarray, n: np.ndarray) -> np.ndarray:
    """round-half-even(s / n) for integer arrays, by integer floor division."""
    q = np.floor_divide(s, n)
    rem = s - q * n  # in [0, n)
    twice = 2 * rem
    up = (twice > n) | ((twice == n) & (q % 2 != 0))
    return q + up.astype(np.int64)


def kmeans_update(X: np.ndarray, labels: np.ndarray, C_old: np.ndarray,
                  grid_log2: int = 0) -> np.ndarray:
    """New centroid of every cluster = mean of its members; an empty cluster
    keeps its previous centroid (R8).  With ``grid_log2 = g > 0`` the mean is
    rounded half-to-even onto multiples of 2**-g, computed as
    round_half_even(sum(2**g * x) / count) in integers; every point must then
    lie on that grid."""
    X = np.asarray(X, dtype=np.float64)
    k, r = C_old.shape
    counts = np.bincount(labels, minlength=k).astype(np.int64)
    C = np.array(C_old, dtype=np.float64, copy=True)
    nz = counts > 0
    if grid_log2 > 0:
        scale = float(1 << grid_log2)
        Xi = X * scale
        if not np.all(Xi == np.round(Xi)):
            raise ValueError("integer-grid k-means needs points on the grid")
        Xi = Xi.astype(np.int64)
        sums = np.zeros((k, r), dtype=np.int64)
        np.add.at(sums, labels, Xi)
        q = _round_half_even_div(sums[nz], counts[nz][:, None])
        C[nz] = q.astype(np.float64) / scale
    else:
        sums = np.zeros((k, r), dtype=np.float64)
        np.add.at(sums, labels, X)
        C[nz] = sums[nz] / counts[nz][:, None]
    return C


def kmeans_init(X: np.ndarray, k: int) -> np.ndarray:
    """Centroid j starts at point floor(j * n / k) (R9)."""
    n = X.shape[0]
    idx = np.array([(j * n) // k for j in range(k)], dtype=np.int64)
    return np.array(X[idx], dtype=np.float64, copy=True)


@dataclass
class KMeansResult:
    labels: np.ndarray          # last assignment, int64 [n]
    centroids: np.ndarray       # last update, float64 [k, r]
    objectives: list            # objective after every assign, len = iters


def kmeans(X: np.ndarray, k: int, iters: int, grid_log2: int = 0, history: list | None = None) -> KMeansResult:
    """``iters`` Lloyd rounds of (assign, update) from the stride init (R9, R10).
    With ``history`` (a list), every round appends (centroids it assigned
    against, labels, centroids after the update), for round-by-round checks."""
    X = np.asarray(X, dtype=np.float64)
    C = kmeans_init(X, k)
    objectives = []
    labels = np.zeros(X.shape[0], dtype=np.int64)
    for _ in range(iters):
        labels, obj = kmeans_assign(X, C)
        objectives.append(obj)
        C_next = kmeans_update(X, labels, C, grid_log2)
        if history is not None:
            history.append((C, labels, C_next))
        C = C_next
    return KMeansResult(labels, C, objectives)


# ---------------------------------------------------------------------------
# The bucket hierarchy  [p2: the tree form of the index; p3 TL;DR: keys are
# clustered level by level; p4 and p5 step 1: the clusters form a hierarchy]
# ---------------------------------------------------------------------------
@dataclass
class Tree:
    """Levels are ordered top first, leaves last.  ``parent[l][j]`` is the node
    at level l-1 that owns node j of level l (parent[0] is None)."""
    pool: int
    sink: int
    level_sizes: list
    centroids: list                     # float64 [n_l, r] per level
    parent: list                        # int64 [n_l] per level (None at top)
    leaf_of_block: np.ndarray           # int64 [Nb]
    objectives: list                    # per level, objective after each assign
    children: list = field(default_factory=list)   # children[l][j] -> ids at l+1
    members: list = field(default_factory=list)    # per leaf, ascending block ids
    minpos: list = field(default_factory=list)     # float64 [n_l] per level

    @property
    def levels(self) -> int:
        return len(self.level_sizes)

    def finish(self) -> "Tree":
        """Derive child lists, leaf member lists and minpos from the labels."""
        L = self.levels
        self.children = [None] * L
        for l in range(L - 1):
            par = self.parent[l + 1]
            self.children[l] = [np.flatnonzero(par == j) for j in range(self.level_sizes[l])]
        nleaf = self.level_sizes[-1]
        order = np.argsort(self.leaf_of_block, kind="stable")
        counts = np.bincount(self.leaf_of_block, minlength=nleaf)
        starts = np.concatenate([[0], np.cumsum(counts)])
        self.members = [order[starts[j]:starts[j + 1]].astype(np.int64) for j in range(nleaf)]
        self.recompute_minpos()
        return self

    def recompute_minpos(self) -> None:
        """minpos(leaf) = smallest start position of a member block that starts
        at or after the sink; minpos(node) = min over its children; +inf when
        there is none (R5, R8)."""
        L = self.levels
        mp = [None] * L
        leaf = np.full(self.level_sizes[-1], INF)
        for j, mem in enumerate(self.members):
            pos = mem * self.pool
            pos = pos[pos >= self.sink]
            if pos.size:
                leaf[j] = float(pos.min())
        mp[L - 1] = leaf
        for l in range(L - 2, -1, -1):
            up = np.full(self.level_sizes[l], INF)
            for j, ch in enumerate(self.children[l]):
                if ch.size:
                    up[j] = mp[l + 1][ch].min()
            mp[l] = up
        self.minpos = mp


def build_tree(Kl: np.ndarray, level_sizes, iters: int, grid_log2: int,
               sink: int, pool: int, leaf_history: list | None = None) -> Tree:
    """Leaf k-means over the latent keys, then k-means of each level's
    centroids into the level above (R10).  ``level_sizes`` is top first.
    ``leaf_history``: see ``kmeans`` (the leaf level's rounds)."""
    level_sizes = list(level_sizes)
    L = len(level_sizes)
    res = kmeans(Kl, level_sizes[-1], iters, grid_log2, leaf_history)
    centroids = [None] * L
    parent = [None] * L
    objectives = [None] * L
    centroids[L - 1] = res.centroids
    objectives[L - 1] = res.objectives
    pts = res.centroids
    for l in range(L - 2, -1, -1):
        up = kmeans(pts, level_sizes[l], iters, grid_log2)
        parent[l + 1] = up.labels
        centroids[l] = up.centroids
        objectives[l] = up.objectives
        pts = up.centroids
    return Tree(pool, sink, level_sizes, centroids, parent, res.labels, objectives).finish()


# ---------------------------------------------------------------------------
# Selection  [p3 TL;DR: the query scores centroids and goes down into a few of
# the best buckets; p1: clusters are scored first, then the keys inside the
# chosen ones; p5 step 3: the chosen far-away keys join the attention sink and
# a local window]
# ---------------------------------------------------------------------------
def top_by_score(ids: np.ndarray, scores: np.ndarray, k: int) -> np.ndarray:
    """The k ids with the highest scores; equal scores go to the lower id (R7)."""
    ids = np.asarray(ids, dtype=np.int64)
    if ids.size <= k:
        return ids.copy()
    order = np.lexsort((ids, -np.asarray(scores, dtype=np.float64)))
    return ids[order[:k]]


def candidate_bound(i: int, window: int, pool: int) -> int:
    """Largest start position a candidate block may have for the query at i (R5)."""
    return i - window - pool + 1


def blocks_per_topk(topk: int, pool: int) -> int:
    """R4: the token budget K buys ceil(K / pool) blocks."""
    return -(-topk // pool)


def beam_search(tree: Tree, qbar: np.ndarray, i: int, beam: int, window: int) -> np.ndarray:
    """Level by level, score the eligible nodes (all top nodes, then the
    children of the kept nodes) by qbar . centroid and keep the best ``beam``.
    Returns the kept leaf ids."""
    bound = candidate_bound(i, window, tree.pool)
    kept = np.arange(tree.level_sizes[0], dtype=np.int64)
    for l in range(tree.levels):
        if l > 0:
            kids = [tree.children[l - 1][j] for j in kept]
            kept = np.concatenate(kids) if kids else np.zeros(0, dtype=np.int64)
        elig = kept[tree.minpos[l][kept] <= bound]
        scores = tree.centroids[l][elig] @ qbar
        kept = top_by_score(elig, scores, beam)
    return kept


def select_blocks(tree: Tree, Kl: np.ndarray, qbar: np.ndarray, i: int, beam: int,
                  topk: int, window: int) -> np.ndarray:
    """Tree search: candidate blocks inside the kept leaves, scored by
    qbar . latent key, top ceil(K/pool) of them; returned ascending."""
    qbar = np.asarray(qbar, dtype=np.float64)
    leaves = beam_search(tree, qbar, i, beam, window)
    bound = candidate_bound(i, window, tree.pool)
    if leaves.size:
        blocks = np.concatenate([tree.members[j] for j in leaves])
    else:
        blocks = np.zeros(0, dtype=np.int64)
    start = blocks * tree.pool
    blocks = blocks[(start >= tree.sink) & (start <= bound)]
    scores = np.asarray(Kl, dtype=np.float64)[blocks] @ qbar
    chosen = top_by_score(blocks, scores, blocks_per_topk(topk, tree.pool))
    return np.sort(chosen)


def fullscan_blocks(Kl: np.ndarray, qbar: np.ndarray, i: int, topk: int, sink: int,
                    window: int, pool: int) -> np.ndarray:
    """The old indexer [p3 flowchart, red path]: score every candidate block,
    keep the top ceil(K/pool); returned ascending."""
    Kl = np.asarray(Kl, dtype=np.float64)
    nb = Kl.shape[0]
    bound = candidate_bound(i, window, pool)
    b = np.arange(nb, dtype=np.int64)
    b = b[(b * pool >= sink) & (b * pool <= bound)]
    scores = Kl[b] @ np.asarray(qbar, dtype=np.float64)
    return np.sort(top_by_score(b, scores, blocks_per_topk(topk, pool)))


def selection_tokens(blocks: np.ndarray, i: int, sink: int, window: int, pool: int) -> np.ndarray:
    """Sorted token set: tokens of the chosen blocks, the sink [0, min(S, i+1))
    and the causal window [max(0, i-W+1), i]."""
    toks = set(range(0, min(sink, i + 1)))
    toks.update(range(max(0, i - window + 1), i + 1))
    for b in np.asarray(blocks, dtype=np.int64):
        toks.update(range(int(b) * pool, int(b) * pool + pool))
    return np.array(sorted(toks), dtype=np.int64)


# ---------------------------------------------------------------------------
# Exact attention over the selected set  [p5 step 3: LSA leaves the attention
# itself as it was; p3 flowchart: exact attention over the subset]
# ---------------------------------------------------------------------------
def sparse_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, sel: np.ndarray):
    """softmax(q . k_j / sqrt(d)) weighted sum of v_j over j in ``sel``.
    q: [G, d] (the query heads that share the selection); K, V: [N, d].
    Returns (O [G, d], lse [G]) with lse the natural log of the softmax
    denominator of the scaled scores (R12)."""
    q = np.asarray(q, dtype=np.float64)
    sel = np.asarray(sel, dtype=np.int64)
    Ks = np.asarray(K, dtype=np.float64)[sel]
    Vs = np.asarray(V, dtype=np.float64)[sel]
    s = (q @ Ks.T) / math.sqrt(q.shape[-1])
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    den = e.sum(axis=1, keepdims=True)
    return (e @ Vs) / den, (m + np.log(den))[:, 0]


# ---------------------------------------------------------------------------
# Decode  [p5 "Prefill, decode and training": every generated token looks at
# all earlier tokens; p4 "Prompt processing is not response generation"]
# ---------------------------------------------------------------------------
def nearest_leaf(tree: Tree, x: np.ndarray) -> int:
    """argmin over all leaves of ||x - c||^2 with frozen centroids (R13, R7)."""
    d2 = squared_distances(np.asarray(x, dtype=np.float64)[None, :], tree.centroids[-1])[0]
    return int(np.argmin(d2))


def refresh_centroids(tree: Tree, Kl: np.ndarray, grid_log2: int = 0) -> None:
    """R19: with every membership fixed, each leaf centroid becomes the mean of
    the latent keys of its blocks (``Kl`` [Nb, r], rows in block order, the
    appended blocks included), then, level by level upwards, each node's the
    mean of its children's new centroids; an empty node keeps its centroid and
    the grid rule of ``kmeans_update`` applies.  Updates ``tree`` in place."""
    Lv = tree.levels
    Kl = np.asarray(Kl, dtype=np.float64)
    if Kl.shape[0] != tree.leaf_of_block.shape[0]:
        raise ValueError("one latent row per labelled block")
    tree.centroids[Lv - 1] = kmeans_update(Kl, tree.leaf_of_block, tree.centroids[Lv - 1], grid_log2)
    for l in range(Lv - 2, -1, -1):
        tree.centroids[l] = kmeans_update(tree.centroids[l + 1], tree.parent[l + 1], tree.centroids[l], grid_log2)


def append_block(tree: Tree, Kl_rows: list, x: np.ndarray) -> int:
    """Index one newly completed block (its latent ``x``): it joins its nearest
    leaf, at the end of that leaf's ascending member list; minpos of the leaf
    and its ancestors is refreshed.  ``Kl_rows`` (a list of latent rows) grows
    by one.  Returns the leaf id."""
    b = len(Kl_rows)
    Kl_rows.append(np.asarray(x, dtype=np.float64))
    leaf = nearest_leaf(tree, x)
    tree.members[leaf] = np.concatenate([tree.members[leaf], [b]]).astype(np.int64)
    tree.leaf_of_block = np.concatenate([tree.leaf_of_block, [leaf]]).astype(np.int64)
    start = b * tree.pool
    if start >= tree.sink:
        node = leaf
        for l in range(tree.levels - 1, -1, -1):
            tree.minpos[l][node] = min(tree.minpos[l][node], float(start))
            if l > 0:
                node = int(tree.parent[l][node])
    return leaf


# ---------------------------------------------------------------------------
# Context parallelism over shards of one sequence  [p5 "What do 22.7x and
# 72.4x actually compare?" and "Can I run LSA?": the 10M-token runs split one
# sequence's context over several GPUs]
#
# Reading R20 (the pages give no algorithm for it): shard s holds the
# contiguous token range [t0_s, t1_s) (block-aligned) and its own tree, built
# from its latent keys alone with the sink rule in global positions (a block is
# a candidate iff it starts at or after S globally).  A query selects in every
# shard the local top ceil(K/P) blocks by the tree search of ``select_blocks``
# (positions shifted by t0_s); the selection is the top ceil(K/P) of the union
# of the shards' picks by (score desc, global block asc), expanded to tokens
# with the sink and the window as in ``selection_tokens``.  Attention over it
# is computed per shard on the shard's rows and merged by the log-sum-exp
# rule, which equals attention over the whole selection.
# ---------------------------------------------------------------------------
def shard_ranges(n_tokens: int, world: int, pool: int):
    """Contiguous token ranges [t0, t1) of ``world`` shards, each starting on a
    block boundary; the first shards get one block more when blocks do not
    divide evenly, and the last one also takes the partial block at the end."""
    nb = n_tokens // pool
    out = []
    b0 = 0
    for s in range(world):
        nbs = nb // world + (1 if s < nb % world else 0)
        t0 = b0 * pool
        t1 = (b0 + nbs) * pool if s < world - 1 else n_tokens
        out.append((t0, t1))
        b0 += nbs
    return out


def local_sink(sink: int, t0: int) -> int:
    """The sink rule of a shard starting at token t0, in its own positions."""
    return max(0, sink - t0)


def scored_blocks(tree: Tree, Kl: np.ndarray, qbar: np.ndarray, i: int, beam: int, topk: int,
                  window: int):
    """``select_blocks`` with the scores of the chosen blocks: returns (blocks,
    scores), blocks ascending.  A position before the tree's first block (i < 0
    in a shard's coordinates) chooses nothing."""
    blocks = select_blocks(tree, Kl, qbar, i, beam, topk, window)
    scores = np.asarray(Kl, dtype=np.float64)[blocks] @ np.asarray(qbar, dtype=np.float64)
    return blocks, scores


def cp_select_blocks(shards, qbar: np.ndarray, i: int, beam: int, topk: int, window: int, pool: int):
    """R20 selection of the query at global position i.  ``shards``: list of
    (t0, tree, Kl) with the tree over that shard's latent keys.  Returns the
    chosen global block ids, ascending."""
    ids, scs = [], []
    for t0, tree, Kl in shards:
        b, s = scored_blocks(tree, Kl, qbar, i - t0, beam, topk, window)
        ids.append(b + t0 // pool)
        scs.append(s)
    ids = np.concatenate(ids) if ids else np.zeros(0, np.int64)
    scs = np.concatenate(scs) if scs else np.zeros(0)
    return np.sort(top_by_score(ids, scs, blocks_per_topk(topk, pool)))


def merge_attention(outs, lses):
    """Attention over a union of disjoint row sets from the parts computed on
    each set: outs[s] [G, d] normalised outputs, lses[s] [G] natural-log
    denominators (-inf for an empty part).  Returns (O [G, d], lse [G]); a query
    whose parts are all empty gets O = 0 and lse = -inf."""
    L = np.stack([np.asarray(x, dtype=np.float64) for x in lses])          # [S, G]
    Os = np.stack([np.asarray(x, dtype=np.float64) for x in outs])         # [S, G, d]
    m = L.max(axis=0)
    G, d = Os.shape[1], Os.shape[2]
    O = np.zeros((G, d))
    lse = np.full(G, -INF)
    for g in range(G):
        if m[g] == -INF:
            continue
        wts = np.exp(L[:, g] - m[g])
        den = wts.sum()
        O[g] = (wts[:, None] * Os[:, g, :]).sum(axis=0) / den
        lse[g] = m[g] + math.log(den)
    return O, lse
