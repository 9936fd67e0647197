"""Helpers shared by the parity tests: run the oracle on seeded inputs and
move its results (never the other way round) into the layouts of the C ABI.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from hierarchical_latent_key_gemm_b200 import lsa
from hierarchical_latent_key_gemm_b200.workloads import Workload


def unit_keys(K: torch.Tensor, b: int, h: int, n: int) -> np.ndarray:
    """K[b, :n, h, :] as float64 numpy."""
    return K[b, :n, h, :].float().cpu().numpy().astype(np.float64)


def unit_queries(Q: torch.Tensor, b: int, h: int, G: int, rows=None) -> np.ndarray:
    """Q[b, rows, h*G:(h+1)*G, :] as float64 numpy [nq, G, d]."""
    q = Q[b, :, h * G:(h + 1) * G, :] if rows is None else Q[b, rows][:, h * G:(h + 1) * G, :]
    return q.float().cpu().numpy().astype(np.float64)


def oracle_latents(inp: dict, w: Workload, n_tokens: int | None = None):
    """Per-unit latent keys (oracle): list over units u = b*hkv + h."""
    n = n_tokens or w.n_tokens
    Wm = inp["W"].double().cpu().numpy()
    out = []
    for b in range(w.batch):
        for h in range(w.hkv):
            out.append(O.project_pool(unit_keys(inp["K"], b, h, n), Wm, w.pool))
    return out


def oracle_trees(Kls: list, w: Workload):
    return [O.build_tree(Kl, w.level_sizes, w.lloyd_iters, w.grid_log2, w.sink, w.pool) for Kl in Kls]


def trees_to_device(trees: list, w: Workload, device="cuda"):
    """Oracle trees -> (leaf_of_block [U, nb], parents[l] [U, n_l], centroids[l] [U, n_l, r])."""
    L = len(w.level_sizes)
    leaf = torch.tensor(np.stack([t.leaf_of_block for t in trees]), dtype=torch.int32, device=device)
    parents = [None] + [torch.tensor(np.stack([t.parent[l] for t in trees]), dtype=torch.int32, device=device)
                        for l in range(1, L)]
    cents = [torch.tensor(np.stack([t.centroids[l] for t in trees]), dtype=torch.float32, device=device)
             for l in range(L)]
    return leaf, parents, cents


def build_params(w: Workload, n_tokens=None, ld_tokens=None, append_capacity=0, dtype=None):
    n = n_tokens or w.n_tokens
    ld = ld_tokens or (w.n_tokens + w.decode_steps)
    dt = dtype if dtype is not None else (lsa.LSA_F32 if w.dtype == "f32" else lsa.LSA_BF16)
    return lsa.make_build_params(w.batch, n, ld, w.hkv, w.d, w.r, w.pool, dt, w.level_sizes, w.lloyd_iters,
                                 w.grid_log2, w.sink, append_capacity)


def select_params(w: Workload, beam=None, topk=None):
    return lsa.make_select_params(w.hq, beam or w.beam, w.topk if topk is None else topk, w.sink, w.window)


def gpu_rows(idx: torch.Tensor, cnt: torch.Tensor, b: int, rows, h: int):
    idx_c = idx[b, rows, h].cpu().numpy()
    cnt_c = cnt[b, rows, h].cpu().numpy()
    return [idx_c[i, : cnt_c[i]].astype(np.int64) for i in range(len(rows))]


def rows_to_idx(selections: list, max_sel: int, device="cuda"):
    """List of token arrays -> idx [n, max_sel] (-1 padded), cnt [n]."""
    n = len(selections)
    idx = np.full((n, max_sel), -1, dtype=np.int32)
    cnt = np.zeros(n, dtype=np.int32)
    for i, s in enumerate(selections):
        idx[i, : len(s)] = s
        cnt[i] = len(s)
    return torch.tensor(idx, device=device), torch.tensor(cnt, device=device)


def explain(tree, Kl, qbar, i, beam, topk, window):
    """Oracle thresholds for one query: per-level B-th kept score and the K-th
    block score, plus fp64 scores of every node/block (for tolerance checks)."""
    bound = O.candidate_bound(i, window, tree.pool)
    kept = np.arange(tree.level_sizes[0])
    level_thr = []
    node_scores = []
    for l in range(tree.levels):
        if l > 0:
            kids = [tree.children[l - 1][j] for j in kept]
            kept = np.concatenate(kids) if kids else np.zeros(0, np.int64)
        elig = kept[tree.minpos[l][kept] <= bound]
        sc = tree.centroids[l][elig] @ qbar
        node_scores.append(dict(zip(elig.tolist(), sc.tolist())))
        kept = O.top_by_score(elig, sc, beam)
        level_thr.append(float(np.min(tree.centroids[l][kept] @ qbar)) if kept.size and elig.size > beam else None)
    chosen = O.select_blocks(tree, Kl, qbar, i, beam, topk, window)
    kth = float(np.min(Kl[chosen] @ qbar)) if chosen.size else None
    return level_thr, kth


def selection_mismatch_ok(tree, Kl, qbar, i, beam, topk, window, gpu_tokens, ora_tokens, rel=1e-3, full=False):
    """True when every token in the symmetric difference belongs to a block whose
    fp64 score is within `rel` of the K-th threshold, or (tree search) to a
    leaf path whose node score is within `rel` of that level's B-th threshold."""
    diff = set(gpu_tokens.tolist()) ^ set(ora_tokens.tolist())
    if not diff:
        return True
    P = tree.pool if tree is not None else 1
    if full:
        chosen = O.fullscan_blocks(Kl, qbar, i, topk, 0, window, P)
        kth = float(np.min(Kl[chosen] @ qbar)) if chosen.size else None
        level_thr = []
    else:
        level_thr, kth = explain(tree, Kl, qbar, i, beam, topk, window)
    for t in diff:
        b = t // P
        s = float(Kl[b] @ qbar)
        if kth is not None and abs(s - kth) <= rel * abs(kth):
            continue
        if tree is not None and not full:
            node = int(tree.leaf_of_block[b])
            ok = False
            for l in range(tree.levels - 1, -1, -1):
                thr = level_thr[l]
                sc = float(tree.centroids[l][node] @ qbar)
                if thr is not None and abs(sc - thr) <= rel * abs(thr):
                    ok = True
                    break
                if l > 0:
                    node = int(tree.parent[l][node])
            if ok:
                continue
        return False
    return True


def recall(gpu_rows_list, ora_rows_list):
    tot = sum(len(o) for o in ora_rows_list)
    hit = sum(len(set(g.tolist()) & set(o.tolist())) for g, o in zip(gpu_rows_list, ora_rows_list))
    return hit / max(1, tot)
