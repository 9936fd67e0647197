"""GPU parity of decode-time index upkeep (lsa_relayout, lsa_refresh_centroids)
against the oracle, whose leaves are unbounded member lists (R18) and whose
refresh recomputes every centroid from its members (R19).

Integer workload: labels, leaf sizes, minpos, centroids and selections
bit-exact.  Float workload (on the oracle's own tree): labels exact, centroids
to 1e-6 relative, selections within the threshold rule of the other tests."""
import numpy as np
import pytest
import torch

import oracle as O
from hierarchical_latent_key_gemm_b200 import lsa
from hierarchical_latent_key_gemm_b200.workloads import WORKLOADS, make_inputs

import lsa_testutil as TU

pytestmark = pytest.mark.gpu

NOPOS = np.iinfo(np.int64).max


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lsa.lib()
    yield
    torch.cuda.synchronize()


def _oracle_append(tree, rows, K, Wm, pool, t0, t1):
    """Blocks completed by tokens [t0, t1) join the oracle tree."""
    for t in range(t0, t1):
        if (t + 1) % pool == 0:
            x = O.project_pool(K[t + 1 - pool:t + 1], Wm, pool)[0]
            O.append_block(tree, rows, x)


def _check_state(ix, tree, rows, exact):
    Kl = np.array(rows)
    np.testing.assert_array_equal(ix.get(lsa.LSA_GET_LEAF_OF_BLOCK).cpu().numpy()[0], tree.leaf_of_block)
    np.testing.assert_array_equal(ix.get(lsa.LSA_GET_LEAF_COUNT).cpu().numpy()[0],
                                  [len(m) for m in tree.members])
    for l in range(tree.levels):
        mp = ix.get(lsa.LSA_GET_MINPOS, l).cpu().numpy()[0]
        np.testing.assert_array_equal(np.where(mp == NOPOS, np.inf, mp.astype(np.float64)), tree.minpos[l])
        c = ix.get(lsa.LSA_GET_CENTROIDS, l).double().cpu().numpy()[0]
        if exact:
            np.testing.assert_array_equal(c, tree.centroids[l])
        else:
            np.testing.assert_allclose(c, tree.centroids[l], rtol=1e-6, atol=1e-6)
    lat = ix.get(lsa.LSA_GET_LATENT).double().cpu().numpy()[0]
    if exact:
        np.testing.assert_array_equal(lat, Kl)
    else:
        np.testing.assert_allclose(lat, Kl, rtol=1e-5, atol=1e-5)


def _check_select(ix, tree, rows, inp, dQ, w, q_rows, pos0, exact):
    Wm = inp["W"].double().numpy()
    Kl = np.array(rows)
    sp = TU.select_params(w)
    q = dQ[:, q_rows[0]:q_rows[-1] + 1].contiguous()
    idx, cnt = lsa.lsa_select(ix, sp, q, q_pos0=pos0)
    qb = O.query_latent(TU.unit_queries(inp["Q"], 0, 0, w.group, list(q_rows)), Wm)
    got = TU.gpu_rows(idx, cnt, 0, list(range(len(q_rows))), 0)
    for k in range(len(q_rows)):
        i = pos0 + k
        blk = O.select_blocks(tree, Kl, qb[k], i, w.beam, w.topk, w.window)
        want = O.selection_tokens(blk, i, w.sink, w.window, w.pool)
        if exact:
            np.testing.assert_array_equal(got[k], want, err_msg=f"query at {i}")
        else:
            assert TU.selection_mismatch_ok(tree, Kl, qb[k], i, w.beam, w.topk, w.window, got[k], want)


def test_relayout_and_refresh_match_the_oracle_exactly():
    """int_exact_16k at 4,096 tokens with a window of 8 (so appended blocks
    become candidates soon): 64 appended keys equal to key 100 all go to one
    leaf, which runs out of free slots; the relayout places them, selections
    then equal the oracle's; 32 more appends, another relayout, a refresh of
    every centroid, 32 more appends under the refreshed leaves."""
    w = WORKLOADS["int_exact_16k"].scaled(n_tokens=4096, decode_steps=128, window=8)
    inp = make_inputs(w, seed=31)
    N = w.n_tokens
    inp["K"][0, N:N + 64] = inp["K"][0, 100]
    dK, dW, dQ = inp["K"].cuda(), inp["W"].cuda(), inp["Q"].cuda()
    ix = lsa.lsa_build_index(TU.build_params(w, append_capacity=w.decode_steps), dK, dW)
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    tree = TU.oracle_trees(TU.oracle_latents(inp, w), w)[0]
    rows = list(TU.oracle_latents(inp, w)[0])
    Wm = inp["W"].double().numpy()
    Kn = TU.unit_keys(inp["K"], 0, 0, N + w.decode_steps)

    lsa.lsa_append(ix, dK, 64)
    assert lsa.lsa_check(ix) == lsa.LSA_ERR_CAPACITY
    _oracle_append(tree, rows, Kn, Wm, w.pool, N, N + 64)
    lead = int(tree.leaf_of_block[N])
    assert np.all(tree.leaf_of_block[N:N + 64] == lead)
    # before the relayout the full leaf holds only what fitted
    assert ix.get(lsa.LSA_GET_LEAF_COUNT).cpu().numpy()[0][lead] < len(tree.members[lead])
    lsa.lsa_relayout(ix)
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    _check_state(ix, tree, rows, exact=True)
    _check_select(ix, tree, rows, inp, dQ, w, range(0, 64), N, exact=True)

    lsa.lsa_append(ix, dK, 32)
    _oracle_append(tree, rows, Kn, Wm, w.pool, N + 64, N + 96)
    lsa.lsa_relayout(ix)   # places whatever did not fit, a no-op otherwise
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    _check_state(ix, tree, rows, exact=True)

    lsa.lsa_refresh_centroids(ix)
    O.refresh_centroids(tree, np.array(rows), w.grid_log2)
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    _check_state(ix, tree, rows, exact=True)
    _check_select(ix, tree, rows, inp, dQ, w, range(64, 96), N + 64, exact=True)

    lsa.lsa_append(ix, dK, 32)
    _oracle_append(tree, rows, Kn, Wm, w.pool, N + 96, N + 128)
    lsa.lsa_relayout(ix)
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    _check_state(ix, tree, rows, exact=True)
    _check_select(ix, tree, rows, inp, dQ, w, range(96, 128), N + 96, exact=True)
    ix.free()


def test_refresh_right_after_a_build_changes_nothing():
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=8192 + 3, level_sizes=(8, 64), needles=0, components=128)
    inp = make_inputs(w, seed=32, device="cuda")
    ix = lsa.lsa_build_index(TU.build_params(w), inp["K"], inp["W"])
    before = [ix.get(lsa.LSA_GET_CENTROIDS, l) for l in range(2)]
    sp = TU.select_params(w)
    i0, c0 = lsa.lsa_select(ix, sp, inp["Q"])
    lsa.lsa_refresh_centroids(ix)
    lsa.lsa_relayout(ix)
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    for l in range(2):
        assert torch.equal(ix.get(lsa.LSA_GET_CENTROIDS, l), before[l])
    i1, c1 = lsa.lsa_select(ix, sp, inp["Q"])
    assert torch.equal(c0, c1) and torch.equal(i0, i1)
    ix.free()


def test_relayout_and_refresh_float_on_the_oracle_tree():
    """flat_4k_f32 (one level of 64 leaves, fp32 keys) imported from the
    oracle's tree; 64 appended keys equal to key 100 overflow one leaf."""
    w = WORKLOADS["flat_4k_f32"].scaled(decode_steps=64, window=8)
    inp = make_inputs(w, seed=33)
    N = w.n_tokens
    inp["K"][0, N:] = inp["K"][0, 100]
    dK, dW, dQ = inp["K"].cuda(), inp["W"].cuda(), inp["Q"].cuda()
    Kls = TU.oracle_latents(inp, w)
    trees = TU.oracle_trees(Kls, w)
    leaf, par, cen = TU.trees_to_device(trees, w)
    ix = lsa.lsa_build_index_from_tree(TU.build_params(w, append_capacity=64), dK, dW, leaf, par, cen)
    tree, rows = trees[0], list(Kls[0])
    Wm = inp["W"].double().numpy()
    lsa.lsa_append(ix, dK, 64)
    assert lsa.lsa_check(ix) == lsa.LSA_ERR_CAPACITY
    _oracle_append(tree, rows, TU.unit_keys(inp["K"], 0, 0, N + 64), Wm, w.pool, N, N + 64)
    lsa.lsa_relayout(ix)
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    _check_state(ix, tree, rows, exact=False)
    _check_select(ix, tree, rows, inp, dQ, w, range(0, 64), N, exact=False)
    lsa.lsa_refresh_centroids(ix)
    O.refresh_centroids(tree, np.array(rows), 0)
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    _check_state(ix, tree, rows, exact=False)
    _check_select(ix, tree, rows, inp, dQ, w, range(32, 64), N + 32, exact=False)
    ix.free()


def test_maintenance_argument_errors():
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=1024, level_sizes=(4, 16), needles=0, components=16)
    inp = make_inputs(w, seed=34, device="cuda")
    ix = lsa.lsa_build_index(TU.build_params(w), inp["K"], inp["W"])
    h = ix.handle
    ix.free()
    assert lsa.lib().lsa_relayout(h, None) == lsa.LSA_ERR_INVALID_ARG
    assert lsa.lib().lsa_refresh_centroids(h, None) == lsa.LSA_ERR_INVALID_ARG
    assert lsa.lib().lsa_relayout(None, None) == lsa.LSA_ERR_INVALID_ARG
