"""Paths that must give the same bits as the per-query search.

Dense-level scoring of large selections (node_scores.cu).  The upper tree
levels whose parents all fit in the beam are scored for tiles of queries
before the per-query search, which then reads one score per node of those
levels.  The selection must be the same, bit for bit, as that of the
per-query search scoring every node itself (the scores are the same fp32
values), with one buffer of scores and with the buffer forced small so that
the queries run in several chunks.  The per-query search is the path the
other parity tests check against the oracle; this pins the dense form to it
on every tree shape the workloads use.  When the leaf level is the only
level below the dense ones, the kept nodes and the kept leaves are chosen by
warp-wide exact selections for all queries and the leaves scored per node
(leaf tiles); the selection must be the same bits with them on and off,
ties included (the integer workload in a three-level tree).

Full scan: calls of 64 or more (query, KV head) pairs filter on the tensor
cores and rank the survivors exactly (a few query tiles split the block range
over CTAs); smaller calls scan every block per query.  All must give the same
selection for the same query."""
import pytest
import torch

from hierarchical_latent_key_gemm_b200 import lsa
from hierarchical_latent_key_gemm_b200.workloads import WORKLOADS, make_inputs

import lsa_testutil as TU

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lsa.lib()
    yield
    lsa.lsa_debug_dense_config(0, 0)
    torch.cuda.synchronize()


def _ways(ix, sp, Q, **kw):
    """per-query search; dense levels + leaf tiles; the same in small chunks;
    dense levels without leaf tiles"""
    out = []
    try:
        for min_pairs, chunk, tiles in ((-1, 0, 1), (1, 0, 1), (1, 1 << 20, 1), (1, 0, 0)):
            lsa.lsa_debug_dense_config(min_pairs, chunk)
            lsa.lsa_debug_leaf_tiles(tiles)
            out.append(lsa.lsa_select(ix, sp, Q, **kw))
    finally:
        lsa.lsa_debug_dense_config(0, 0)
        lsa.lsa_debug_leaf_tiles(1)
    return out


def _same(outs):
    (i0, c0) = outs[0]
    for k, (i, c) in enumerate(outs[1:], 1):
        assert torch.equal(c0, c), f"counts differ (way {k})"
        assert torch.equal(i0, i), f"rows differ (way {k})"


@pytest.mark.parametrize("name,over,beam", [
    ("int_exact_16k", {}, None),                                        # 16 x 256, r = 16, beam 16: both levels dense
    ("flat_4k_f32", {}, None),                                          # one level of 64, r = 32
    ("gqa_128k", dict(n_tokens=16384 + 5, needles=0, components=512), None),   # 32 x 1024, beam 32, 4 KV heads
    ("gqa_128k", dict(n_tokens=16384 + 5, needles=0, components=512), 31),     # beam below the top level: one level
    ("prefill_1m", dict(n_tokens=65536 + 7, level_sizes=(16, 128, 1024), needles=0, components=1024,
                        drift_every=1 << 14), None),                    # three levels, leaf tiles
    ("prefill_1m", dict(n_tokens=32768 + 3, level_sizes=(16, 512, 4096), needles=0, components=1024,
                        drift_every=1 << 13), None),                    # the bench's upper levels, leaf tiles
    ("int_exact_16k", dict(level_sizes=(4, 16, 256)), 4),               # integer scores: ties at every level
    ("gqa_128k", dict(n_tokens=65536 + 5, level_sizes=(8, 1024, 8192), needles=0, components=512), None),
                                                                        # 1,024 kept-node candidates: 32 keys a lane
    ("gqa_128k", dict(n_tokens=65536 + 5, level_sizes=(8, 2048, 8192), needles=0, components=512), None),
                                                                        # 2,048: keys in shared memory
])
def test_dense_levels_match_the_per_query_search(name, over, beam):
    w = WORKLOADS[name].scaled(**over)
    inp = make_inputs(w, seed=31, device="cuda")
    ix = lsa.lsa_build_index(TU.build_params(w), inp["K"], inp["W"])
    sp = TU.select_params(w, beam=beam)
    outs = _ways(ix, sp, inp["Q"])
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    _same(outs)
    ix.free()


def test_leaf_tiles_rows_that_fall_back():
    """Kept nodes with about 3,072 leaves between them: some rows exceed the
    leaf-score slots of the leaf tiles and search every level themselves,
    the others use the tiles; every row must equal the per-query search."""
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=32768 + 5, level_sizes=(4, 8, 6144), needles=0, components=512)
    inp = make_inputs(w, seed=35, device="cuda")
    ix = lsa.lsa_build_index(TU.build_params(w), inp["K"], inp["W"])
    # children per level-1 node: the 4 largest hold more than the 3,072 slots,
    # the 4 smallest fewer, so both kinds of rows can occur
    par = ix.get(lsa.LSA_GET_PARENT, 2).long().cpu()
    kids = torch.stack([torch.bincount(par[u], minlength=8) for u in range(par.shape[0])]).sort(dim=1).values
    assert bool((kids[:, -4:].sum(1) > 3072).any()) and bool((kids[:, :4].sum(1) <= 3072).any()), kids
    sp = TU.select_params(w, beam=4)
    outs = _ways(ix, sp, inp["Q"])
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    _same(outs)
    ix.free()


def test_dense_levels_batch_and_given_positions():
    """Several sequences (row index (b * nq + qi) * hkv + h in the score
    buffer) and query positions given per query."""
    w = WORKLOADS["decode_10m_x4"].scaled(n_tokens=8192 + 3, level_sizes=(8, 64, 512), needles=0, components=512,
                                          decode_steps=0)
    inp = make_inputs(w, seed=32, device="cuda")
    ix = lsa.lsa_build_index(TU.build_params(w), inp["K"], inp["W"])
    sp = TU.select_params(w)
    nq = 1500
    g = torch.Generator().manual_seed(5)
    pos = torch.randint(0, w.n_tokens, (w.batch, nq), generator=g).to(torch.int64).cuda()
    Q = inp["Q"][:, :nq].contiguous()
    outs = _ways(ix, sp, Q, q_pos=pos)
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    _same(outs)
    # three levels with a sparse leaf level (leaf tiles) over several sequences
    w2 = w.scaled(level_sizes=(8, 32, 256))
    ix2 = lsa.lsa_build_index(TU.build_params(w2), inp["K"], inp["W"])
    outs = _ways(ix2, TU.select_params(w2, beam=16), Q, q_pos=pos)
    assert lsa.lsa_check(ix2) == lsa.LSA_OK
    _same(outs)
    ix.free()
    ix2.free()


def test_dense_levels_scored_blocks():
    """The scored-blocks form (context-parallel shards) through the dense path
    and the leaf tiles (three levels, the leaf level sparse)."""
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=8192 + 1, level_sizes=(8, 64, 512), needles=0, components=256)
    inp = make_inputs(w, seed=33, device="cuda")
    ix = lsa.lsa_build_index(TU.build_params(w), inp["K"], inp["W"])
    sp = TU.select_params(w)
    outs = []
    try:
        for min_pairs, chunk, tiles in ((-1, 0, 1), (1, 0, 1), (1, 1 << 18, 1), (1, 0, 0)):
            lsa.lsa_debug_dense_config(min_pairs, chunk)
            lsa.lsa_debug_leaf_tiles(tiles)
            sc, bl, ct = lsa.lsa_select_blocks(ix, sp, inp["Q"], 0)
            # the kept blocks come in no particular order: sort each row by block id
            key = torch.where(bl >= 0, bl, torch.full_like(bl, 2 ** 31 - 1))
            key, order = torch.sort(key, dim=-1)
            outs.append((torch.gather(sc, -1, order), key, ct))
    finally:
        lsa.lsa_debug_dense_config(0, 0)
        lsa.lsa_debug_leaf_tiles(1)
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    for o in outs[1:]:
        for a, b in zip(outs[0], o):
            assert torch.equal(a, b)
    ix.free()


@pytest.mark.parametrize("name,over", [
    ("int_exact_16k", {}),
    ("gqa_128k", dict(n_tokens=16384 + 5, needles=0, components=512)),
])
def test_fullscan_tensor_core_filter_matches_per_query_scan(name, over):
    w = WORKLOADS[name].scaled(**over)
    inp = make_inputs(w, seed=34, device="cuda")
    ix = lsa.lsa_build_index(TU.build_params(w), inp["K"], inp["W"])
    sp = TU.select_params(w)
    big_i, big_c = lsa.lsa_fullscan_select(ix, sp, inp["Q"])          # tensor-core filter, whole tiles
    small = 60 // w.hkv                                                # under 64 pairs: per-query scan
    for q0 in (0, 5000, w.n_tokens - 300):
        for n in (small, 300):                                         # 300: tensor cores, split block range
            Q = inp["Q"][:, q0:q0 + n].contiguous()
            i, c = lsa.lsa_fullscan_select(ix, sp, Q, q_pos0=q0)
            assert torch.equal(c, big_c[:, q0:q0 + n]) and torch.equal(i, big_i[:, q0:q0 + n])
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    ix.free()
