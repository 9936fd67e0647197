"""GPU parity of the banded attention entry point (lsa_sparse_attn_banded):
dense sink/window band per tile of consecutive queries plus per-query
gathered long-range rows, merged by their maxima.  Checked against the oracle
on the oracle's own selections, against dense causal attention, on row lists
that are not of the selection form, and against lsa_sparse_attn on the GPU's
selection over every query.
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


def _oracle_attn(inp, w, sels, q0, nq):
    """fp64 oracle attention of queries q0..q0+nq-1 over given row lists."""
    Kn = inp["K"][0].float().numpy().astype(np.float64)
    Vn = inp["V"][0].float().numpy().astype(np.float64)
    G = w.group
    out = np.zeros((nq, w.hq, w.d))
    lse = np.zeros((nq, w.hq))
    for h in range(w.hkv):
        qs = TU.unit_queries(inp["Q"], 0, h, G, list(range(q0, q0 + nq)))
        for k in range(nq):
            o, l = O.sparse_attention(qs[k], Kn[:, h], Vn[:, h], sels[h][k])
            out[k, h * G:(h + 1) * G] = o
            lse[k, h * G:(h + 1) * G] = l
    return out, lse


def _check(w, got, glse, want, wlse):
    e = np.abs(got - want)
    le = np.abs(glse - wlse)
    if w.dtype == "f32":
        assert e.max() <= 1e-4 and le.max() <= 1e-4
    elif w.kind == "int":
        # one bf16 ulp of the oracle value plus fp32 accumulation slack
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(want), 1e-30))) - 7)
        assert np.all(e <= ulp + 1e-3) and e.max() <= BF16_MAX_ABS
        assert le.max() <= 1e-2
    else:
        assert e.max() <= BF16_MAX_ABS and e.mean() <= BF16_MEAN_ABS
        assert le.max() <= 1e-2


CASES = [
    ("flat_4k_f32", {}),
    ("int_exact_16k", {"n_tokens": 4096 + 3}),
    ("gqa_128k", {"n_tokens": 8192 + 1, "level_sizes": (8, 64), "needles": 0, "components": 256}),
    ("decode_10m_x4", {"n_tokens": 8192 + 2, "batch": 1, "level_sizes": (4, 16, 64), "needles": 0,
                       "components": 256, "decode_steps": 0}),
]


@pytest.mark.parametrize("name,over", CASES)
def test_banded_on_oracle_selections(name, over):
    """Consecutive query runs (from position 0, so sink and window overlap at
    first, and from inside the sequence with a ragged tail) on the oracle's
    selections."""
    w = WORKLOADS[name].scaled(**over)
    inp = make_inputs(w, seed=7)
    d = _dev(inp)
    Kls = TU.oracle_latents(inp, w)
    trees = TU.oracle_trees(Kls, w)
    Wm = inp["W"].double().numpy()
    n_end = w.n_tokens
    for q0, nq in [(0, 37), (n_end - 203, 203)]:
        sels = {}
        for h in range(w.hkv):
            qb = O.query_latent(TU.unit_queries(inp["Q"], 0, h, w.group, list(range(q0, q0 + nq))), Wm)
            sels[h] = [O.selection_tokens(O.select_blocks(trees[h], Kls[h], qb[k], q0 + k, w.beam, w.topk, w.window),
                                          q0 + k, w.sink, w.window, w.pool) for k in range(nq)]
        idx = torch.full((1, nq, w.hkv, w.max_sel), -1, dtype=torch.int32, device="cuda")
        cnt = torch.zeros((1, nq, w.hkv), dtype=torch.int32, device="cuda")
        for h in range(w.hkv):
            ii, cc = TU.rows_to_idx(sels[h], w.max_sel)
            idx[0, :, h] = ii
            cnt[0, :, h] = cc
        Qs = d["Q"][:, q0:q0 + nq].contiguous()
        O_, lse = lsa.lsa_sparse_attn_banded(Qs, d["K"], d["V"], idx, cnt, w.hkv, w.sink, w.window, q_pos0=q0)
        assert lsa.lsa_check(None) == lsa.LSA_OK
        want, wlse = _oracle_attn(inp, w, sels, q0, nq)
        _check(w, O_[0].double().cpu().numpy(), lse[0].double().cpu().numpy(), want, wlse)


@pytest.mark.parametrize("sink,window", [(0, 1), (4, 8), (40, 8), (0, 300), (7, 129)])
def test_banded_dense_causal(sink, window):
    """pool 1 and top-K >= N select every earlier token, so the banded result
    is dense causal attention (checked against a direct fp64 softmax)."""
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=333, pool=1, level_sizes=(2, 8), topk=4096, sink=sink,
                                     window=window, needles=0, components=16)
    inp = make_inputs(w, seed=8)
    d = _dev(inp)
    ix = lsa.lsa_build_index(TU.build_params(w), d["K"], d["W"])
    idx, cnt = lsa.lsa_select(ix, TU.select_params(w, beam=1024), d["Q"])
    O_, lse = lsa.lsa_sparse_attn_banded(d["Q"], d["K"], d["V"], idx, cnt, w.hkv, w.sink, w.window)
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    Kn = inp["K"][0].float().double().numpy()
    Vn = inp["V"][0].float().double().numpy()
    errs = []
    for i in range(0, w.n_tokens, 7):
        for h in range(w.hkv):
            assert idx[0, i, h, : cnt[0, i, h]].tolist() == list(range(i + 1))
            q = TU.unit_queries(inp["Q"], 0, h, w.group, [i])[0]
            s = q @ Kn[: i + 1, h].T / math.sqrt(w.d)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            dense = (p @ Vn[: i + 1, h]) / p.sum(axis=1, keepdims=True)
            got = O_[0, i, h * w.group:(h + 1) * w.group].double().cpu().numpy()
            errs.append(np.abs(got - dense).ravel())
    e = np.concatenate(errs)
    assert e.max() <= BF16_MAX_ABS and e.mean() <= BF16_MEAN_ABS
    ix.free()


def test_banded_rows_not_of_selection_form():
    """Ascending lists without the sink/window structure (and some with it)
    are attended whole: same result as the oracle on those lists."""
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=2048, level_sizes=(4, 16), needles=0, components=64)
    inp = make_inputs(w, seed=9)
    d = _dev(inp)
    rng = np.random.default_rng(9)
    q0, nq = 1500, 150
    sels = {}
    for h in range(w.hkv):
        rows = []
        for k in range(nq):
            i = q0 + k
            kind = k % 5
            if kind == 0:      # random subset of [0, i]
                s = np.unique(rng.integers(0, i + 1, rng.integers(1, 300)))
            elif kind == 1:    # selection form
                lo = max(w.sink, i - w.window + 1)
                mid = np.unique(rng.integers(w.sink, i - w.window + 1, 40)) if i - w.window + 1 > w.sink else []
                s = np.concatenate([np.arange(min(w.sink, i + 1)), mid, np.arange(lo, i + 1)])
            elif kind == 2:    # window only, no sink
                s = np.arange(max(0, i - w.window + 1), i + 1)
            elif kind == 3:    # sink only
                s = np.arange(min(w.sink, i + 1))
            else:              # empty row
                s = np.array([], dtype=np.int64)
            rows.append(np.asarray(s, dtype=np.int64))
        sels[h] = rows
    idx = torch.full((1, nq, w.hkv, w.max_sel + 300), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros((1, nq, w.hkv), dtype=torch.int32, device="cuda")
    for h in range(w.hkv):
        ii, cc = TU.rows_to_idx(sels[h], w.max_sel + 300)
        idx[0, :, h] = ii
        cnt[0, :, h] = cc
    Qs = d["Q"][:, q0:q0 + nq].contiguous()
    O_, lse = lsa.lsa_sparse_attn_banded(Qs, d["K"], d["V"], idx, cnt, w.hkv, w.sink, w.window, q_pos0=q0)
    assert lsa.lsa_check(None) == lsa.LSA_OK
    got = O_[0].double().cpu().numpy()
    glse = lse[0].double().cpu().numpy()
    empty = np.array([[len(sels[h][k]) == 0 for h in range(w.hkv)] for k in range(nq)])
    want, wlse = np.zeros_like(got), np.full_like(glse, -np.inf)
    nz = {h: [s if len(s) else np.array([0]) for s in sels[h]] for h in sels}
    w2, l2 = _oracle_attn(inp, w, nz, q0, nq)
    G = w.group
    for k in range(nq):
        for h in range(w.hkv):
            if not empty[k, h]:
                want[k, h * G:(h + 1) * G] = w2[k, h * G:(h + 1) * G]
                wlse[k, h * G:(h + 1) * G] = l2[k, h * G:(h + 1) * G]
    assert np.all(got[np.repeat(empty, G, axis=1)] == 0)
    assert np.all(np.isneginf(glse[np.repeat(empty, G, axis=1)]))
    ne = ~np.repeat(empty, G, axis=1)
    e = np.abs(got - want)[ne]
    assert e.max() <= BF16_MAX_ABS and e.mean() <= BF16_MEAN_ABS
    assert np.abs(glse[ne] - wlse[ne]).max() <= 1e-2


@pytest.mark.parametrize("name,over", [
    ("gqa_128k", {"n_tokens": 20000 + 5, "level_sizes": (8, 64), "needles": 4, "components": 256}),
    ("int_exact_16k", {}),
])
def test_banded_equals_generic_on_gpu_selection(name, over):
    """Every query of the sequence: banded and per-row attention over the
    GPU's own selection agree to rounding."""
    w = WORKLOADS[name].scaled(**over)
    inp = make_inputs(w, seed=10, device="cuda")
    ix = lsa.lsa_build_index(TU.build_params(w), inp["K"], inp["W"])
    idx, cnt = lsa.lsa_select(ix, TU.select_params(w), inp["Q"])
    O1, l1 = lsa.lsa_sparse_attn(inp["Q"], inp["K"], inp["V"], idx, cnt, w.hkv)
    O2, l2 = lsa.lsa_sparse_attn_banded(inp["Q"], inp["K"], inp["V"], idx, cnt, w.hkv, w.sink, w.window)
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    diff = (O1.float() - O2.float()).abs()
    ref = O1.float().abs()
    # two bf16 roundings of nearly the same fp32 value: within 2 ulps
    assert bool((diff <= ref * 2.0 ** -6 + 1e-3).all())
    assert float((l1 - l2).abs().max()) <= 1e-3
    ix.free()


def test_banded_argument_errors():
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=256, level_sizes=(2, 8), needles=0, components=16)
    inp = make_inputs(w, seed=11, device="cuda")
    idx = torch.zeros((1, 256, w.hkv, w.max_sel), dtype=torch.int32, device="cuda")
    cnt = torch.ones((1, 256, w.hkv), dtype=torch.int32, device="cuda")
    for kw in [dict(q_pos0=1), dict(q_pos0=-1)]:
        with pytest.raises(lsa.LsaError):
            lsa.lsa_sparse_attn_banded(inp["Q"], inp["K"], inp["V"], idx, cnt, w.hkv, w.sink, w.window, **kw)
    with pytest.raises(lsa.LsaError):
        lsa.lsa_sparse_attn_banded(inp["Q"], inp["K"], inp["V"], idx, cnt, w.hkv, w.sink, 0)
    with pytest.raises(lsa.LsaError):
        lsa.lsa_sparse_attn_banded(inp["Q"], inp["K"], inp["V"], idx, cnt, w.hkv, -1, w.window)
    assert lsa.lsa_check(None) == lsa.LSA_OK


def test_attention_rejects_unaligned_bf16_buffers():
    """bf16 attention moves rows in 16-byte pieces: a buffer that is not
    16-byte aligned is refused before anything is launched."""
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=256, level_sizes=(2, 8), needles=0, components=16)
    inp = make_inputs(w, seed=13, device="cuda")
    idx = torch.zeros((1, 256, w.hkv, w.max_sel), dtype=torch.int32, device="cuda")
    cnt = torch.ones((1, 256, w.hkv), dtype=torch.int32, device="cuda")
    K = inp["K"]
    flat = torch.empty(K.numel() + 4, dtype=K.dtype, device="cuda")
    Kmis = flat[4:].view(K.shape)          # 8-byte offset
    Kmis.copy_(K)
    with pytest.raises(lsa.LsaError):
        lsa.lsa_sparse_attn(inp["Q"], Kmis, inp["V"], idx, cnt, w.hkv)
    with pytest.raises(lsa.LsaError):
        lsa.lsa_sparse_attn_banded(inp["Q"], Kmis, inp["V"], idx, cnt, w.hkv, w.sink, w.window)
    assert lsa.lsa_check(None) == lsa.LSA_OK


def test_host_prefill_pipeline_matches_device_path():
    """The overlapped host-to-host layer (K, V, W up; Q up and O down in
    chunks around select + banded attention on three streams) gives the
    device path's output: the same selections, attention within 2 bf16 ulps
    (band tiles start at each chunk's first query)."""
    from hierarchical_latent_key_gemm_b200.pipeline import HostPrefill
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=6000 + 7, level_sizes=(8, 64), needles=0, components=256)
    inp = make_inputs(w, seed=14)
    hQ, hK, hV, hW = (inp[k].pin_memory() for k in ("Q", "K", "V", "W"))
    hO = torch.empty(hQ.shape, dtype=hQ.dtype, pin_memory=True)
    bp, sp = TU.build_params(w), TU.select_params(w)
    hp = HostPrefill(bp, sp, hQ, hK, hV, hW, hO, w.sink, w.window, chunks=5)
    for _ in range(2):
        hp.run().free()
        torch.cuda.synchronize()
    d = _dev(inp)
    ix = lsa.lsa_build_index(bp, d["K"], d["W"])
    idx, cnt = lsa.lsa_select(ix, sp, d["Q"])
    O_, _ = lsa.lsa_sparse_attn_banded(d["Q"], d["K"], d["V"], idx, cnt, w.hkv, w.sink, w.window)
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    ref = O_.float().cpu()
    got = hO.float()
    assert bool(((got - ref).abs() <= ref.abs() * 2.0 ** -6 + 1e-3).all())
    ix.free()


def test_host_prefill_c_entry_matches_the_stream_pipeline():
    """lsa_prefill_run (one C-ABI call from host buffers: copies overlapped
    with the build, select and banded attention in chunks) writes the same
    bits as the same layer driven from Python on three streams with the same
    chunks, on two runs of one context; its lse matches the device path's."""
    from hierarchical_latent_key_gemm_b200.pipeline import HostPrefill
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=6000 + 7, level_sizes=(8, 64), needles=0, components=256)
    inp = make_inputs(w, seed=15)
    hQ, hK, hV, hW = (inp[k].pin_memory() for k in ("Q", "K", "V", "W"))
    bp, sp = TU.build_params(w), TU.select_params(w)
    hO_py = torch.empty(hQ.shape, dtype=hQ.dtype, pin_memory=True)
    hp = HostPrefill(bp, sp, hQ, hK, hV, hW, hO_py, w.sink, w.window, chunks=5)
    hp.run().free()
    torch.cuda.synchronize()
    pf = lsa.Prefill(bp, sp, w.n_tokens, chunks=5)
    for _ in range(2):
        hO = torch.full(hQ.shape, float("nan"), dtype=hQ.dtype).pin_memory()
        hlse = torch.full((1, w.n_tokens, w.hq), float("nan")).pin_memory()
        ix = pf.run(hQ, hK, hV, hW, hO, hlse=hlse)
        torch.cuda.synchronize()
        assert lsa.lsa_check(ix) == lsa.LSA_OK
        ix.free()
        assert torch.equal(hO.view(torch.int16), hO_py.view(torch.int16))
    pf.free()
    d = _dev(inp)
    ix = lsa.lsa_build_index(bp, d["K"], d["W"])
    idx, cnt = lsa.lsa_select(ix, sp, d["Q"])
    _, lse = lsa.lsa_sparse_attn_banded(d["Q"], d["K"], d["V"], idx, cnt, w.hkv, w.sink, w.window)
    ix.free()
    ref = lse.cpu()
    assert bool(((hlse - ref).abs() <= 1e-3 * ref.abs() + 1e-3).all())


def test_select_and_banded_attention_capture_in_a_cuda_graph():
    """Selection runs on the device and every call is stream-ordered (scratch
    from the stream-ordered pool), so select + banded attention of a prefill
    can be captured in a CUDA graph; a replay writes the eager outputs bit for
    bit."""
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=20000 + 5, level_sizes=(8, 64), needles=0, components=256)
    inp = make_inputs(w, seed=30, device="cuda")
    bp, sp = TU.build_params(w), TU.select_params(w)
    ix = lsa.lsa_build_index(bp, inp["K"], inp["W"])
    idx = torch.empty((1, w.n_tokens, w.hkv, w.max_sel), dtype=torch.int32, device="cuda")
    cnt = torch.empty((1, w.n_tokens, w.hkv), dtype=torch.int32, device="cuda")
    O_ = torch.empty_like(inp["Q"])
    lse = torch.empty((1, w.n_tokens, w.hq), dtype=torch.float32, device="cuda")

    def run():
        lsa.lsa_select(ix, sp, inp["Q"], idx=idx, cnt=cnt)
        lsa.lsa_sparse_attn_banded(inp["Q"], inp["K"], inp["V"], idx, cnt, w.hkv, w.sink, w.window, O=O_, lse=lse)

    run()
    torch.cuda.synchronize()
    ref_o, ref_i, ref_c = O_.clone(), idx.clone(), cnt.clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run()
    O_.zero_()
    idx.zero_()
    cnt.zero_()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(O_, ref_o) and torch.equal(idx, ref_i) and torch.equal(cnt, ref_c)
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    del g
    ix.free()


def test_decode_graph_steps_match_plain_calls():
    """Decode with the captured select + attention graph gives, step by step,
    the rows and outputs of the plain calls (appends cross several blocks)."""
    from hierarchical_latent_key_gemm_b200.pipeline import DecodeStep
    w = WORKLOADS["decode_10m_x4"].scaled(n_tokens=8192 + 2, batch=2, level_sizes=(4, 16, 64), needles=0,
                                          components=256, decode_steps=24)
    inp = make_inputs(w, seed=31, device="cuda")
    bp = TU.build_params(w, append_capacity=w.decode_steps)
    sp = TU.select_params(w)
    ix_a = lsa.lsa_build_index(bp, inp["K"], inp["W"])
    ix_b = lsa.lsa_build_index(bp, inp["K"], inp["W"])
    ds = DecodeStep(ix_b, sp, inp["K"], inp["V"], w.hq, w.max_sel)
    for s in range(w.decode_steps):
        t = w.n_tokens + s
        q = inp["Q"][:, s:s + 1].contiguous()
        lsa.lsa_append(ix_a, inp["K"], 1)
        ia, ca = lsa.lsa_select(ix_a, sp, q, q_pos0=t, max_sel=w.max_sel)
        oa, la = lsa.lsa_sparse_attn(q, inp["K"], inp["V"], ia, ca, w.hkv)
        ob, lb = ds.step(q, t)
        torch.cuda.synchronize()
        assert torch.equal(ia, ds.idx) and torch.equal(ca, ds.cnt), f"step {s}"
        assert torch.equal(oa, ob) and torch.equal(la, lb), f"step {s}"
    assert lsa.lsa_check(ix_a) == lsa.LSA_OK and lsa.lsa_check(ix_b) == lsa.LSA_OK
    del ds
    ix_a.free()
    ix_b.free()
