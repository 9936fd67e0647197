"""Allocation-free selection (lsa_select_noalloc), for callers that cannot
allocate device memory while they serve.  Called through the C ABI; its
output must equal lsa_select's (bit-exact, the same kernels), on two calls in
a row that share the fixed buffer.  Kept in its own file so it runs last."""
import ctypes as C

import pytest
import torch

from hierarchical_latent_key_gemm_b200 import lsa
from hierarchical_latent_key_gemm_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def test_select_noalloc_matches_select_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    L = lsa.lib()
    w = WORKLOADS["prefill_1m"].scaled(n_tokens=16384 + 7, level_sizes=(4, 32, 256), beam=16, topk=512,
                                       window=256, needles=0, components=256, drift_every=4096)
    inp = make_inputs(w, seed=31)
    K, Q, W = inp["K"].cuda(), inp["Q"].cuda(), inp["W"].cuda()
    bp = lsa.make_build_params(1, w.n_tokens, w.n_tokens, w.hkv, w.d, w.r, w.pool, lsa.LSA_BF16, w.level_sizes,
                               w.lloyd_iters, w.grid_log2, w.sink)
    sp = lsa.make_select_params(w.hq, w.beam, w.topk, w.sink, w.window)
    ix = lsa.lsa_build_index(bp, K, W)
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    nq = 4096  # 1 x 4096 x 2 x 64 = 524,288 floats: inside the fixed buffer
    for q0 in (1000, 9000):
        Qc = Q[:, q0:q0 + nq].contiguous()
        ref_idx, ref_cnt = lsa.lsa_select(ix, sp, Qc, q_pos0=q0)
        idx = torch.full_like(ref_idx, -7)
        cnt = torch.full_like(ref_cnt, -7)
        st = L.lsa_select_noalloc(ix.handle, C.byref(sp), C.c_void_p(Qc.data_ptr()), nq, None, q0,
                                  C.c_void_p(idx.data_ptr()), C.c_void_p(cnt.data_ptr()), idx.shape[-1], stream)
        assert st == lsa.LSA_OK, lsa.strerror(st)
        assert lsa.lsa_check(ix) == lsa.LSA_OK
        assert torch.equal(cnt, ref_cnt)
        assert torch.equal(idx, ref_idx)
    # it allocates nothing: with the library's next device allocation set to
    # fail, lsa_select_noalloc still succeeds with the same rows, while
    # lsa_select (which takes its scratch from the pool) reports the failure
    Qc = Q[:, 1000:1000 + nq].contiguous()
    ref_idx, ref_cnt = lsa.lsa_select(ix, sp, Qc, q_pos0=1000)
    idx = torch.full_like(ref_idx, -7)
    cnt = torch.full_like(ref_cnt, -7)
    lsa.lsa_debug_fail_alloc_after(1)
    try:
        st = L.lsa_select_noalloc(ix.handle, C.byref(sp), C.c_void_p(Qc.data_ptr()), nq, None, 1000,
                                  C.c_void_p(idx.data_ptr()), C.c_void_p(cnt.data_ptr()), idx.shape[-1], stream)
        assert st == lsa.LSA_OK, lsa.strerror(st)
        st = L.lsa_select(ix.handle, C.byref(sp), C.c_void_p(Qc.data_ptr()), nq, None, 1000,
                          C.c_void_p(idx.data_ptr()), C.c_void_p(cnt.data_ptr()), idx.shape[-1], stream)
        assert st == lsa.LSA_ERR_OOM
    finally:
        lsa.lsa_debug_fail_alloc_after(0)
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    assert torch.equal(cnt, ref_cnt) and torch.equal(idx, ref_idx)
    # a request beyond the fixed buffer is refused before anything runs
    big = Q[:, :9000].contiguous()  # 9000 x 2 x 64 = 1,152,000 floats
    bidx = torch.empty((1, 9000, w.hkv, w.max_sel), dtype=torch.int32, device="cuda")
    bcnt = torch.empty((1, 9000, w.hkv), dtype=torch.int32, device="cuda")
    st = L.lsa_select_noalloc(ix.handle, C.byref(sp), C.c_void_p(big.data_ptr()), 9000, None, 0,
                              C.c_void_p(bidx.data_ptr()), C.c_void_p(bcnt.data_ptr()), w.max_sel, stream)
    assert st == lsa.LSA_ERR_INVALID_ARG
    ix.free()
