"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/lsa.h declares, and the binding's structs match the C
layout (compiled here with gcc)."""
import ctypes as C
import os
import subprocess
import tempfile

import pytest

from hierarchical_latent_key_gemm_b200 import lsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lsa.h")


def test_library_exports_every_declared_symbol():
    L = lsa.lib()
    names = lsa.exported_symbols_from_header(HEADER)
    assert len(names) >= 15
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing
    # the binding declares a signature for each of them
    assert sorted(names) == sorted(lsa._SIGS)


def test_status_strings_and_null_handles():
    for s in range(8):
        assert lsa.strerror(s) and lsa.strerror(s) != "unknown status"
    assert lsa.strerror(99) == "unknown status"
    L = lsa.lib()
    info = lsa.IndexInfo()
    assert L.lsa_index_info(None, C.byref(info)) == lsa.LSA_ERR_INVALID_ARG
    L.lsa_free_index(None)  # no-op
    bogus = C.c_void_p(0x1234)
    L.lsa_free_index(bogus)  # not a live index: ignored, never dereferenced
    assert L.lsa_index_info(bogus, C.byref(info)) == lsa.LSA_ERR_INVALID_ARG
    # index upkeep refuses handles that are not live indexes before any CUDA call
    for f in (L.lsa_relayout, L.lsa_refresh_centroids):
        assert f(None, None) == lsa.LSA_ERR_INVALID_ARG
        assert f(bogus, None) == lsa.LSA_ERR_INVALID_ARG


def test_struct_layout_matches_c_header():
    src = r'''
#include <stddef.h>
#include <stdio.h>
#include "lsa.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu\n", sizeof(lsa_build_params), offsetof(lsa_build_params, level_sizes),
         offsetof(lsa_build_params, append_capacity), sizeof(lsa_select_params), sizeof(lsa_index_info_t));
  printf("%zu %zu\n", offsetof(lsa_index_info_t, level_sizes), offsetof(lsa_index_info_t, grid_log2));
  return 0;
}
'''
    with tempfile.TemporaryDirectory() as td:
        c = os.path.join(td, "t.c")
        exe = os.path.join(td, "t")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-I", os.path.dirname(HEADER), c, "-o", exe], check=True)
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split()
    got = [int(x) for x in out]
    want = [C.sizeof(lsa.BuildParams), lsa.BuildParams.level_sizes.offset, lsa.BuildParams.append_capacity.offset,
            C.sizeof(lsa.SelectParams), C.sizeof(lsa.IndexInfo), lsa.IndexInfo.level_sizes.offset,
            lsa.IndexInfo.grid_log2.offset]
    assert got == want


def test_binding_rejects_host_tensors():
    import torch
    with pytest.raises(ValueError):
        lsa._ptr(torch.zeros(4))


def test_binding_checks_element_types_before_the_call():
    """The binding refuses tensors of the wrong element type (the C ABI takes
    untyped pointers) before anything reaches the library."""
    import torch
    with pytest.raises(ValueError, match="idx must be torch.int32"):
        lsa._typed(torch.zeros(4, dtype=torch.int64), torch.int32, "idx")
    assert lsa._typed(None, torch.int32, "idx") is None
    q = torch.zeros(1, 2, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="share one dtype"):
        lsa._same_dtype(q, q.float(), q, None)
    with pytest.raises(ValueError, match="unsupported dtype"):
        lsa._same_dtype(q.half(), q.half(), q.half(), None)
    lsa._same_dtype(q, q, q, None)
    bp = lsa.make_build_params(1, 8, 8, 1, 64, 16, 1, lsa.LSA_BF16, (2, 4), 1, 0, 0, 0)
    with pytest.raises(ValueError, match="build parameters"):
        lsa.lsa_build_index(bp, torch.zeros(1, 8, 1, 64, dtype=torch.float32), torch.zeros(64, 16))


def test_binding_checks_shapes_before_the_call():
    """The C ABI cannot see buffer sizes, so the binding checks every shape
    against the index and the call's parameters before the library is called:
    a mismatched tensor raises instead of reaching a kernel as an
    out-of-bounds read or write.  (Host tensors: each case must fail on its
    shape, before the device-pointer check.)"""
    import torch
    bp = lsa.make_build_params(1, 64, 64, 2, 64, 16, 1, lsa.LSA_BF16, (2, 4), 1, 0, 0, 0)
    ix = lsa.Index(C.c_void_p(None), bp)
    sp = lsa.make_select_params(4, 2, 8, 0, 4)
    bf = torch.bfloat16
    Q = torch.zeros(1, 8, 4, 64, dtype=bf)
    ms = 8 + 0 + 4
    idx = torch.zeros(1, 8, 2, ms, dtype=torch.int32)
    cnt = torch.zeros(1, 8, 2, dtype=torch.int32)
    cases = [
        (dict(Q=torch.zeros(1, 8, 3, 64, dtype=bf)), "Q must have shape"),
        (dict(Q=torch.zeros(2, 8, 4, 64, dtype=bf)), "Q must have shape"),
        (dict(Q=torch.zeros(1, 8, 4, 128, dtype=bf)), "Q must have shape"),
        (dict(Q=Q.float()), "built for dtype"),
        (dict(idx=torch.zeros(1, 7, 2, ms, dtype=torch.int32)), "idx must have shape"),
        (dict(idx=torch.zeros(1, 8, 1, ms, dtype=torch.int32)), "idx must have shape"),
        (dict(cnt=torch.zeros(1, 8, 1, dtype=torch.int32)), "cnt must have shape"),
        (dict(cnt=torch.zeros(1, 8, 2, dtype=torch.int64)), "cnt must be"),
        (dict(q_pos=torch.zeros(1, 9, dtype=torch.int64)), "q_pos must have shape"),
        (dict(q_pos=torch.zeros(1, 8, dtype=torch.int32)), "q_pos must be"),
    ]
    for over, msg in cases:
        a = dict(Q=Q, idx=idx, cnt=cnt, q_pos=None)
        a.update(over)
        with pytest.raises(ValueError, match=msg):
            lsa.lsa_select(ix, sp, a["Q"], idx=a["idx"], cnt=a["cnt"], q_pos=a["q_pos"])
        with pytest.raises(ValueError, match=msg):
            lsa.lsa_select_noalloc(ix, sp, a["Q"], a["idx"], a["cnt"], q_pos=a["q_pos"])
    # well-formed host tensors get past the shape checks and stop at the
    # device-pointer check
    with pytest.raises(ValueError, match="CUDA device"):
        lsa.lsa_select(ix, sp, Q, idx=idx, cnt=cnt)
    # attention
    K = torch.zeros(1, 64, 2, 64, dtype=bf)
    O = torch.zeros_like(Q)
    lse = torch.zeros(1, 8, 4)
    att = [
        (dict(K=torch.zeros(1, 64, 1, 64, dtype=bf)), "K must have shape"),
        (dict(V=torch.zeros(1, 63, 2, 64, dtype=bf)), "V must have shape"),
        (dict(idx=torch.zeros(1, 8, 1, ms, dtype=torch.int32)), "idx must have shape"),
        (dict(cnt=torch.zeros(1, 7, 2, dtype=torch.int32)), "cnt must have shape"),
        (dict(O=torch.zeros(1, 8, 4, 32, dtype=bf)), "O must have shape"),
        (dict(lse=torch.zeros(1, 8, 2)), "lse must have shape"),
        (dict(lse=torch.zeros(1, 8, 4, dtype=torch.float64)), "lse must be"),
        (dict(V=K.float()), "share one dtype"),
    ]
    for over, msg in att:
        a = dict(Q=Q, K=K, V=K, idx=idx, cnt=cnt, O=O, lse=lse)
        a.update(over)
        for fn in (lambda a: lsa.lsa_sparse_attn(a["Q"], a["K"], a["V"], a["idx"], a["cnt"], 2, O=a["O"],
                                                 lse=a["lse"]),
                   lambda a: lsa.lsa_sparse_attn_banded(a["Q"], a["K"], a["V"], a["idx"], a["cnt"], 2, 0, 4,
                                                        O=a["O"], lse=a["lse"])):
            with pytest.raises(ValueError, match=msg):
                fn(a)


def test_host_prefill_refuses_bad_arguments_before_any_cuda_call():
    """lsa_prefill_create / run check their arguments on the host first
    (batch 1, 1 <= nq <= n_tokens, chunks >= 1, hq a multiple of hkv, a valid
    dtype, non-null buffers), and the binding checks the host tensors' types
    and shapes before the call."""
    import torch
    L = lsa.lib()
    bp = lsa.make_build_params(1, 64, 64, 2, 64, 16, 1, lsa.LSA_BF16, (2, 4), 1, 0, 0, 0)
    sp = lsa.make_select_params(4, 2, 8, 0, 4)
    out = C.c_void_p(0x1)
    for over, nq, chunks in ((dict(batch=2), 64, 4), ({}, 0, 4), ({}, 65, 4), ({}, 64, 0),
                             (dict(dtype=7), 64, 4), (dict(ld_tokens=32), 64, 4)):
        b = lsa.BuildParams.from_buffer_copy(bp)
        for k, v in over.items():
            setattr(b, k, v)
        assert L.lsa_prefill_create(C.byref(b), C.byref(sp), nq, chunks, C.byref(out)) == lsa.LSA_ERR_INVALID_ARG
        assert not out.value
        out = C.c_void_p(0x1)
    sp3 = lsa.SelectParams.from_buffer_copy(sp)
    sp3.hq = 3
    assert L.lsa_prefill_create(C.byref(bp), C.byref(sp3), 64, 4, C.byref(out)) == lsa.LSA_ERR_INVALID_ARG
    h = C.c_void_p()
    assert L.lsa_prefill_run(None, None, None, None, None, None, None, None, C.byref(h)) == lsa.LSA_ERR_INVALID_ARG
    assert not h.value
    L.lsa_prefill_free(None)   # no-op
    # the binding: host tensors of the right type and shape only
    pf = lsa.Prefill.__new__(lsa.Prefill)
    pf.params, pf.sp, pf.nq, pf.handle = bp, sp, 64, C.c_void_p(None)
    bf = torch.bfloat16
    ok = dict(hQ=torch.zeros(1, 64, 4, 64, dtype=bf), hK=torch.zeros(1, 64, 2, 64, dtype=bf),
              hV=torch.zeros(1, 64, 2, 64, dtype=bf), hW=torch.zeros(64, 16), hO=torch.zeros(1, 64, 4, 64, dtype=bf))
    cases = [
        (dict(hQ=torch.zeros(1, 63, 4, 64, dtype=bf)), "hQ must have shape"),
        (dict(hK=torch.zeros(1, 64, 2, 64)), "hK must be"),
        (dict(hV=torch.zeros(1, 64, 1, 64, dtype=bf)), "hV must have shape"),
        (dict(hW=torch.zeros(64, 32)), "hW must have shape"),
        (dict(hO=torch.zeros(1, 64, 4, 64, dtype=bf)[:, ::2]), "hO must be contiguous"),
        (dict(hlse=torch.zeros(1, 64, 2)), "hlse must have shape"),
    ]
    for over, msg in cases:
        a = dict(ok, hlse=None)
        a.update(over)
        with pytest.raises(ValueError, match=msg):
            pf.run(a["hQ"], a["hK"], a["hV"], a["hW"], a["hO"], hlse=a["hlse"], stream=0)
