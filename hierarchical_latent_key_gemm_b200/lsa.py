"""Python binding of liblsa.so (the C ABI declared in include/lsa.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors are torch tensors used as device memory; the stream is
torch's current stream unless one is given.  The binding refuses to run
without the compiled library (there is no fallback).
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblsa.so")

LSA_OK, LSA_ERR_INVALID_ARG, LSA_ERR_CUDA, LSA_ERR_OOM = 0, 1, 2, 3
LSA_ERR_INEXACT, LSA_ERR_TIMEOUT, LSA_ERR_DEVICE, LSA_ERR_CAPACITY = 4, 5, 6, 7
LSA_F32, LSA_BF16 = 0, 1
LSA_MAX_LEVELS = 4
(LSA_GET_CENTROIDS, LSA_GET_PARENT, LSA_GET_LEAF_OF_BLOCK, LSA_GET_MINPOS,
 LSA_GET_OBJECTIVE, LSA_GET_LATENT, LSA_GET_LEAF_COUNT) = range(7)


class LsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {strerror(status)} (status {status})")


class BuildParams(C.Structure):
    _fields_ = [("batch", C.c_int64), ("n_tokens", C.c_int64), ("ld_tokens", C.c_int64),
                ("hkv", C.c_int32), ("d", C.c_int32), ("r", C.c_int32), ("pool", C.c_int32),
                ("dtype", C.c_int32), ("levels", C.c_int32), ("level_sizes", C.c_int32 * LSA_MAX_LEVELS),
                ("lloyd_iters", C.c_int32), ("grid_log2", C.c_int32), ("sink", C.c_int32),
                ("append_capacity", C.c_int64)]


class SelectParams(C.Structure):
    _fields_ = [("hq", C.c_int32), ("beam", C.c_int32), ("topk", C.c_int32), ("sink", C.c_int32),
                ("window", C.c_int32)]


class IndexInfo(C.Structure):
    _fields_ = [("units", C.c_int64), ("n_tokens", C.c_int64), ("n_blocks", C.c_int64),
                ("block_capacity", C.c_int64), ("device_bytes", C.c_int64), ("levels", C.c_int32),
                ("level_sizes", C.c_int32 * LSA_MAX_LEVELS), ("r", C.c_int32), ("pool", C.c_int32),
                ("sink", C.c_int32), ("grid_log2", C.c_int32)]


_vp, _i64, _i32 = C.c_void_p, C.c_int64, C.c_int32
_SIGS = {
    "lsa_build_index": (_i32, [C.POINTER(BuildParams), _vp, _vp, _vp, C.POINTER(_vp)]),
    "lsa_build_index_from_tree": (_i32, [C.POINTER(BuildParams), _vp, _vp, _vp, C.POINTER(_vp), C.POINTER(_vp),
                                         _vp, C.POINTER(_vp)]),
    "lsa_select": (_i32, [_vp, C.POINTER(SelectParams), _vp, _i64, _vp, _i64, _vp, _vp, _i32, _vp]),
    "lsa_fullscan_select": (_i32, [_vp, C.POINTER(SelectParams), _vp, _i64, _vp, _i64, _vp, _vp, _i32, _vp]),
    "lsa_select_work": (_i32, [_vp, C.POINTER(SelectParams), _vp, _i64, _vp, _i64, _vp, _vp, _i32, _vp, _vp]),
    "lsa_select_noalloc": (_i32, [_vp, C.POINTER(SelectParams), _vp, _i64, _vp, _i64, _vp, _vp, _i32, _vp]),
    "lsa_sparse_attn": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i32, _i32, _i32, _i32, _i32, _i64, _vp, _vp,
                               _vp]),
    "lsa_sparse_attn_banded": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32, _i32, _i32,
                                      _i64, _i32, _i32, _vp, _vp, _vp]),
    "lsa_append": (_i32, [_vp, _vp, _i64, _vp]),
    "lsa_relayout": (_i32, [_vp, _vp]),
    "lsa_refresh_centroids": (_i32, [_vp, _vp]),
    "lsa_pca_map": (_i32, [_vp, _i64, _i64, _i64, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "lsa_project_pool": (_i32, [_vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32, _i32, _i32, _vp, _vp]),
    "lsa_query_latent": (_i32, [_vp, _vp, _i64, _i64, _i32, _i32, _i32, _i32, _i32, _vp, _vp]),
    "lsa_kmeans": (_i32, [_vp, _i64, _i64, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp]),
    "lsa_index_get": (_i32, [_vp, _i32, _i32, _vp, _i64, _vp]),
    "lsa_index_info": (_i32, [_vp, C.POINTER(IndexInfo)]),
    "lsa_check": (_i32, [_vp, _vp]),
    "lsa_free_index": (None, [_vp]),
    "lsa_strerror": (C.c_char_p, [_i32]),
    "lsa_debug_fail_alloc_after": (None, [_i32]),
    "lsa_debug_dense_config": (None, [_i64, _i64]),
    "lsa_debug_leaf_tiles": (None, [_i32]),
    "lsa_launch_count": (_i64, []),
    "lsa_select_blocks": (_i32, [_vp, C.POINTER(SelectParams), _vp, _i64, _vp, _i64, _i64, _vp, _vp, _vp, _i32,
                                 _vp]),
    "lsa_merge_selection": (_i32, [_i32, _vp, _vp, _vp, _i32, _i64, _i64, _i32, _vp, _i64, _i32, _i32, _i32, _i32,
                                   _vp, _vp, _i32, _vp]),
    "lsa_localize_rows": (_i32, [_vp, _vp, _i64, _i32, _i64, _i64, _vp, _vp, _vp]),
    "lsa_merge_attn": (_i32, [_i32, _vp, _vp, _i64, _i32, _i32, _i32, _vp, _vp, _vp]),
    "lsa_prefill_create": (_i32, [C.POINTER(BuildParams), C.POINTER(SelectParams), _i64, _i32, _vp]),
    "lsa_prefill_run": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "lsa_prefill_free": (None, [_vp]),
}

_lib = None


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m hierarchical_latent_key_gemm_b200.build` "
                               "(the LSA path has no CPU fallback)")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def strerror(status: int) -> str:
    return lib().lsa_strerror(int(status)).decode()


def _ok(status, where):
    if status != LSA_OK:
        raise LsaError(status, where)


def _stream(stream):
    if stream is None:
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return C.c_void_p(stream.cuda_stream)
    return C.c_void_p(int(stream))


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return C.c_void_p(t.data_ptr())


def _same_dtype(*ts):
    """Q, K, V and O share one element type (float32 or bfloat16)."""
    dt = ts[0].dtype
    dtype_code(ts[0])
    for t in ts[1:]:
        if t is not None and t.dtype != dt:
            raise ValueError(f"Q, K, V and O must share one dtype, got {dt} and {t.dtype}")


def _typed(t, dtype, name):
    """_ptr after checking the element type the C call expects."""
    if t is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return _ptr(t)


def dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return LSA_F32
    if t.dtype == torch.bfloat16:
        return LSA_BF16
    raise ValueError(f"unsupported dtype {t.dtype}")


@dataclass
class Index:
    """Owner of an lsa_index handle (freed by free() or garbage collection)."""
    handle: C.c_void_p
    params: BuildParams

    def free(self):
        if self.handle:
            lib().lsa_free_index(self.handle)
            self.handle = C.c_void_p(None)

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass

    def info(self) -> IndexInfo:
        out = IndexInfo()
        _ok(lib().lsa_index_info(self.handle, C.byref(out)), "lsa_index_info")
        return out

    def get(self, what: int, level: int = 0, device="cuda") -> torch.Tensor:
        """Copy one index array out (see LSA_GET_*)."""
        inf = self.info()
        U, r, nb = inf.units, inf.r, inf.n_blocks
        sizes = list(inf.level_sizes)[: inf.levels]
        L = sizes[-1]
        it = self.params.lloyd_iters
        shape, dt = {
            LSA_GET_CENTROIDS: ((U, sizes[level], r), torch.float32),
            LSA_GET_PARENT: ((U, sizes[level]), torch.int32),
            LSA_GET_LEAF_OF_BLOCK: ((U, nb), torch.int32),
            LSA_GET_MINPOS: ((U, sizes[level]), torch.int64),
            LSA_GET_OBJECTIVE: ((it, U), torch.float64),
            LSA_GET_LATENT: ((U, nb, r), torch.float32),
            LSA_GET_LEAF_COUNT: ((U, L), torch.int32),
        }[what]
        out = torch.empty(shape, dtype=dt, device=device)
        nbytes = out.numel() * out.element_size()
        _ok(lib().lsa_index_get(self.handle, what, level, C.c_void_p(out.data_ptr()), nbytes, _stream(None)),
            "lsa_index_get")
        return out


def make_build_params(batch, n_tokens, ld_tokens, hkv, d, r, pool, dtype, level_sizes, lloyd_iters, grid_log2,
                      sink, append_capacity=0) -> BuildParams:
    p = BuildParams()
    p.batch, p.n_tokens, p.ld_tokens = int(batch), int(n_tokens), int(ld_tokens)
    p.hkv, p.d, p.r, p.pool, p.dtype = int(hkv), int(d), int(r), int(pool), int(dtype)
    p.levels = len(level_sizes)
    for i, s in enumerate(level_sizes):
        p.level_sizes[i] = int(s)
    p.lloyd_iters, p.grid_log2, p.sink = int(lloyd_iters), int(grid_log2), int(sink)
    p.append_capacity = int(append_capacity)
    return p


def make_select_params(hq, beam, topk, sink, window) -> SelectParams:
    s = SelectParams()
    s.hq, s.beam, s.topk, s.sink, s.window = int(hq), int(beam), int(topk), int(sink), int(window)
    return s


def _check_keys(params: BuildParams, K: torch.Tensor):
    if dtype_code(K) != params.dtype:
        raise ValueError(f"K is {K.dtype} but the build parameters say dtype {params.dtype}")


def lsa_build_index(params: BuildParams, K: torch.Tensor, W: torch.Tensor, stream=None) -> Index:
    h = C.c_void_p()
    _check_keys(params, K)
    _ok(lib().lsa_build_index(C.byref(params), _ptr(K), _typed(W, torch.float32, "W"), _stream(stream), C.byref(h)),
        "lsa_build_index")
    return Index(h, params)


def lsa_build_index_from_tree(params: BuildParams, K, W, leaf_of_block, parents, centroids, stream=None) -> Index:
    """parents[l] for l >= 1 and centroids[l] for every level are device tensors."""
    L = params.levels
    par = (C.c_void_p * L)(*([None] + [C.c_void_p(parents[l].data_ptr()) for l in range(1, L)]))
    cen = (C.c_void_p * L)(*[C.c_void_p(centroids[l].data_ptr()) for l in range(L)])
    _check_keys(params, K)
    for t in parents[1:]:
        _typed(t, torch.int32, "parents")
    for t in centroids:
        _typed(t, torch.float32, "centroids")
    _typed(leaf_of_block, torch.int32, "leaf_of_block")
    _typed(W, torch.float32, "W")
    h = C.c_void_p()
    _ok(lib().lsa_build_index_from_tree(C.byref(params), _ptr(K), _ptr(W), _ptr(leaf_of_block), par, cen,
                                        _stream(stream), C.byref(h)), "lsa_build_index_from_tree")
    return Index(h, params)


def _shape(t, want, name):
    if t is not None and tuple(t.shape) != tuple(int(x) for x in want):
        raise ValueError(f"{name} must have shape {tuple(int(x) for x in want)}, got {tuple(t.shape)}")


def _check_select_args(p, sp, Q, q_pos, idx, cnt, max_sel):
    """The C ABI takes untyped pointers and cannot see sizes: every buffer's
    element type and shape is checked here, before anything is enqueued, so a
    wrong tensor is an error and never an out-of-bounds device access."""
    if Q.dim() != 4:
        raise ValueError(f"Q must be [batch, nq, hq, d], got shape {tuple(Q.shape)}")
    if dtype_code(Q) != p.dtype:
        raise ValueError(f"Q is {Q.dtype} but the index was built for dtype {p.dtype}")
    nq = Q.shape[1]
    _shape(Q, (p.batch, nq, sp.hq, p.d), "Q")
    _shape(q_pos, (p.batch, nq), "q_pos")
    _shape(idx, (p.batch, nq, p.hkv, max_sel), "idx")
    _shape(cnt, (p.batch, nq, p.hkv), "cnt")
    for t, dt, nm in ((q_pos, torch.int64, "q_pos"), (idx, torch.int32, "idx"), (cnt, torch.int32, "cnt")):
        if t is not None and t.dtype != dt:
            raise ValueError(f"{nm} must be {dt}, got {t.dtype}")


def _select(fn, name, index, sp, Q, q_pos=None, q_pos0=0, idx=None, cnt=None, max_sel=None, stream=None):
    p = index.params
    B, nq = Q.shape[0], Q.shape[1]
    kb = -(-sp.topk // p.pool)
    if max_sel is None:
        max_sel = idx.shape[-1] if idx is not None else kb * p.pool + p.sink + sp.window
    _check_select_args(p, sp, Q, q_pos, idx, cnt, max_sel)
    if idx is None:
        idx = torch.empty((B, nq, p.hkv, max_sel), dtype=torch.int32, device=Q.device)
    if cnt is None:
        cnt = torch.empty((B, nq, p.hkv), dtype=torch.int32, device=Q.device)
    st = fn(index.handle, C.byref(sp), _ptr(Q), int(nq), _typed(q_pos, torch.int64, "q_pos"), int(q_pos0),
            _typed(idx, torch.int32, "idx"), _typed(cnt, torch.int32, "cnt"), int(max_sel), _stream(stream))
    _ok(st, name)
    return idx, cnt


def lsa_select(index, sp, Q, **kw):
    return _select(lib().lsa_select, "lsa_select", index, sp, Q, **kw)


LSA_SELECT_NOALLOC_MAX_FLOATS = 1 << 20


def lsa_select_noalloc(index, sp, Q, idx, cnt, q_pos=None, q_pos0=0, stream=None):
    """Allocation-free selection: the caller passes idx and cnt, and the latent
    queries use the library's fixed 4 MiB device buffer (see include/lsa.h).
    batch * nq * hkv * r must not exceed LSA_SELECT_NOALLOC_MAX_FLOATS."""
    p = index.params
    _check_select_args(p, sp, Q, q_pos, idx, cnt, idx.shape[-1])
    need = p.batch * Q.shape[1] * p.hkv * p.r
    if need > LSA_SELECT_NOALLOC_MAX_FLOATS:
        raise ValueError(f"lsa_select_noalloc: {need} latent-query floats exceed the fixed buffer of "
                         f"{LSA_SELECT_NOALLOC_MAX_FLOATS}; select in smaller query chunks")
    st = lib().lsa_select_noalloc(index.handle, C.byref(sp), _ptr(Q), int(Q.shape[1]),
                                  _typed(q_pos, torch.int64, "q_pos"), int(q_pos0), _typed(idx, torch.int32, "idx"),
                                  _typed(cnt, torch.int32, "cnt"), int(idx.shape[-1]), _stream(stream))
    _ok(st, "lsa_select_noalloc")
    return idx, cnt


def lsa_select_work(index, sp, Q, q_pos=None, q_pos0=0, idx=None, cnt=None, max_sel=None, stream=None):
    """lsa_select plus the numbers of eligible tree nodes and of candidate
    blocks whose latent rows were scored: returns (idx, cnt, nodes, blocks),
    the counts as Python ints (synchronises the stream)."""
    scored = torch.zeros(2, dtype=torch.int64, device=Q.device)

    def fn(h, spp, q, nq, qp, qp0, ii, cc, ms, st):
        return lib().lsa_select_work(h, spp, q, nq, qp, qp0, ii, cc, ms, _ptr(scored), st)

    idx, cnt = _select(fn, "lsa_select_work", index, sp, Q, q_pos=q_pos, q_pos0=q_pos0, idx=idx, cnt=cnt,
                       max_sel=max_sel, stream=stream)
    return idx, cnt, int(scored[0].item()), int(scored[1].item())


def lsa_fullscan_select(index, sp, Q, **kw):
    return _select(lib().lsa_fullscan_select, "lsa_fullscan_select", index, sp, Q, **kw)


def _check_attn_args(Q, K, V, idx, cnt, hkv, O, lse):
    """Shapes and element types of an attention call (see _check_select_args)."""
    if Q.dim() != 4 or K.dim() != 4:
        raise ValueError("Q must be [batch, nq, hq, d] and K, V [batch, ld_tokens, hkv, d]")
    B, nq, hq, d = Q.shape
    _shape(K, (B, K.shape[1], hkv, d), "K")
    _shape(V, tuple(K.shape), "V")
    if idx.dim() != 4:
        raise ValueError(f"idx must be [batch, nq, hkv, max_sel], got shape {tuple(idx.shape)}")
    _shape(idx, (B, nq, hkv, idx.shape[-1]), "idx")
    _shape(cnt, (B, nq, hkv), "cnt")
    _shape(O, tuple(Q.shape), "O")
    _shape(lse, (B, nq, hq), "lse")
    _same_dtype(Q, K, V, O)
    for t, dt, nm in ((idx, torch.int32, "idx"), (cnt, torch.int32, "cnt"), (lse, torch.float32, "lse")):
        if t is not None and t.dtype != dt:
            raise ValueError(f"{nm} must be {dt}, got {t.dtype}")


def lsa_sparse_attn(Q, K, V, idx, cnt, hkv, O=None, lse=None, want_lse=True, stream=None):
    _check_attn_args(Q, K, V, idx, cnt, hkv, O, lse)
    B, nq, hq, d = Q.shape
    ld_tokens = K.shape[1]
    max_sel = idx.shape[-1]
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty((B, nq, hq), dtype=torch.float32, device=Q.device)
    st = lib().lsa_sparse_attn(_ptr(Q), _ptr(K), _ptr(V), _typed(idx, torch.int32, "idx"),
                               _typed(cnt, torch.int32, "cnt"), int(B), int(nq), int(hq), int(hkv),
                               int(d), dtype_code(Q), int(max_sel), int(ld_tokens), _ptr(O),
                               _typed(lse, torch.float32, "lse"), _stream(stream))
    _ok(st, "lsa_sparse_attn")
    return O, lse


def lsa_sparse_attn_banded(Q, K, V, idx, cnt, hkv, sink, window, q_pos0=0, O=None, lse=None, want_lse=True,
                           stream=None):
    _check_attn_args(Q, K, V, idx, cnt, hkv, O, lse)
    B, nq, hq, d = Q.shape
    ld_tokens = K.shape[1]
    max_sel = idx.shape[-1]
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty((B, nq, hq), dtype=torch.float32, device=Q.device)
    st = lib().lsa_sparse_attn_banded(_ptr(Q), _ptr(K), _ptr(V), _typed(idx, torch.int32, "idx"),
                                      _typed(cnt, torch.int32, "cnt"), int(B), int(nq), int(q_pos0),
                                      int(hq), int(hkv), int(d), dtype_code(Q), int(max_sel), int(ld_tokens),
                                      int(sink), int(window), _ptr(O), _typed(lse, torch.float32, "lse"),
                                      _stream(stream))
    _ok(st, "lsa_sparse_attn_banded")
    return O, lse


def lsa_append(index: Index, K: torch.Tensor, n_new: int, stream=None):
    _ok(lib().lsa_append(index.handle, _ptr(K), int(n_new), _stream(stream)), "lsa_append")


def lsa_relayout(index: Index, stream=None):
    _ok(lib().lsa_relayout(index.handle, _stream(stream)), "lsa_relayout")


def lsa_refresh_centroids(index: Index, stream=None):
    _ok(lib().lsa_refresh_centroids(index.handle, _stream(stream)), "lsa_refresh_centroids")


def lsa_pca_map(K, n_tokens, pool, r, W=None, eigvals=None, stream=None):
    """Training-free latent map of the pooled keys: returns (W [d, r] float32,
    eigenvalues [r] float64), both on K's device."""
    B, ld, hkv, d = K.shape
    if W is None:
        W = torch.empty((d, r), dtype=torch.float32, device=K.device)
    if eigvals is None:
        eigvals = torch.empty(r, dtype=torch.float64, device=K.device)
    _ok(lib().lsa_pca_map(_ptr(K), int(B), int(n_tokens), int(ld), int(hkv), int(d), int(pool), dtype_code(K),
                          int(r), _ptr(W), _ptr(eigvals), _stream(stream)), "lsa_pca_map")
    return W, eigvals


def lsa_project_pool(K, W, n_tokens, pool, Kl=None, stream=None):
    B, ld, hkv, d = K.shape
    r = W.shape[1]
    nb = n_tokens // pool
    if Kl is None:
        Kl = torch.empty((B * hkv, nb, r), dtype=torch.float32, device=K.device)
    _ok(lib().lsa_project_pool(_ptr(K), _ptr(W), int(B), int(n_tokens), int(ld), int(hkv), int(d), int(r),
                               int(pool), dtype_code(K), _ptr(Kl), _stream(stream)), "lsa_project_pool")
    return Kl


def lsa_query_latent(Q, W, hkv, qbar=None, stream=None):
    B, nq, hq, d = Q.shape
    r = W.shape[1]
    if qbar is None:
        qbar = torch.empty((B, nq, hkv, r), dtype=torch.float32, device=Q.device)
    _ok(lib().lsa_query_latent(_ptr(Q), _ptr(W), int(B), int(nq), int(hq), int(hkv), int(d), int(r),
                               dtype_code(Q), _ptr(qbar), _stream(stream)), "lsa_query_latent")
    return qbar


def lsa_kmeans(X, k, iters, grid_log2=0, C_init=None, stream=None):
    """Lloyd k-means of X [units, n, r] (float32); C_init [units, k, r] float32
    or None for the stride init.  Returns (labels, centroids, objectives)."""
    U, n, r = X.shape
    _typed(X, torch.float32, "X")
    _shape(C_init, (U, k, r), "C_init")
    labels = torch.empty((U, n), dtype=torch.int32, device=X.device)
    Cc = torch.empty((U, k, r), dtype=torch.float32, device=X.device)
    obj = torch.empty((iters, U), dtype=torch.float64, device=X.device)
    _ok(lib().lsa_kmeans(_ptr(X), int(U), int(n), int(r), int(k), int(iters), int(grid_log2), _ptr(labels),
                         _ptr(Cc), _typed(C_init, torch.float32, "C_init"), _ptr(obj), _stream(stream)), "lsa_kmeans")
    return labels, Cc, obj


# ------------------------------------------------------------ context parallelism
def lsa_select_blocks(index, sp, Q, token_offset, q_pos=None, q_pos0=0, kb_cap=None, stream=None):
    """A shard's tree search: (scores [B, nq, hkv, kb_cap] float32, blocks
    [B, nq, hkv, kb_cap] int32 in whole-sequence block ids, count [B, nq, hkv]
    int32); positions are whole-sequence positions."""
    p = index.params
    if Q.dim() != 4:
        raise ValueError(f"Q must be [batch, nq, hq, d], got shape {tuple(Q.shape)}")
    if dtype_code(Q) != p.dtype:
        raise ValueError(f"Q is {Q.dtype} but the index was built for dtype {p.dtype}")
    B, nq = p.batch, Q.shape[1]
    _shape(Q, (B, nq, sp.hq, p.d), "Q")
    _shape(q_pos, (B, nq), "q_pos")
    kb = -(-sp.topk // p.pool)
    kb_cap = kb if kb_cap is None else int(kb_cap)
    scores = torch.empty((B, nq, p.hkv, kb_cap), dtype=torch.float32, device=Q.device)
    blocks = torch.empty((B, nq, p.hkv, kb_cap), dtype=torch.int32, device=Q.device)
    count = torch.empty((B, nq, p.hkv), dtype=torch.int32, device=Q.device)
    _ok(lib().lsa_select_blocks(index.handle, C.byref(sp), _ptr(Q), int(nq), _typed(q_pos, torch.int64, "q_pos"),
                                int(q_pos0), int(token_offset), _ptr(scores), _ptr(blocks), _ptr(count), int(kb_cap),
                                _stream(stream)), "lsa_select_blocks")
    return scores, blocks, count


def lsa_merge_selection(scores, blocks, count, pool, topk, sink, window, q_pos=None, q_pos0=0, max_sel=None,
                        idx=None, cnt=None, stream=None):
    """Merge of the shards' picks (scores/blocks [parts, B, nq, hkv, kb_cap],
    count [parts, B, nq, hkv]) into selection rows (idx, cnt) as lsa_select
    writes them."""
    parts, B, nq, hkv, kb_cap = scores.shape
    _shape(blocks, scores.shape, "blocks")
    _shape(count, scores.shape[:4], "count")
    _shape(q_pos, (B, nq), "q_pos")
    kb = -(-int(topk) // int(pool))
    if max_sel is None:
        max_sel = idx.shape[-1] if idx is not None else kb * pool + sink + window
    _shape(idx, (B, nq, hkv, max_sel), "idx")
    _shape(cnt, (B, nq, hkv), "cnt")
    if idx is None:
        idx = torch.empty((B, nq, hkv, max_sel), dtype=torch.int32, device=scores.device)
    if cnt is None:
        cnt = torch.empty((B, nq, hkv), dtype=torch.int32, device=scores.device)
    _ok(lib().lsa_merge_selection(int(parts), _typed(scores, torch.float32, "scores"),
                                  _typed(blocks, torch.int32, "blocks"), _typed(count, torch.int32, "count"),
                                  int(kb_cap), int(B), int(nq), int(hkv), _typed(q_pos, torch.int64, "q_pos"),
                                  int(q_pos0), int(pool), int(topk), int(sink), int(window),
                                  _typed(idx, torch.int32, "idx"), _typed(cnt, torch.int32, "cnt"), int(max_sel),
                                  _stream(stream)), "lsa_merge_selection")
    return idx, cnt


def lsa_localize_rows(idx, cnt, lo, hi, idx_out=None, cnt_out=None, stream=None):
    """The entries of each selection row in [lo, hi), shifted by -lo."""
    max_sel = idx.shape[-1]
    rows = idx.numel() // max_sel
    _shape(cnt, idx.shape[:-1], "cnt")
    if idx_out is None:
        idx_out = torch.empty_like(idx)
    if cnt_out is None:
        cnt_out = torch.empty_like(cnt)
    _shape(idx_out, idx.shape, "idx_out")
    _shape(cnt_out, cnt.shape, "cnt_out")
    _ok(lib().lsa_localize_rows(_typed(idx, torch.int32, "idx"), _typed(cnt, torch.int32, "cnt"), int(rows),
                                int(max_sel), int(lo), int(hi), _typed(idx_out, torch.int32, "idx_out"),
                                _typed(cnt_out, torch.int32, "cnt_out"), _stream(stream)), "lsa_localize_rows")
    return idx_out, cnt_out


def lsa_merge_attn(O_parts, lse_parts, O=None, lse=None, want_lse=True, stream=None):
    """Attention over the union of the parts' disjoint row sets: O_parts
    [parts, B, nq, hq, d], lse_parts [parts, B, nq, hq] -> (O, lse)."""
    parts, B, nq, hq, d = O_parts.shape
    _shape(lse_parts, O_parts.shape[:4], "lse_parts")
    if O is None:
        O = torch.empty(O_parts.shape[1:], dtype=O_parts.dtype, device=O_parts.device)
    if lse is None and want_lse:
        lse = torch.empty((B, nq, hq), dtype=torch.float32, device=O_parts.device)
    _shape(O, O_parts.shape[1:], "O")
    _shape(lse, (B, nq, hq), "lse")
    _same_dtype(O_parts, O)
    _ok(lib().lsa_merge_attn(int(parts), _ptr(O_parts), _typed(lse_parts, torch.float32, "lse_parts"), int(B * nq),
                             int(hq), int(d), dtype_code(O), _ptr(O), _typed(lse, torch.float32, "lse"),
                             _stream(stream)), "lsa_merge_attn")
    return O, lse


def _host_ptr(t, dtype, shape, name):
    """Pointer of a host tensor after checking its type and shape (the C call
    cannot see either)."""
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    _shape(t, shape, name)
    return C.c_void_p(t.data_ptr())


class Prefill:
    """Owner of an lsa_prefill context: one prefill layer from host memory per
    run, the host-device copies overlapped with the build, select and
    attention (lsa_prefill_create / run / free)."""

    def __init__(self, params: BuildParams, sp: SelectParams, nq: int, chunks: int = 16):
        self.params, self.sp, self.nq = params, sp, int(nq)
        self.handle = C.c_void_p()
        _ok(lib().lsa_prefill_create(C.byref(params), C.byref(sp), self.nq, int(chunks), C.byref(self.handle)),
            "lsa_prefill_create")

    def run(self, hQ, hK, hV, hW, hO, hlse=None, stream=None) -> Index:
        """Enqueue one layer after the work on `stream` (default: the current
        stream), which then waits for it; returns the layer's index (free it
        once the stream has passed the run)."""
        p, sp, nq = self.params, self.sp, self.nq
        dt = {LSA_F32: torch.float32, LSA_BF16: torch.bfloat16}[p.dtype]
        kv = (1, p.ld_tokens, p.hkv, p.d)
        args = (_host_ptr(hQ, dt, (1, nq, sp.hq, p.d), "hQ"), _host_ptr(hK, dt, kv, "hK"),
                _host_ptr(hV, dt, kv, "hV"), _host_ptr(hW, torch.float32, (p.d, p.r), "hW"),
                _host_ptr(hO, dt, (1, nq, sp.hq, p.d), "hO"), _host_ptr(hlse, torch.float32, (1, nq, sp.hq), "hlse"))
        h = C.c_void_p()
        _ok(lib().lsa_prefill_run(self.handle, *args, _stream(stream), C.byref(h)), "lsa_prefill_run")
        return Index(h, p)

    def free(self):
        if self.handle:
            lib().lsa_prefill_free(self.handle)
            self.handle = C.c_void_p(None)

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def lsa_check(index: Index | None = None, stream=None) -> int:
    return int(lib().lsa_check(index.handle if index is not None else None, _stream(stream)))


def lsa_launch_count() -> int:
    return int(lib().lsa_launch_count())


def lsa_debug_fail_alloc_after(n: int):
    lib().lsa_debug_fail_alloc_after(int(n))


def lsa_debug_dense_config(min_pairs: int = 0, chunk_bytes: int = 0):
    """Test hook: min_pairs < 0 turns the dense-level scoring of large
    selections off, 0 restores its default threshold; chunk_bytes bounds its
    score buffer (0: default)."""
    lib().lsa_debug_dense_config(int(min_pairs), int(chunk_bytes))


def lsa_debug_leaf_tiles(on: bool = True):
    """Test hook: turn the leaf tiles of large selections on or off."""
    lib().lsa_debug_leaf_tiles(1 if on else 0)


def exported_symbols_from_header(header_path: str) -> list:
    """Function names declared in include/lsa.h (used by the ABI test)."""
    import re
    txt = open(header_path).read()
    return sorted(set(re.findall(r"^\s*(?:int|void|int64_t|const char\*)\s+(lsa_\w+)\s*\(", txt, re.M)))
