"""GPU parity of the training-free latent map (lsa_pca_map) against the
oracle's pca_map: eigenvalues to fp64 rounding, columns of W where the
eigenvalue gaps make them unique; at the 1M-token size, by the property that
the latent keys under W have a diagonal covariance equal to the eigenvalues."""
import numpy as np
import pytest
import torch

import oracle as O
from hierarchical_latent_key_gemm_b200 import lsa
from hierarchical_latent_key_gemm_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lsa.lib()
    yield
    torch.cuda.synchronize()


def _units(K, n_tokens):
    B, _, hkv, _ = K.shape
    return [K[b, :n_tokens, h].double().numpy() for b in range(B) for h in range(hkv)]


@pytest.mark.parametrize("name,over,r", [
    ("gqa_128k", {"n_tokens": 8192 + 3, "needles": 0, "components": 256}, 64),
    ("int_exact_16k", {"n_tokens": 4096 + 5}, 16),
    ("flat_4k_f32", {}, 32),
    ("decode_10m_x4", {"n_tokens": 4096 + 2, "batch": 2, "needles": 0, "components": 128, "decode_steps": 0}, 128),
])
def test_pca_map_matches_oracle(name, over, r):
    w = WORKLOADS[name].scaled(**over)
    inp = make_inputs(w, seed=21)
    Wg, evg = lsa.lsa_pca_map(inp["K"].cuda(), w.n_tokens, w.pool, r)
    assert lsa.lsa_check(None) == lsa.LSA_OK
    Wo, evo = O.pca_map(_units(inp["K"], w.n_tokens), w.pool, r)
    evg = evg.cpu().numpy()
    assert np.allclose(evg, evo, rtol=1e-9, atol=1e-12 * abs(evo[0]))
    # a column is unique (up to the sign convention) when its eigenvalue is
    # apart from its neighbours; compare those, and the whole subspace when
    # the r-th eigenvalue is apart from the next one
    Wg = Wg.double().cpu().numpy()
    _, evall = O.pca_map(_units(inp["K"], w.n_tokens), w.pool, w.d)
    gaps = np.abs(np.diff(evall))
    scale = abs(evall[0])
    for c in range(r):
        left = gaps[c - 1] if c > 0 else np.inf
        right = gaps[c] if c < len(gaps) else np.inf
        if min(left, right) > 1e-4 * scale:
            assert np.abs(Wg[:, c] - Wo[:, c]).max() <= 1e-5, f"column {c}"
    if r == w.d or gaps[r - 1] > 1e-4 * scale:
        assert np.abs(Wg @ Wg.T - Wo @ Wo.T).max() <= 1e-5
    assert np.abs(Wg.T @ Wg - np.eye(r)).max() <= 1e-5


def test_pca_map_full_size_latent_covariance_is_diagonal():
    """prefill_1m: 2 KV heads x 262,144 blocks.  Under the map, the latent keys
    (computed by the build's own projection kernel) have covariance
    diag(eigenvalues): checked in fp64 on the device's latents."""
    w = WORKLOADS["prefill_1m"]
    inp = make_inputs(w, seed=0, device="cuda")
    Wg, evg = lsa.lsa_pca_map(inp["K"], w.n_tokens, w.pool, w.r)
    Kl = lsa.lsa_project_pool(inp["K"], Wg, w.n_tokens, w.pool)      # [units, nb, r]
    assert lsa.lsa_check(None) == lsa.LSA_OK
    X = Kl.reshape(-1, w.r).double()
    Xc = X - X.mean(dim=0)
    C = (Xc.T @ Xc / X.shape[0]).cpu().numpy()
    ev = evg.cpu().numpy()
    assert np.all(np.diff(ev) <= 0)
    assert np.allclose(np.diag(C), ev, rtol=1e-4)
    off = C - np.diag(np.diag(C))
    assert np.abs(off).max() <= 1e-4 * ev[0]
    # and the map feeds the build unchanged
    bp = lsa.make_build_params(w.batch, w.n_tokens, w.n_tokens, w.hkv, w.d, w.r, w.pool, lsa.LSA_BF16,
                               w.level_sizes, w.lloyd_iters, 0, w.sink, 0)
    ix = lsa.lsa_build_index(bp, inp["K"], Wg)
    assert lsa.lsa_check(ix) == lsa.LSA_OK
    ix.free()


def test_pca_map_argument_errors():
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=512, needles=0, components=16)
    K = make_inputs(w, seed=22, device="cuda")["K"]
    for r in (0, w.d + 1):
        with pytest.raises(lsa.LsaError):
            lsa.lsa_pca_map(K, w.n_tokens, w.pool, r)
    with pytest.raises(lsa.LsaError):
        lsa.lsa_pca_map(K, 2, 4, 8)          # no complete block
    assert lsa.lsa_check(None) == lsa.LSA_OK
