"""The seeded input generators produce what their recipes state (CPU only)."""
import numpy as np
import pytest
import torch

from hierarchical_latent_key_gemm_b200.workloads import WORKLOADS, make_inputs, make_map


def test_integer_workload_recipe():
    w = WORKLOADS["int_exact_16k"].scaled(n_tokens=512)
    a = make_inputs(w, seed=0)
    for k in ("K", "Q", "V"):
        x = a[k].float()
        assert a[k].dtype == torch.bfloat16
        assert torch.equal(x, x.round()) and x.min() >= -4 and x.max() <= 4
    assert a["K"].shape == (1, 512, 1, 64) and a["Q"].shape == (1, 512, 4, 64)
    W = a["W"]
    assert W.shape == (64, 16)
    assert torch.all((W != 0).sum(dim=1) == 4)
    assert set(W.unique().tolist()) <= {-1.0, 0.0, 1.0}


def test_float_map_is_orthonormal_and_seeded():
    w = WORKLOADS["gqa_128k"]
    W = make_map(w, seed=1).double()
    np.testing.assert_allclose((W.T @ W).numpy(), np.eye(w.r), atol=1e-6)
    assert torch.equal(make_map(w, seed=1), make_map(w, seed=1))
    assert not torch.equal(make_map(w, seed=1), make_map(w, seed=2))


def test_mixture_workload_is_deterministic_and_shaped():
    w = WORKLOADS["gqa_128k"].scaled(n_tokens=3000, needles=4, needle_gap=1000, components=32)
    a = make_inputs(w, seed=5)
    b = make_inputs(w, seed=5)
    for k in ("K", "Q", "V"):
        assert torch.equal(a[k], b[k])
    assert a["K"].shape == (1, 3000, 4, 128) and a["Q"].shape == (1, 3000, 32, 128)
    assert len(a["needles"]) == 4
    for (bb, h, p, qp) in a["needles"]:
        assert qp >= p + 1000 and p >= w.sink
        kn = a["K"][bb, p, h].float().norm()
        assert kn > 1.5 * a["K"][bb, :100].float().norm(dim=-1).median()


def test_decode_workload_layout():
    w = WORKLOADS["decode_10m_x4"].scaled(n_tokens=1000, batch=2, decode_steps=8, needles=2, needle_gap=100,
                                          components=16)
    a = make_inputs(w, seed=0)
    assert a["K"].shape == (2, 1008, 1, 128)
    assert a["Q"].shape == (2, 8, 16, 128)
    for (bb, h, p, qp) in a["needles"]:
        assert 1000 <= qp < 1008


def test_drift_changes_component_weights():
    w = WORKLOADS["prefill_1m"].scaled(n_tokens=4096, drift_every=1024, components=8, needles=0)
    a = make_inputs(w, seed=0)
    assert a["K"].shape == (1, 4096, 2, 128)
