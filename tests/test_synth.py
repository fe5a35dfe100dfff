"""Checks of the seeded input generators (CPU only)."""
import math

import numpy as np
import pytest

from decode_lr_linear_b200 import synth


def test_normals_reproducible_and_chunk_independent(monkeypatch):
    a = synth.normals((3, 1 << 21), seed=0, key=(1, 2))
    monkeypatch.setattr(synth, "_threads", lambda: 1)
    b = synth.normals((3, 1 << 21), seed=0, key=(1, 2))
    assert np.array_equal(a, b)
    c = synth.normals((3, 1 << 21), seed=0, key=(1, 3))
    assert not np.array_equal(a, c)
    assert abs(a.mean()) < 5e-3 and abs(a.std() - 1) < 5e-3


def test_attention_rank_vector():
    r = synth.attention_ranks(0)
    assert r.shape == (32, 4)
    assert (r % 32 == 0).all() and r.min() >= 512 and r.max() <= 1536
    params = (r * 8192).sum()
    budget = 0.6 * 128 * 4096 ** 2
    assert params <= budget and budget - params < 32 * 8192
    assert abs(1 - params / (128 * 4096 ** 2) - 0.4) < 1e-4
    assert r.std() > 50  # non-uniform
    assert np.array_equal(r, synth.attention_ranks(0))


def test_prefill_rank_vector():
    r = synth.prefill_ranks(0)
    shp = synth.prefill_shapes()
    assert r.shape == (40, 7) and (r % 32 == 0).all()
    d_in = np.array([shp[p][0] for p in synth.PREFILL_PROJ])
    d_out = np.array([shp[p][1] for p in synth.PREFILL_PROJ])
    be = d_in * d_out / (d_in + d_out)
    assert (r >= 0.3 * be - 1e-9).all() and (r <= 0.9 * be + 1e-9).all()
    params = (r * (d_in + d_out)).sum()
    budget = 0.6 * 40 * (d_in * d_out).sum()
    assert params <= budget and budget - params < 32 * (d_in + d_out).max()


def test_rtn_error_bound_and_range():
    rng = np.random.default_rng(0)
    W = rng.standard_normal((64, 300)) * np.linspace(0.01, 3, 64)[:, None]
    W[5] = 0.0
    q, s = synth.rtn_int8_rows(W)
    deq = q.astype(np.float64) * s.astype(np.float64)[:, None]
    assert (np.abs(W - deq) <= s.astype(np.float64)[:, None] / 2 + 1e-12).all() or \
        (np.abs(q) == 127).any()
    inside = np.abs(W) <= 127 * s.astype(np.float64)[:, None]
    assert (np.abs(W - deq)[inside] <= (s.astype(np.float64)[:, None] / 2 + 1e-12).repeat(300, 1)[inside]).all()
    assert not q[5].any() and s[5] == 0
    assert np.abs(q).max() <= 127


def test_rotation_orthogonal_and_folding_invariant():
    R = synth.make_rotation(1536, seed=0)
    assert np.abs(R @ R.T - np.eye(1536)).max() < 1e-12
    rng = np.random.default_rng(1)
    A = rng.standard_normal((40, 1536))
    B = rng.standard_normal((1536, 30))
    assert np.abs((A @ R) @ (R.T @ B) - A @ B).max() < 1e-9
    H = synth.hadamard(8)
    assert np.array_equal(H @ H.T, 8 * np.eye(8))


def test_haar_columns_orthonormal():
    Q = synth.haar_orthogonal(50, np.random.default_rng(0), 20)
    assert np.abs(Q.T @ Q - np.eye(20)).max() < 1e-12


def test_latent_factor_spectrum():
    B = synth.make_latent_factors(3, 32, 128, seed=0, key=(1,))
    c = math.sqrt(128 / synth.harmonic(32))
    for h in range(3):
        s = np.linalg.svd(B[h], compute_uv=False)
        assert np.abs(s - c / np.sqrt(np.arange(1, 33))).max() < 1e-10
        assert abs((s ** 2).sum() - 128) < 1e-9


def test_hybrid_ffn_shapes():
    d = synth.make_hybrid_ffn(seed=0, hidden=128, inter=96, n_lr=64, rank=512)
    assert tuple(d["A_q"].shape) == (512, 128)
    assert tuple(d["B_q"].shape) == (512, 128)
    assert tuple(d["D_q"].shape) == (64, 128)
    assert tuple(d["Wd_q"].shape) == (96, 128)
    assert d["s_A"].dtype.itemsize == 2


@pytest.mark.parametrize("batch", [1, 3])
def test_activations_outliers(batch):
    x = synth.make_activations(batch, 4096, seed=0, key=(7,), outliers=4).float().numpy()
    big = (np.abs(x).max(axis=0) > 8).sum()
    assert 1 <= big <= 4 + 2
