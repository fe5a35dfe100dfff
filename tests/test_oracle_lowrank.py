"""Pins for oracle.lowrank: closed forms, identities and brute force (CPU only)."""
import math
from fractions import Fraction

import numpy as np
import pytest

from decode_lr_linear_b200 import synth
from oracle import lowrank as L


def harmonic_exact(n):
    return float(sum(Fraction(1, i) for i in range(1, n + 1)))


@pytest.fixture(scope="module")
def single():
    return synth.make_single_linear(0)


def test_eckart_young_closed_form(single):
    """sigma_i = i^-1/2: the rank-32 truncation error is sqrt(H_256 - H_32) (Frobenius)
    and 33^-1/2 (spectral) -- the truncated SVD reaches the theoretical minimum."""
    W = single["W"]
    A, B = L.truncated_svd(W, 32)
    err = L.truncation_error(W, A, B)
    closed = math.sqrt(harmonic_exact(256) - harmonic_exact(32))
    assert abs(err - closed) < 1e-10
    assert abs(closed - 1.4373064) < 1e-6
    rel = err / np.linalg.norm(W)
    assert abs(rel - closed / math.sqrt(harmonic_exact(256))) < 1e-10
    assert abs(rel - 0.580791) < 1e-6
    spec = np.linalg.norm(W - A @ B, 2)
    assert abs(spec - 33 ** -0.5) < 1e-10
    assert abs(L.eckart_young_error(single["sigma"], 32) - closed) < 1e-12


def test_truncation_matches_construction(single):
    """The oracle's SVD factors give the same product as the generator's U_r S_r V_r^T."""
    A, B = L.truncated_svd(single["W"], 32)
    assert np.abs(A @ B - single["A"] @ single["B"]).max() < 1e-10


def test_rank_r_alternatives_are_not_better(single):
    W = single["W"]
    best = L.eckart_young_error(single["sigma"], 32)
    rng = np.random.default_rng(5)
    A, B = L.truncated_svd(W, 32)
    for _ in range(5):
        Ap = A + 1e-3 * rng.standard_normal(A.shape)
        assert L.truncation_error(W, Ap, B) >= best - 1e-12
    # another rank-32 subspace: the 32 smallest-indexed-after-the-first components
    U, s, Vt = np.linalg.svd(W)
    idx = np.arange(1, 33)
    assert L.truncation_error(W, U[:, idx] * s[idx], Vt[idx]) > best


def test_retained_energy_ratio(single):
    """RER_32 = H_32 / H_256, and 1 - RER = ||W - A B||_F^2 / ||W||_F^2."""
    s = single["sigma"]
    rer = L.retained_energy_ratio(s, 32)
    assert abs(rer - harmonic_exact(32) / harmonic_exact(256)) < 1e-12
    assert abs(rer - 0.6626823) < 1e-6
    A, B = L.truncated_svd(single["W"], 32)
    W = single["W"]
    assert abs((1 - rer) - L.truncation_error(W, A, B) ** 2 / np.linalg.norm(W) ** 2) < 1e-12


def test_generated_spectrum(single):
    s = L.singular_values(single["W"])
    assert np.abs(s - 1 / np.sqrt(np.arange(1, 257))).max() < 1e-12
    U, V = single["U"], single["V"]
    assert np.abs(U.T @ U - np.eye(256)).max() < 1e-12
    assert np.abs(V.T @ V - np.eye(256)).max() < 1e-12


def test_exact_rank_identity():
    """When W has exact rank r, the factored path equals the dense path."""
    d = synth.make_single_linear(0, exact_rank=True)
    x = d["x"].double().numpy()
    y_lr = L.lr_linear(x, d["A"], d["B"])
    y_dn = L.dense_linear(x, d["W"])
    assert np.linalg.norm(y_lr - y_dn) / np.linalg.norm(y_dn) < 1e-12
    assert L.truncation_error(d["W"], d["A"], d["B"]) < 1e-12


def _brute_lr(x, A, B, r=None):
    nb, din = x.shape
    rank = A.shape[1] if r is None else r
    dout = B.shape[1]
    y = np.zeros((nb, dout))
    for b in range(nb):
        for k in range(dout):
            acc = 0.0
            for j in range(rank):
                zj = 0.0
                for i in range(din):
                    zj += x[b, i] * A[i, j]
                acc += zj * B[j, k]
            y[b, k] = acc
    return y


def test_lr_linear_brute_force_nonsquare():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, 7))
    A = rng.standard_normal((7, 4))
    B = rng.standard_normal((4, 5))
    assert np.abs(L.lr_linear(x, A, B) - _brute_lr(x, A, B)).max() < 1e-12
    assert np.abs(L.lr_linear(x, A, B, active_rank=2) - _brute_lr(x, A, B, 2)).max() < 1e-12


def test_eigh_route_gives_output_spectrum():
    """Swift-SVD: eigenvalues of Y^T Y are the squared singular values of Y = X W."""
    rng = np.random.default_rng(2)
    X = rng.standard_normal((40, 12))
    W = rng.standard_normal((12, 9))
    s_ref = np.linalg.svd(X @ W, compute_uv=False)
    s = L.output_spectrum_by_eigh(X, W)
    assert np.abs(s - s_ref).max() < 1e-9
