"""Oracle: truncated-SVD factorised linear layers (test infrastructure only).

Notation: activations are row vectors, x is [batch, d_in]; the effective
weight W is d_in x d_out and a layer computes y = x W.  A compressed layer
holds factors A (d_in x r) and B (r x d_out) and computes y = (x A) B without
forming W.  (SAES-SVD writes the same pair as A_l B_l acting on column
activations, CEALC objective; Swift-SVD writes Y = X W with row activations;
WSVD writes W_Kh = A_Kh B_Kh.)
"""
from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.asarray(a, dtype=np.float64)


def lr_linear(x, A, B, active_rank: int | None = None) -> np.ndarray:
    """y = (x A) B in float64: first the r-dim latent z = x A, then z B.

    Follows the factor pair that replaces the weight in SAES-SVD (technical
    summary, CEALC: the local term || A_l B_l X_l - W_l X_l ||) and WSVD
    ("Fine-Grained Per-Head SVD", W_Kh = A_Kh B_Kh).  ``active_rank`` keeps
    only the leading r' latent components (FLRC "progressive low-rank
    decoding": the rank used for token t is r(t) <= r).
    """
    x, A, B = _f64(x), _f64(A), _f64(B)
    if active_rank is not None:
        A = A[:, :active_rank]
        B = B[:active_rank, :]
    z = x @ A
    return z @ B


def dense_linear(x, W) -> np.ndarray:
    """y = x W in float64 (the uncompressed layer)."""
    return _f64(x) @ _f64(W)


def truncated_svd(W, r: int):
    """Rank-r truncated SVD factors of W (d_in x d_out): A = U_r S_r^1/2, B = S_r^1/2 V_r^T.

    The truncation keeps the r largest singular components (SAES-SVD
    technical summary, "low-rank compression via truncated SVD"; WSVD
    problem statement).  The split of S_r between the factors does not
    change A B.
    """
    W = _f64(W)
    U, s, Vt = np.linalg.svd(W, full_matrices=False)
    sr = np.sqrt(s[:r])
    return U[:, :r] * sr[None, :], sr[:, None] * Vt[:r, :]


def singular_values(W) -> np.ndarray:
    return np.linalg.svd(_f64(W), compute_uv=False)


def truncation_error(W, A, B) -> float:
    """|| W - A B ||_F in float64."""
    return float(np.linalg.norm(_f64(W) - _f64(A) @ _f64(B)))


def eckart_young_error(sigma, r: int) -> float:
    """Minimum Frobenius error of any rank-r approximation: sqrt(sum_{i>r} sigma_i^2).

    This is the "theoretical minimum loss" that Swift-SVD's numerical-stability
    experiment compares reconstruction errors against.
    """
    s = np.sort(_f64(sigma))[::-1]
    return float(np.sqrt(np.sum(s[r:] ** 2)))


def retained_energy_ratio(sigma, k: int) -> float:
    """RER = sum of the top-k squared singular values over the sum of all of them
    (SAES-SVD technical summary, ACES optimisation target)."""
    s = np.sort(_f64(sigma))[::-1]
    return float(np.sum(s[:k] ** 2) / np.sum(s ** 2))


def output_spectrum_by_eigh(X, W) -> np.ndarray:
    """Singular values of Y = X W from one eigendecomposition of Y^T Y.

    Swift-SVD methodology: instead of an SVD of Y, aggregate Y^T Y and take
    its eigendecomposition; the eigenvalues are the squared singular values
    of Y.  Returned in descending order, clipped at zero before the root.
    """
    Y = _f64(X) @ _f64(W)
    lam = np.linalg.eigh(Y.T @ Y)[0][::-1]
    return np.sqrt(np.clip(lam, 0.0, None))
