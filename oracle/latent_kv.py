"""Oracle: single-query decode attention over per-head latent K/V caches (test infrastructure only).

WSVD "Fine-Grained Per-Head SVD": each head's key projection is factored as
W_Kh = A_Kh B_Kh at a small rank r, and the cache keeps the per-head latent
CK_h instead of the full key; likewise for values.  WSVD "Quantization-Aware
Training (QAT) en Fused Kernel" reconstructs K and V inside the
flash-decoding pipeline without writing them to global memory.

Shapes: q [batch, heads, head_dim]; C_K, C_V [batch, heads, ctx, r];
B_K, B_V [heads, r, head_dim]; seq_lens [batch].  Key t of head h is
K_t = C_K[t] B_K[h] (a 1 x head_dim row), value V_t = C_V[t] B_V[h].
The single query attends to positions 0 .. seq_len-1 (it sits after them,
so the causal mask removes nothing).  No rotary embedding is applied.
"""
from __future__ import annotations

import numpy as np

from .lowrank import _f64


def _softmax(s: np.ndarray) -> np.ndarray:
    e = np.exp(s - s.max())
    return e / e.sum()


def decode_head(q, CK, CV, BK, BV, n: int, scale: float) -> np.ndarray:
    """One (batch, head): reconstruct K, V for the first n positions, then softmax attention.

    An empty context (n = 0) has no softmax; the library's reading is a zero output.
    """
    if n <= 0:
        return np.zeros(_f64(BV).shape[1])
    K = _f64(CK)[:n] @ _f64(BK)          # n x head_dim
    V = _f64(CV)[:n] @ _f64(BV)          # n x head_dim
    p = _softmax((K @ _f64(q)) * scale)  # n
    return p @ V


def _pairs_and_lens(q, seq_lens, pairs):
    seq_lens = np.asarray(seq_lens.cpu() if hasattr(seq_lens, "cpu") else seq_lens).astype(np.int64)
    nb, nh = q.shape[0], q.shape[1]
    todo = pairs if pairs is not None else [(b, h) for b in range(nb) for h in range(nh)]
    return seq_lens, todo


def latent_kv_decode(q, C_K, C_V, B_K, B_V, seq_lens, scale: float, pairs=None) -> np.ndarray:
    """o [batch, heads, head_dim] in float64 (reconstruct-then-attend form).

    ``pairs``: optional list of (b, h) to evaluate; other entries stay NaN.
    Inputs are converted to float64 one (batch, head) at a time.
    """
    seq_lens, todo = _pairs_and_lens(q, seq_lens, pairs)
    nb, nh, hd = q.shape
    out = np.full((nb, nh, hd), np.nan)
    for b, h in todo:
        out[b, h] = decode_head(q[b, h], C_K[b, h], C_V[b, h], B_K[h], B_V[h], int(seq_lens[b]), scale)
    return out


def decode_head_absorbed(q, CK, CV, BK, BV, n: int, scale: float) -> np.ndarray:
    """Same result with the factors moved onto the query and the output:
    s_t = C_K[t] (B_K q) * scale, acc = sum_t p_t C_V[t] (r-vector), o = acc B_V."""
    if n <= 0:
        return np.zeros(_f64(BV).shape[1])
    qt = _f64(BK) @ _f64(q)              # r
    p = _softmax((_f64(CK)[:n] @ qt) * scale)
    return (p @ _f64(CV)[:n]) @ _f64(BV)


def latent_kv_decode_absorbed(q, C_K, C_V, B_K, B_V, seq_lens, scale: float, pairs=None) -> np.ndarray:
    seq_lens, todo = _pairs_and_lens(q, seq_lens, pairs)
    nb, nh, hd = q.shape
    out = np.full((nb, nh, hd), np.nan)
    for b, h in todo:
        out[b, h] = decode_head_absorbed(q[b, h], C_K[b, h], C_V[b, h], B_K[h], B_V[h],
                                         int(seq_lens[b]), scale)
    return out


def dequantize_cache(Cq, s) -> np.ndarray:
    """int8 latent cache with one scale per (batch, head, position): C[..., t, j] = Cq[..., t, j] * s[..., t]."""
    return _f64(Cq) * _f64(s)[..., None]


def latent_kv_decode_q8(q, CKq, sK, CVq, sV, B_K, B_V, seq_lens, scale: float, pairs=None) -> np.ndarray:
    """Decode attention over int8 latent caches with per-token scales (LASER results:
    the KV cache kept in 8 bits under W8A8): dequantize, then the reconstructed form."""
    return latent_kv_decode(q, dequantize_cache(CKq, sK), dequantize_cache(CVq, sV), B_K, B_V, seq_lens, scale,
                            pairs)
