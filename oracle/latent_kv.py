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
so the causal mask removes nothing).  latent_kv_decode and the absorbed form
apply no rotary embedding; latent_kv_decode_rope rotates the reconstructed
keys and the query (LLaMA rotary convention, a reading: the pages do not
write it out).  append_latents is the producer that writes new latents.
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


# --------------------------------------------------------------------------
# Rotary positions and the reconstruct-on-chip form; the latent producer.
#
# The pages' models (LLaVA-v1.5, LLaVA-Next, SmolVLM in WSVD "Resultaten")
# are LLaMA-family decoders, whose keys and queries carry a rotary position
# embedding.  The pages never write it out; the reading taken here is the
# LLaMA convention: head_dim/2 frequencies theta_i = base^(-2i/head_dim),
# and dimension i is rotated together with dimension i + head_dim/2 by the
# angle pos * theta_i.  A rotation applied to the reconstructed key K_t is
# why the query can no longer be absorbed into B_K: the key must be
# reconstructed (WSVD "Quantization-Aware Training (QAT) en Fused Kernel",
# reconstruction inside the flash-decoding pipeline) before it is rotated.
# --------------------------------------------------------------------------
def rope_freqs(head_dim: int, base: float) -> np.ndarray:
    """theta_i = base^(-2i / head_dim), i = 0 .. head_dim/2 - 1, in float64."""
    return np.asarray(base, np.float64) ** (-2.0 * np.arange(head_dim // 2) / head_dim)


def rope(x, pos, base: float) -> np.ndarray:
    """Rotate x [..., head_dim] at positions pos (broadcast over the leading dims):
    out[i] = x[i] cos(pos theta_i) - x[i+h] sin(pos theta_i),
    out[i+h] = x[i+h] cos(pos theta_i) + x[i] sin(pos theta_i), h = head_dim / 2."""
    x = _f64(x)
    half = x.shape[-1] // 2
    ang = np.asarray(pos, np.float64)[..., None] * rope_freqs(x.shape[-1], base)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def decode_head_rope(q, CK, CV, BK, BV, n: int, scale: float, base: float) -> np.ndarray:
    """One (batch, head) with rotary positions: reconstruct K_t = C_K[t] B_K, rotate it
    to position t and the query to position n - 1 (the newest cached token, whose
    latents the producer appended before the attention step), softmax attention over
    t < n; values are not rotated, V_t = C_V[t] B_V.  n = 0 gives a zero row."""
    if n <= 0:
        return np.zeros(_f64(BV).shape[1])
    K = rope(_f64(CK)[:n] @ _f64(BK), np.arange(n), base)
    qr = rope(_f64(q), n - 1, base)
    V = _f64(CV)[:n] @ _f64(BV)
    p = _softmax((K @ qr) * scale)
    return p @ V


def latent_kv_decode_rope(q, C_K, C_V, B_K, B_V, seq_lens, scale: float, base: float, pairs=None) -> np.ndarray:
    """o [batch, heads, head_dim] in float64 with rotary positions (decode_head_rope per pair)."""
    seq_lens, todo = _pairs_and_lens(q, seq_lens, pairs)
    nb, nh, hd = q.shape
    out = np.full((nb, nh, hd), np.nan)
    for b, h in todo:
        out[b, h] = decode_head_rope(q[b, h], C_K[b, h], C_V[b, h], B_K[h], B_V[h], int(seq_lens[b]), scale, base)
    return out


def append_latents(x, A_KV, heads: int, rank: int, C_K, C_V, pos):
    """The latent producer (WSVD "Fine-Grained Per-Head SVD": the cache keeps the
    per-head latent x A_Kh instead of the key).  A_KV [2 * heads * rank, hidden] holds
    the per-head first factors latent-major, keys (head 0 .. heads-1) then values:
    row h * rank + j is column j of A_Kh, row (heads + h) * rank + j column j of A_Vh.
    Returns float64 copies of C_K, C_V [batch, heads, ctx, rank] with position pos[b]
    of sequence b overwritten by x[b] A_Kh and x[b] A_Vh; a position outside
    [0, ctx) leaves that sequence's caches unchanged."""
    x, A = _f64(x), _f64(A_KV)
    CK, CV = _f64(C_K).copy(), _f64(C_V).copy()
    ctx = CK.shape[2]
    lat = x @ A.T                                   # [batch, 2 * heads * rank]
    for b in range(x.shape[0]):
        p = int(pos[b])
        if not 0 <= p < ctx:
            continue
        CK[b, :, p, :] = lat[b, :heads * rank].reshape(heads, rank)
        CV[b, :, p, :] = lat[b, heads * rank:].reshape(heads, rank)
    return CK, CV
