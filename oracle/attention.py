"""Oracle: single-query decode attention over full K/V caches (test infrastructure only).

The uncompressed baseline the latent-KV pages measure against: standard
flash-decoding attention reads every cached key and value in full (WSVD
"Resultaten": speed-up over FlashDecoding; LASER results: speed-up over Flash
Decoding).  For one (batch, head), the query attends to positions
0 .. seq_len-1:  s_t = (q . K_t) * scale,  p = softmax(s),  o = sum_t p_t V_t.

Shapes: q [batch, heads, head_dim]; K, V [batch, heads, ctx, head_dim];
seq_lens [batch].  An empty context (seq_len 0) has no softmax; the reading is
a zero output row, as for the latent form.
"""
from __future__ import annotations

import numpy as np

from .lowrank import _f64


def decode_head(q, K, V, n: int, scale: float) -> np.ndarray:
    """One (batch, head) in float64: max-subtracted softmax over the first n keys."""
    if n <= 0:
        return np.zeros(_f64(V).shape[-1])
    K = _f64(K)[:n]
    V = _f64(V)[:n]
    s = (K @ _f64(q)) * scale
    e = np.exp(s - s.max())
    return (e / e.sum()) @ V


def decode_attention(q, K, V, seq_lens, scale: float, pairs=None) -> np.ndarray:
    """o [batch, heads, head_dim] in float64; `pairs` limits the (b, h) evaluated (others NaN)."""
    seq_lens = np.asarray(seq_lens.cpu() if hasattr(seq_lens, "cpu") else seq_lens).astype(np.int64)
    nb, nh, hd = q.shape
    todo = pairs if pairs is not None else [(b, h) for b in range(nb) for h in range(nh)]
    out = np.full((nb, nh, hd), np.nan)
    for b, h in todo:
        out[b, h] = decode_head(q[b, h], K[b, h], V[b, h], int(seq_lens[b]), scale)
    return out
