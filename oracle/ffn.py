"""Oracle: hybrid low-rank / dense SwiGLU FFN with int8 RTN weights (test infrastructure only).

LASER methodology, "Hybrid SVD-Quantization for FFNs": the hidden channels
chosen as SVD-friendly are compressed by SVD (one latent shared by gate and
up over those channels), the rest stay dense; both branches are RTN
quantised after an orthogonal rotation is inserted between the SVD factors.
LASER "System Implementation" fuses the input projection, the latent
activation, SwiGLU and the (de)quantisation.

Stored layout consumed here (the library's), every scale per output channel:
  A_q  [r, hidden]         int8, s_A [r]        A' = (A_q * s_A[:,None]).T   (hidden x r)
  B_q  [r, 2 n_lr]         int8, s_B [2 n_lr]   B' = B_q * s_B[None,:]; columns gate_0, up_0, gate_1, ...
  D_q  [2 n_dense, hidden] int8, s_D            dense gate/up rows, interleaved the same way
  Wd_q [inter, hidden]     int8, s_d [hidden]   down_proj W_down = Wd_q * s_d[None,:]; rows in [S; D] order
"""
from __future__ import annotations

import numpy as np

from .lowrank import _f64


def dequantize_rows(q, s) -> np.ndarray:
    """w = q * s with one scale per stored row (= per output channel), in float64."""
    q, s = _f64(q), _f64(s)
    return q * s[:, None]


def dequantize_cols(q, s) -> np.ndarray:
    """w = q * s with one scale per column (= per output channel), in float64."""
    q, s = _f64(q), _f64(s)
    return q * s[None, :]


def silu(t) -> np.ndarray:
    """silu(t) = t / (1 + e^-t), the gate nonlinearity of SwiGLU."""
    t = _f64(t)
    with np.errstate(over="ignore"):  # e^-t = inf for t << 0 gives the exact limit -0
        return t / (1.0 + np.exp(-t))


def swiglu_ffn_math(x, A, B_gate, B_up, W_gate_D, W_up_D, W_down) -> np.ndarray:
    """The hybrid FFN in math layout (all float64, row activations).

    z = x A; g_S = z B_gate, u_S = z B_up (low-rank channels);
    g_D = x W_gate_D, u_D = x W_up_D (dense channels);
    h = [silu(g_S) u_S, silu(g_D) u_D]; y = h W_down.
    """
    x = _f64(x)
    parts = []
    if B_gate is not None and B_gate.shape[1] > 0:
        z = x @ _f64(A)
        parts.append(silu(z @ _f64(B_gate)) * (z @ _f64(B_up)))
    if W_gate_D is not None and W_gate_D.shape[1] > 0:
        parts.append(silu(x @ _f64(W_gate_D)) * (x @ _f64(W_up_D)))
    h = np.concatenate(parts, axis=1)
    return h @ _f64(W_down)


def hybrid_swiglu_ffn(x, A_q, s_A, B_q, s_B, D_q, s_D, Wd_q, s_d, n_lr: int, n_dense: int):
    """The hybrid FFN on the stored int8 tensors: dequantise, de-interleave, evaluate.

    Returns (y, h) with y [batch, hidden] and h [batch, n_lr + n_dense].
    """
    A = dequantize_rows(A_q, s_A).T                   # hidden x r
    Bs = dequantize_cols(B_q, s_B) if n_lr else None  # r x 2 n_lr
    Ds = dequantize_rows(D_q, s_D).T if n_dense else None  # hidden x 2 n_dense
    Wdown = dequantize_cols(Wd_q, s_d)                # inter x hidden
    x = _f64(x)
    parts = []
    if n_lr:
        z = x @ A
        gu = z @ Bs
        parts.append(silu(gu[:, 0::2]) * gu[:, 1::2])
    if n_dense:
        gu = x @ Ds
        parts.append(silu(gu[:, 0::2]) * gu[:, 1::2])
    h = np.concatenate(parts, axis=1)
    return h @ Wdown, h
