"""Oracle: W8A8 low-rank linear for prefill (test infrastructure only).

Both the activations and the factor weights are 8-bit (LASER results, the
W8A8 setting; WSVD "Quantization-Aware Training (QAT) en Fused Kernel",
weights and activations quantised, e.g. W8A8).  Activations get one scale
per token; weights one scale per output channel.  The latent z = x A is
re-quantised per token before the second factor.

The pipeline is specified down to the fp32 operation so that integer
results and the requantised latent can be compared bit for bit:
  acc1[t,j] = sum_i xq[t,i] Aq[j,i]                       (exact integer)
  z[t,j]    = fp32( fp32( (float)acc1[t,j] * s_x[t] ) * s_A[j] )
  s_z[t]    = fp32( max_j |z[t,j]| / 127 )   (1 if that is 0, then z_q = 0)
  zq[t,j]   = clamp( rint_even( fp32( z[t,j] / s_z[t] ) ), -127, 127 )
  acc2[t,k] = sum_j zq[t,j] Bq[j,k]                       (exact integer)
  y[t,k]    = bf16_rn( fp32( fp32( (float)acc2[t,k] * s_z[t] ) * s_B[k] ) )
Storage is latent-major: Aq [r, d_in] (row j = latent channel j), Bq [r, d_out].
"""
from __future__ import annotations

import numpy as np
import torch


def _np(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu")
        if a.dtype == torch.bfloat16:
            a = a.float()
        a = a.numpy()
    return np.asarray(a)


def quantize_per_token(x):
    """Symmetric per-row int8: s = max|x| / 127 in fp32, q = clamp(rint(x / s), -127, 127).

    x is read as fp32 (bf16 converts exactly).  A row of zeros gets s = 1, q = 0.
    Returns (q int8 [rows, cols], s float32 [rows]).
    """
    x32 = _np(x).astype(np.float32)
    amax = np.abs(x32).max(axis=1)
    s = amax / np.float32(127.0)
    zero = s == np.float32(0.0)
    s_safe = np.where(zero, np.float32(1.0), s).astype(np.float32)
    q = np.rint(x32 / s_safe[:, None])
    q = np.clip(q, -127, 127)
    q[zero, :] = 0
    return q.astype(np.int8), s_safe


def int_matmul_nt(a_q, b_q) -> np.ndarray:
    """C[t,k] = sum_i a[t,i] b[k,i] for int8 inputs, exact, as int64.

    The products are evaluated in float64 BLAS: every term is at most 127^2
    and every partial sum stays below 2^53 for inner sizes under 2^38, so
    each sum is an exact integer whatever the summation order.
    """
    a = _np(a_q).astype(np.float64)
    b = _np(b_q).astype(np.float64)
    assert a.shape[1] < (1 << 38)
    return (a @ b.T).astype(np.int64)


def requant_latent(acc1, s_x, s_A):
    """z = (acc1 * s_x[t]) * s_A[j] in fp32, one rounding per product, then per-token int8."""
    z = (acc1.astype(np.float32) * _np(s_x).astype(np.float32)[:, None]).astype(np.float32)
    z = (z * _np(s_A).astype(np.float32)[None, :]).astype(np.float32)
    zq, s_z = quantize_per_token(z)
    return z, zq, s_z


def bf16_round(a32: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returned as fp32 values."""
    return torch.from_numpy(np.ascontiguousarray(a32, np.float32)).to(torch.bfloat16).float().numpy()


def w8a8_lr_linear(xq, s_x, Aq, s_A, Bq, s_B) -> dict:
    """The full W8A8 low-rank pipeline; returns every intermediate."""
    acc1 = int_matmul_nt(xq, Aq)
    z, zq, s_z = requant_latent(acc1, s_x, s_A)
    acc2 = int_matmul_nt(zq, _np(Bq).T)
    y32 = (acc2.astype(np.float32) * s_z[:, None]).astype(np.float32)
    y32 = (y32 * _np(s_B).astype(np.float32)[None, :]).astype(np.float32)
    return {"acc1": acc1, "z": z, "zq": zq, "s_z": s_z, "acc2": acc2, "y": bf16_round(y32)}


def w8a8_fp64_reference(xq, s_x, Aq, s_A, Bq, s_B) -> np.ndarray:
    """The same W8A8 method evaluated in float64: z = (X A) in float64, per-token
    requant of z with the same rule (s_z = max|z| / 127, rint ties to even,
    clamp to +-127), y = (z_q s_z) B, all in float64 (no fp32 or bf16 rounding).
    """
    X = _np(xq).astype(np.float64) * _np(s_x).astype(np.float64)[:, None]
    A = (_np(Aq).astype(np.float64) * _np(s_A).astype(np.float64)[:, None]).T
    B = _np(Bq).astype(np.float64) * _np(s_B).astype(np.float64)[None, :]
    z = X @ A
    s_z = np.abs(z).max(axis=1) / 127.0
    zero = s_z == 0.0
    s_safe = np.where(zero, 1.0, s_z)
    zq = np.clip(np.rint(z / s_safe[:, None]), -127, 127)
    zq[zero, :] = 0.0
    return (zq * s_safe[:, None]) @ B


def w8a8_dequant_reference(xq, s_x, Aq, s_A, Bq, s_B) -> np.ndarray:
    """Float64 definition without the latent requant: y = (X A) B with X = xq s_x,
    A = (Aq s_A)^T, B = Bq s_B (column scales)."""
    X = _np(xq).astype(np.float64) * _np(s_x).astype(np.float64)[:, None]
    A = (_np(Aq).astype(np.float64) * _np(s_A).astype(np.float64)[:, None]).T
    B = _np(Bq).astype(np.float64) * _np(s_B).astype(np.float64)[None, :]
    return (X @ A) @ B
