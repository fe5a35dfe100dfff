"""Shared helpers for the parity tests (no method arithmetic here)."""
import numpy as np
import torch

# Parity bar for floating-point outputs: max over rows of ||y - y_ref||_2 / ||y_ref||_2
# against the float64 oracle.
NORMWISE_TOL = 1e-2


def normwise_rel(y, ref) -> float:
    y = y.detach().float().cpu().double().numpy() if hasattr(y, "detach") else np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    y = y.reshape(-1, y.shape[-1])
    ref = ref.reshape(-1, ref.shape[-1])
    num = np.linalg.norm(y - ref, axis=1)
    den = np.linalg.norm(ref, axis=1)
    den = np.where(den == 0, 1.0, den)
    return float((num / den).max())


def dev(t, device="cuda"):
    return t.to(device).contiguous()
