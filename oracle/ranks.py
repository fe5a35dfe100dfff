"""Oracle: FLRC rank allocation from per-projection importances (test infrastructure only).

FLRC "Fisher-based layer-wise rank allocation": with importances alpha_{l,p}
and their total S, projection p gets r_{l,p} = round(alpha_{l,p} / S * R_budget).
FLRC "progressive low-rank decoding": token t uses
r_{l,p}(t) = round(alpha_{l,p} / S * R_budget(t)) with a non-increasing
budget schedule R_budget(t).

Readings where the pages are silent: "round" is to nearest with ties to even;
S is summed in index order; each rank is clamped to [1, cap_p], the rank the
stored factors hold (a zero rank would drop the projection).
"""
from __future__ import annotations

import numpy as np


def flrc_ranks(alpha, r_budget: float, caps) -> np.ndarray:
    """r_p = clamp(rint(alpha_p / S * r_budget), 1, caps_p), S = sum of alpha in index order."""
    alpha = [float(a) for a in alpha]
    S = 0.0
    for a in alpha:
        S += a
    out = []
    for a, cap in zip(alpha, caps):
        r = float(np.rint((a / S) * float(r_budget)))
        out.append(int(min(max(r, 1.0), float(cap))))
    return np.asarray(out, np.int64)


def progressive_ranks(alpha, budgets, caps) -> np.ndarray:
    """[tokens, n] ranks for a budget schedule R_budget(t), t = 0, 1, ..."""
    return np.stack([flrc_ranks(alpha, b, caps) for b in budgets])
