"""Writes the closed-form fixtures in this folder.

Only exact rational arithmetic (``fractions``) and ``math`` are used: no
oracle call is needed for a closed form, and nothing here touches the CUDA
library.  Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import math
import os
from fractions import Fraction

HERE = os.path.dirname(os.path.abspath(__file__))


def harmonic(n):
    return sum(Fraction(1, i) for i in range(1, n + 1))


def eckart_young(d=256, r=32):
    h_d, h_r = harmonic(d), harmonic(r)
    return {
        "citation": ("SAES-SVD technical summary (low-rank compression via truncated SVD, CEALC local "
                     "objective; ACES retained energy ratio) and Swift-SVD results (numerical stability: "
                     "reconstruction error against the theoretical minimum). Spectrum sigma_i = i^-1/2, i=1..d."),
        "d": d, "rank": r,
        "frobenius_error": math.sqrt(float(h_d - h_r)),
        "relative_frobenius_error": math.sqrt(float((h_d - h_r) / h_d)),
        "spectral_error": 1.0 / math.sqrt(r + 1),
        "retained_energy_ratio": float(h_r / h_d),
        "derivation": "||W - W_r||_F^2 = sum_{i>r} 1/i = H_d - H_r; ||W||_F^2 = H_d; RER = H_r / H_d.",
    }


def two_token_attention():
    return {
        "citation": "WSVD, per-head latent cache attention (single query, softmax over cached tokens).",
        "scores": [0.0, math.log(3.0)], "values": [2.0, -6.0],
        "output": 0.25 * 2.0 + 0.75 * -6.0,
        "derivation": "softmax(0, ln 3) = (1/4, 3/4); o = v0/4 + 3 v1/4.",
    }


if __name__ == "__main__":
    with open(os.path.join(HERE, "eckart_young_256_r32.json"), "w") as f:
        json.dump(eckart_young(), f, indent=1)
    with open(os.path.join(HERE, "attention_two_tokens.json"), "w") as f:
        json.dump(two_token_attention(), f, indent=1)
