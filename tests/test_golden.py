"""The oracle against the closed-form fixtures in tests/golden (CPU only)."""
import json
import os

import numpy as np

from decode_lr_linear_b200 import synth
from oracle import latent_kv, lowrank

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def test_eckart_young_fixture():
    g = _load("eckart_young_256_r32.json")
    d = synth.make_single_linear(0, d=g["d"], rank=g["rank"])
    A, B = lowrank.truncated_svd(d["W"], g["rank"])
    err = lowrank.truncation_error(d["W"], A, B)
    assert abs(err - g["frobenius_error"]) < 1e-10
    assert abs(err / np.linalg.norm(d["W"]) - g["relative_frobenius_error"]) < 1e-10
    assert abs(np.linalg.norm(d["W"] - A @ B, 2) - g["spectral_error"]) < 1e-10
    assert abs(lowrank.retained_energy_ratio(lowrank.singular_values(d["W"]), g["rank"])
               - g["retained_energy_ratio"]) < 1e-12


def test_two_token_fixture():
    g = _load("attention_two_tokens.json")
    q = np.ones((1, 1, 1))
    CK = np.array(g["scores"]).reshape(1, 1, 2, 1)
    CV = np.array(g["values"]).reshape(1, 1, 2, 1)
    one = np.ones((1, 1, 1))
    for fn in (latent_kv.latent_kv_decode, latent_kv.latent_kv_decode_absorbed):
        o = fn(q, CK, CV, one, one, np.array([2]), 1.0)
        assert abs(o[0, 0, 0] - g["output"]) < 1e-14
