"""Pins for oracle.ffn: brute force, library reductions and invariants (CPU only)."""
import math

import numpy as np
import torch
import torch.nn.functional as F

from decode_lr_linear_b200 import synth
from oracle import ffn as O


def _rand_q(rng, shape):
    return rng.integers(-127, 128, size=shape).astype(np.int8)


def _tiny_case(seed=0, hidden=5, n_lr=2, n_dense=3, r=2):
    rng = np.random.default_rng(seed)
    inter = n_lr + n_dense
    return dict(
        x=rng.standard_normal((2, hidden)),
        A_q=_rand_q(rng, (r, hidden)), s_A=rng.uniform(0.001, 0.01, r),
        B_q=_rand_q(rng, (r, 2 * n_lr)), s_B=rng.uniform(0.001, 0.01, 2 * n_lr),
        D_q=_rand_q(rng, (2 * n_dense, hidden)), s_D=rng.uniform(0.001, 0.01, 2 * n_dense),
        Wd_q=_rand_q(rng, (inter, hidden)), s_d=rng.uniform(0.001, 0.01, hidden),
        n_lr=n_lr, n_dense=n_dense,
    )


def _brute_ffn(c):
    """Element-by-element loops over the stored tensors, with math.exp."""
    x = c["x"]
    nb, hidden = x.shape
    r = c["A_q"].shape[0]
    n_lr, n_dense = c["n_lr"], c["n_dense"]
    y = np.zeros((nb, hidden))
    for b in range(nb):
        h = []
        z = [sum(x[b, i] * float(c["A_q"][j, i]) * c["s_A"][j] for i in range(hidden)) for j in range(r)]
        for ch in range(n_lr):
            g = sum(z[j] * float(c["B_q"][j, 2 * ch]) * c["s_B"][2 * ch] for j in range(r))
            u = sum(z[j] * float(c["B_q"][j, 2 * ch + 1]) * c["s_B"][2 * ch + 1] for j in range(r))
            h.append(g / (1 + math.exp(-g)) * u)
        for ch in range(n_dense):
            g = sum(x[b, i] * float(c["D_q"][2 * ch, i]) * c["s_D"][2 * ch] for i in range(hidden))
            u = sum(x[b, i] * float(c["D_q"][2 * ch + 1, i]) * c["s_D"][2 * ch + 1] for i in range(hidden))
            h.append(g / (1 + math.exp(-g)) * u)
        for k in range(hidden):
            y[b, k] = sum(h[c2] * float(c["Wd_q"][c2, k]) * c["s_d"][k] for c2 in range(len(h)))
    return y


def test_brute_force_tiny():
    for seed in range(3):
        c = _tiny_case(seed)
        y, _ = O.hybrid_swiglu_ffn(**c)
        ref = _brute_ffn(c)
        assert np.abs(y - ref).max() < 1e-12 * max(1.0, np.abs(ref).max())


def test_silu_against_torch():
    t = np.linspace(-30, 30, 1001)
    ref = F.silu(torch.from_numpy(t)).numpy()
    assert np.abs(O.silu(t) - ref).max() < 1e-14
    assert O.silu(np.array([0.0]))[0] == 0.0


def test_no_lowrank_channels_is_dense_swiglu():
    """S empty: the hybrid FFN reduces to a dense SwiGLU FFN (torch fp64, F.silu)."""
    d = synth.make_hybrid_ffn(seed=0, hidden=64, inter=48, n_lr=0, rank=512, rotate=False)
    x = np.random.default_rng(3).standard_normal((3, 64))
    y, _ = O.hybrid_swiglu_ffn(x, d["A_q"], d["s_A"], d["B_q"], d["s_B"], d["D_q"], d["s_D"],
                               d["Wd_q"], d["s_d"], 0, 48)
    Dq = d["D_q"].double() * d["s_D"].double()[:, None]      # [2*48, 64]
    Wg, Wu = Dq[0::2].T, Dq[1::2].T                           # 64 x 48 each
    Wdown = d["Wd_q"].double() * d["s_d"].double()[None, :]  # 48 x 64
    xt = torch.from_numpy(x)
    ref = (F.silu(xt @ Wg) * (xt @ Wu)) @ Wdown
    assert np.abs(y - ref.numpy()).max() < 1e-12


def test_integer_preactivations_exact():
    """Integer x, unit scales: every pre-activation is an exact integer sum."""
    rng = np.random.default_rng(4)
    c = _tiny_case(7, hidden=16, n_lr=3, n_dense=2, r=4)
    c["x"] = rng.integers(-3, 4, size=(2, 16)).astype(np.float64)
    for k in ("s_A", "s_B", "s_D", "s_d"):
        c[k] = np.ones_like(c[k])
    _, h = O.hybrid_swiglu_ffn(**c)
    z = c["x"].astype(np.int64) @ c["A_q"].astype(np.int64).T
    gu = z @ c["B_q"].astype(np.int64)
    g, u = gu[:, 0::2].astype(np.float64), gu[:, 1::2].astype(np.float64)
    with np.errstate(over="ignore"):
        ref = g / (1 + np.exp(-g)) * u
    assert np.abs(h[:, :3] - ref).max() <= 1e-9 * max(1, np.abs(ref).max())


def test_channel_permutation_invariance():
    """Permuting low-rank channels consistently in B (row pairs) and down_proj columns leaves y unchanged."""
    c = _tiny_case(11, hidden=6, n_lr=4, n_dense=2, r=3)
    y0, _ = O.hybrid_swiglu_ffn(**c)
    perm = np.array([2, 0, 3, 1])
    rows = np.stack([2 * perm, 2 * perm + 1], axis=1).reshape(-1)
    c2 = dict(c)
    c2["B_q"] = c["B_q"][:, rows]
    c2["s_B"] = c["s_B"][rows]
    cols = np.concatenate([perm, np.arange(4, 6)])
    c2["Wd_q"] = c["Wd_q"][cols, :]
    y1, _ = O.hybrid_swiglu_ffn(**c2)
    assert np.abs(y0 - y1).max() < 1e-12
    # swapping gate and up of one channel changes the result (silu is not symmetric)
    c3 = dict(c)
    sw = np.arange(8); sw[[0, 1]] = [1, 0]
    c3["B_q"] = c["B_q"][:, sw]; c3["s_B"] = c["s_B"][sw]
    y3, _ = O.hybrid_swiglu_ffn(**c3)
    assert np.abs(y0 - y3).max() > 1e-6


def test_math_layout_matches_stored_layout():
    c = _tiny_case(13, hidden=6, n_lr=2, n_dense=2, r=3)
    y, _ = O.hybrid_swiglu_ffn(**c)
    A = O.dequantize_rows(c["A_q"], c["s_A"]).T
    Bs = O.dequantize_cols(c["B_q"], c["s_B"])
    Ds = O.dequantize_rows(c["D_q"], c["s_D"]).T
    Wd = O.dequantize_cols(c["Wd_q"], c["s_d"])
    y2 = O.swiglu_ffn_math(c["x"], A, Bs[:, 0::2], Bs[:, 1::2], Ds[:, 0::2], Ds[:, 1::2], Wd)
    assert np.abs(y - y2).max() < 1e-12
