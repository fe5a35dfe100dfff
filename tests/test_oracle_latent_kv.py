"""Pins for oracle.latent_kv: brute force, closed forms and a library reduction (CPU only)."""
import math

import numpy as np
import torch
import torch.nn.functional as F

from oracle import latent_kv as O


def _brute(q, CK, CV, BK, BV, seq_lens, scale):
    nb, nh, hd = q.shape
    r = CK.shape[-1]
    out = np.zeros((nb, nh, hd))
    for b in range(nb):
        for h in range(nh):
            n = int(seq_lens[b])
            s = []
            for t in range(n):
                kt = [sum(CK[b, h, t, j] * BK[h, j, d] for j in range(r)) for d in range(hd)]
                s.append(scale * sum(q[b, h, d] * kt[d] for d in range(hd)))
            m = max(s)
            w = [math.exp(v - m) for v in s]
            tot = sum(w)
            for d in range(hd):
                out[b, h, d] = sum(w[t] / tot * sum(CV[b, h, t, j] * BV[h, j, d] for j in range(r))
                                   for t in range(n))
    return out


def _case(rng, nb=2, nh=2, L=9, r=3, hd=4):
    return (rng.standard_normal((nb, nh, hd)), rng.standard_normal((nb, nh, L, r)),
            rng.standard_normal((nb, nh, L, r)), rng.standard_normal((nh, r, hd)),
            rng.standard_normal((nh, r, hd)))


def test_brute_force_ragged():
    rng = np.random.default_rng(0)
    q, CK, CV, BK, BV = _case(rng)
    seq = np.array([5, 9])
    ref = _brute(q, CK, CV, BK, BV, seq, 0.37)
    o1 = O.latent_kv_decode(q, CK, CV, BK, BV, seq, 0.37)
    o2 = O.latent_kv_decode_absorbed(q, CK, CV, BK, BV, seq, 0.37)
    assert np.abs(o1 - ref).max() < 1e-12
    assert np.abs(o2 - ref).max() < 1e-12


def test_absorbed_equals_reconstructed():
    rng = np.random.default_rng(1)
    q, CK, CV, BK, BV = _case(rng, nb=3, nh=4, L=257, r=32, hd=128)
    seq = np.array([257, 100, 1])
    o1 = O.latent_kv_decode(q, CK, CV, BK, BV, seq, 1 / math.sqrt(128))
    o2 = O.latent_kv_decode_absorbed(q, CK, CV, BK, BV, seq, 1 / math.sqrt(128))
    assert np.abs(o1 - o2).max() < 1e-12


def test_single_token_returns_its_value():
    rng = np.random.default_rng(2)
    q, CK, CV, BK, BV = _case(rng, L=4)
    o = O.latent_kv_decode(q, CK, CV, BK, BV, np.array([1, 1]), 0.5)
    for b in range(2):
        for h in range(2):
            assert np.abs(o[b, h] - CV[b, h, 0] @ BV[h]).max() < 1e-12


def test_zero_keys_give_mean_value():
    rng = np.random.default_rng(3)
    q, CK, CV, BK, BV = _case(rng, L=6)
    CK[:] = 0.0
    o = O.latent_kv_decode(q, CK, CV, BK, BV, np.array([6, 4]), 0.5)
    for b, n in ((0, 6), (1, 4)):
        for h in range(2):
            assert np.abs(o[b, h] - (CV[b, h, :n] @ BV[h]).mean(axis=0)).max() < 1e-12


def test_two_token_closed_form():
    """Scores 0 and ln 3 give weights 1/4 and 3/4."""
    q = np.ones((1, 1, 1))
    CK = np.array([0.0, math.log(3.0)]).reshape(1, 1, 2, 1)
    CV = np.array([2.0, -6.0]).reshape(1, 1, 2, 1)
    one = np.ones((1, 1, 1))
    o = O.latent_kv_decode(q, CK, CV, one, one, np.array([2]), 1.0)
    assert abs(o[0, 0, 0] - (0.25 * 2.0 + 0.75 * -6.0)) < 1e-14


def test_identity_factors_reduce_to_sdpa():
    """B_K = B_V = [I_32 | 0]: latent attention is plain attention with head_dim 32."""
    rng = np.random.default_rng(4)
    nb, nh, L, r, hd = 2, 3, 50, 32, 128
    q = rng.standard_normal((nb, nh, hd))
    CK = rng.standard_normal((nb, nh, L, r))
    CV = rng.standard_normal((nb, nh, L, r))
    I = np.zeros((nh, r, hd))
    I[:, :, :r] = np.eye(r)
    scale = 1 / math.sqrt(hd)
    o = O.latent_kv_decode(q, CK, CV, I, I, np.array([L, L]), scale)
    ref = F.scaled_dot_product_attention(torch.from_numpy(q[:, :, None, :r]), torch.from_numpy(CK),
                                         torch.from_numpy(CV), scale=scale)[:, :, 0]
    assert np.abs(o[..., :r] - ref.numpy()).max() < 1e-12
    assert np.abs(o[..., r:]).max() == 0.0


def test_int8_cache_dequantization_and_invariants():
    from decode_lr_linear_b200 import synth
    d = synth.make_latent_kv_int8(batch=2, heads=2, ctx=40, seed=3, seq_lens=[40, 13])
    # dequantization is the elementwise product with the per-position scale
    from oracle import latent_kv
    C = latent_kv.dequantize_cache(d["C_Kq"], d["s_K"])
    t = 7
    assert np.array_equal(C[1, 0, t], d["C_Kq"][1, 0, t].double().numpy() * float(d["s_K"][1, 0, t]))
    o = latent_kv.latent_kv_decode_q8(d["q"], d["C_Kq"], d["s_K"], d["C_Vq"], d["s_V"], d["B_K"], d["B_V"],
                                      d["seq_lens"], d["scale"])
    # scaling every key scale by c and the query by 1/c leaves the scores unchanged
    o2 = latent_kv.latent_kv_decode_q8(d["q"].double() / 8.0, d["C_Kq"], d["s_K"].double() * 8.0, d["C_Vq"],
                                       d["s_V"], d["B_K"], d["B_V"], d["seq_lens"], d["scale"])
    assert np.abs(o - o2).max() < 1e-12
    # scaling every value scale by c scales the output by c
    o3 = latent_kv.latent_kv_decode_q8(d["q"], d["C_Kq"], d["s_K"], d["C_Vq"], d["s_V"].double() * 3.0, d["B_K"],
                                       d["B_V"], d["seq_lens"], d["scale"])
    assert np.abs(o3 - 3.0 * o).max() < 1e-12
    # brute force on one head, written out
    b, h, n = 1, 1, 13
    K = (d["C_Kq"][b, h, :n].double().numpy() * d["s_K"][b, h, :n].double().numpy()[:, None]) @ d["B_K"][h].double().numpy()
    V = (d["C_Vq"][b, h, :n].double().numpy() * d["s_V"][b, h, :n].double().numpy()[:, None]) @ d["B_V"][h].double().numpy()
    s = np.array([K[i] @ d["q"][b, h].double().numpy() for i in range(n)]) * d["scale"]
    p = np.exp(s - s.max()) / np.exp(s - s.max()).sum()
    assert np.abs(o[b, h] - sum(p[i] * V[i] for i in range(n))).max() < 1e-12
