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


# ---- rotary positions, the reconstruct-on-chip form and the producer -------
def test_rope_matches_complex_rotation():
    # RoFormer's complex form: pair (x_i, x_{i+h}) as x_i + i x_{i+h}, multiplied by e^{i pos theta_i}
    rng = np.random.default_rng(10)
    x = rng.standard_normal((5, 16))
    pos = np.array([0, 1, 7, 1000, 32767])
    base = 10000.0
    theta = base ** (-np.arange(8) * 2.0 / 16.0)
    z = (x[:, :8] + 1j * x[:, 8:]) * np.exp(1j * pos[:, None] * theta[None, :])
    want = np.concatenate([z.real, z.imag], axis=1)
    assert np.abs(O.rope(x, pos, base) - want).max() < 1e-12
    assert np.abs(O.rope(x[:1], 0, base) - x[:1]).max() == 0.0          # position 0: identity
    assert np.allclose(np.linalg.norm(O.rope(x, pos, base), axis=1), np.linalg.norm(x, axis=1))


def test_rope_matches_llama_library_routine():
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb
    rng = np.random.default_rng(11)
    hd, L, base = 128, 40, 10000.0
    q = torch.from_numpy(rng.standard_normal((1, 1, L, hd)))
    k = torch.from_numpy(rng.standard_normal((1, 1, L, hd)))
    inv = 1.0 / (base ** (torch.arange(0, hd, 2, dtype=torch.float64) / hd))
    ang = torch.arange(L, dtype=torch.float64)[:, None] * inv[None, :]
    emb = torch.cat([ang, ang], dim=-1)
    qr, kr = apply_rotary_pos_emb(q, k, emb.cos()[None], emb.sin()[None])
    pos = np.arange(L)
    assert np.abs(O.rope(q[0, 0].numpy(), pos, base) - qr[0, 0].numpy()).max() < 1e-12
    assert np.abs(O.rope(k[0, 0].numpy(), pos, base) - kr[0, 0].numpy()).max() < 1e-12


def test_rope_scores_depend_on_relative_position_only():
    rng = np.random.default_rng(12)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for a, b, c in ((3, 10, 5), (100, 7, 4000), (0, 0, 31)):
        s1 = O.rope(q, a, 500.0) @ O.rope(k, b, 500.0)
        s2 = O.rope(q, a + c, 500.0) @ O.rope(k, b + c, 500.0)
        assert abs(s1 - s2) < 1e-9


def _brute_rope(q, CK, CV, BK, BV, seq_lens, scale, base):
    nb, nh, hd = q.shape
    r, half = CK.shape[-1], hd // 2
    out = np.zeros((nb, nh, hd))

    def rot(v, pos):
        w = [0.0] * hd
        for i in range(half):
            a = pos * base ** (-2.0 * i / hd)
            w[i] = v[i] * math.cos(a) - v[i + half] * math.sin(a)
            w[i + half] = v[i + half] * math.cos(a) + v[i] * math.sin(a)
        return w

    for b in range(nb):
        for h in range(nh):
            n = int(seq_lens[b])
            if n == 0:
                continue
            qr = rot(list(q[b, h]), n - 1)
            s = []
            for t in range(n):
                kt = rot([sum(CK[b, h, t, j] * BK[h, j, d] for j in range(r)) for d in range(hd)], t)
                s.append(scale * sum(qr[d] * kt[d] for d in range(hd)))
            m = max(s)
            w = [math.exp(v - m) for v in s]
            tot = sum(w)
            for d in range(hd):
                out[b, h, d] = sum(w[t] / tot * sum(CV[b, h, t, j] * BV[h, j, d] for j in range(r))
                                   for t in range(n))
    return out


def test_rope_decode_brute_force_ragged():
    rng = np.random.default_rng(13)
    q, CK, CV, BK, BV = _case(rng, nb=3, nh=2, L=11, r=3, hd=6)
    seq = np.array([11, 4, 0])
    ref = _brute_rope(q, CK, CV, BK, BV, seq, 0.41, 50.0)
    got = O.latent_kv_decode_rope(q, CK, CV, BK, BV, seq, 0.41, 50.0)
    assert np.abs(got - ref).max() < 1e-12
    assert np.all(got[2] == 0.0)


def test_rope_decode_special_cases():
    rng = np.random.default_rng(14)
    q, CK, CV, BK, BV = _case(rng, nb=2, nh=2, L=6, r=4, hd=8)
    # one cached token: query and key both at position 0, no rotation; output V_0
    one = np.array([1, 1])
    assert np.abs(O.latent_kv_decode_rope(q, CK, CV, BK, BV, one, 0.3, 10000.0)
                  - O.latent_kv_decode(q, CK, CV, BK, BV, one, 0.3)).max() < 1e-12
    # rotation changes the scores of a longer context (the absorbed form is not exact any more)
    full = np.array([6, 6])
    d = np.abs(O.latent_kv_decode_rope(q, CK, CV, BK, BV, full, 0.3, 10.0)
               - O.latent_kv_decode(q, CK, CV, BK, BV, full, 0.3)).max()
    assert d > 1e-3
    # keys rotated explicitly, then the unrotated oracle on a cache whose factor is the identity
    b, h, n, base = 0, 1, 6, 10.0
    K = O.rope(CK[b, h, :n] @ BK[h], np.arange(n), base)
    qr = O.rope(q[b, h], n - 1, base)
    ref = O.decode_head(qr, K, CV[b, h, :n], np.eye(8), BV[h], n, 0.3)
    assert np.abs(O.decode_head_rope(q[b, h], CK[b, h], CV[b, h], BK[h], BV[h], n, 0.3, base) - ref).max() < 1e-12


def test_append_latents_brute_force_and_exact_rank_key():
    rng = np.random.default_rng(15)
    nb, nh, r, hidden, ctx, hd = 3, 2, 3, 10, 5, 4
    x = rng.standard_normal((nb, hidden))
    A = rng.standard_normal((2 * nh * r, hidden))
    CK, CV = rng.standard_normal((nb, nh, ctx, r)), rng.standard_normal((nb, nh, ctx, r))
    pos = np.array([2, 4, 5])                     # the last one is outside the cache: unchanged
    ck, cv = O.append_latents(x, A, nh, r, CK, CV, pos)
    for b in range(nb):
        for h in range(nh):
            for t in range(ctx):
                for j in range(r):
                    if t == pos[b]:
                        wk = sum(x[b, i] * A[h * r + j, i] for i in range(hidden))
                        wv = sum(x[b, i] * A[(nh + h) * r + j, i] for i in range(hidden))
                    else:
                        wk, wv = CK[b, h, t, j], CV[b, h, t, j]
                    assert abs(ck[b, h, t, j] - wk) < 1e-12 and abs(cv[b, h, t, j] - wv) < 1e-12
    # the appended latent reconstructs the key of the exactly-rank-r per-head projection W_Kh = A_Kh B_Kh
    BK = rng.standard_normal((nh, r, hd))
    for h in range(nh):
        W = A[h * r:(h + 1) * r].T @ BK[h]         # hidden x head_dim
        assert np.abs(ck[0, h, pos[0]] @ BK[h] - x[0] @ W).max() < 1e-12
