"""Pins for oracle.w8a8: integer exactness, rounding rule, error bounds (CPU only)."""
import numpy as np

from decode_lr_linear_b200 import synth
from oracle import w8a8 as O


def test_int_matmul_exact_against_integer_arithmetic():
    rng = np.random.default_rng(0)
    a = rng.integers(-127, 128, size=(5, 300)).astype(np.int8)
    b = rng.integers(-127, 128, size=(7, 300)).astype(np.int8)
    ref = np.einsum("ti,ki->tk", a.astype(np.int64), b.astype(np.int64))
    assert np.array_equal(O.int_matmul_nt(a, b), ref)


def test_int_matmul_extreme_values():
    k = 13824
    a = np.full((2, k), 127, np.int8); a[1] = -127
    b = np.full((3, k), -127, np.int8); b[2, ::2] = 127
    c = O.int_matmul_nt(a, b)
    assert c[0, 0] == -127 * 127 * k and c[1, 0] == 127 * 127 * k
    assert c[0, 2] == 0 and abs(c[0, 0]) < 2 ** 31


def test_quantize_ties_to_even_and_extremes():
    x = np.array([[127.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, 0.0]], np.float32)
    q, s = O.quantize_per_token(x)
    assert s[0] == np.float32(1.0)
    assert q.tolist() == [[127, 2, 4, -2, 0, 0, 2, 0]]
    q0, s0 = O.quantize_per_token(np.zeros((1, 4), np.float32))
    assert s0[0] == 1.0 and not q0.any()
    q1, s1 = O.quantize_per_token(np.array([[-3.0, 1.0]], np.float32))
    assert q1[0, 0] == -127


def test_quantize_reconstruction_bound():
    x = synth.make_activations(16, 512, seed=0, key=(9,), outliers=3).float().numpy()
    q, s = O.quantize_per_token(x)
    err = np.abs(x - q.astype(np.float64) * s[:, None].astype(np.float64))
    assert (err <= s[:, None] * (0.5 + 1e-5)).all()
    assert (np.abs(q).max(axis=1) == 127).all()


def test_requant_rounding_order_is_fp32():
    rng = np.random.default_rng(2)
    acc = rng.integers(-2 ** 27, 2 ** 27, size=(4, 64)).astype(np.int64)
    sx = rng.uniform(1e-3, 1e-2, 4).astype(np.float32)
    sa = rng.uniform(1e-4, 1e-3, 64).astype(np.float32)
    z, zq, sz = O.requant_latent(acc, sx, sa)
    assert z.dtype == np.float32
    exact = acc.astype(np.float64) * sx[:, None].astype(np.float64) * sa[None, :].astype(np.float64)
    # conversion + two products: at most 3 roundings of 2^-24 relative each
    assert (np.abs(z - exact) <= 3.01 * 2.0 ** -24 * np.abs(exact) + 1e-30).all()
    assert (np.abs(zq).max(axis=1) == 127).all()


def test_pipeline_close_to_fp64_definition():
    rng = np.random.default_rng(3)
    d_in, d_out, r, T = 256, 192, 64, 40
    p = synth.make_prefill_projection(d_in, d_out, r, seed=0, key=(0,))
    x = synth.make_activations(T, d_in, seed=0, key=(10,), outliers=1)
    xq, sx = O.quantize_per_token(x)
    res = O.w8a8_lr_linear(xq, sx, p["A_q"], p["s_A"], p["B_q"], p["s_B"])
    ref = O.w8a8_dequant_reference(xq, sx, p["A_q"], p["s_A"], p["B_q"], p["s_B"])
    rel = np.linalg.norm(res["y"] - ref, axis=1) / np.linalg.norm(ref, axis=1)
    assert rel.max() < 1e-2
    ref2 = np.einsum("tj,jk->tk", res["zq"].astype(np.int64), p["B_q"].numpy().astype(np.int64))
    assert np.array_equal(res["acc2"], ref2)
    del rng


def test_unit_scale_integer_pipeline():
    """With unit weight scales and an activation scale of 1, z equals acc1 exactly."""
    rng = np.random.default_rng(4)
    xq = rng.integers(-5, 6, size=(3, 32)).astype(np.int8)
    Aq = rng.integers(-5, 6, size=(8, 32)).astype(np.int8)
    Bq = rng.integers(-5, 6, size=(8, 6)).astype(np.int8)
    one = np.ones
    res = O.w8a8_lr_linear(xq, one(3, np.float32), Aq, one(8, np.float32), Bq, one(6, np.float32))
    acc1 = xq.astype(np.int64) @ Aq.astype(np.int64).T
    assert np.array_equal(res["z"], acc1.astype(np.float32))


def _brute_fp64_method(xq, sx, Aq, sA, Bq, sB):
    T, d_in = xq.shape
    r, d_out = Aq.shape[0], Bq.shape[1]
    y = np.zeros((T, d_out))
    for t in range(T):
        z = [sum(float(xq[t, i]) * float(sx[t]) * float(Aq[j, i]) * float(sA[j]) for i in range(d_in))
             for j in range(r)]
        sz = max(abs(v) for v in z) / 127.0
        if sz == 0.0:
            continue
        zq = [min(127.0, max(-127.0, float(np.rint(v / sz)))) for v in z]
        for k in range(d_out):
            y[t, k] = sum(zq[j] * sz * float(Bq[j, k]) * float(sB[k]) for j in range(r))
    return y


def test_fp64_method_brute_force_and_zero_row():
    rng = np.random.default_rng(8)
    xq = rng.integers(-127, 128, size=(3, 9)).astype(np.int8)
    xq[1] = 0
    sx = rng.uniform(0.01, 0.1, 3)
    Aq = rng.integers(-127, 128, size=(5, 9)).astype(np.int8)
    sA = rng.uniform(0.001, 0.01, 5)
    Bq = rng.integers(-127, 128, size=(5, 4)).astype(np.int8)
    sB = rng.uniform(0.001, 0.01, 4)
    y = O.w8a8_fp64_reference(xq, sx, Aq, sA, Bq, sB)
    assert np.abs(y - _brute_fp64_method(xq, sx, Aq, sA, Bq, sB)).max() < 1e-12
    assert not y[1].any()


def test_fp64_method_agrees_with_fp32_pipeline():
    """The fp32-exact pipeline and the float64 method differ only by rounding."""
    p = synth.make_prefill_projection(384, 256, 96, seed=2, key=(2,))
    x = synth.make_activations(64, 384, seed=2, key=(11,), outliers=1)
    xq, sx = O.quantize_per_token(x)
    res = O.w8a8_lr_linear(xq, sx, p["A_q"], p["s_A"], p["B_q"], p["s_B"])
    y64 = O.w8a8_fp64_reference(xq, sx, p["A_q"], p["s_A"], p["B_q"], p["s_B"])
    rel = np.linalg.norm(res["y"] - y64, axis=1) / np.linalg.norm(y64, axis=1)
    assert rel.max() < 5e-3
