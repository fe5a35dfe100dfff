"""CPU pins of the full-K/V decode-attention oracle (the uncompressed baseline)."""
import numpy as np
import torch

from oracle import attention, latent_kv


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_matches_torch_sdpa():
    q = _rand((2, 3, 16), 0)
    K = _rand((2, 3, 40, 16), 1)
    V = _rand((2, 3, 40, 16), 2)
    o = attention.decode_attention(q, K, V, [40, 40], 0.25)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[:, :, None, :], torch.from_numpy(K), torch.from_numpy(V), scale=0.25)[:, :, 0, :]
    assert np.abs(o - ref.numpy()).max() < 1e-12


def test_single_token_zero_keys_and_empty():
    q = _rand((1, 1, 8), 3)
    K = _rand((1, 1, 5, 8), 4)
    V = _rand((1, 1, 5, 8), 5)
    assert np.allclose(attention.decode_attention(q, K, V, [1], 1.0)[0, 0], V[0, 0, 0], atol=1e-15)
    o = attention.decode_attention(q, np.zeros_like(K), V, [5], 1.0)
    assert np.allclose(o[0, 0], V[0, 0].mean(0), atol=1e-14)
    assert (attention.decode_attention(q, K, V, [0], 1.0) == 0).all()


def test_ragged_lengths_ignore_the_tail():
    q = _rand((2, 1, 8), 6)
    K = _rand((2, 1, 20, 8), 7)
    V = _rand((2, 1, 20, 8), 8)
    o = attention.decode_attention(q, K, V, [7, 20], 0.5)
    K2, V2 = K.copy(), V.copy()
    K2[0, :, 7:] = 1e6      # keys past the length must not matter
    V2[0, :, 7:] = -1e6
    assert np.array_equal(o, attention.decode_attention(q, K2, V2, [7, 20], 0.5))


def test_equals_latent_form_on_reconstructed_caches():
    # K = C_K B_K, V = C_V B_V: the full-cache oracle and the latent oracle agree
    rng = np.random.default_rng(9)
    CK, CV = rng.standard_normal((2, 2, 30, 4)), rng.standard_normal((2, 2, 30, 4))
    BK, BV = rng.standard_normal((2, 4, 12)), rng.standard_normal((2, 4, 12))
    q = rng.standard_normal((2, 2, 12))
    K = np.einsum("bhtr,hrd->bhtd", CK, BK)
    V = np.einsum("bhtr,hrd->bhtd", CV, BV)
    a = attention.decode_attention(q, K, V, [30, 17], 0.3)
    b = latent_kv.latent_kv_decode(q, CK, CV, BK, BV, [30, 17], 0.3)
    assert np.abs(a - b).max() < 1e-12
