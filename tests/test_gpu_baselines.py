"""GPU parity: the uncompressed baselines (dense GEMV, flash decoding over full K/V)
against the float64 oracle, and the latent path against full-K/V decoding."""
import numpy as np
import pytest
import torch

import decode_lr_linear_b200 as lr
from decode_lr_linear_b200 import synth
from oracle import attention, lowrank
from tests._helpers import NORMWISE_TOL, dev, normwise_rel

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d_in,d_out,batch", [(4096, 12288, 1), (4096, 4096, 3), (1040, 1000, 8), (512, 24, 11)])
def test_dense_bf16(cuda_device, d_in, d_out, batch):
    rng = np.random.default_rng(d_in + d_out + batch)
    W = torch.from_numpy((rng.standard_normal((d_out, d_in)) / np.sqrt(d_in)).astype(np.float32)).to(torch.bfloat16)
    x = synth.make_activations(batch, d_in, seed=1, key=(100, d_in, batch))
    y = lr.lr_dense_linear(dev(W), dev(x))
    ref = lowrank.dense_linear(x.double().numpy(), W.double().numpy().T)
    assert normwise_rel(y, ref) < NORMWISE_TOL


@pytest.mark.parametrize("scale_dtype", [torch.float16, torch.float32])
def test_dense_int8(cuda_device, scale_dtype):
    rng = np.random.default_rng(7)
    Wf = rng.standard_normal((5632, 4096)) / 64.0
    q, s = synth.rtn_int8_rows(Wf, np.float16 if scale_dtype == torch.float16 else np.float32)
    x = synth.make_activations(4, 4096, seed=2, key=(101,), outliers=4)
    y = lr.lr_dense_linear(dev(torch.from_numpy(q)), dev(x), dev(torch.from_numpy(s)))
    W = q.astype(np.float64) * s.astype(np.float64)[:, None]
    assert normwise_rel(y, lowrank.dense_linear(x.double().numpy(), W.T)) < NORMWISE_TOL


def _full_caches(d):
    """K = C_K B_K, V = C_V B_V (per head), rounded to bf16, as full caches."""
    K = torch.einsum("bhtr,hrd->bhtd", d["C_K"].float(), d["B_K"].float()).to(torch.bfloat16)
    V = torch.einsum("bhtr,hrd->bhtd", d["C_V"].float(), d["B_V"].float()).to(torch.bfloat16)
    return K, V


@pytest.mark.parametrize("split", [0, 64, 256])
def test_flash_ragged_all_pairs(cuda_device, split):
    seq = [1, 63, 64, 65, 300, 1000, 0, 777]
    d = synth.make_latent_kv(batch=8, heads=4, ctx=1000, seed=12, seq_lens=seq)
    K, V = _full_caches(d)
    o = lr.lr_flash_decode(dev(d["q"]), dev(K), dev(V), dev(d["seq_lens"]), d["scale"], split_tokens=split)
    ref = attention.decode_attention(d["q"], K, V, d["seq_lens"], d["scale"])
    o = o.float().cpu().numpy()
    for b in range(8):
        if seq[b] == 0:
            assert np.abs(o[b]).max() == 0.0
            continue
        assert normwise_rel(o[b], ref[b]) < NORMWISE_TOL, (b, seq[b])


def test_flash_full_size_sampled_and_equal_to_latent(cuda_device):
    d = synth.make_latent_kv(batch=8, heads=32, ctx=4096, seed=0)
    K, V = _full_caches(d)
    o = lr.lr_flash_decode(dev(d["q"]), dev(K), dev(V), dev(d["seq_lens"]), d["scale"]).float().cpu().numpy()
    kv = lr.LatentKv(8, 32, 4096, dev(d["B_K"]), dev(d["B_V"]), d["scale"])
    ol = lr.lr_latent_kv_decode(kv, dev(d["q"]), dev(d["C_K"]), dev(d["C_V"]), dev(d["seq_lens"])).float().cpu().numpy()
    rng = np.random.default_rng(3)
    pairs = [(int(b), int(h)) for b, h in zip(rng.integers(0, 8, 10), rng.integers(0, 32, 10))]
    ref = attention.decode_attention(d["q"], K, V, d["seq_lens"], d["scale"], pairs)
    for b, h in pairs:
        assert normwise_rel(o[b, h][None], ref[b, h][None]) < NORMWISE_TOL
    # same attention from the latent caches (K, V differ only by the bf16 rounding of the reconstruction)
    assert normwise_rel(ol, o) < NORMWISE_TOL
    assert lr.lr_check_device_error() == 0
