"""GPU parity: hybrid SwiGLU FFN, latent-KV decode attention and per-token quantisation."""

import numpy as np
import pytest
import torch

import decode_lr_linear_b200 as lr
from decode_lr_linear_b200 import synth
from oracle import ffn as offn
from oracle import latent_kv as okv
from oracle import w8a8 as ow8
from tests._helpers import NORMWISE_TOL, dev, normwise_rel

pytestmark = pytest.mark.gpu


def _ffn_dev(d):
    return lr.FfnWeights(d["hidden"], d["inter"], d["n_lr"], d["rank"], dev(d["A_q"]), dev(d["s_A"]),
                         dev(d["B_q"]), dev(d["s_B"]), dev(d["D_q"]), dev(d["s_D"]), dev(d["Wd_q"]), dev(d["s_d"]))


def _ffn_oracle(d, x):
    y, _ = offn.hybrid_swiglu_ffn(x.double().numpy(), d["A_q"], d["s_A"], d["B_q"], d["s_B"], d["D_q"], d["s_D"],
                                  d["Wd_q"], d["s_d"], d["n_lr"], d["n_dense"])
    return y


@pytest.fixture(scope="module")
def ffn7b():
    return synth.make_hybrid_ffn(seed=0)


@pytest.mark.parametrize("batch", [1, 8, 32])
def test_hybrid_ffn_llama7b(cuda_device, ffn7b, batch):
    x = synth.make_activations(batch, 4096, seed=0, key=(30, batch), outliers=4)
    y = lr.lr_swiglu_ffn(_ffn_dev(ffn7b), dev(x))
    err = normwise_rel(y, _ffn_oracle(ffn7b, x))
    assert err < NORMWISE_TOL, err


def test_hybrid_ffn_long_down_slices(cuda_device):
    # inter 20480: each unit of the down projection stages an 18-block slice of h, which at
    # 8 tokens takes more than one round of loads per pass (pieces read again for the codes)
    d = synth.make_hybrid_ffn(seed=2, hidden=4096, inter=20480, n_lr=16384, rank=256, rotate=False)
    x = synth.make_activations(8, 4096, seed=2, key=(31, 8), outliers=4)
    y = lr.lr_swiglu_ffn(_ffn_dev(d), dev(x))
    assert normwise_rel(y, _ffn_oracle(d, x)) < NORMWISE_TOL


@pytest.mark.parametrize("batch", [1, 5])
def test_hybrid_ffn_cuda_core_path(cuda_device, ffn7b, batch):
    # the CUDA-core FFN kernels (the tensor cores take every batch by default)
    lr.lr_set_tensor_core_min_batch(64, 64)
    try:
        x = synth.make_activations(batch, 4096, seed=0, key=(32, batch), outliers=4)
        assert normwise_rel(lr.lr_swiglu_ffn(_ffn_dev(ffn7b), dev(x)), _ffn_oracle(ffn7b, x)) < NORMWISE_TOL
        d = synth.make_hybrid_ffn(seed=1, hidden=512, inter=1000, n_lr=512, rank=512)
        xs = synth.make_activations(batch, 512, seed=1, key=(33, batch), outliers=1)
        assert normwise_rel(lr.lr_swiglu_ffn(_ffn_dev(d), dev(xs)), _ffn_oracle(d, xs)) < NORMWISE_TOL
    finally:
        lr.lr_set_tensor_core_min_batch(0, 0)


@pytest.mark.parametrize("n_lr", [0, 512, 1000])
def test_hybrid_ffn_small_and_degenerate(cuda_device, n_lr):
    d = synth.make_hybrid_ffn(seed=1, hidden=512, inter=1000, n_lr=n_lr, rank=512, rotate=n_lr > 0)
    x = synth.make_activations(3, 512, seed=1, key=(31, n_lr), outliers=1)
    y = lr.lr_swiglu_ffn(_ffn_dev(d), dev(x))
    assert normwise_rel(y, _ffn_oracle(d, x)) < NORMWISE_TOL


def _kv_run(d, split=0, mode=0):
    kv = lr.LatentKv(d["batch"], d["heads"], d["ctx"], dev(d["B_K"]), dev(d["B_V"]), d["scale"], mode, split)
    return lr.lr_latent_kv_decode(kv, dev(d["q"]), dev(d["C_K"]), dev(d["C_V"]), dev(d["seq_lens"]))


def _kv_oracle(d, pairs=None):
    return okv.latent_kv_decode(d["q"], d["C_K"], d["C_V"], d["B_K"], d["B_V"], d["seq_lens"], d["scale"], pairs)


@pytest.mark.parametrize("ctx", [4096, 16384, 32768])
def test_latent_kv_full_size_sampled(cuda_device, ctx):
    d = synth.make_latent_kv(batch=8, heads=32, ctx=ctx, seed=0)
    o = _kv_run(d).float().cpu().numpy()
    rng = np.random.default_rng(ctx)
    pairs = [(int(b), int(h)) for b, h in zip(rng.integers(0, 8, 12), rng.integers(0, 32, 12))]
    ref = _kv_oracle(d, pairs)
    for b, h in pairs:
        assert normwise_rel(o[b, h][None], ref[b, h][None]) < NORMWISE_TOL, (b, h)
    assert np.isfinite(o).all()


@pytest.mark.parametrize("split", [0, 64, 512])
def test_latent_kv_ragged_all_pairs(cuda_device, split):
    seq = [1, 63, 64, 65, 300, 1000, 0, 777]
    d = synth.make_latent_kv(batch=8, heads=4, ctx=1000, seed=2, seq_lens=seq)
    o = _kv_run(d, split).float().cpu().numpy()
    ref = _kv_oracle(d)
    for b in range(8):
        if seq[b] == 0:
            assert np.abs(o[b]).max() == 0.0
            continue
        assert normwise_rel(o[b], ref[b]) < NORMWISE_TOL, (b, seq[b])


def test_latent_kv_single_token_is_value(cuda_device):
    d = synth.make_latent_kv(batch=2, heads=3, ctx=128, seed=3, seq_lens=[1, 1])
    o = _kv_run(d).float().cpu().numpy()
    for b in range(2):
        for h in range(3):
            v0 = d["C_V"][b, h, 0].double().numpy() @ d["B_V"][h].double().numpy()
            assert normwise_rel(o[b, h][None], v0[None]) < NORMWISE_TOL


def test_latent_kv_peaky_softmax(cuda_device):
    d = synth.make_latent_kv(batch=2, heads=8, ctx=2048, seed=4, peak=4.0)
    o = _kv_run(d).float().cpu().numpy()
    assert normwise_rel(o, _kv_oracle(d)) < NORMWISE_TOL


# 40976 and 49152 columns: rows longer than the pieces a block holds in registers
@pytest.mark.parametrize("rows,cols", [(4, 512), (2048, 5120), (7, 13824), (5, 40976), (3, 49152)])
def test_quantize_per_token_bit_exact(cuda_device, rows, cols):
    x = synth.make_activations(rows, cols, seed=5, key=(40, rows), outliers=max(1, cols // 1000))
    xq, s = lr.lr_quantize_per_token(dev(x))
    q_ref, s_ref = ow8.quantize_per_token(x)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(xq.cpu().numpy(), q_ref)


def test_quantize_dense_ties(cuda_device):
    # max 63.5 gives s = 0.5 exactly, so every multiple of 0.25 divides to an exact
    # half-integer (a tie, rounded to even); the other rows mix in scales that are
    # not powers of two
    rng = np.random.default_rng(11)
    x = torch.from_numpy(rng.integers(-254, 255, size=(64, 2048)).astype(np.float32) * 0.25)
    x[:, 0] = 63.5
    x[32:] *= 1.171875   # (rounded to bf16 below) s no longer a power of two
    x = x.to(torch.bfloat16)
    xq, s = lr.lr_quantize_per_token(dev(x))
    q_ref, s_ref = ow8.quantize_per_token(x)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    assert s[0].item() == 0.5


def test_quantize_zero_row_and_ties(cuda_device):
    x = torch.zeros(3, 32, dtype=torch.bfloat16)
    x[1, :8] = torch.tensor([127.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, -127.0])
    x[2] = torch.linspace(-3, 3, 32)
    xq, s = lr.lr_quantize_per_token(dev(x))
    q_ref, s_ref = ow8.quantize_per_token(x)
    assert np.array_equal(xq.cpu().numpy(), q_ref) and np.array_equal(s.cpu().numpy(), s_ref)
    assert s[0].item() == 1.0 and int(xq[0].abs().max()) == 0



def _kv8_run(d, split=0):
    kv = lr.LatentKv(d["q"].shape[0], d["q"].shape[1], d["ctx"], dev(d["B_K"]), dev(d["B_V"]), d["scale"], 0, split)
    return lr.lr_latent_kv_decode_q8(kv, dev(d["q"]), dev(d["C_Kq"]), dev(d["s_K"]), dev(d["C_Vq"]), dev(d["s_V"]),
                                     dev(d["seq_lens"]))


def _kv8_oracle(d, pairs=None):
    return okv.latent_kv_decode_q8(d["q"], d["C_Kq"], d["s_K"], d["C_Vq"], d["s_V"], d["B_K"], d["B_V"],
                                   d["seq_lens"], d["scale"], pairs)


@pytest.mark.parametrize("split,scale_dtype", [(0, np.float16), (64, np.float32), (512, np.float16)])
def test_latent_kv_int8_ragged_all_pairs(cuda_device, split, scale_dtype):
    seq = [1, 63, 64, 65, 300, 1000, 0, 777]
    d = synth.make_latent_kv_int8(batch=8, heads=4, ctx=1000, seed=13, seq_lens=seq, scale_dtype=scale_dtype)
    o = _kv8_run(d, split).float().cpu().numpy()
    ref = _kv8_oracle(d)
    for b in range(8):
        if seq[b] == 0:
            assert np.abs(o[b]).max() == 0.0
            continue
        assert normwise_rel(o[b], ref[b]) < NORMWISE_TOL, (b, seq[b])


def test_latent_kv_int8_full_size_sampled(cuda_device):
    d = synth.make_latent_kv_int8(batch=8, heads=32, ctx=16384, seed=0)
    o = _kv8_run(d).float().cpu().numpy()
    rng = np.random.default_rng(16384)
    pairs = [(int(b), int(h)) for b, h in zip(rng.integers(0, 8, 12), rng.integers(0, 32, 12))]
    ref = _kv8_oracle(d, pairs)
    for b, h in pairs:
        assert normwise_rel(o[b, h][None], ref[b, h][None]) < NORMWISE_TOL, (b, h)
    assert np.isfinite(o).all()
    assert lr.lr_check_device_error() == 0
