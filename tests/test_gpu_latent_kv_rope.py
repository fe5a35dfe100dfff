"""GPU parity: latent-KV decode with keys reconstructed on the tensor cores and
rotated (LR_KV_RECONSTRUCT), and the latent producer (lr_latent_kv_append),
against the float64 oracle."""
import numpy as np
import pytest
import torch

import decode_lr_linear_b200 as lr
from decode_lr_linear_b200 import synth
from oracle import latent_kv as okv
from tests._helpers import NORMWISE_TOL, dev, normwise_rel

pytestmark = pytest.mark.gpu

REC = 1  # LR_KV_RECONSTRUCT


def _run(d, base, ws=None):
    kv = lr.LatentKv(d["batch"], d["heads"], d["ctx"], dev(d["B_K"]), dev(d["B_V"]), d["scale"], REC, 0, base)
    return lr.lr_latent_kv_decode(kv, dev(d["q"]), dev(d["C_K"]), dev(d["C_V"]), dev(d["seq_lens"]), ws=ws)


def _oracle(d, base, pairs=None):
    return okv.latent_kv_decode_rope(d["q"], d["C_K"], d["C_V"], d["B_K"], d["B_V"], d["seq_lens"], d["scale"], base,
                                     pairs)


@pytest.mark.parametrize("base", [10000.0, 10.0])
def test_reconstruct_rope_ragged_all_pairs(cuda_device, base):
    # 3 splits of 256 with a ragged tail, a length inside the first tile, a single token and an empty sequence
    d = synth.make_latent_kv(batch=4, heads=4, ctx=700, seed=3, seq_lens=[700, 129, 1, 0])
    o = _run(d, base)
    ref = _oracle(d, base)
    assert normwise_rel(o[:3], ref[:3]) < NORMWISE_TOL
    assert torch.count_nonzero(o[3]).item() == 0


def test_reconstruct_without_rotation_equals_absorbed_definition(cuda_device):
    d = synth.make_latent_kv(batch=2, heads=3, ctx=513, seed=4, seq_lens=[513, 300])
    o = _run(d, 0.0)
    ref = okv.latent_kv_decode(d["q"], d["C_K"], d["C_V"], d["B_K"], d["B_V"], d["seq_lens"], d["scale"])
    assert normwise_rel(o, ref) < NORMWISE_TOL


def test_reconstruct_rope_peaky_scores(cuda_device):
    d = synth.make_latent_kv(batch=2, heads=2, ctx=1024, seed=5, peak=4.0, seq_lens=[1024, 777])
    assert normwise_rel(_run(d, 10000.0), _oracle(d, 10000.0)) < NORMWISE_TOL


@pytest.mark.parametrize("ctx", [4096, 32768])
def test_reconstruct_rope_full_size_sampled(cuda_device, ctx):
    d = synth.make_latent_kv(batch=8, heads=32, ctx=ctx, seed=0)
    o = _run(d, 10000.0).float().cpu().numpy()
    rng = np.random.default_rng(ctx + 1)
    pairs = [(int(b), int(h)) for b, h in zip(rng.integers(0, 8, 12), rng.integers(0, 32, 12))]
    ref = _oracle(d, 10000.0, pairs)
    for b, h in pairs:
        assert normwise_rel(o[b, h][None], ref[b, h][None]) < NORMWISE_TOL, (b, h)
    assert np.isfinite(o).all()
    assert lr.lr_check_device_error() == 0


@pytest.mark.parametrize("use_ws", [True, False])
def test_append_writes_only_the_new_positions(cuda_device, use_ws):
    # with a workspace: tensor-core product + scatter; without: the CUDA-core GEMV
    heads, rank, hidden, ctx, batch = 32, 32, 4096, 64, 5
    pr = synth.make_latent_producer(heads, rank, hidden, seed=1)
    d = synth.make_latent_kv(batch=batch, heads=heads, ctx=ctx, seed=6)
    x = synth.make_activations(batch, hidden, seed=1, key=(40,))
    pos = torch.tensor([0, 17, 63, 64, -1], dtype=torch.int32)   # the last two are outside the cache
    CK, CV = dev(d["C_K"]), dev(d["C_V"])
    kv = lr.LatentKv(batch, heads, ctx, dev(d["B_K"]), dev(d["B_V"]), d["scale"])
    lr.lr_latent_kv_append(kv, dev(pr["A_KV"]), dev(x), dev(pos), CK, CV, use_ws=use_ws)
    rk, rv = okv.append_latents(x, pr["A_KV"], heads, rank, d["C_K"], d["C_V"], pos.numpy())
    ck, cv = CK.cpu(), CV.cpu()
    for b in range(batch):
        p = int(pos[b])
        keep = torch.ones(ctx, dtype=torch.bool)
        if 0 <= p < ctx:
            keep[p] = False
            assert normwise_rel(ck[b, :, p], rk[b, :, p]) < NORMWISE_TOL
            assert normwise_rel(cv[b, :, p], rv[b, :, p]) < NORMWISE_TOL
        assert torch.equal(ck[b][:, keep], d["C_K"][b][:, keep])
        assert torch.equal(cv[b][:, keep], d["C_V"][b][:, keep])


def test_append_repeated_on_one_workspace(cuda_device):
    # three appends through the same workspace: every call writes the right latents, and the
    # workspace (the product's accumulator) is all zero again afterwards
    heads, rank, hidden, ctx, batch = 32, 32, 4096, 64, 3
    pr = synth.make_latent_producer(heads, rank, hidden, seed=4)
    d = synth.make_latent_kv(batch=batch, heads=heads, ctx=ctx, seed=8)
    kv = lr.LatentKv(batch, heads, ctx, dev(d["B_K"]), dev(d["B_V"]), d["scale"])
    CK, CV = dev(d["C_K"]), dev(d["C_V"])
    ws = lr.workspace(lr.lr_latent_kv_append_workspace_size(kv, hidden), CK.device)
    ck_ref, cv_ref = d["C_K"].clone(), d["C_V"].clone()
    for call in range(3):
        x = synth.make_activations(batch, hidden, seed=4, key=(41, call))
        pos = torch.tensor([call, 10 + call, 30 + 2 * call], dtype=torch.int32)
        lr.lr_latent_kv_append(kv, dev(pr["A_KV"]), dev(x), dev(pos), CK, CV, ws=ws)
        rk, rv = okv.append_latents(x, pr["A_KV"], heads, rank, ck_ref, cv_ref, pos.numpy())
        for b in range(batch):
            p = int(pos[b])
            assert normwise_rel(CK.cpu()[b, :, p], rk[b, :, p]) < NORMWISE_TOL
            assert normwise_rel(CV.cpu()[b, :, p], rv[b, :, p]) < NORMWISE_TOL
        ck_ref, cv_ref = CK.cpu(), CV.cpu()
    torch.cuda.synchronize()
    assert int(ws.abs().max()) == 0
    assert lr.lr_check_device_error() == 0


def test_decode_step_append_then_rotated_attention(cuda_device):
    # one decode step of a layer's attention: write the new token's latents, then attend with rotation
    heads, rank, hidden, ctx, batch, base = 32, 32, 4096, 2048, 4, 10000.0
    pr = synth.make_latent_producer(heads, rank, hidden, seed=2)
    lens = np.array([2048, 1000, 257, 1], np.int32)
    d = synth.make_latent_kv(batch=batch, heads=heads, ctx=ctx, seed=7, seq_lens=lens)
    x = synth.make_activations(batch, hidden, seed=2, key=(41,))
    pos = torch.from_numpy(lens - 1)
    CK, CV = dev(d["C_K"]), dev(d["C_V"])
    kv = lr.LatentKv(batch, heads, ctx, dev(d["B_K"]), dev(d["B_V"]), d["scale"], REC, 0, base)
    lr.lr_latent_kv_append(kv, dev(pr["A_KV"]), dev(x), dev(pos), CK, CV)
    o = lr.lr_latent_kv_decode(kv, dev(d["q"]), CK, CV, dev(d["seq_lens"]))
    # the oracle attends over the caches the GPU wrote (their bf16 values), checked above against append_latents
    ref = okv.latent_kv_decode_rope(d["q"], CK.cpu(), CV.cpu(), d["B_K"], d["B_V"], d["seq_lens"], d["scale"], base)
    assert normwise_rel(o, ref) < NORMWISE_TOL
    rk, _ = okv.append_latents(x, pr["A_KV"], heads, rank, d["C_K"], d["C_V"], pos.numpy())
    for b in range(batch):
        assert normwise_rel(CK.cpu()[b, :, int(pos[b])], rk[b, :, int(pos[b])]) < NORMWISE_TOL
