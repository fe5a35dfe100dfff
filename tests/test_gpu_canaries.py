"""GPU: every entry point writes exactly its output, nothing around it.

The library's kernels write outputs and workspaces only; each test places the
output (and, where the call takes one, the workspace) inside a larger buffer
filled with a sentinel and checks, after two calls, that the guard regions
before and after are untouched and the workspace is zero again.  Shapes are
ragged (ranks, widths and lengths off the tile grids) so that the edge paths
of the kernels run.  With compute-sanitizer unavailable, this and the oracle
comparisons are the library's bounds checks on the GPU."""
import pytest
import torch

import decode_lr_linear_b200 as lr
from decode_lr_linear_b200 import synth
from tests._helpers import dev

pytestmark = pytest.mark.gpu

G = 256          # guard elements on each side (a multiple of 16 bytes for every dtype used)
SENT = {torch.bfloat16: -1234.0, torch.float32: -98765.0}


def _guarded(shape, dtype):
    n = 1
    for s in shape:
        n *= s
    buf = torch.full((n + 2 * G,), SENT[dtype], dtype=dtype, device="cuda")
    return buf, buf[G:G + n].view(*shape)


def _guards_intact(buf, dtype):
    torch.cuda.synchronize()
    return bool((buf[:G] == SENT[dtype]).all()) and bool((buf[-G:] == SENT[dtype]).all())


def _guarded_ws(nbytes):
    buf = torch.full((nbytes + 2 * G,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = buf[G:G + nbytes]
    ws.zero_()
    return buf, ws


def _ws_intact(buf, nbytes):
    torch.cuda.synchronize()
    return bool((buf[:G] == 0xA5).all()) and bool((buf[-G:] == 0xA5).all()) and int(buf[G:G + nbytes].count_nonzero()) == 0


@pytest.mark.parametrize("batch", [1, 3, 6, 19])
def test_linear_outputs_and_workspace(cuda_device, batch):
    At, B = synth._lr_factors(264, 392, 100, 5, (120, batch))
    f = lr.Factor(dev(torch.from_numpy(At).to(torch.bfloat16)), dev(torch.from_numpy(B).to(torch.bfloat16)))
    x = dev(synth.make_activations(batch, 264, seed=5, key=(121, batch)))
    ybuf, y = _guarded((batch, 392), torch.bfloat16)
    nws = lr.lr_linear_workspace_size(f, batch)
    wbuf, ws = _guarded_ws(nws)
    for _ in range(2):
        lr.lr_linear(f, x, y, ws)
    assert _guards_intact(ybuf, torch.bfloat16)
    assert _ws_intact(wbuf, nws)
    assert lr.lr_check_device_error() == 0


@pytest.mark.parametrize("batch", [1, 9])
def test_ffn_outputs_and_workspace(cuda_device, batch):
    d = synth.make_hybrid_ffn(seed=2, hidden=512, inter=1000, n_lr=504, rank=328, rotate=False)
    w = lr.FfnWeights(d["hidden"], d["inter"], d["n_lr"], d["rank"], dev(d["A_q"]), dev(d["s_A"]), dev(d["B_q"]),
                      dev(d["s_B"]), dev(d["D_q"]), dev(d["s_D"]), dev(d["Wd_q"]), dev(d["s_d"]))
    x = dev(synth.make_activations(batch, 512, seed=2, key=(122, batch), outliers=1))
    ybuf, y = _guarded((batch, 512), torch.bfloat16)
    nws = lr.lr_swiglu_ffn_workspace_size(w, batch)
    wbuf, ws = _guarded_ws(nws)
    for _ in range(2):
        lr.lr_swiglu_ffn(w, x, y, ws)
    assert _guards_intact(ybuf, torch.bfloat16)
    assert _ws_intact(wbuf, nws)


@pytest.mark.parametrize("mode,base", [(0, 0.0), (1, 10000.0)])
def test_latent_kv_outputs(cuda_device, mode, base):
    d = synth.make_latent_kv(batch=3, heads=3, ctx=333, seed=8, seq_lens=[333, 129, 0])
    kv = lr.LatentKv(3, 3, 333, dev(d["B_K"]), dev(d["B_V"]), d["scale"], mode, 0, base)
    obuf, o = _guarded((3, 3, 128), torch.bfloat16)
    nws = lr.lr_latent_kv_workspace_size(kv)
    wbuf, ws = _guarded_ws(nws)
    for _ in range(2):
        lr.lr_latent_kv_decode(kv, dev(d["q"]), dev(d["C_K"]), dev(d["C_V"]), dev(d["seq_lens"]), o, ws)
    assert _guards_intact(obuf, torch.bfloat16)
    torch.cuda.synchronize()
    assert bool((wbuf[:G] == 0xA5).all()) and bool((wbuf[-G:] == 0xA5).all())   # partials stay in the workspace


def test_dense_and_flash_outputs(cuda_device):
    W = dev((torch.randn(136, 272) / 16).to(torch.bfloat16))
    x = dev(synth.make_activations(5, 272, seed=9, key=(123,)))
    ybuf, y = _guarded((5, 136), torch.bfloat16)
    lr.lr_dense_linear(W, x, y=y)
    assert _guards_intact(ybuf, torch.bfloat16)
    K = dev(torch.randn(2, 2, 300, 128).to(torch.bfloat16))
    V = dev(torch.randn(2, 2, 300, 128).to(torch.bfloat16))
    q = dev(torch.randn(2, 2, 128).to(torch.bfloat16))
    obuf, o = _guarded((2, 2, 128), torch.bfloat16)
    lr.lr_flash_decode(q, K, V, dev(torch.tensor([300, 77], dtype=torch.int32)), 128 ** -0.5, out=o)
    assert _guards_intact(obuf, torch.bfloat16)
