"""GPU parity: batched decode of bf16 factorised linears on the tensor cores
(batch above 8: every weight streams once per pass of up to 32 tokens), against
the float64 oracle."""
import pytest
import torch

import decode_lr_linear_b200 as lr
from decode_lr_linear_b200 import synth
from oracle import lowrank
from tests._helpers import NORMWISE_TOL, dev, normwise_rel

pytestmark = pytest.mark.gpu


def _fac(f, active=0):
    return lr.Factor(dev(f["At"]), dev(f["B"]), active_rank=active)


def _oracle(f, x64, active=None):
    At, B = f["At"].double().numpy(), f["B"].double().numpy()
    return lowrank.lr_linear(x64, At.T, B, active)


@pytest.fixture(scope="module")
def layers4():
    ranks = synth.attention_ranks(0)
    return [synth.make_attention_layer(l, ranks, seed=0) for l in range(4)]


@pytest.mark.parametrize("batch", [9, 16, 32, 40])
def test_linear_batched(cuda_device, layers4, batch):
    f = layers4[0]["q"]
    x = synth.make_activations(batch, 4096, seed=8, key=(100, batch))
    ws = lr.workspace(lr.lr_linear_workspace_size(_fac(f), batch), torch.device("cuda"))
    y = lr.lr_linear(_fac(f), dev(x), ws=ws)
    torch.cuda.synchronize()
    assert normwise_rel(y, _oracle(f, x.double().numpy())) < NORMWISE_TOL
    assert int(ws.count_nonzero()) == 0
    assert lr.lr_check_device_error() == 0


def test_grouped_qkv_batched(cuda_device, layers4):
    L = layers4[1]
    x = synth.make_activations(16, 4096, seed=9, key=(101,))
    ys = lr.lr_linear_grouped([_fac(L[n]) for n in ("q", "k", "v")], dev(x))
    for y, n in zip(ys, ("q", "k", "v")):
        assert normwise_rel(y, _oracle(L[n], x.double().numpy())) < NORMWISE_TOL


def test_ragged_shapes_batched(cuda_device):
    # reduction lengths and row counts off the 64 / 128 tile grid, ragged batch
    for (d_in, d_out, r, batch) in ((264, 392, 100, 12), (4096, 11008, 256, 17), (520, 136, 1, 9)):
        At, B = synth._lr_factors(d_in, d_out, r, 4, (102, d_in))
        f = {"At": torch.from_numpy(At).to(torch.bfloat16), "B": torch.from_numpy(B).to(torch.bfloat16)}
        x = synth.make_activations(batch, d_in, seed=4, key=(103, d_in))
        y = lr.lr_linear(_fac(f), dev(x))
        assert normwise_rel(y, _oracle(f, x.double().numpy())) < NORMWISE_TOL, (d_in, d_out, r)


@pytest.mark.parametrize("active", [1, 130, 500])
def test_active_rank_batched(cuda_device, layers4, active):
    f = layers4[2]["v"]                 # stored rank >= 512 (ranks lie in [512, 1536])
    x = synth.make_activations(16, 4096, seed=10, key=(104, active))
    y = lr.lr_linear(_fac(f, active), dev(x))
    assert normwise_rel(y, _oracle(f, x.double().numpy(), active)) < NORMWISE_TOL


@pytest.mark.parametrize("batch", [16, 33])
def test_decode_stack_chain_batched(cuda_device, layers4, batch):
    x = synth.make_activations(batch, 4096, seed=11, key=(105, batch))
    steps = []
    for l, L in enumerate(layers4):
        steps.append(lr.ChainStep([_fac(L["q"]), _fac(L["k"]), _fac(L["v"])], -1 if l == 0 else 2 * l - 1, 0))
        steps.append(lr.ChainStep([_fac(L["o"])], 2 * l, 2))
    # an extra step reading an older step's stored output (layer 0's K)
    steps.append(lr.ChainStep([_fac(layers4[0]["o"])], 0, 1))
    ws = lr.workspace(lr.lr_linear_chain_workspace_size(steps, batch), torch.device("cuda"))
    outs = lr.lr_linear_chain(steps, dev(x), ws=ws)
    torch.cuda.synchronize()
    x64 = x.double().numpy()
    k0 = None
    for l, L in enumerate(layers4):
        q, k, v = (_oracle(L[n], x64) for n in ("q", "k", "v"))
        if l == 0:
            k0 = outs[0][1].double().cpu().numpy()   # the stored (bf16) output the extra step reads
        o = _oracle(L["o"], v)
        for got, ref in zip(outs[2 * l] + outs[2 * l + 1], (q, k, v, o)):
            assert normwise_rel(got, ref) < NORMWISE_TOL, l
        x64 = o
    assert normwise_rel(outs[-1][0], _oracle(layers4[0]["o"], k0)) < NORMWISE_TOL
    assert int(ws.count_nonzero()) == 0
    assert lr.lr_check_device_error() == 0


# ---- int8 factors and the hybrid FFN on the tensor cores (kind::i8) ----
from oracle import ffn as offn  # noqa: E402


def test_int8_factors_batched(cuda_device):
    p = synth.make_prefill_projection(4096, 4096, 512, seed=3, key=(106,))
    x = synth.make_activations(16, 4096, seed=3, key=(107,), outliers=4)
    for sA, sB in ((p["s_A"], p["s_B"]), (p["s_A"].half(), p["s_B"].half())):
        y = lr.lr_linear(lr.Factor(dev(p["A_q"]), dev(p["B_q"]), dev(sA), dev(sB)), dev(x))
        A = (p["A_q"].double() * sA.double()[:, None]).numpy().T
        B = (p["B_q"].double() * sB.double()[None, :]).numpy()
        assert normwise_rel(y, lowrank.lr_linear(x.double().numpy(), A, B)) < NORMWISE_TOL


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


@pytest.mark.parametrize("batch", [12, 40])
def test_hybrid_ffn_batched(cuda_device, ffn7b, batch):
    x = synth.make_activations(batch, 4096, seed=0, key=(108, batch), outliers=4)
    ws = lr.workspace(lr.lr_swiglu_ffn_workspace_size(_ffn_dev(ffn7b), batch), torch.device("cuda"))
    y = lr.lr_swiglu_ffn(_ffn_dev(ffn7b), dev(x), ws=ws)
    torch.cuda.synchronize()
    assert normwise_rel(y, _ffn_oracle(ffn7b, x)) < NORMWISE_TOL
    assert int(ws.count_nonzero()) == 0
    assert lr.lr_check_device_error() == 0


@pytest.mark.parametrize("n_lr", [0, 512, 1000])
def test_hybrid_ffn_batched_degenerate(cuda_device, n_lr):
    d = synth.make_hybrid_ffn(seed=1, hidden=512, inter=1000, n_lr=n_lr, rank=512, rotate=n_lr > 0)
    x = synth.make_activations(17, 512, seed=1, key=(109, n_lr), outliers=1)
    assert normwise_rel(lr.lr_swiglu_ffn(_ffn_dev(d), dev(x)), _ffn_oracle(d, x)) < NORMWISE_TOL


@pytest.mark.parametrize("batch", [1, 8])
def test_tensor_core_path_at_small_batch(cuda_device, ffn7b, layers4, batch):
    # the threshold knob sends small batches to the tensor cores too; results stay within the bar
    lr.lr_set_tensor_core_min_batch(1, 1)
    try:
        x = synth.make_activations(batch, 4096, seed=2, key=(110, batch), outliers=4)
        assert normwise_rel(lr.lr_swiglu_ffn(_ffn_dev(ffn7b), dev(x)), _ffn_oracle(ffn7b, x)) < NORMWISE_TOL
        f = layers4[3]["o"]
        y = lr.lr_linear(_fac(f), dev(x))
        assert normwise_rel(y, _oracle(f, x.double().numpy())) < NORMWISE_TOL
    finally:
        lr.lr_set_tensor_core_min_batch(0, 0)
