"""GPU parity at full size, in the launch the bench times: the 32-layer
Llama-2-7B-shaped low-rank Q/K/V/O decode stack as one lr_linear_chain call
(64 dependent steps, Q/K/V then O per layer, as the bench times it) at batch
1 (CUDA cores) and 16 (tensor cores), every
output of every layer against the fp64 oracle run layer by layer on the same
stored factors.
"""
import pytest
import torch

import decode_lr_linear_b200 as lr
from decode_lr_linear_b200 import synth
from oracle import lowrank
from tests._helpers import NORMWISE_TOL, dev, normwise_rel

pytestmark = pytest.mark.gpu

LAYERS, HIDDEN = 32, 4096


def _fac(f):
    return lr.Factor(dev(f["At"]), dev(f["B"]))


def _oracle(f, x64):
    return lowrank.lr_linear(x64, f["At"].double().numpy().T, f["B"].double().numpy())


@pytest.fixture(scope="module")
def layers32():
    ranks = synth.attention_ranks(0)
    return [synth.make_attention_layer(l, ranks, seed=0) for l in range(LAYERS)]


@pytest.mark.parametrize("batch", [1, 16])
def test_full_decode_stack_chain(cuda_device, layers32, batch):
    layers = layers32
    x = synth.make_activations(batch, HIDDEN, seed=0, key=(90,) if batch == 1 else (90, batch))
    qkv = [[torch.empty(batch, HIDDEN, dtype=torch.bfloat16, device="cuda") for _ in range(3)] for _ in range(LAYERS)]
    outs = [torch.empty(batch, HIDDEN, dtype=torch.bfloat16, device="cuda") for _ in range(LAYERS)]
    steps = []
    for l, L in enumerate(layers):
        steps.append(lr.ChainStep([_fac(L["q"]), _fac(L["k"]), _fac(L["v"])], -1 if l == 0 else 2 * l - 1, 0,
                                  qkv[l]))
        steps.append(lr.ChainStep([_fac(L["o"])], 2 * l, 2, [outs[l]]))
    ws = lr.workspace(lr.lr_linear_chain_workspace_size(steps, batch), torch.device("cuda"))
    lr.lr_linear_chain(steps, dev(x), ws=ws)
    torch.cuda.synchronize()
    assert lr.lr_check_device_error() == 0

    x64 = x.double().numpy()
    worst = 0.0
    for l, L in enumerate(layers):
        q, k, v = (_oracle(L[n], x64) for n in ("q", "k", "v"))
        o = _oracle(L["o"], v)          # attention over one cached token returns V
        for got, ref in zip(qkv[l] + [outs[l]], (q, k, v, o)):
            err = normwise_rel(got, ref)
            worst = max(worst, err)
            assert err < NORMWISE_TOL, (l, err)
        x64 = o                          # the next layer reads O (fp64 here, fp32 in the chain)
    assert int(ws.count_nonzero()) == 0
    print(f"batch {batch}: worst normwise error over 128 outputs: {worst:.2e}")
