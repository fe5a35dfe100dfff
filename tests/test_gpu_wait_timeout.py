"""GPU: a wait of a persistent kernel on its other CTAs gives up, reports
through the device error word, and leaves the context usable.

The CTAs of one chain launch meet at a grid-wide barrier per step.  With the
bound of those waits set far below the time the other CTAs need to arrive,
the waits run out (nothing is faulted, no wait is unbounded); the kernel
records code 3, finishes, and lr_check_device_error reports it.  After restoring the bound and
re-zeroing the workspace, the same call matches the float64 oracle again.
"""
import pytest
import torch

import decode_lr_linear_b200 as lr
from decode_lr_linear_b200 import _lib as L
from decode_lr_linear_b200 import synth
from oracle import lowrank
from tests._helpers import NORMWISE_TOL, dev, normwise_rel

pytestmark = pytest.mark.gpu


def _stack(layers):
    steps = []
    for l, Lr in enumerate(layers):
        steps.append(lr.ChainStep([lr.Factor(dev(Lr[n]["At"]), dev(Lr[n]["B"])) for n in ("q", "k", "v")],
                                  -1 if l == 0 else 2 * l - 1, 0))
        steps.append(lr.ChainStep([lr.Factor(dev(Lr["o"]["At"]), dev(Lr["o"]["B"]))], 2 * l, 2))
    return steps


def test_grid_wait_runs_out_and_recovers(cuda_device):
    ranks = synth.attention_ranks(0)
    layers = [synth.make_attention_layer(l, ranks, seed=0) for l in range(4)]
    x = synth.make_activations(1, 4096, seed=9, key=(74,))
    steps = _stack(layers)
    ws = lr.workspace(lr.lr_linear_chain_workspace_size(steps, 1), torch.device("cuda"))
    assert lr.lr_check_device_error() == 0
    try:
        lr.lr_set_wait_timeout_us(1)
        lr.lr_linear_chain(steps, dev(x), ws=ws)
        err = lr.lr_check_device_error()
    finally:
        lr.lr_set_wait_timeout_us(0)
    assert err == L.DEVICE_ERR_GRID_WAIT
    assert lr.lr_check_device_error() == 0          # the word was cleared by the check
    lr.lr_workspace_init(ws)
    outs = lr.lr_linear_chain(steps, dev(x), ws=ws)
    assert lr.lr_check_device_error() == 0
    x64 = x.double().numpy()
    for l, Lr in enumerate(layers):
        ref = [lowrank.lr_linear(x64, Lr[n]["At"].double().numpy().T, Lr[n]["B"].double().numpy())
               for n in ("q", "k", "v")]
        o = lowrank.lr_linear(ref[2], Lr["o"]["At"].double().numpy().T, Lr["o"]["B"].double().numpy())
        for got, r in zip(outs[2 * l] + outs[2 * l + 1], ref + [o]):
            assert normwise_rel(got, r) < NORMWISE_TOL
        x64 = o
    assert int(ws.count_nonzero()) == 0
