"""GPU parity: lr_linear_chain (a stack of dependent factorised projections in one launch)."""
import numpy as np
import pytest
import torch

import decode_lr_linear_b200 as lr
from decode_lr_linear_b200 import synth
from oracle import lowrank
from tests._helpers import NORMWISE_TOL, dev, normwise_rel

pytestmark = pytest.mark.gpu


def _fac(f):
    return lr.Factor(dev(f["At"]), dev(f["B"]))


def _oracle(f, x64):
    return lowrank.lr_linear(x64, f["At"].double().numpy().T, f["B"].double().numpy())


@pytest.fixture(scope="module")
def layers4():
    ranks = synth.attention_ranks(0)
    return [synth.make_attention_layer(l, ranks, seed=0) for l in range(4)]


def _decode_stack_steps(layers):
    steps = []
    for l, L in enumerate(layers):
        steps.append(lr.ChainStep([_fac(L["q"]), _fac(L["k"]), _fac(L["v"])], -1 if l == 0 else 2 * l - 1, 0))
        steps.append(lr.ChainStep([_fac(L["o"])], 2 * l, 2))
    return steps


@pytest.mark.parametrize("batch", [1, 3])
def test_decode_stack_chain(cuda_device, layers4, batch):
    x = synth.make_activations(batch, 4096, seed=5, key=(70, batch))
    steps = _decode_stack_steps(layers4)
    ws = lr.workspace(lr.lr_linear_chain_workspace_size(steps, batch), torch.device("cuda"))
    outs = lr.lr_linear_chain(steps, dev(x), ws=ws)
    torch.cuda.synchronize()
    x64 = x.double().numpy()
    for l, L in enumerate(layers4):
        q, k, v = (_oracle(L[n], x64) for n in ("q", "k", "v"))
        o = _oracle(L["o"], v)
        for got, ref in zip(outs[2 * l] + outs[2 * l + 1], (q, k, v, o)):
            assert normwise_rel(got, ref) < NORMWISE_TOL, l
        x64 = o
    assert int(ws.count_nonzero()) == 0


def test_chain_older_inputs_against_oracle(cuda_device, layers4):
    L0, L1 = layers4[0], layers4[1]
    x = synth.make_activations(2, 4096, seed=6, key=(71,))
    # step 1 reads step 0's second output, step 2 step 0's first output two steps
    # back (both at fp32, from step 0's accumulators)
    steps = [lr.ChainStep([_fac(L0["q"]), _fac(L0["v"])]), lr.ChainStep([_fac(L0["o"])], 0, 1),
             lr.ChainStep([_fac(L1["k"])], 0, 0)]
    outs = lr.lr_linear_chain(steps, dev(x))
    x64 = x.double().numpy()
    q, v = _oracle(L0["q"], x64), _oracle(L0["v"], x64)
    o, k = _oracle(L0["o"], v), _oracle(L1["k"], q)
    for got, ref in ((outs[0][0], q), (outs[0][1], v), (outs[1][0], o), (outs[2][0], k)):
        assert normwise_rel(got, ref) < NORMWISE_TOL


def test_chain_four_projections_one_consumed(cuda_device, layers4):
    # three steps of four projections each; only the last projection of a step
    # feeds the next, so the other three are scheduled as fillers
    x = synth.make_activations(1, 4096, seed=8, key=(73,))
    names = ("q", "k", "v", "o")
    steps = [lr.ChainStep([_fac(layers4[l][n]) for n in names], -1 if l == 0 else l - 1, 3) for l in range(3)]
    outs = lr.lr_linear_chain(steps, dev(x))
    x64 = x.double().numpy()
    for l in range(3):
        refs = [_oracle(layers4[l][n], x64) for n in names]
        for got, ref in zip(outs[l], refs):
            assert normwise_rel(got, ref) < NORMWISE_TOL, l
        x64 = refs[3]


def test_chain_int8_and_fp32(cuda_device):
    p1 = synth.make_prefill_projection(1024, 768, 160, seed=1, key=(1,))
    p2 = synth.make_prefill_projection(768, 1024, 96, seed=1, key=(2,))
    f = [lr.Factor(dev(p["A_q"]), dev(p["B_q"]), dev(p["s_A"].half()), dev(p["s_B"].half())) for p in (p1, p2)]
    x = synth.make_activations(2, 1024, seed=1, key=(72,))
    outs = lr.lr_linear_chain([lr.ChainStep([f[0]]), lr.ChainStep([f[1]], 0, 0)], dev(x))

    def deq(p):
        A = (p["A_q"].double() * p["s_A"].half().double()[:, None]).numpy().T
        B = (p["B_q"].double() * p["s_B"].half().double()[None, :]).numpy()
        return A, B
    A1, B1 = deq(p1)
    A2, B2 = deq(p2)
    y1 = lowrank.lr_linear(x.double().numpy(), A1, B1)
    y2 = lowrank.lr_linear(y1, A2, B2)
    assert normwise_rel(outs[0][0], y1) < NORMWISE_TOL and normwise_rel(outs[1][0], y2) < NORMWISE_TOL
    d = synth.make_single_linear(0)
    g = lr.Factor(dev(d["At"]), dev(d["B32"]))
    outs = lr.lr_linear_chain([lr.ChainStep([g]), lr.ChainStep([g], 0, 0)], dev(d["x"]))
    r1 = lowrank.lr_linear(d["x"].double().numpy(), d["At"].double().numpy().T, d["B32"].double().numpy())
    r2 = lowrank.lr_linear(r1, d["At"].double().numpy().T, d["B32"].double().numpy())
    assert normwise_rel(outs[1][0], r2) < 1e-5
    assert lr.lr_check_device_error() == 0


def test_ranked_chain_progressive_schedule(cuda_device, layers4):
    # FLRC progressive decoding: per-token budgets, ranks from the library's
    # allocation rule, applied to a 2-layer chain; every output against the
    # oracle on factors truncated to the same ranks
    from oracle import ranks as oranks
    steps = _decode_stack_steps(layers4[:2])
    caps = [layers4[l][n]["rank"] for l in range(2) for n in ("q", "k", "v", "o")]
    alpha = np.random.default_rng(3).lognormal(0.0, 0.35, len(caps))
    ws = lr.workspace(lr.lr_linear_chain_workspace_size(steps, 1), torch.device("cuda"))
    for t, budget in enumerate((9000.0, 6000.0, 2500.0)):
        active = lr.lr_rank_allocate(alpha, budget, caps)
        assert active == oranks.flrc_ranks(alpha, budget, caps).tolist()
        x = synth.make_activations(1, 4096, seed=10, key=(75, t))
        outs = lr.lr_linear_chain_ranked(steps, dev(x), active, ws=ws)
        x64, k = x.double().numpy(), 0
        for l in range(2):
            L_ = layers4[l]
            ref = {}
            for n in ("q", "k", "v"):
                ref[n] = lowrank.lr_linear(x64, L_[n]["At"].double().numpy().T, L_[n]["B"].double().numpy(), active[k])
                k += 1
            ref["o"] = lowrank.lr_linear(ref["v"], L_["o"]["At"].double().numpy().T, L_["o"]["B"].double().numpy(),
                                         active[k])
            k += 1
            for got, n in zip(outs[2 * l] + outs[2 * l + 1], ("q", "k", "v", "o")):
                assert normwise_rel(got, ref[n]) < NORMWISE_TOL, (t, l, n)
            x64 = ref["o"]
    assert int(ws.count_nonzero()) == 0


def test_chain_split_layout_waits_only_for_inputs(cuda_device, layers4):
    # V, then Q and K, then O (reads V two steps back) per layer: O waits only for V
    x = synth.make_activations(2, 4096, seed=12, key=(76,))
    steps = []
    for l, L in enumerate(layers4):
        src = -1 if l == 0 else 3 * l - 1
        steps.append(lr.ChainStep([_fac(L["v"])], src, 0))
        steps.append(lr.ChainStep([_fac(L["q"]), _fac(L["k"])], src, 0))
        steps.append(lr.ChainStep([_fac(L["o"])], 3 * l, 0))
    ws = lr.workspace(lr.lr_linear_chain_workspace_size(steps, 2), torch.device("cuda"))
    outs = lr.lr_linear_chain(steps, dev(x), ws=ws)
    torch.cuda.synchronize()
    x64 = x.double().numpy()
    for l, L in enumerate(layers4):
        v, q, k = (_oracle(L[n], x64) for n in ("v", "q", "k"))
        o = _oracle(L["o"], v)
        for got, ref in zip(outs[3 * l] + outs[3 * l + 1] + outs[3 * l + 2], (v, q, k, o)):
            assert normwise_rel(got, ref) < NORMWISE_TOL, l
        x64 = o
    assert int(ws.count_nonzero()) == 0
    assert lr.lr_check_device_error() == 0
