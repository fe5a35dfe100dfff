"""GPU parity: factorised linear (lr_linear / lr_linear_grouped) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import decode_lr_linear_b200 as lr
from decode_lr_linear_b200 import synth
from oracle import lowrank
from tests._helpers import NORMWISE_TOL, dev, normwise_rel

pytestmark = pytest.mark.gpu


def _oracle(f_cpu: dict, x_cpu, active=None):
    """fp64 oracle on the stored (rounded) factors: A = At^T, B = B."""
    return lowrank.lr_linear(x_cpu, f_cpu["At"].double().numpy().T, f_cpu["B"].double().numpy(), active)


def _factor_dev(f_cpu, active=0, sA=None, sB=None):
    return lr.Factor(dev(f_cpu["At"]), dev(f_cpu["B"]), None if sA is None else dev(sA),
                     None if sB is None else dev(sB), active)


def test_single_linear_fp32(cuda_device):
    d = synth.make_single_linear(0)
    f = lr.Factor(dev(d["At"]), dev(d["B32"]))
    y = lr.lr_linear(f, dev(d["x"]))
    ref = lowrank.lr_linear(d["x"].double().numpy(), d["At"].double().numpy().T, d["B32"].double().numpy())
    err = normwise_rel(y, ref)
    assert err < 1e-5, err  # fp32 storage and accumulation: far inside the 1e-2 bar


def test_single_linear_exact_rank_matches_dense(cuda_device):
    d = synth.make_single_linear(0, exact_rank=True)
    y = lr.lr_linear(lr.Factor(dev(d["At"]), dev(d["B32"])), dev(d["x"]))
    ref = lowrank.dense_linear(d["x"].double().numpy(), d["W"])
    assert normwise_rel(y, ref) < 1e-5


@pytest.fixture(scope="module")
def layer0():
    ranks = synth.attention_ranks(0)
    return synth.make_attention_layer(0, ranks, seed=0)


@pytest.mark.parametrize("batch", [1, 4, 16])
def test_attention_projections_bf16(cuda_device, layer0, batch):
    x = synth.make_activations(batch, 4096, seed=0, key=(20, batch))
    xd = dev(x)
    for name in synth.ATTN_PROJ:
        f = layer0[name]
        y = lr.lr_linear(_factor_dev(f), xd)
        err = normwise_rel(y, _oracle(f, x.double().numpy()))
        assert err < NORMWISE_TOL, (name, err)
        assert err < 1e-2 and np.isfinite(err)


@pytest.mark.parametrize("batch", [1, 3, 8])
def test_grouped_qkv_matches_oracle(cuda_device, layer0, batch):
    x = synth.make_activations(batch, 4096, seed=1, key=(21, batch))
    fs = [_factor_dev(layer0[n]) for n in ("q", "k", "v")]
    ys = lr.lr_linear_grouped(fs, dev(x))
    for n, y in zip(("q", "k", "v"), ys):
        assert normwise_rel(y, _oracle(layer0[n], x.double().numpy())) < NORMWISE_TOL


def test_ragged_shapes(cuda_device):
    # d_in, d_out not multiples of the 256-element line; odd rank; several CTAs
    rng = np.random.default_rng(3)
    for d_in, d_out, r in ((1288, 1000, 97), (136, 24, 1), (8, 8, 3), (4104, 4096, 1531)):
        At = torch.from_numpy(rng.standard_normal((r, d_in)).astype(np.float32) / np.sqrt(d_in)).to(torch.bfloat16)
        B = torch.from_numpy(rng.standard_normal((r, d_out)).astype(np.float32) / np.sqrt(r)).to(torch.bfloat16)
        x = torch.from_numpy(rng.standard_normal((2, d_in)).astype(np.float32)).to(torch.bfloat16)
        y = lr.lr_linear(lr.Factor(dev(At), dev(B)), dev(x))
        ref = lowrank.lr_linear(x.double().numpy(), At.double().numpy().T, B.double().numpy())
        assert normwise_rel(y, ref) < NORMWISE_TOL, (d_in, d_out, r)


@pytest.mark.parametrize("active", [1, 512, 1000])
def test_progressive_active_rank(cuda_device, layer0, active):
    f = layer0["q"]
    x = synth.make_activations(1, 4096, seed=2, key=(22,))
    y = lr.lr_linear(_factor_dev(f, active=active), dev(x))
    ref = _oracle(f, x.double().numpy(), active)
    assert normwise_rel(y, ref) < NORMWISE_TOL


@pytest.mark.parametrize("scale_dtype", [torch.float16, torch.float32])
def test_int8_weight_only(cuda_device, scale_dtype):
    p = synth.make_prefill_projection(2048, 1536, 352, seed=0, key=(7,))
    sA, sB = p["s_A"].to(scale_dtype), p["s_B"].to(scale_dtype)
    x = synth.make_activations(2, 2048, seed=0, key=(23,))
    y = lr.lr_linear(lr.Factor(dev(p["A_q"]), dev(p["B_q"]), dev(sA), dev(sB)), dev(x))
    A = (p["A_q"].double() * sA.double()[:, None]).numpy().T
    B = (p["B_q"].double() * sB.double()[None, :]).numpy()
    assert normwise_rel(y, lowrank.lr_linear(x.double().numpy(), A, B)) < NORMWISE_TOL


@pytest.mark.parametrize("batch", [5, 8, 11])
def test_batch_pieces_wide_output_and_int8(cuda_device, batch):
    # a wide bf16 output (11008 columns: 4 lines per warp) takes 2 batch rows per
    # launch, int8 (16 elements per lane) takes 4: the batch is split into pieces
    At, B = synth._lr_factors(4096, 11008, 256, 3, (80,))
    f = {"At": torch.from_numpy(At).to(torch.bfloat16), "B": torch.from_numpy(B).to(torch.bfloat16)}
    x = synth.make_activations(batch, 4096, seed=3, key=(81, batch))
    y = lr.lr_linear(_factor_dev(f), dev(x))
    assert normwise_rel(y, _oracle(f, x.double().numpy())) < NORMWISE_TOL
    p = synth.make_prefill_projection(4096, 4096, 512, seed=3, key=(82,))
    xi = synth.make_activations(batch, 4096, seed=3, key=(83, batch))
    yi = lr.lr_linear(lr.Factor(dev(p["A_q"]), dev(p["B_q"]), dev(p["s_A"]), dev(p["s_B"])), dev(xi))
    A = (p["A_q"].double() * p["s_A"].double()[:, None]).numpy().T
    Bq = (p["B_q"].double() * p["s_B"].double()[None, :]).numpy()
    assert normwise_rel(yi, lowrank.lr_linear(xi.double().numpy(), A, Bq)) < NORMWISE_TOL


def test_workspace_left_zeroed_and_reusable(cuda_device, layer0):
    f = _factor_dev(layer0["v"])
    x = dev(synth.make_activations(2, 4096, seed=3, key=(24,)))
    ws = lr.workspace(lr.lr_linear_workspace_size(f, 2), x.device)
    y1 = lr.lr_linear(f, x, ws=ws)
    y2 = lr.lr_linear(f, x, ws=ws)
    torch.cuda.synchronize()
    assert int(ws.count_nonzero()) == 0
    # split reductions may add in a different order: equal to rounding
    assert normwise_rel(y2, y1.double().cpu().numpy()) < 1e-3


def test_errors_raise(cuda_device, layer0):
    f = _factor_dev(layer0["o"])
    x = dev(synth.make_activations(1, 4096, seed=4, key=(25,)))
    ws = lr.workspace(64, x.device)
    with pytest.raises(lr.LrError):
        lr.lr_linear(f, x, ws=ws)
    assert lr.lr_check_device_error() == 0


@pytest.mark.parametrize("batch", [5, 8])
def test_cuda_core_path_multi_row(cuda_device, layer0, batch):
    # the CUDA-core kernels at several rows per pass (the tensor cores take these batches by default)
    lr.lr_set_tensor_core_min_batch(64, 64)
    try:
        x = synth.make_activations(batch, 4096, seed=13, key=(26, batch))
        fs = [_factor_dev(layer0[n]) for n in ("q", "k", "v")]
        ys = lr.lr_linear_grouped(fs, dev(x))
        for y, n in zip(ys, ("q", "k", "v")):
            assert normwise_rel(y, _oracle(layer0[n], x.double().numpy())) < NORMWISE_TOL
    finally:
        lr.lr_set_tensor_core_min_batch(0, 0)
