"""GPU: lr_linear_noalloc, the factorised linear that allocates nothing.

Some callers cannot hand the library a workspace: a plugin inside a host
framework that owns every device allocation, or a serving loop that must not
call cudaMalloc after start-up (it can synchronise the device and stall other
work).  lr_linear_noalloc serves them from a fixed scratch array inside the
library.  This file calls it through the C ABI and checks, on two calls in a
row and more, that it gives what lr_linear gives with a caller workspace and
what the float64 oracle gives (to the parity tolerance), that a call needing
more scratch than the array holds is refused, and that the array is clean
again after a kernel gave up a wait.  It is named so that pytest collects it
last.
"""
import ctypes

import numpy as np
import pytest
import torch

import decode_lr_linear_b200 as lr
from decode_lr_linear_b200 import _lib as L
from decode_lr_linear_b200 import synth
from oracle import lowrank
from tests._helpers import NORMWISE_TOL, dev, normwise_rel

pytestmark = pytest.mark.gpu


def _call_noalloc(factor: lr.Factor, x: torch.Tensor) -> torch.Tensor:
    y = torch.empty(x.shape[0], factor.d_out, dtype=factor.out_dtype(), device=x.device)
    d = factor.desc()
    st = L.load().lr_linear_noalloc(ctypes.byref(d), x.data_ptr(), x.shape[0], y.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)
    L.check("lr_linear_noalloc", st)
    return y


def _oracle_bf16(f, x):
    return lowrank.lr_linear(x.double().numpy(), f["At"].double().numpy().T, f["B"].double().numpy())


@pytest.fixture(scope="module")
def layer0():
    ranks = synth.attention_ranks(0)
    return synth.make_attention_layer(0, ranks, seed=0)


@pytest.mark.parametrize("batch", [1, 3, 16])
def test_noalloc_matches_workspace_path_and_oracle_twice(cuda_device, layer0, batch):
    f = layer0["k"]
    factor = lr.Factor(dev(f["At"]), dev(f["B"]))
    x = synth.make_activations(batch, 4096, seed=7, key=(50, batch))
    ref64 = _oracle_bf16(f, x)
    ref = lr.lr_linear(factor, dev(x)).double().cpu().numpy()
    # batch 16 runs as two launches of 8 rows that reuse the same scratch
    y1 = _call_noalloc(factor, dev(x))
    y2 = _call_noalloc(factor, dev(x))
    torch.cuda.synchronize()
    for y in (y1, y2):
        assert normwise_rel(y, ref) < NORMWISE_TOL
        assert normwise_rel(y, ref64) < NORMWISE_TOL


def test_noalloc_fp32_small(cuda_device):
    d = synth.make_single_linear(0)
    factor = lr.Factor(dev(d["At"]), dev(d["B32"]))
    x = dev(d["x"])
    ref64 = lowrank.lr_linear(d["x"].double().numpy(), d["At"].double().numpy().T, d["B32"].double().numpy())
    for _ in range(2):
        assert normwise_rel(_call_noalloc(factor, x), ref64) < 1e-5


def test_noalloc_int8_then_other_width(cuda_device, layer0):
    # int8 weights with fp16 scales, then a call with a different d_out into the same scratch
    p = synth.make_prefill_projection(2048, 1536, 352, seed=0, key=(7,))
    sA, sB = p["s_A"].half(), p["s_B"].half()
    x = synth.make_activations(5, 2048, seed=0, key=(51,))
    factor = lr.Factor(dev(p["A_q"]), dev(p["B_q"]), dev(sA), dev(sB))
    A = (p["A_q"].double() * sA.double()[:, None]).numpy().T
    B = (p["B_q"].double() * sB.double()[None, :]).numpy()
    ref = lowrank.lr_linear(x.double().numpy(), A, B)
    for _ in range(2):
        assert normwise_rel(_call_noalloc(factor, dev(x)), ref) < NORMWISE_TOL
    f = layer0["o"]
    xo = synth.make_activations(2, 4096, seed=7, key=(52,))
    y = _call_noalloc(lr.Factor(dev(f["At"]), dev(f["B"])), dev(xo))
    assert normwise_rel(y, _oracle_bf16(f, xo)) < NORMWISE_TOL


def test_noalloc_refuses_oversized_but_valid_request(cuda_device):
    # int8, d_out 32768 (a 32 KiB row, the widest lr_linear takes), batch 8:
    # 256 + 3 * 8 * 32768 * 4 bytes of scratch, more than the fixed array holds
    rng = np.random.default_rng(11)
    At = torch.from_numpy(rng.integers(-127, 128, size=(32, 64)).astype(np.int8))
    B = torch.from_numpy(rng.integers(-127, 128, size=(32, 32768)).astype(np.int8))
    sA = torch.full((32,), 1.0 / 64, dtype=torch.float32)
    sB = torch.full((32768,), 1.0 / 512, dtype=torch.float32)
    x = synth.make_activations(8, 64, seed=11, key=(53,))
    factor = lr.Factor(dev(At), dev(B), dev(sA), dev(sB))
    y = torch.empty(8, 32768, dtype=torch.bfloat16, device="cuda")
    d = factor.desc()
    xd = dev(x)
    st = L.load().lr_linear_noalloc(ctypes.byref(d), xd.data_ptr(), 8, y.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)
    assert st == L.LR_ERR_WORKSPACE
    # lr_linear with its own workspace takes the same shape
    yw = lr.lr_linear(factor, xd)
    ref = lowrank.lr_linear(x.double().numpy(), (At.double() * sA.double()[:, None]).numpy().T,
                            (B.double() * sB.double()[None, :]).numpy())
    assert normwise_rel(yw, ref) < NORMWISE_TOL


def test_noalloc_scratch_clean_after_a_wait_gave_up(cuda_device, layer0):
    # a bound far below the CTAs' arrival time makes the kernel's grid-barrier waits give up;
    # once lr_check_device_error has reported it, the next call re-zeroes the scratch
    f = layer0["v"]
    factor = lr.Factor(dev(f["At"]), dev(f["B"]))
    x = synth.make_activations(4, 4096, seed=7, key=(54,))
    try:
        lr.lr_set_wait_timeout_us(1)
        for _ in range(3):
            _call_noalloc(factor, dev(x))
        err = lr.lr_check_device_error()
    finally:
        lr.lr_set_wait_timeout_us(0)
    assert err in (0, L.DEVICE_ERR_GRID_WAIT)
    ref = _oracle_bf16(f, x)
    for _ in range(2):
        assert normwise_rel(_call_noalloc(factor, dev(x)), ref) < NORMWISE_TOL
    assert lr.lr_check_device_error() == 0
