"""GPU: lr_linear_noalloc, the factorised linear that allocates nothing.

Callers inside a framework that owns all device memory, or a serving loop
that must not allocate after start-up, cannot hand the library a workspace.
lr_linear_noalloc serves them from a fixed scratch array inside the library.
This file checks, through the C ABI, that two calls in a row give what
lr_linear gives with a caller workspace (to the parity tolerance), and that a
call needing more scratch than the array holds is refused.  It is named so
that pytest collects it last.
"""
import ctypes

import pytest
import torch

import decode_lr_linear_b200 as lr
from decode_lr_linear_b200 import _lib as L
from decode_lr_linear_b200 import synth
from tests._helpers import NORMWISE_TOL, dev, normwise_rel

pytestmark = pytest.mark.gpu


def _call_noalloc(factor: lr.Factor, x: torch.Tensor) -> torch.Tensor:
    y = torch.empty(x.shape[0], factor.d_out, dtype=factor.out_dtype(), device=x.device)
    d = factor.desc()
    st = L.load().lr_linear_noalloc(ctypes.byref(d), x.data_ptr(), x.shape[0], y.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)
    L.check("lr_linear_noalloc", st)
    return y


@pytest.mark.parametrize("batch", [1, 3])
def test_noalloc_matches_workspace_path_twice(cuda_device, batch):
    ranks = synth.attention_ranks(0)
    layer = synth.make_attention_layer(0, ranks, seed=0)
    f = layer["k"]
    factor = lr.Factor(dev(f["At"]), dev(f["B"]))
    x = dev(synth.make_activations(batch, 4096, seed=7, key=(50, batch)))
    ref = lr.lr_linear(factor, x).double().cpu().numpy()
    y1 = _call_noalloc(factor, x)
    y2 = _call_noalloc(factor, x)
    torch.cuda.synchronize()
    assert normwise_rel(y1, ref) < NORMWISE_TOL
    assert normwise_rel(y2, ref) < NORMWISE_TOL


def test_noalloc_fp32_small(cuda_device):
    d = synth.make_single_linear(0)
    factor = lr.Factor(dev(d["At"]), dev(d["B32"]))
    x = dev(d["x"])
    ref = lr.lr_linear(factor, x).double().cpu().numpy()
    for _ in range(2):
        assert normwise_rel(_call_noalloc(factor, x), ref) < NORMWISE_TOL


def test_noalloc_refuses_oversized_request(cuda_device):
    # 8 batch rows x 40000 outputs x 4 bytes exceeds the fixed scratch
    At = torch.zeros(32, 64, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(32, 40000, dtype=torch.bfloat16, device="cuda")
    x = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(8, 40000, dtype=torch.bfloat16, device="cuda")
    d = lr.Factor(At, B).desc()
    st = L.load().lr_linear_noalloc(ctypes.byref(d), x.data_ptr(), 8, y.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)
    assert st == L.LR_ERR_WORKSPACE
