"""The polynomial exponential that shares each score tile with the special-function
unit, checked on the device against float64 2^x and against CUDA's exp2f (torch.exp2
on the GPU in float32)."""
import numpy as np
import pytest
import torch

import exact_tiled_attention_34_b200 as fa

pytestmark = pytest.mark.gpu


def test_poly_exp2_error_bound(cuda_device):
    x = torch.cat([torch.linspace(-126.0, 10.0, 2_000_001), torch.linspace(-1.0, 1.0, 200_001),
                   torch.arange(-126, 11, dtype=torch.float32)]).to(cuda_device)
    y = fa.debug_exp2(x, 1).double().cpu().numpy()
    ref = np.exp2(x.double().cpu().numpy())
    rel = np.abs(y / ref - 1.0)
    # fit bound 1.02e-4 plus fp32 rounding of the few operations
    assert float(rel.max()) < 1.1e-4
    ints = torch.arange(-126, 11, dtype=torch.float32, device=cuda_device)
    assert torch.equal(fa.debug_exp2(ints, 1), torch.exp2(ints.double()).float())  # 2^n exact


def test_poly_vs_cuda_exp2f(cuda_device):
    x = torch.linspace(-60.0, 8.0, 1_000_001, device=cuda_device)
    y = fa.debug_exp2(x, 1)
    ref = torch.exp2(x)  # CUDA's exp2f
    assert float((y.double() / ref.double() - 1).abs().max()) < 1.1e-4
    m = fa.debug_exp2(x, 0)  # the special-function path against exp2f too
    assert float((m.double() / ref.double() - 1).abs().max()) < 1e-6


def test_poly_tiny_inputs_do_not_wrap(cuda_device):
    x = torch.tensor([-1e4, -500.0, -200.0, -127.0, -126.4, -126.0], device=cuda_device)
    y = fa.debug_exp2(x, 1)
    assert torch.all(y >= 0) and torch.all(y < 1e-37)
