"""The kernels' FMA-pipe exp2 (Cody-Waite reduction + degree-4 minimax
polynomial) against CUDA's own exp2f on the range the softmax uses."""
import numpy as np
import pytest
import torch

import causal_flash_attention_attn_b200 as fa

pytestmark = pytest.mark.gpu


def test_exp2_poly_matches_cuda_exp2f():
    g = torch.Generator().manual_seed(5)
    x = torch.cat([torch.linspace(-125.0, 8.0, 1_000_001),
                   torch.rand(1_000_000, generator=g) * 20.0 - 12.0,
                   torch.tensor([0.0, -0.5, 0.5, -1.0, 1.0, 7.999, -124.5])]).to("cuda")
    y = torch.empty_like(x)
    yr = torch.empty_like(x)
    assert fa.forge_attn_selftest_exp2(x, y, yr, x.numel()) == fa.FORGE_OK
    torch.cuda.synchronize()
    y, yr, xd = y.double().cpu().numpy(), yr.double().cpu().numpy(), x.double().cpu().numpy()
    exact = np.exp2(xd)
    rel = np.abs(y - exact) / exact
    # the polynomial's f32 Horner bound (2.7e-6) plus a few ulps of rounding
    assert rel.max() < 4e-6, rel.max()
    # and CUDA's exp2f agrees with the exact value to its documented ulp bound
    assert (np.abs(yr - exact) / exact).max() < 1e-6
