"""GPU test of the FMA-pipe exp2 the prefill softmax uses for a share of its
probabilities: its relative error against CUDA's exp2f (torch.exp2 on the
device) and against float64 stays within the bound of its minimax fit
(exp2_poly_fit.py: 7.5e-5, plus float32 rounding) over the arguments the
softmax produces, and the clamp below -126 gives values that no sum notices."""
import numpy as np
import pytest
import torch

import split_kv_merge_attn_b200 as skv

pytestmark = pytest.mark.gpu

BOUND = 7.5e-5 + 3 * 2.0 ** -24


def test_exp2_fma_error_bound():
    g = torch.Generator().manual_seed(0)
    # the softmax's arguments lie in [-inf, 8]; the bound holds down to -125 (below it results are subnormal-sized)
    x = torch.cat([torch.linspace(-125.0, 8.0, 2_000_001), (torch.rand(1_000_000, generator=g) - 0.5) * 40,
                   torch.tensor([0.0, -0.5, 0.5, 1.0, -1.0, 7.999, 100.25, -124.75])]).float().cuda()
    y = skv.exp2_fma(x)
    ref32 = torch.exp2(x)
    torch.cuda.synchronize()
    rel32 = ((y.double() - ref32.double()).abs() / ref32.double()).max().item()
    x64 = x.double().cpu().numpy()
    rel64 = np.max(np.abs(y.double().cpu().numpy() - np.exp2(x64)) / np.exp2(x64))
    assert rel32 <= BOUND + 2.0 ** -22, rel32
    assert rel64 <= BOUND, rel64
    # nearly unbiased (a biased error would shift every row sum the same way)
    mean = ((y.double().cpu().numpy() - np.exp2(x64)) / np.exp2(x64)).mean()
    assert abs(mean) < 2e-5, mean
    assert skv.device_error() == 0


def test_exp2_fma_clamp_and_odd_length():
    x = torch.tensor([-125.5, -126.0, -127.0, -200.0, -1e30, 3.0], dtype=torch.float32, device="cuda")
    y = skv.exp2_fma(x).cpu()
    assert torch.isfinite(y).all() and (y >= 0).all()
    assert (y[:5] <= 2.0 ** -124).all()
    assert abs(y[5].item() - 8.0) <= 8.0 * BOUND
