"""The FMA-pipe exponential the prefill kernel uses for part of its probabilities,
against the library exp2 (fp64 reference of the same fp32 inputs)."""

import numpy as np
import pytest
import torch

import attn_fwd_05_b200 as ab

pytestmark = pytest.mark.gpu


def test_exp2_poly_relative_error(cuda_device):
    # the range the softmax feeds it: scores minus the row maximum, up to the 2^8 slack
    x = torch.cat([torch.linspace(-125.0, 9.0, 1 << 20), torch.tensor([0.0, -0.5, 0.5, 1.0, -1.0, 8.0, -124.5])])
    x = x.to(torch.float32).to(cuda_device)
    y = torch.empty_like(x)
    ab.attn_debug_exp2(x, y)
    ref = np.exp2(x.double().cpu().numpy())
    got = y.double().cpu().numpy()
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1e-4, rel.max()
    assert got[-7] == 1.0 or abs(got[-7] - 1.0) < 1e-4


def test_exp2_poly_clamps_below_range(cuda_device):
    x = torch.tensor([-126.0, -200.0, -1e30, -300.5], device=cuda_device)
    y = torch.empty_like(x)
    ab.attn_debug_exp2(x, y)
    got = y.cpu().numpy()
    assert np.all(got > 0) and np.all(got < 4e-38)  # about 2^-125: negligible next to the row maximum's 1
