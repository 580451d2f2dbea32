"""The kernels' FMA-pipe cubic 2^x against the definition and the oracle's model."""
import numpy as np
import pytest
import torch

from oracle import exp2_cubic

pytestmark = pytest.mark.gpu


def test_exp2_poly_error_bound():
    import attention_attn_fwd_10_b200 as attn

    # every fp32 in (-2, -1] (its fraction f runs over every multiple of 2^-23 in [0, 1))
    # plus a dense sweep of [-125, 16]
    x1 = np.arange(0xBF800000, 0xC0000000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    x2 = np.linspace(-125.0, 16.0, 4_000_001, dtype=np.float32)
    x = np.concatenate([x1, x2]).astype(np.float32)
    y = attn.exp2_poly_eval(torch.from_numpy(x).cuda()).cpu().numpy().astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    # minimax relative error of the cubic is 7.48e-5; fp32 evaluation adds a few ulp
    assert rel.max() < 7.48e-5 + 4e-7, rel.max()
    # and it matches the oracle's independently fitted model of the same scheme
    c, _ = exp2_cubic.remez_cubic()
    ym = exp2_cubic.exp2_cubic_f32(x, c).astype(np.float64)
    assert np.max(np.abs(y / ym - 1.0)) < 2e-6


def test_exp2_poly_tiny_inputs():
    import attention_attn_fwd_10_b200 as attn

    x = torch.tensor([-1e30, -1000.0, -200.0, -127.0, -126.0, -125.5], dtype=torch.float32, device="cuda")
    y = attn.exp2_poly_eval(x).cpu()
    assert torch.all(y >= 0) and torch.all(y < 2.0 ** -124)
