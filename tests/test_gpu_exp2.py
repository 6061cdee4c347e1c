"""GPU: the softmax's FMA-pipe exponential (exp2_fma2, reached through the
sma_selftest_exp2 diagnostic) against CUDA's exp2 and the float64 value.

The forward softmax computes part of each row's 2^t on the FMA pipe: t is
split into round(t) + f, 2^f comes from a cubic fitted for relative error
(fit_exp2_poly.py: at most 7.5e-5 on [-1/2, 1/2] in float32), and 2^round(t)
is added to the exponent field.  Arguments at or below -125, -inf included,
come out as 2^-125 (the softmax tells an empty row by its max)."""
import numpy as np
import pytest
import torch

import structured_mask_attention_analytic_b200 as sma

pytestmark = pytest.mark.gpu

REL_BOUND = 7.5e-5 + 2.0 ** -22   # the cubic's bound plus float32 rounding of the last steps


def test_exp2_fma_relative_error_over_the_softmax_range():
    # softmax arguments lie in [-inf, +8] (the row max is rescaled lazily by up to 2^8)
    t = torch.cat([torch.linspace(-125.0, 8.0, 1 << 21), torch.tensor([0.0, -0.5, 0.5, -1.0, 7.99])])
    t = t[: t.numel() // 2 * 2].cuda()
    got = sma.selftest_exp2(t).double()
    exact = torch.exp2(t.double())
    rel = ((got - exact).abs() / exact).max().item()
    assert rel <= REL_BOUND, rel
    # CUDA's own float32 exp2 is within a few ulp of the exact value; ours
    # differs from it by no more than the cubic's bound plus those ulp
    cuda32 = torch.exp2(t).double()
    assert ((got - cuda32).abs() / cuda32).max().item() <= REL_BOUND + 2.0 ** -21


def test_exp2_fma_clamps_below_minus_125():
    t = torch.tensor([-float("inf"), -1e30, -200.0, -125.5, -125.0, 100.0], device="cuda")
    got = sma.selftest_exp2(t).double().cpu().numpy()
    floor = 2.0 ** -125
    assert np.all(np.abs(got[:5] / floor - 1.0) <= REL_BOUND)
    assert abs(got[5] / 2.0 ** 100 - 1.0) <= REL_BOUND
