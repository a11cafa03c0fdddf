"""The attention kernel's FMA-pipe 2^x against 2^x itself.

Stage 2 evaluates three of every eight pairs of its softmax exponentials
with its own polynomial (a Cody-Waite split x = n + f, |f| <= 1/2, and a
degree-3 polynomial for 2^f fitted by iteratively reweighted least squares
for minimum maximum relative error, 7.5e-5) instead of the special-function
unit.  Its arguments are s * scale + bias - m with a lazily updated running
maximum m, which may trail the block maximum by up to 8 (in log2 units), so
they lie in (-inf, 8].  This checks the polynomial element by element over
a dense grid of that range against the exact 2^x (fp64) and against CUDA's
exp2f (torch.exp2 on the device), and pins the clamp: every argument below
-125 (-inf included) gives the value at -125, about 2^-125, which is
negligible next to the row maximum's 1 but not zero.
"""

import numpy as np
import pytest
import torch

from sparse_hierarchical_attention_chunk_b200 import dash

pytestmark = pytest.mark.gpu

REL_BOUND = 7.5e-5          # the fit's stated maximum relative error
FP32_SLACK = 4 * 2.0 ** -24  # rounding of the fp32 evaluation itself


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_hierarchical_attention_chunk_b200 import build
    build.build()
    dash.lib()


def _poly(x):
    xd = x.cuda()
    y = torch.empty_like(xd)
    dash.dash_selftest_exp2_poly(xd, y)
    assert dash.dash_get_error() == dash.DASH_OK
    return y


def test_relative_error_within_the_fit_bound():
    # every float32 step of 1/4096 over [-125, 8], plus the odd count that
    # leaves a last element unpaired
    x = torch.arange(-125 * 4096, 8 * 4096 + 1, dtype=torch.float64) / 4096.0
    x = torch.cat([x, torch.tensor([0.3])]).float()
    y = _poly(x).double().cpu().numpy()
    exact = np.exp2(x.double().numpy())
    rel = np.abs(y - exact) / exact
    assert rel.max() <= REL_BOUND + FP32_SLACK, float(rel.max())
    # and against CUDA's exp2f on the same inputs (itself within 2 ulp of 2^x)
    cuda = torch.exp2(x.cuda()).double().cpu().numpy()
    assert (np.abs(y - cuda) / cuda).max() <= REL_BOUND + FP32_SLACK + 2 * 2.0 ** -23


def test_random_arguments_and_integers():
    g = torch.Generator().manual_seed(5)
    x = (torch.rand(1 << 20, generator=g, dtype=torch.float64) * 133.0 - 125.0).float()
    y = _poly(x).double().cpu().numpy()
    exact = np.exp2(x.double().numpy())
    assert (np.abs(y - exact) / exact).max() <= REL_BOUND + FP32_SLACK
    # integer arguments: 2^n times the polynomial at f = 0 (0.99992806)
    n = torch.arange(-125, 9, dtype=torch.float32)
    yn = _poly(n).double().cpu().numpy()
    np.testing.assert_allclose(yn / np.exp2(n.double().numpy()), 0.99992806, rtol=1e-7)


def test_clamp_below_minus_125():
    x = torch.tensor([-125.0, -125.5, -126.0, -200.0, -1e30, -float("inf")])
    y = _poly(x).double().cpu().numpy()
    # all equal to the value at the clamp, within the bound of 2^-125
    assert np.all(y == y[0])
    assert abs(y[0] / 2.0 ** -125 - 1.0) <= REL_BOUND + FP32_SLACK
    assert y[0] > 0.0
