"""The software exponent of the attention softmax (one pair of scores in four
takes it instead of the special-function unit) against the CUDA math
library's exp2f, which this test computes with torch on the device, and
against the hardware ex2.approx.

The stated bound is a relative error of at most 7.6e-5 for x in [-125, 8]
(the range that matters to the softmax: scores minus a reference maximum
that is never more than 8 below the block maximum).  Below -125 the input is
clamped, so the result is at most 2^-125, against a smaller true value.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_39_b200 import pbsa as K

pytestmark = pytest.mark.gpu

BOUND = 7.6e-5


def _eval(x):
    yp = torch.empty_like(x)
    yh = torch.empty_like(x)
    K.check_exp2(x, yp, yh)
    torch.cuda.synchronize()
    return yp, yh


def test_exp2_poly_within_its_bound_over_the_softmax_range():
    assert torch.cuda.is_available()
    # a dense grid over [-125, 8], every integer and half-integer (the range
    # split's boundaries), and odd sizes (the last pair half empty)
    grid = torch.linspace(-125.0, 8.0, 2_000_001, dtype=torch.float64)
    edges = torch.arange(-125.0, 8.01, 0.5, dtype=torch.float64)
    near = torch.cat([edges - 1e-4, edges + 1e-4])
    x = torch.cat([grid, edges, near]).clamp(-125.0, 8.0).float().cuda()
    yp, yh = _eval(x)
    ref = torch.exp2(x.double())                 # float64 reference of the float32 inputs
    lib = torch.exp2(x)                           # CUDA math library, float32
    rel_poly = ((yp.double() - ref) / ref).abs()
    rel_lib = ((lib.double() - ref) / ref).abs()
    assert float(rel_poly.max()) <= BOUND, float(rel_poly.max())
    # the library routine is far more accurate; the polynomial stays within the
    # bound of it as well
    assert float(rel_lib.max()) < 1e-6
    assert float(((yp.double() - lib.double()) / lib.double()).abs().max()) <= BOUND + 1e-6
    # the hardware unit it stands in for is within its own documented 2 ulp
    rel_hw = ((yh.double() - ref) / ref).abs()
    assert float(rel_hw.max()) < 1e-6
    # the bf16 P it feeds has 8 significant bits: the polynomial error is at
    # least 25 times smaller than half a bf16 ulp
    assert BOUND * 25 < 2.0 ** -9


def test_exp2_poly_special_points_and_odd_length():
    x = torch.tensor([0.0, 1.0, -1.0, 8.0, -125.0, 0.5, -0.5, 3.25, -126.0, -200.0],
                     device="cuda")
    yp, _ = _eval(x)
    ref = torch.exp2(x.double()).cpu().numpy()
    got = yp.double().cpu().numpy()
    np.testing.assert_allclose(got[:8], ref[:8], rtol=BOUND, atol=0)
    # below the range the input is clamped at -125: a normal float of at most 2^-125
    for g in got[8:]:
        assert 2.0 ** -126 <= g <= 2.0 ** -125 * (1 + BOUND)
