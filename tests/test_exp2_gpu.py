"""The forward's FMA-pipe exponential against the exponential unit and 2^x.

The kernels may take part of their exponentials as 2^x = 2^j * p(f),
j = round(x), f = x - j in [-1/2, 1/2], with p a Remez polynomial of degree 3
(forward, 16-bit inputs), 2 (forward, FP8 inputs, whose P is rounded to a
3-bit mantissa) or 5 (backward, whose P also enters dS in fp32).
Over the range the softmax feeds it (x <= the rescale threshold, and clamped
at -125 below), its relative error must stay within the fit's bound, which
csrc/gen_exp2_poly.py reports for the fp32 Horner evaluation: 7.49e-5 for
degree 3, 1.73e-3 for degree 2, 2.20e-7 for degree 5 (checked here with 1 %
of slack for points between the fit's grid and 4 fp32 ulps of rounding).
"""

import numpy as np
import pytest
import torch

from exact_attention_136_b200 import _lib

pytestmark = pytest.mark.gpu

FIT = {3: 7.49e-5, 2: 1.725e-3, 5: 2.197e-7}   # the fit's own worst relative error
BOUND = {d: e * 1.01 + 4 * 2.0 ** -24 for d, e in FIT.items()}


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    _lib.lib()


def _run(x_np: np.ndarray, degree: int):
    dev = torch.device("cuda", 0)
    x = torch.from_numpy(x_np.astype(np.float32)).to(dev)
    poly = torch.empty_like(x)
    mufu = torch.empty_like(x)
    rc = _lib.lib().fa_exp2_check(x.data_ptr(), poly.data_ptr(), mufu.data_ptr(), x.numel(), degree,
                                  torch.cuda.current_stream().cuda_stream)
    assert rc == _lib.FA_OK, _lib.status_string(rc)
    torch.cuda.synchronize()
    return x.cpu().numpy().astype(np.float64), poly.cpu().numpy().astype(np.float64), mufu.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("degree", [3, 2, 5])
def test_polynomial_exp2_within_its_bound(degree):
    grid = np.linspace(-125.0, 8.0, 400001)
    edges = np.concatenate([np.arange(-125, 9), np.arange(-125, 8) + 0.5, np.arange(-125, 8) + 0.5 - 2.0 ** -20,
                            np.arange(-125, 8) + 0.5 + 2.0 ** -20])
    x, poly, mufu = _run(np.concatenate([grid, edges]), degree)
    exact = np.exp2(x)
    rel = np.abs(poly - exact) / exact
    assert rel.max() <= BOUND[degree], f"max relative error {rel.max():.3e} at x = {x[np.argmax(rel)]}"
    # and against the exponential unit, which the rest of the softmax uses
    rel_mufu = np.abs(poly - mufu) / mufu
    assert rel_mufu.max() <= BOUND[degree] + 2.0 ** -21
    # the fit is not loose: its worst point reaches half the fit's error (at
    # degree 5 the rounding slack is as large as the fit's error)
    assert rel.max() >= 0.5 * FIT[degree]


@pytest.mark.parametrize("degree", [3, 2, 5])
def test_polynomial_exp2_clamps_far_below(degree):
    """x below -125 (a score far under the row's maximum) gives a tiny
    non-negative value instead of a wrapped exponent."""
    x, poly, _ = _run(np.array([-125.5, -126.0, -127.0, -150.0, -300.0, -1000.0, -1e6, -3.0e38]), degree)
    assert np.all(poly >= 0.0) and np.all(poly <= 2.0 ** -124), poly


def test_exp2_check_rejects_bad_arguments():
    f = _lib.lib().fa_exp2_check
    assert f(None, None, None, -1, 3, None) == _lib.FA_ERR_ARG
    assert f(None, None, None, 4, 3, None) == _lib.FA_ERR_ARG
    assert f(None, None, None, 4, 4, None) == _lib.FA_ERR_ARG
    assert f(None, None, None, 0, 2, None) == _lib.FA_OK
