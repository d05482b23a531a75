"""Pins of the oracle's FFN activation, GELU in its tanh form (no GPU).

The DiT's transformer blocks are attention and FFN (171host.com LongLive-2.0
teardown, usage section "训练管线": LoRA on Attn/FFN); the pages name no
activation form, and the reading taken is the tanh form,
0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))).  The oracle evaluates it in
binary64.  Pinned here against torch's own float64 GELU (approximate="tanh"),
which fixes the inner polynomial, and against identities that hold for any odd
inner function: GELU(y) - GELU(-y) = y, GELU(0) = 0, GELU(y) -> y and -> 0 far
out.  The slope bound used by the GPU tolerance (|GELU'| <= 1.13) is checked on
a fine grid.
"""
import numpy as np
import pytest
import torch

from _util import GELU_SLOPE_MAX


def _grid():
    g = np.random.default_rng(7)
    return np.concatenate([np.linspace(-12, 12, 4801), g.standard_normal(4000) * 3,
                           [0.0, -0.0, 1e-300, -1e-300, 1e-8, -1e-8, 40.0, -40.0, 1e6, -1e6]])


def test_matches_torch_float64_tanh_gelu(orc):
    y = _grid()
    ref = torch.nn.functional.gelu(torch.from_numpy(y), approximate="tanh").numpy()
    got = orc.gelu_tanh(y)
    # where y < 0 the two sides cancel in 1 + tanh(.): compare on the scale of |y|
    assert np.all(np.abs(got - ref) <= 1e-15 * (np.abs(y) + np.abs(ref)))
    # a wrong coefficient (0.0447 for 0.044715) is far outside that
    y1 = np.array([1.0, 2.0, -1.5])
    bad = 0.5 * y1 * (1 + np.tanh(np.sqrt(2 / np.pi) * (y1 + 0.0447 * y1 ** 3)))
    assert np.all(np.abs(orc.gelu_tanh(y1) - bad) > 1e-7)


def test_odd_part_is_identity(orc):
    y = _grid()
    d = orc.gelu_tanh(y) - orc.gelu_tanh(-y)
    np.testing.assert_allclose(d, y, rtol=1e-15, atol=1e-300)


def test_zero_and_tails(orc):
    assert orc.gelu_tanh(np.array([0.0]))[0] == 0.0
    far = np.array([40.0, 1e6, -40.0, -1e6])
    out = orc.gelu_tanh(far)
    assert out[0] == 40.0 and out[1] == 1e6
    assert out[2] == 0.0 and out[3] == 0.0
    # below zero the function dips to its minimum near y = -0.75 and is never below -0.171
    y = np.linspace(-5, 0, 50001)
    assert orc.gelu_tanh(y).min() > -0.171


def test_slope_bound(orc):
    y = np.linspace(-10, 10, 400001)
    g = orc.gelu_tanh(y)
    slope = np.diff(g) / np.diff(y)
    assert slope.max() <= GELU_SLOPE_MAX
    assert slope.max() > 1.12  # the bound is tight, not a loose guess
    assert slope.min() > -0.2


def test_rejects_non_finite(orc):
    with pytest.raises(Exception):
        orc.gelu_tanh(np.array([1.0, np.nan]))
