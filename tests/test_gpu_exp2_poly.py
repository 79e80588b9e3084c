"""The tensor-core forward's polynomial exponential (2^x on the FMA pipe, used
for part of the softmax at head dims up to 64), evaluated through its test
hook and checked against the exact 2^x in fp64 over its whole input range:
relative error at most 7.5e-5 (the bound its fit states) for x in
[-125, 127], inputs below -125 (and -inf) clamped to -125."""

import numpy as np
import pytest
import torch

from tests._helpers import gpu

pytestmark = gpu

BOUND = 7.5e-5


@pytest.fixture(scope="module")
def rm():
    from sequence_attention_rm_b200 import rm as mod
    return mod


def _eval(rm, x: np.ndarray) -> np.ndarray:
    y = rm.debug_exp2_poly(torch.from_numpy(x.astype(np.float32)).cuda())
    return y.cpu().numpy().astype(np.float64)


def test_exp2_poly_relative_error_over_the_softmax_range(rm):
    # the softmax's arguments: s - m <= 0, or up to +8 while a row's max is
    # allowed to run ahead of the stored one; a dense grid of 2^-12 steps plus
    # the points where the nearest integer changes (odd multiples of 1/2) and
    # their float neighbours
    grid = np.arange(-125.0, 8.0, 2.0 ** -12)
    halves = np.arange(-124.5, 8.0, 1.0)
    near = np.concatenate([np.nextafter(halves.astype(np.float32), np.float32(-np.inf)),
                           halves.astype(np.float32),
                           np.nextafter(halves.astype(np.float32), np.float32(np.inf))])
    x = np.concatenate([grid.astype(np.float32), near, np.float32([0.0, -0.0, -125.0, 8.0])])
    y = _eval(rm, x)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(y - exact) / exact
    worst = int(np.argmax(rel))
    assert rel.max() <= BOUND, f"relative error {rel.max():.3e} at x = {x[worst]!r}"


def test_exp2_poly_full_exponent_range(rm):
    # every integer and half-integer exponent the function accepts, and a
    # random sample between them
    rng = np.random.default_rng(7)
    x = np.concatenate([np.arange(-125.0, 127.5, 0.5), rng.uniform(-125.0, 127.0, 200000)])
    x = x.astype(np.float32)
    y = _eval(rm, x)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(y - exact) / exact
    assert np.isfinite(y).all()
    assert rel.max() <= BOUND, f"relative error {rel.max():.3e} at x = {x[int(np.argmax(rel))]!r}"


def test_exp2_poly_clamps_below_minus_125(rm):
    x = np.float32([-125.0, -125.5, -126.0, -130.0, -1000.0, -3.0e38, -np.inf])
    y = _eval(rm, x)
    # everything below -125 gives exactly the value at -125: normal, positive,
    # within the bound of 2^-125
    assert (y == y[0]).all()
    assert y[0] > 0 and abs(y[0] - 2.0 ** -125) <= BOUND * 2.0 ** -125


def test_exp2_poly_odd_length_and_empty(rm):
    x = np.float32([-1.0, 0.5, 3.0])
    y = _eval(rm, x)
    assert np.all(np.abs(y - np.exp2(x.astype(np.float64))) <= BOUND * np.exp2(x.astype(np.float64)))
    assert rm.debug_exp2_poly(torch.empty(0, device="cuda")).numel() == 0
