"""Pins of the oracle's binary16 conversions against numpy's IEEE float16 (a
library routine with round-to-nearest-even), over every bit pattern and over
edge and random binary32 inputs."""
import numpy as np
import pytest

import oracle


def test_half_to_double_all_bit_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = oracle.half_to_double(bits)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zeros keep their sign
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


EDGE = [0.0, -0.0, 1.0, -1.0, 65504.0, 65519.99, 65520.0, 1e9, -1e9, 2.0 ** -24, 2.0 ** -25,
        1.5 * 2.0 ** -25, 2.0 ** -26, 2.0 ** -14, 2.0 ** -14 - 2.0 ** -25, 2.0 ** -14 * (1 - 2 ** -11),
        1 + 2 ** -11, 1 + 3 * 2 ** -11, 1 + 2 ** -11 + 2 ** -20, 2048.0 + 1.0, 2048.0 + 3.0,
        3.0 * 2.0 ** -24 / 2, 5.0 * 2.0 ** -24 / 2, 1e-30, -1e-30, float("inf"), float("-inf"),
        1.0 / 127.0, 0.3, 1.0 / 3.0, 6.1e-5, 6.0e-8, 5.9e-8, 2.9e-8, 3.0e-8]


@pytest.mark.parametrize("x", EDGE)
def test_float_to_half_edges(x):
    f = np.float32(x)
    ref = np.array([f], np.float32).astype(np.float16).view(np.uint16)[0]
    assert int(oracle.float_to_half(f)) == int(ref), hex(int(ref))


def test_float_to_half_nan():
    h = int(oracle.float_to_half(np.float32("nan")))
    assert (h & 0x7c00) == 0x7c00 and (h & 0x3ff) != 0


def test_float_to_half_random():
    rng = np.random.default_rng(123)
    mag = np.exp2(rng.uniform(-30, 17, 40000)).astype(np.float32)
    sgn = np.where(rng.random(40000) < 0.5, -1, 1).astype(np.float32)
    f = (mag * sgn).astype(np.float32)
    # plus exact ties between neighbouring halves
    h = rng.integers(0, 0x7bff, 2000, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float32)
    hi = (h + 1).astype(np.uint16).view(np.float16).astype(np.float32)
    ties = ((lo.astype(np.float64) + hi.astype(np.float64)) / 2).astype(np.float32)
    f = np.concatenate([f, ties])
    ref = f.astype(np.float16).view(np.uint16)
    got = oracle.float_to_half(f)
    assert np.array_equal(got, ref)
