"""Pins of the FP8 oracle: e4m3 values fixed by the OCP 8-bit floating-point format,
its round-to-nearest-even rule checked by brute force, and the block quantizer's
properties."""

import numpy as np
import pytest

from oracle import block_quantize, dequantize, e4m3_value, quantize_e4m3


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6), (0x38, 1.0), (0x39, 1.125),
    (0x3F, 1.875), (0x40, 2.0), (0x7E, 448.0), (0x77, 240.0), (0xB8, -1.0), (0xFE, -448.0), (0x80, -0.0),
])
def test_e4m3_values_from_the_format(code, value):
    assert e4m3_value(code) == value


def test_e4m3_nan_codes():
    assert np.isnan(e4m3_value(0x7F)) and np.isnan(e4m3_value(0xFF))


def test_every_finite_code_round_trips():
    for c in list(range(0x7F)) + list(range(0x80, 0xFF)):
        v = e4m3_value(c)
        got = int(quantize_e4m3(np.array([v], dtype=np.float32))[0])
        assert got == c, (hex(c), v, hex(got))


def test_rounding_is_nearest_with_ties_to_even_by_brute_force():
    finite = np.array([e4m3_value(c) for c in range(0x7F)])
    rng = np.random.default_rng(3)
    y = np.concatenate([rng.uniform(-460, 460, 20000), rng.uniform(-2.0 ** -6, 2.0 ** -6, 20000),
                        (finite[1:] + finite[:-1]) / 2])        # every midpoint: a tie
    y = y.astype(np.float32).astype(np.float64)
    codes = quantize_e4m3(y.astype(np.float32))
    for yi, c in zip(y, codes):
        a = min(abs(yi), 448.0)
        dist = np.abs(finite - a)
        best = np.flatnonzero(dist == dist.min())
        want = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        assert (int(c) & 0x7F) == want, (yi, hex(int(c)), want)
        assert bool(int(c) & 0x80) == bool(np.signbit(yi))


def test_saturation():
    assert int(quantize_e4m3(np.array([1e6], dtype=np.float32))[0]) == 0x7E
    assert int(quantize_e4m3(np.array([-500.0], dtype=np.float32))[0]) == 0xFE


def test_block_quantizer():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((2, 3, 300, 16)).astype(np.float32)
    x[0, 1, 128:256] = 0.0  # an all-zero block keeps scale 1
    codes, scales = block_quantize(x)
    assert codes.dtype == np.uint8 and scales.shape == (2, 3, 3)
    assert scales[0, 1, 1] == 1.0 and np.all(codes[0, 1, 128:256] == 0)
    # the block maximum lands on the largest code and every value is within half a unit
    # of the format (relative 2^-4) after scaling back
    back = dequantize(codes, scales)
    err = np.abs(back - x)
    assert np.all(err <= np.abs(x) * 2.0 ** -4 + np.repeat(scales, 128, axis=-1)[..., :300, None] * 2.0 ** -10)
    for idx in np.ndindex(2, 3):
        for j in range(3):
            blk = x[idx][j * 128:(j + 1) * 128]
            if np.abs(blk).max() > 0:
                assert (int(np.abs(codes[idx][j * 128:(j + 1) * 128].astype(np.int64) & 0x7F).max())) == 0x7E
