"""Pins of the oracle's e4m3 quantiser against the format definition.

Every expected value below follows from the OCP e4m3 definition (sign,
4-bit exponent with bias 7, 3-bit mantissa, subnormals m * 2^-9, largest
finite 448, 0x7F NaN) by hand arithmetic, not from the encoder under test.
"""
import numpy as np
import pytest

from oracle.fp8 import E4M3_MAX, dequantize_e4m3, e4m3_decode, e4m3_encode, quantize_e4m3


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6),
    (0x38, 1.0), (0x3C, 1.5), (0x3F, 1.875), (0x40, 2.0), (0x7E, 448.0),
    (0x77, 240.0), (0xB8, -1.0), (0xFE, -448.0),
])
def test_decode_hand_values(code, value):
    assert e4m3_decode(code) == value


def test_decode_nan_and_negative_zero():
    assert np.isnan(e4m3_decode(0x7F)) and np.isnan(e4m3_decode(0xFF))
    v = e4m3_decode(0x80)
    assert v == 0.0 and np.signbit(v)


def test_every_finite_code_round_trips():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = e4m3_decode(codes)
    assert np.array_equal(e4m3_encode(vals), codes)


@pytest.mark.parametrize("x,code", [
    (1.0625, 0x38),            # halfway 1.0 / 1.125: ties to the even mantissa (1.0)
    (1.1875, 0x3A),            # halfway 1.125 / 1.25: ties to even (1.25)
    (1.06, 0x38), (1.07, 0x39),   # either side of the midpoint 1.0625
    (1.07 + 0.0625, 0x39),
    (3 * 2.0 ** -10, 0x02),    # halfway 1 / 2 subnormal steps: even (2)
    (2.0 ** -10, 0x00),        # halfway 0 / smallest subnormal: even (0)
    (2.0 ** -10 * 1.01, 0x01),
    (15.5 * 2.0 ** -10, 0x08), # 7.75 subnormal steps: rounds to 8 = smallest normal
    (464.0, 0x7E),             # halfway 448 / 480 would be NaN: saturates
    (500.0, 0x7E), (1e30, 0x7E), (-1000.0, 0xFE),
    (-0.0, 0x80),
])
def test_encode_hand_values(x, code):
    assert int(e4m3_encode(np.array([x]))[0]) == code


def test_encode_is_monotone_and_within_half_ulp():
    rng = np.random.default_rng(0)
    x = np.sort(np.concatenate([rng.uniform(0, 448, 4000), 2.0 ** rng.uniform(-12, 8.8, 4000)]))
    c = e4m3_encode(x)
    v = e4m3_decode(c)
    assert np.all(np.diff(v) >= 0)
    normal = (x >= 2.0 ** -6) & (x <= E4M3_MAX)
    # 3 mantissa bits: the nearest code is within half a unit, 2^-4 relative
    assert np.all(np.abs(v[normal] - x[normal]) <= 2.0 ** -4 * x[normal])
    sub = x < 2.0 ** -6
    assert np.all(np.abs(v[sub] - x[sub]) <= 2.0 ** -10)


def test_quantize_scales_and_codes():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((2, 3, 50, 8)).astype(np.float32)
    x[1, 2] = 0.0
    codes, scale = quantize_e4m3(x)
    assert scale.dtype == np.float32 and scale.shape == (2, 3)
    for b in range(2):
        for h in range(3):
            amax = np.float32(np.abs(x[b, h]).max())
            if amax == 0:
                assert scale[b, h] == 1.0 and not codes[b, h].any()
                continue
            assert scale[b, h] == np.float32(amax / np.float32(448.0))
            # the largest magnitude lands on the largest code
            i = np.unravel_index(np.abs(x[b, h]).argmax(), x[b, h].shape)
            assert codes[b, h][i] & 0x7F == 0x7E
    deq = dequantize_e4m3(codes, scale)
    big = np.abs(x) >= 2.0 ** -6 * scale[:, :, None, None]
    assert np.all(np.abs(deq - x)[big] <= 2.0 ** -4 * np.abs(x)[big] * (1 + 1e-6))
