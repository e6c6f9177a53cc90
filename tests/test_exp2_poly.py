"""The FMA-pipe exp2 of the bf16 attention kernel, emulated step by step in float32 on the CPU
(same coefficients, same range reduction, same exponent insertion), against exact 2^x."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "scaled_dot_product_16_b200", "csrc", "fwd_bf16_sm100.cu")


def _coeffs():
    text = open(SRC).read()
    body = text[text.index("exp2_poly2"):]
    return [np.float32(float(re.search(rf"c{i} = ([0-9.e+-]+)f", body).group(1))) for i in range(4)]


def _emulate(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    shift = np.float32(12582912.0)
    with np.errstate(invalid="ignore", over="ignore"):
        t = (x + shift).astype(np.float32)
        j = (t - shift).astype(np.float32)
        f = (x - j).astype(np.float32)        # fma(j, -1, x) is exact here
        q = (c3 * f + c2).astype(np.float32)  # separate rounding is within the fma's error
        q = (q * f + c1).astype(np.float32)
        q = (q * f + c0).astype(np.float32)
        bits = (q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    return bits.view(np.float32)


def test_relative_error_over_the_used_range():
    x = np.concatenate([np.linspace(-125.0, 8.5, 2_000_001, dtype=np.float32),
                        np.arange(-125, 9, dtype=np.float32),           # integers (f = 0)
                        np.arange(-125, 9, dtype=np.float32) + 0.5])    # ties (f = +-1/2)
    y = _emulate(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 8e-5, rel.max()


def test_masked_and_underflow_stay_below_2_to_minus_125():
    """Scores set to -inf by a mask and anything under -125.5 land on a non-negative value below
    2^-125 (never NaN, never an overflowed exponent); from -125.5 up the error bound holds."""
    x = np.concatenate([np.array([-np.inf, -1e30, -200.0, -127.0, -126.0], dtype=np.float32),
                        np.linspace(-130.0, -125.5, 10_001, dtype=np.float32)])
    y = _emulate(x)
    assert np.all(np.isfinite(y)) and np.all(y >= 0.0)
    assert np.all(y.astype(np.float64) < 2.0 ** -125)
    x = np.linspace(-125.5, -120.0, 100_001, dtype=np.float32)
    rel = np.abs(_emulate(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 8e-5, rel.max()
