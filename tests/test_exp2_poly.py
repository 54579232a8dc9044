"""The FMA-pipe 2^y kept beside the softmax (off by default: measured slower):
replay its float32 operation sequence, with the coefficients of our own fit
read from rola_common.cuh, and check it against 2^y in float64.  P is rounded to bf16 (relative 2^-9)
afterwards, so a relative error below 1e-4 is invisible in the output."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "sparse_linear_attention_mean_b200", "csrc", "rola_common.cuh")


def coeffs():
    text = open(HDR).read()
    return [np.float32(float(re.search(rf"kExp2C{i} = ([0-9.e+-]+)f", text).group(1))) for i in range(4)]


def emulate(y):
    c0, c1, c2, c3 = coeffs()
    y = np.maximum(np.asarray(y, np.float32), np.float32(-126))
    t = (y + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (y - n).astype(np.float32)              # fma(n, -1, y) is exact here
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_range_reduction_is_rint_and_fraction_bounded():
    y = np.linspace(-125, 9, 100001).astype(np.float32)
    t = (y + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    assert np.array_equal(n, np.rint(y))
    assert np.abs(y - n).max() <= 0.5


def test_relative_error_below_1e4():
    y = np.concatenate([np.linspace(-125, 9, 400001), np.arange(-125, 10) + 0.5,
                        np.arange(-125, 10) - 0.5, np.arange(-125, 10)]).astype(np.float32)
    got = emulate(y).astype(np.float64)
    want = np.exp2(y.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1e-4, rel.max()


def test_exact_powers_close_and_clamp():
    y = np.arange(-120, 9).astype(np.float32)
    got = emulate(y).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(y.astype(np.float64)) - 1) < 1e-4)
    # masked scores (-inf) become negligible, never negative or NaN
    tiny = emulate(np.array([-np.inf, -1e30, -200.0], np.float32))
    assert np.all(np.isfinite(tiny)) and np.all(tiny >= 0) and np.all(tiny < 2.0 ** -120)
