"""The FMA-pipe exponential used for part of the softmax (common.cuh): the
coefficients are read out of the kernel source and the whole algorithm
(shifter rounding x = n + f, degree-3 polynomial, n added to the exponent
field) is emulated step by step in fp32 and compared with the exact 2^x.
CPU only."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "mqa_kv_cache_b200", "csrc",
                   "common.cuh")


def _coeffs():
    text = open(SRC).read()
    vals = {k: np.float32(v) for k, v in re.findall(r"(kP[0-3]) = ([0-9.eE+-]+)f", text)}
    shifter = np.float32(re.search(r"kShifter = ([0-9.]+)f", text).group(1))
    return [vals[f"kP{i}"] for i in range(4)], shifter


def _exp2_fma(x):
    (c0, c1, c2, c3), S = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + S).astype(np.float32)
    n = (t - S).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.float32(c3) * f + c2
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_shifter_is_one_and_a_half_times_2_pow_23():
    _, S = _coeffs()
    assert S == np.float32(1.5 * 2 ** 23)


def test_relative_error_over_the_softmax_range():
    x = np.linspace(-120.0, 10.0, 2_000_001).astype(np.float32)
    got = _exp2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1.0e-4  # far below the bf16 spacing (2^-8) that P is rounded to


def test_integers_and_underflow():
    for k in range(-100, 9):
        v = _exp2_fma(np.array([k], np.float32))[0]
        assert abs(v / 2.0 ** k - 1.0) < 1.0e-4
    tiny = _exp2_fma(np.array([-np.inf, -1e30, -200.0], np.float32))
    assert np.all(tiny >= 0) and np.all(tiny < 1e-37)
