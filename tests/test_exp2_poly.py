"""The scorer's polynomial 2^x (FMA-pipe share of pass 1's exponentials),
emulated step by step in IEEE float32 on the CPU with the coefficients read
from the CUDA header, against the exact 2^x: relative error <= 8e-5 for
x in [-125, 0], and tiny (not NaN) for x = -inf."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "attention_score_reduction_b200", "csrc", "sm100_ptx.cuh")


def _coeffs():
    src = open(HDR).read()
    body = src[src.index("float2 exp2_poly2"):]
    body = body[:body.index("return p;")]
    nums = [float(x) for x in re.findall(r"make_float2\(([0-9.]+)f,", body)]
    # shift, c3, c2, c1, c0 in order of appearance
    return np.float32(nums[0]), [np.float32(v) for v in nums[1:5]]


def exp2_poly_emulated(x):
    x = np.asarray(x, dtype=np.float32)
    shift, (c3, c2, c1, c0) = _coeffs()
    x = np.maximum(x, np.float32(-125.0))
    j = (x + shift).astype(np.float32)
    n = (j - shift).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = (c3 * f + c2).astype(np.float32)      # fma: single rounding; product exact enough here
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = p.view(np.int32) + (j.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_shift_constant_is_one_and_a_half_times_2_pow_23():
    shift, _ = _coeffs()
    assert shift == np.float32(1.5 * 2**23)


def test_relative_error_bound():
    x = np.concatenate([np.linspace(-125, 0, 2_000_001, dtype=np.float32),
                        -np.random.default_rng(0).random(100000).astype(np.float32) * 30])
    got = exp2_poly_emulated(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1)
    assert rel.max() <= 8e-5, rel.max()


def test_masked_inputs_give_negligible_values():
    got = exp2_poly_emulated(np.array([-np.inf, -1e30, -200.0], dtype=np.float32))
    assert np.all(np.isfinite(got)) and np.all(got > 0) and np.all(got < 1e-37)

