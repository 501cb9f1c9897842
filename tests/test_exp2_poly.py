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


def _sat_consts():
    src = open(HDR).read()
    span = np.float32(float(re.search(r"kSatSpan = ([0-9.]+)f", src).group(1)))
    body = src[src.index("float2 exp2_poly_sat2"):]
    body = body[:body.index("return p;")]
    nums = [float(x) for x in re.findall(r"make_float2\(([0-9.]+)f,", body)]
    return span, np.float32(nums[0]), [np.float32(v) for v in nums[1:5]]


def _fma32(a, b, c):
    """float32 fused multiply-add: exact product and sum in float64, one rounding."""
    return (np.asarray(a, np.float64) * np.asarray(b, np.float64)
            + np.asarray(c, np.float64)).astype(np.float32)


def exp2_poly_sat_emulated(v, c, m):
    """The pass-1 fast path for one logit v: y = sat(v * c/span + (125 - m)/span),
    then 2^(span * y - 125) by the split and polynomial of exp2_poly_sat2."""
    span, base, (c3, c2, c1, c0) = _sat_consts()
    cs = np.float32(np.float32(c) * np.float32(1.0 / span))
    bs = np.float32((np.float32(125.0) - np.float32(m)) * np.float32(1.0 / span))
    y = np.clip(_fma32(v, cs, bs), 0.0, 1.0).astype(np.float32)
    j = _fma32(y, span, base)
    t = (base - j).astype(np.float32)
    f = _fma32(y, span, t)
    p = _fma32(c3, f, c2)
    p = _fma32(p, f, c1)
    p = _fma32(p, f, c0)
    bits = p.view(np.int32) + (j.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_saturated_form_constants():
    span, base, _ = _sat_consts()
    assert base == np.float32(1.5 * 2**23 - 125)
    assert span == np.float32(251.0)       # x = span * y - 125 covers [-125, 126]


def test_saturated_form_relative_error_bound():
    """Against the exact 2^(c v - m) over the whole unclamped range, for the
    scale of head dim 128 and references m from -40 to 60."""
    c = np.float32(1.4426950408889634 / np.sqrt(128.0))
    rng = np.random.default_rng(1)
    for m in (-40.0, 0.0, 7.25, 60.0):
        x = np.concatenate([np.linspace(-124.5, 125.5, 500_001),
                            rng.uniform(-30, 30, 100_000)])
        v = ((x + m) / c).astype(np.float32)
        xe = np.float64(c) * v.astype(np.float64) - m          # the exact exponent of this v
        keep = (xe > -124.9) & (xe < 125.9)
        got = exp2_poly_sat_emulated(v[keep], c, m).astype(np.float64)
        rel = np.abs(got / np.exp2(xe[keep]) - 1)
        assert rel.max() <= 1e-4, (m, rel.max())


def test_saturated_form_clamps_both_ways():
    """Logits far above the reference give 2^126 (finite, and above the 2^100
    that sends a chunk to the exact path); far below and masked (-inf) give
    2^-125, negligible next to a row sum >= 1."""
    c = np.float32(0.1275)
    got = exp2_poly_sat_emulated(np.array([1e4, 3e3, -1e4, -np.inf], np.float32), c, 0.0)
    assert np.all(np.isfinite(got)) and np.all(got > 0)
    assert got[0] >= 2.0**100 and got[1] >= 2.0**100
    assert got[2] < 1e-37 and got[3] < 1e-37
