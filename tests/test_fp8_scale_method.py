"""The FP8 kernels' arithmetic shortcuts, checked on the host against exact
rational arithmetic (no GPU).

- The group scale RN(amax/448) is computed as the product with RN(1/448),
  corrected once by its exact remainder (P. Markstein, IBM J. Res. Dev.
  34(1), 1990). amax is the largest magnitude of a group of bf16 values, so
  the check runs over every finite non-negative bf16 value.
- The bracketed-reciprocal quantiser only needs the reciprocal of the scale
  to within 2^-22 relative (the approximate reciprocal is within 1 ulp): the
  products by RN(inv*(1-2^-20)) and RN(inv*(1+2^-20)) must enclose x/s.

Reading: "DeepSeek开源周第二天：DeepEP深度分析", section 性能 (FP8 dispatch with
per-128-channel scales); the scale is amax/448 in fp32, the code
e4m3(RN(x/scale)).
"""
import os
import re
from fractions import Fraction

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
QUANT = os.path.join(ROOT, "combine_ep_layout_09_b200", "csrc", "ep_quant.cuh")


def rn32(x: Fraction) -> Fraction:
    """x rounded to the nearest fp32 value, ties to even, gradual underflow
    (no overflow handling: the values here stay finite)."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    x = abs(x)
    e = x.numerator.bit_length() - x.denominator.bit_length()
    if Fraction(2) ** e > x:
        e -= 1
    elif Fraction(2) ** (e + 1) <= x:
        e += 1
    ulp = Fraction(2) ** (max(e, -126) - 23)
    m = x / ulp
    n = m.numerator // m.denominator
    rem = m - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * n * ulp


def test_rn32_matches_numpy_fp32():
    # the emulated rounding agrees with numpy's fp32 arithmetic
    rng = np.random.default_rng(0)
    a = rng.standard_normal(2000).astype(np.float32) * np.float32(2.0) ** \
        rng.integers(-140, 100, 2000).astype(np.float32)
    b = rng.standard_normal(2000).astype(np.float32)
    for x, y in zip(a, b):
        want = np.float32(x) * np.float32(y)
        assert float(rn32(Fraction(float(x)) * Fraction(float(y)))) == float(want)


def kernel_inv448() -> Fraction:
    src = open(QUANT).read()
    m = re.search(r"kInv448\s*=\s*(0x[0-9a-fA-F.]+p-?\d+)f", src)
    assert m, "kInv448 not found"
    return Fraction(float.fromhex(m.group(1)))


def test_scale_of_amax_is_the_correctly_rounded_quotient():
    c = kernel_inv448()
    assert c == rn32(Fraction(1, 448))
    vals = (np.arange(0, 0x7f80, dtype=np.uint32) << 16).view(np.float32)
    wrong_plain = wrong_corrected = 0
    for v in vals:
        a = Fraction(float(v))
        want = rn32(a / 448)
        q = rn32(a * c)
        r = rn32(a - q * 448)      # one fused multiply-add: exact, then rounded
        q1 = rn32(r * c + q)       # fused multiply-add
        wrong_plain += q != want
        wrong_corrected += q1 != want
    assert wrong_corrected == 0
    assert wrong_plain > 10000     # the correction is what makes it exact


def test_bracket_encloses_the_quotient_with_a_one_ulp_reciprocal():
    rng = np.random.default_rng(1)
    lo_m, hi_m = Fraction(1) - Fraction(1, 2 ** 20), Fraction(1) + Fraction(1, 2 ** 20)
    for _ in range(3000):
        s = Fraction(float(np.float32(rng.uniform(1, 2) * 2.0 ** rng.integers(-125, 125))))
        x = Fraction(float(np.float32(rng.standard_normal() * 2.0 ** rng.integers(-30, 30))))
        for err in (-1, 1):
            inv = rn32(1 / s)
            inv = inv + err * (Fraction(2) ** (inv.numerator.bit_length()
                                                 - inv.denominator.bit_length() - 24))
            lo = rn32(x * rn32(inv * lo_m))
            hi = rn32(x * rn32(inv * hi_m))
            q = rn32(x / s)
            assert min(lo, hi) <= q <= max(lo, hi)
