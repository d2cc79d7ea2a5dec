"""CPU model of the dequantize kernel's rounding, checked against exact
rational arithmetic.

The kernel forms r = scale * q + bias with one fused multiply-add (the
product is exact in binary32, so r is the exact sum rounded once to
binary32) and converts r to bf16 with round-to-nearest-even, except when r
lies exactly halfway between two bf16 values: then the two-sum error of the
addition says on which side the exact sum lies.  This test applies exactly
those steps with numpy and Python fractions (no GPU, no kernel code) and
asserts that the result is the exact sum rounded once to bf16, on random
inputs and on constructed ties; without the tie step some of those cases
round the wrong way, so the check is not vacuous.
"""
from fractions import Fraction

import numpy as np

from tests._codes import exact_bf16 as _exact_bf16


def _f32(x: Fraction) -> Fraction:
    # binary32 rounding of an exact value (via binary64, exact for these
    # inputs: a bf16 times a code below 256 plus a bf16 within 2^40 of it)
    d = float(x)
    assert Fraction(d) == x
    return Fraction(float(np.float32(d)))


def _bf16_rne_of_f32(r: Fraction) -> int:
    u = int(np.array([float(r)], dtype=np.float32).view(np.uint32)[0])
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) & 0xFFFF


def _model(s: Fraction, q: int, b: Fraction, tie_step=True) -> int:
    exact = s * q + b
    r = _f32(exact)
    u = int(np.array([float(r)], dtype=np.float32).view(np.uint32)[0])
    if tie_step and (u & 0xFFFF) == 0x8000 and exact != r:
        away = (exact > r) == (r > 0)
        return ((u >> 16) + (1 if away else 0)) & 0xFFFF
    return _bf16_rne_of_f32(r)


def _bf16(v) -> Fraction:
    return Fraction(float(v))


def test_model_rounds_like_the_exact_sum_on_random_inputs():
    rng = np.random.default_rng(17)
    for _ in range(4000):
        s = _bf16(np.ldexp(float(rng.integers(128, 256)) * rng.choice([-1, 1]),
                           int(rng.integers(-30, 10))))
        b = _bf16(np.ldexp(float(rng.integers(128, 256)) * rng.choice([-1, 1]),
                           int(rng.integers(-30, 10))))
        q = int(rng.integers(0, 256))
        assert _model(s, q, b) == _exact_bf16(s * q + b)


def test_model_on_binary32_ties():
    # s * q exactly halfway between two bf16 values, with a bias small
    # enough that binary32 rounds the sum back onto the halfway point
    cases = 0
    wrong_without = 0
    for m in range(129, 256, 2):                 # odd 8-bit significands
        s = Fraction(m, 128)
        for q in (3, 5, 7, 9, 129, 255):
            p = s * q
            for eb in (-40, -35, -30):
                for sign in (1, -1, 0):
                    b = Fraction(sign) * Fraction(2) ** eb
                    exact = p + b
                    if _f32(exact) != _f32(p):
                        continue
                    cases += 1
                    want = _exact_bf16(exact)
                    assert _model(s, q, b) == want
                    wrong_without += _model(s, q, b, tie_step=False) != want
    assert cases > 100 and wrong_without > 0
