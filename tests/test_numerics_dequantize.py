"""CPU checks of the dequantize kernel's arithmetic.

The kernel forms each output with one bf16 fused multiply-add,
bf16(scale * q + bias) with a single rounding (nearest, ties to even), which
is the definition of the dequantized weight itself.  Its only other step is
turning a code q into an exact bf16 operand:
  * codes below 128 (2- to 6-bit): the bits 0x4300 | q are the bf16 number
    128 + q, and subtracting 128 is exact;
  * 8-bit codes: the binary32 bits 0x4b000000 | q are 2^23 + q, subtracting
    2^23 is exact, and the integer (below 256) converts to bf16 exactly.
These tests check both encodings for every code with plain bit arithmetic
and exact rationals, and that the exact value rounded once to bf16 is what
the oracle's dequantizer returns (so a kernel computing it matches the
oracle bit for bit).
"""
from fractions import Fraction

import numpy as np

import oracle
from tests._codes import exact_bf16 as _exact_bf16


def _bf16_value(bits: int) -> Fraction:
    return Fraction(float(np.array([bits << 16], dtype=np.uint32).view(np.float32)[0]))


def test_small_codes_encode_exactly_in_bf16():
    for q in range(128):
        assert _bf16_value(0x4300 | q) == 128 + q
        # the difference with 128 is exactly q, so the subtraction is exact
        assert _exact_bf16(_bf16_value(0x4300 | q) - 128) == _exact_bf16(Fraction(q))
    assert _bf16_value(0x4300) == 128


def test_eight_bit_codes_encode_exactly_via_binary32():
    for q in range(256):
        f = np.array([0x4B000000 | q], dtype=np.uint32).view(np.float32)[0]
        v = np.float32(f - np.float32(8388608.0))
        assert Fraction(float(v)) == q
        # an integer below 256 has at most 8 significant bits: exact in bf16
        assert _bf16_value(_exact_bf16(Fraction(q))) == q


def test_single_rounding_is_the_oracles_dequantized_value():
    # the oracle's dequantizer rounds the exact scale * q + bias once to bf16;
    # so does one bf16 fused multiply-add, whatever the inputs
    rng = np.random.default_rng(17)
    N, K, bits, gs = 4, 64, 4, 32
    G = K // gs
    codes = rng.integers(0, 1 << bits, size=(N, K))
    sb = rng.integers(0, 1 << 16, size=(N, G)).astype(np.uint16)
    bb = rng.integers(0, 1 << 16, size=(N, G)).astype(np.uint16)
    # keep finite, moderate magnitudes (exponent field 100..150)
    sb = (sb & 0x807F) | (rng.integers(100, 150, size=(N, G)).astype(np.uint16) << 7)
    bb = (bb & 0x807F) | (rng.integers(100, 150, size=(N, G)).astype(np.uint16) << 7)
    from tests._codes import pack
    w = pack(codes, bits)
    got = oracle.dequantize_bf16(w, sb, bb, N, K, bits, gs)
    for n in range(N):
        for k in range(K):
            g = k // gs
            exact = _bf16_value(int(sb[n, g])) * int(codes[n, k]) + _bf16_value(int(bb[n, g]))
            assert int(got[n, k]) == _exact_bf16(exact), (n, k)
