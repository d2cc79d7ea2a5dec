"""CPU checks of the many-row tensor-core path's arithmetic (qmv_qmm.cu).

1. The natural-order unpack.  Each pair of consecutive codes becomes a bf16
   pair by byte permutes, a mask and the exponent of 128: 128 + 2^i q in each
   half, with 2^i q kept below the exponent field's lowest bit; one pair FMA
   with exact constants then gives q.  8-bit codes go through binary32 (2^23 +
   q, minus 2^23).  The test repeats the kernel's integer steps in Python
   (byte permute as the PTX prmt instruction defines it, default mode) for
   every byte value, reads the halves as bf16 numbers, applies the constants
   in exact rational arithmetic and checks that the result is the code: an
   exact result needs no rounding, so the hardware FMA returns it too.
2. The rounding model: W_hat = bf16(s q + b) once (the dequantized weight),
   x exact in bf16, products and sums in fp32, one bf16 rounding of y.  The
   model meets the acceptance bound against the fp64 oracle on the prefill
   input distribution and on extreme activations.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

from affine_group_quantized_b200 import synth
import oracle
from tests import _codes
from tests._parity import ABS_COEF, REL_TOL


def prmt(a: int, b: int, sel: int) -> int:
    src = [(a >> (8 * i)) & 0xFF for i in range(4)] + [(b >> (8 * i)) & 0xFF for i in range(4)]
    out = 0
    for i in range(4):
        out |= src[(sel >> (4 * i)) & 7] << (8 * i)
    return out


def bf16(bits16: int) -> Fraction:
    return Fraction(float(np.array([bits16 << 16], dtype=np.uint32).view(np.float32)[0]))


def halves(v: int):
    return bf16(v & 0xFFFF), bf16(v >> 16)


def _pair_fma(v: int, mul: int, add: int):
    lo, hi = halves(v)
    ml, mh = halves(mul)
    al, ah = halves(add)
    return lo * ml + al, hi * mh + ah


MAGIC = 0x43004300


def test_bf16_constants():
    assert halves(0x3E003F80) == (1, Fraction(1, 8))
    assert halves(0xC180C300) == (-128, -16)
    assert halves(0x3E803F80) == (1, Fraction(1, 4))
    assert halves(0xC200C300) == (-128, -32)
    assert halves(0x3D803E80) == (Fraction(1, 4), Fraction(1, 16))
    assert halves(0xC100C200) == (-32, -8)


def test_four_bit_pairs_are_exact_for_every_byte():
    rng = np.random.default_rng(5)
    for byte in range(256):
        for pr in range(4):
            # the byte at position pr of a word with random neighbours
            others = int(rng.integers(0, 1 << 32))
            w = (others & ~(0xFF << (8 * pr))) | (byte << (8 * pr))
            w1 = w >> 1
            sel = pr | (pr << 4) | ((4 + pr) << 8) | ((4 + pr) << 12)
            t = (prmt(w, w1, sel) & 0x0078000F) | MAGIC
            lo, hi = _pair_fma(t, 0x3E003F80, 0xC180C300)
            assert (lo, hi) == (byte & 15, byte >> 4), (byte, pr)


def test_two_bit_pairs_are_exact_for_every_byte():
    rng = np.random.default_rng(6)
    for byte in range(256):
        for pr in range(4):
            others = int(rng.integers(0, 1 << 32))
            w = (others & ~(0xFF << (8 * pr))) | (byte << (8 * pr))
            w2 = w >> 2
            sel = pr | (pr << 4) | (pr << 8) | (pr << 12)
            ta = (prmt(w, w, sel) & 0x000C0003) | MAGIC
            tb = (prmt(w2, w2, sel) & 0x0030000C) | MAGIC
            q = [(byte >> (2 * i)) & 3 for i in range(4)]
            assert _pair_fma(ta, 0x3E803F80, 0xC200C300) == (q[0], q[1]), (byte, pr)
            assert _pair_fma(tb, 0x3D803E80, 0xC100C200) == (q[2], q[3]), (byte, pr)


def test_eight_bit_codes_are_exact_via_binary32():
    for byte in range(256):
        for j in range(4):
            w = byte << (8 * j)
            f = prmt(w, 0x4B000000, 0x7440 | j)
            v = np.array([f], dtype=np.uint32).view(np.float32)[0]
            q = np.float32(v - np.float32(8388608.0))
            assert Fraction(float(q)) == byte
            # an integer below 256 has at most 8 significant bits: exact in bf16
            assert float(torch.tensor(float(q)).to(torch.bfloat16)) == byte


def test_halves_stay_below_the_exponent_field():
    # every masked field sits in mantissa bits 0..6 of its half, so the
    # exponent (bits 7..14) stays that of 128
    for mask in (0x0078000F, 0x000C0003, 0x0030000C):
        for half in (mask & 0xFFFF, mask >> 16):
            assert half < 0x80


def _model(x_bits, codes, s_bits, b_bits, gs):
    x = synth.bits_to_float(x_bits).astype(np.float64)
    s = synth.bits_to_float(s_bits).astype(np.float64)
    b = synth.bits_to_float(b_bits).astype(np.float64)
    g = np.arange(codes.shape[1]) // gs
    w_hat = s[:, g] * codes + b[:, g]
    wb = torch.from_numpy(w_hat).to(torch.bfloat16).to(torch.float32).numpy()
    acc = x.astype(np.float32) @ wb.T                       # fp32 products and sums
    return torch.from_numpy(acc).to(torch.bfloat16).to(torch.float64).numpy()


def _inputs(M, N, K, bits, gs, seed):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 1 << bits, size=(N, K), dtype=np.int64)
    w = _codes.pack(codes, bits)
    x, _, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=seed)
    return x, codes, w, s, b


def _check(y, y_ref, a_ref, what):
    err = np.abs(y - y_ref)
    bound = REL_TOL * np.abs(y_ref) + ABS_COEF * a_ref
    assert np.all(err <= bound), f"{what}: max err/bound {np.max(err / bound)}"


@pytest.mark.parametrize("bits, gs", [(4, 32), (4, 128), (8, 64), (2, 32)])
def test_bf16_operand_roundings_meet_the_bound(bits, gs):
    M, N, K = 32, 40, 4096
    x, codes, w, s, b = _inputs(M, N, K, bits, gs, seed=900 + bits + gs)
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs, nthreads=4)
    _check(_model(x, codes, s, b, gs), y_ref, a_ref, f"bits={bits} gs={gs}")


def test_bf16_operand_roundings_extreme_activations():
    M, N, K, bits, gs = 8, 40, 1024, 4, 32
    x, codes, w, s, b = _inputs(M, N, K, bits, gs, seed=921)
    s = s ^ np.where(np.arange(s.size).reshape(s.shape) % 3 == 0,
                     np.uint16(0x8000), np.uint16(0))
    xf = synth.bits_to_float(x).astype(np.float32).copy()
    xf[0, :256] *= np.float32(2.0 ** 40)
    xf[0, 256:512] *= np.float32(2.0 ** -40)
    xf[2, 512:544] = 0.0
    xf[3, :] *= np.float32(2.0 ** -60)
    x = synth.bf16_bits(torch.from_numpy(xf))
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs)
    _check(_model(x, codes, s, b, gs), y_ref, a_ref, "extreme activations")
