"""Test-side packing helpers, written independently of the oracle.

The oracle reads a packed row one bit at a time.  These helpers use two other
formulations of the same layout (code i of a row sits at bits
[i*bits, (i+1)*bits) of the row's little-endian byte string):

* ``pack`` expands every code into its bits (numpy), lays the bits out
  LSB-first and lets ``np.packbits(bitorder="little")`` form the bytes;
* ``pack_digits`` reads packs as base-2**bits numbers (numpy integer shifts),
  used for the exhaustive unpack checks.

Tests build inputs from known codes with ``pack`` and compute expected values
from the codes directly, so a layout mistake in the oracle cannot cancel.

``exact_bf16`` rounds an exact rational (``fractions.Fraction``) to bf16, the
reference for every rounding-to-bf16 check.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np


def pack(codes: np.ndarray, bits: int) -> np.ndarray:
    """codes [N, K] (values < 2**bits) -> packed uint32 [N, K*bits/32]."""
    codes = np.asarray(codes, dtype=np.uint64)
    N, K = codes.shape
    assert (K * bits) % 32 == 0
    assert int(codes.max(initial=0)) < (1 << bits)
    shifts = np.arange(bits, dtype=np.uint64)
    bitplanes = ((codes[:, :, None] >> shifts) & 1).astype(np.uint8)  # [N,K,bits]
    flat = bitplanes.reshape(N, K * bits)
    by = np.packbits(flat, axis=1, bitorder="little")  # [N, K*bits/8]
    return np.ascontiguousarray(by).view("<u4").astype(np.uint32)


def digits(values: np.ndarray, bits: int, ncodes: int) -> np.ndarray:
    """Base-2**bits digits (least significant first) of integer packs."""
    v = np.asarray(values, dtype=np.uint64)
    mask = np.uint64((1 << bits) - 1)
    out = np.empty(v.shape + (ncodes,), dtype=np.uint8)
    for i in range(ncodes):
        out[..., i] = ((v >> np.uint64(bits * i)) & mask).astype(np.uint8)
    return out


def bf16_value(h) -> np.ndarray:
    """bf16 bit patterns -> float64 values (binary32 upper half, exact)."""
    h = np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16
    return h.view(np.float32).astype(np.float64)


def to_bf16_bits(v) -> np.ndarray:
    """float64 values that are exactly representable in bf16 -> bit patterns.
    Raises if a value is not exact (tests only pass exact dyadic values)."""
    f = np.asarray(v, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("value not exactly representable in bf16")
    if np.any(f.astype(np.float64) != np.asarray(v, dtype=np.float64)):
        raise ValueError("value not exactly representable in fp32")
    return (u >> 16).astype(np.uint16)


def exact_bf16(v: Fraction) -> int:
    """bf16 bit pattern nearest to the rational v (ties to even)."""
    if v == 0:
        return 0
    neg = v < 0
    a = -v if neg else v
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1                                  # now 2^e <= a < 2^(e+1)
    ue = max(e - 7, -133)                       # 8 significant bits
    n = round(a / Fraction(2) ** ue)            # Fraction rounds half to even
    r = n * Fraction(2) ** ue
    if r >= Fraction(2) ** 128:
        return 0xff80 if neg else 0x7f80
    if r == 0:
        return 0x8000 if neg else 0
    u = int(np.array([float(r)], dtype=np.float32).view(np.uint32)[0])
    assert u & 0xffff == 0
    return (u >> 16) | (0x8000 if neg else 0)
