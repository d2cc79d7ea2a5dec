"""Pins of the oracle's producer side (affine_quantize, affine_dequantize to
bf16 and the bf16 rounding under both) against facts fixed outside it.

* bf16 rounding and dequantization: exact rational arithmetic (Python
  ``fractions``), including exact ties, the sticky case where a tiny bias
  breaks a tie, bf16 subnormals and overflow.
* The quantizer: groups worked out by hand from the pages' rules
  (``tests/golden/quantize.txt``), which separate every choice the rules make
  (the edge's side, halves away from zero, w_max starting at 0, w_min not,
  binary32 decisions, the clamp, the 1e-7 floor, the snap to edge/q0); and
  properties of any output: the edge is code 0 and is the bias, codes are
  monotone in the weight, each group is quantized on its own, and the
  reconstruction through the (separately pinned) fp64 dequantizer stays
  within the rounding bound.
"""
from fractions import Fraction
import os

import numpy as np
import pytest

import oracle
from tests._codes import bf16_value, exact_bf16 as _exact_bf16, pack, to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
ALL_BITS = (2, 3, 4, 5, 6, 8)


# --------------------------------------------------------------------------
# bf16 rounding
# --------------------------------------------------------------------------

def _bf16_fraction(h: int) -> Fraction:
    return Fraction(float(bf16_value(np.uint16(h))))


def test_bf16_round_random_doubles():
    rng = np.random.default_rng(11)
    for _ in range(3000):
        e = int(rng.integers(-140, 130))
        v = float(np.ldexp(rng.uniform(-1.0, 1.0), e))
        assert oracle.bf16_round(v) == _exact_bf16(Fraction(v)), v


def test_bf16_round_ties_and_sticky():
    for m in range(128, 256):               # every 8-bit significand
        for e in (-140, -134, -126, -20, 0, 7, 127):
            mid = Fraction(2 * m + 1, 2) * Fraction(2) ** (e - 7)   # a tie
            hi = float(mid)
            if Fraction(hi) != mid:
                continue                     # not a double (tiny exponents)
            assert oracle.bf16_round(hi) == _exact_bf16(mid)
            tiny = float(mid) * 2.0 ** -60
            for lo in (tiny, -tiny):
                want = _exact_bf16(mid + Fraction(lo))
                assert oracle.bf16_round(hi, lo) == want, (m, e, lo)


def test_bf16_round_overflow_and_zero():
    big = Fraction(2) ** 128 - Fraction(2) ** (127 - 8)   # tie above the max
    assert oracle.bf16_round(float(big)) == 0x7f80 == _exact_bf16(big)
    below = Fraction(2) ** 128 - Fraction(2) ** (127 - 7) - Fraction(2) ** 100
    assert oracle.bf16_round(float(below)) == 0x7f7f
    assert oracle.bf16_round(-0.0) == 0x8000 and oracle.bf16_round(0.0) == 0
    assert oracle.bf16_round(2.0 ** -134) == 0            # half of the spacing
    assert oracle.bf16_round(-(2.0 ** -134) * 1.5) == 0x8001


# --------------------------------------------------------------------------
# Dequantize to bf16
# --------------------------------------------------------------------------

def _random_bf16(rng, shape, emin, emax):
    m = rng.integers(128, 256, size=shape)
    e = rng.integers(emin, emax, size=shape)
    sgn = rng.choice([-1.0, 1.0], size=shape)
    return to_bf16_bits(sgn * np.ldexp(m.astype(np.float64), e - 7))


@pytest.mark.parametrize("bits", ALL_BITS)
def test_dequantize_bf16_exact_rationals(bits):
    rng = np.random.default_rng(100 + bits)
    N, K, gs = 4, 128, 32
    codes = rng.integers(0, 1 << bits, size=(N, K))
    # scale and bias exponents far apart too, so the sum is not exact in fp64
    s = _random_bf16(rng, (N, K // gs), -60, 20)
    b = _random_bf16(rng, (N, K // gs), -120, 60)
    out = oracle.dequantize_bf16(pack(codes, bits), s, b, N, K, bits, gs)
    for n in range(N):
        for k in range(K):
            g = k // gs
            v = _bf16_fraction(s[n, g]) * int(codes[n, k]) + _bf16_fraction(b[n, g])
            assert out[n, k] == _exact_bf16(v), (n, k)


def test_dequantize_bf16_tie_broken_by_tiny_bias():
    # scale 129/128 times code 3 is 387/128, halfway between two bf16 values;
    # a bias of +-2^-60 decides the direction, a zero bias ties to even
    bits, gs, K = 2, 32, 32
    codes = np.full((3, K), 3)
    s = to_bf16_bits(np.full((3, 1), 129 / 128))
    b = to_bf16_bits(np.array([[2.0 ** -60], [-(2.0 ** -60)], [0.0]]))
    out = oracle.dequantize_bf16(pack(codes, bits), s, b, 3, K, bits, gs)
    up, down = to_bf16_bits([3.03125])[0], to_bf16_bits([3.015625])[0]
    assert (out[0] == up).all() and (out[1] == down).all()
    assert (out[2] == up).all()              # 3.03125 has the even significand


@pytest.mark.parametrize("bits", (3, 4, 8))
def test_dequantize_bf16_is_the_rounded_fp64_dequant(bits):
    # where the fp64 w_hat is exact (close exponents), rounding it once gives
    # the same bf16 values
    rng = np.random.default_rng(7 + bits)
    N, K, gs = 8, 256, 64
    codes = rng.integers(0, 1 << bits, size=(N, K))
    s = _random_bf16(rng, (N, K // gs), -8, -2)
    b = _random_bf16(rng, (N, K // gs), -3, 2)
    w = pack(codes, bits)
    hat = oracle.dequant(w, s, b, N, K, bits, gs)
    want = np.array([[_exact_bf16(Fraction(v)) for v in row] for row in hat])
    assert (oracle.dequantize_bf16(w, s, b, N, K, bits, gs) == want).all()


# --------------------------------------------------------------------------
# Quantize
# --------------------------------------------------------------------------

def _golden_groups():
    rows = []
    with open(os.path.join(GOLDEN, "quantize.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            c = [x.strip() for x in line.split("|")]
            rows.append(dict(bits=int(c[0]), gs=int(c[1]),
                             lead=[float(v) for v in c[2].split()],
                             fill=float(c[3]), scale=int(c[4], 16),
                             bias=int(c[5], 16),
                             lead_codes=[int(v) for v in c[6].split()],
                             fill_code=int(c[7])))
    return rows


def test_quantize_golden_groups():
    cases = _golden_groups()
    assert len(cases) == 12
    for c in cases:
        gs, bits = c["gs"], c["bits"]
        vals = c["lead"] + [c["fill"]] * (gs - len(c["lead"]))
        codes = c["lead_codes"] + [c["fill_code"]] * (gs - len(c["lead"]))
        # two rows, the second with the group reversed: rows are independent
        w = to_bf16_bits(np.array([vals, vals[::-1]]))
        wq, s, b = oracle.affine_quantize(w, 2, gs, bits, gs)
        assert (s == c["scale"]).all(), (c, s)
        assert (b == c["bias"]).all(), (c, b)
        assert (wq == pack(np.array([codes, codes[::-1]]), bits)).all(), c


def _groups(a, gs):
    N, K = a.shape
    return a.reshape(N, K // gs, gs)


def _weights(rng, N, K, kind):
    if kind == "normal":
        v = rng.normal(0.0, 0.02, size=(N, K))
    elif kind == "positive":
        v = np.abs(rng.normal(0.5, 0.2, size=(N, K))) + 0.01
    else:                                       # heavy tails and exact zeros
        v = rng.standard_t(2.0, size=(N, K)) * 0.05
        v[rng.random(size=(N, K)) < 0.1] = 0.0
    v32 = v.astype(np.float32).view(np.uint32)
    return (v32 >> 16).astype(np.uint16)       # truncate to bf16 bit patterns


@pytest.mark.parametrize("bits", ALL_BITS)
@pytest.mark.parametrize("gs", [32, 64, 128])
@pytest.mark.parametrize("kind", ["normal", "positive", "heavy"])
def test_quantize_properties(bits, gs, kind):
    seed = 1000 * bits + gs + {"normal": 0, "positive": 1, "heavy": 2}[kind]
    rng = np.random.default_rng(seed)
    N, K = 6, 512
    w = _weights(rng, N, K, kind)
    wq, s, b = oracle.affine_quantize(w, N, K, bits, gs)
    q = _groups(oracle.unpack(wq, N, K, bits).astype(np.int64), gs)
    wv = _groups(bf16_value(w), gs)
    sv, bv = bf16_value(s), bf16_value(b)
    n_bins = (1 << bits) - 1
    assert q.max() <= n_bins
    for n in range(N):
        for g in range(K // gs):
            x, c = wv[n, g], q[n, g]
            lo, hi = x.min(), max(x.max(), 0.0)   # w_max starts at 0
            edge = lo if abs(lo) > abs(hi) else hi
            # the bias is the larger-magnitude edge (kept exactly), coded 0
            assert bv[n, g] == edge
            assert (c[x == edge] == 0).all()
            # codes are monotone in the weight, upward for a positive scale
            order = np.argsort(x, kind="stable")
            d = np.diff(c[order])
            assert (d >= 0).all() if sv[n, g] > 0 else (d <= 0).all()
    # reconstruction through the fp64 dequantizer: within one code step at the
    # clamped far edge (half a step elsewhere) plus the scale's bf16 rounding
    hat = _groups(oracle.dequant(wq, s, b, N, K, bits, gs), gs)
    step = np.abs(sv)[:, :, None]
    bound = (1.0001 + n_bins * 2.0 ** -8) * step / (1 - 2.0 ** -8)
    assert (np.abs(hat - wv) <= bound).all()


def test_quantize_each_group_on_its_own():
    rng = np.random.default_rng(5)
    N, K, bits, gs = 3, 256, 5, 64
    w = _weights(rng, N, K, "heavy")
    wq, s, b = oracle.affine_quantize(w, N, K, bits, gs)
    codes = oracle.unpack(wq, N, K, bits)
    for n in range(N):
        for g in range(K // gs):
            one = np.ascontiguousarray(w[n:n + 1, g * gs:(g + 1) * gs])
            wq1, s1, b1 = oracle.affine_quantize(one, 1, gs, bits, gs)
            assert s1[0, 0] == s[n, g] and b1[0, 0] == b[n, g]
            assert (oracle.unpack(wq1, 1, gs, bits)[0] ==
                    codes[n, g * gs:(g + 1) * gs]).all()


def test_quantize_then_dequantize_keeps_zero_near_zero():
    # zero is code -q0 (|q0| <= n_bins) because scale = edge / q0 in binary32;
    # after the scale's bf16 rounding (at most 2^-8 relative) it decodes to
    # within |q0| * 2^-8 * |scale| of 0, plus the binary32 quotient's rounding
    rng = np.random.default_rng(9)
    N, K, bits, gs = 4, 256, 4, 32
    w = _weights(rng, N, K, "heavy")
    wq, s, b = oracle.affine_quantize(w, N, K, bits, gs)
    hat = _groups(oracle.dequant(wq, s, b, N, K, bits, gs), gs)
    wv = _groups(bf16_value(w), gs)
    sv = np.abs(bf16_value(s))[:, :, None]
    ev = np.abs(bf16_value(b))[:, :, None]
    zeros = wv == 0.0
    assert zeros.sum() > 10
    lim = (1 << bits) * 2.0 ** -8 * sv * (1 + 2.0 ** -7) + 2.0 ** -23 * ev
    assert (np.abs(hat[zeros]) <= np.broadcast_to(lim, hat.shape)[zeros]).all()


def test_quantize_rejects_bad_shapes():
    w = np.zeros((2, 64), dtype=np.uint16)
    with pytest.raises(ValueError):
        oracle.affine_quantize(w, 2, 64, 7, 32)      # bits
    with pytest.raises(ValueError):
        oracle.affine_quantize(w, 2, 64, 4, 48)      # group size
    with pytest.raises(ValueError):
        oracle.affine_quantize(w[:, :48], 2, 48, 4, 32)   # K % gs


# --------------------------------------------------------------------------
# Generated groups (hypothesis): zeros, subnormals, tiny spans, large values
# --------------------------------------------------------------------------

from hypothesis import given, settings, strategies as st  # noqa: E402

_BF16_FINITE = st.integers(0, 0xFFFF).filter(lambda h: (h & 0x7F80) != 0x7F80)


def _small_magnitude(h):
    # finite and below 2^100 in magnitude (far inside the definition's range)
    return ((h >> 7) & 0xFF) < 127 + 100


@settings(max_examples=300, deadline=None)
@given(bits=st.sampled_from(ALL_BITS),
       vals=st.lists(_BF16_FINITE.filter(_small_magnitude), min_size=32, max_size=32),
       base=_BF16_FINITE.filter(_small_magnitude),
       spread=st.integers(0, 3))
def test_quantize_generated_groups(bits, vals, base, spread):
    gs = 32
    if spread == 0:      # a near-constant group: every value within a few ulps of base
        vals = [(base & 0xFF80) | (v & 0x3) for v in vals]
    w = np.array([vals], dtype=np.uint16)
    wq, s, b = oracle.affine_quantize(w, 1, gs, bits, gs)
    q = oracle.unpack(wq, 1, gs, bits)[0].astype(np.int64)
    x = bf16_value(w)[0]
    n_bins = (1 << bits) - 1
    lo, hi = x.min(), max(x.max(), 0.0)
    edge = lo if abs(lo) > abs(hi) else hi
    bias = bf16_value(b)[0, 0]
    scale = bf16_value(s)[0, 0]
    assert q.max() <= n_bins
    assert bias == edge or bias == 0.0
    if bias == 0.0 and edge != 0.0:
        assert (q == 0).all()            # q0 rounded to 0: every code is 0
    else:
        assert (q[x == edge] == 0).all()
    order = np.argsort(x, kind="stable")
    d = np.diff(q[order])
    assert (d >= 0).all() if scale > 0 else (d <= 0).all()
