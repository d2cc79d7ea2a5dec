"""CPU model of the streaming kernel's integer path (2/4/8-bit codes),
checked against the oracle.

Per unit of 32 consecutive activations (always inside one group): the unit's
largest magnitude sets a power of two 2^s that brings it just below 2^22;
X = rint(x * 2^s) is split into three byte digits (two unsigned, the top one
signed); each digit's dot product with the codes is an exact integer; the
three are combined in fp32, scaled by the group's scale, the bias term uses
the unit's fp32 activation sum, 2^-s is applied, and the units' partials are
added in fp32 before one bf16 rounding.  These are the kernel's roundings,
applied here with numpy only.  The test asserts the acceptance bound against
the fp64 oracle on the decode distribution and on a unit whose largest value
dwarfs the rest (the case that rules out two-byte digits), and shows that
two digits would fail there, so the check is not vacuous.
"""
import numpy as np
import pytest
import torch

from affine_group_quantized_b200 import synth
import oracle
from tests import _codes
from tests._parity import ABS_COEF, REL_TOL

f32 = np.float32


def _bf16_round(v):
    return torch.from_numpy(np.asarray(v, np.float32)).to(torch.bfloat16).to(
        torch.float64).numpy()


def _model(x_bits, codes, s_bits, b_bits, gs, ndigits=3):
    x = synth.bits_to_float(x_bits).astype(np.float32)[0]      # one activation row
    s = synth.bits_to_float(s_bits).astype(np.float32)
    b = synth.bits_to_float(b_bits).astype(np.float32)
    N, K = codes.shape
    top = 8 * ndigits - 2                  # magnitude bits of the fixed point
    y = np.zeros(N, np.float32)
    for u in range(K // 32):
        xu = x[32 * u:32 * u + 32]
        mx = float(np.max(np.abs(xu)))
        eb = int(np.frexp(np.float32(mx))[1]) + 126 if mx > 0 else 0  # mx < 2^(eb-126)
        sh = int(np.clip(top + 126 - eb, -126, 126))
        X = np.rint(xu.astype(np.float64) * 2.0 ** sh).astype(np.int64)
        assert np.all(np.abs(X) <= 2 ** top)
        # byte digits, top one signed: X = d[-1] * 256^(n-1) + ... + d[0]
        d, rest = [], X.copy()
        for i in range(ndigits - 1):
            d.append(rest & 0xFF)
            rest = rest >> 8
        d.append(rest)
        q = codes[:, 32 * u:32 * u + 32].astype(np.int64)
        sums = [q @ di for di in d]        # exact integers
        # fp32 FMAs from the low digit up, one rounding each:
        # r = d2 * 65536 + (d1 * 256 + d0)
        r = sums[0].astype(np.float32)
        for i in range(1, ndigits):
            r = f32(sums[i].astype(np.float64) * 256.0 ** i + r.astype(np.float64))
        vs = f32(0.0)
        for v in xu:                       # fp32 activation sum
            vs = f32(vs + v)
        vs = f32(vs * f32(2.0 ** sh))
        g = (32 * u) // gs
        part = f32(b[:, g].astype(np.float64) * float(vs) +
                   f32(s[:, g] * r).astype(np.float64))
        y = f32(y + f32(part * f32(2.0 ** -sh)))
    return _bf16_round(y.astype(np.float64))[None, :]


def _inputs(N, K, bits, gs, seed):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 1 << bits, size=(N, K), dtype=np.int64)
    x, _, s, b = synth.qmv_inputs(1, N, K, bits, gs, seed=seed)
    return x, codes, _codes.pack(codes, bits), s, b


def _ratio(y, y_ref, a_ref):
    bound = REL_TOL * np.abs(y_ref) + ABS_COEF * a_ref
    return np.max(np.abs(y - y_ref) / bound)


@pytest.mark.parametrize("bits, gs", [(4, 64), (2, 32), (8, 128)])
def test_integer_path_roundings_meet_the_bound(bits, gs):
    N, K = 32, 2048
    x, codes, w, s, b = _inputs(N, K, bits, gs, seed=500 + bits + gs)
    y_ref, a_ref = oracle.qmv(x, w, s, b, 1, N, K, bits, gs)
    assert _ratio(_model(x, codes, s, b, gs), y_ref, a_ref) <= 1.0


def _outlier_case():
    # in every unit one activation is about 2^10 times the others and meets
    # a zero weight: the rows' sums come from the small activations alone
    N, K, bits, gs = 16, 256, 4, 32
    x, codes, w, s, b = _inputs(N, K, bits, gs, seed=777)
    xf = synth.bits_to_float(x).astype(np.float32).copy()
    xf[0, ::32] = np.float32(2.0 ** 10)
    x = synth.bf16_bits(torch.from_numpy(xf))
    codes = codes.copy()
    codes[:, ::32] = 0
    # w_hat = scale * 0 + bias vanishes at the outliers only with a zero bias
    b = synth.bf16_bits(torch.zeros(b.shape, dtype=torch.float32))
    w = _codes.pack(codes, bits)
    return x, codes, w, s, b, N, K, bits, gs


def test_integer_path_outlier_unit_meets_the_bound():
    x, codes, w, s, b, N, K, bits, gs = _outlier_case()
    y_ref, a_ref = oracle.qmv(x, w, s, b, 1, N, K, bits, gs)
    assert _ratio(_model(x, codes, s, b, gs), y_ref, a_ref) <= 1.0


def test_two_digit_fixed_point_would_fail_the_outlier_unit():
    x, codes, w, s, b, N, K, bits, gs = _outlier_case()
    y_ref, a_ref = oracle.qmv(x, w, s, b, 1, N, K, bits, gs)
    assert _ratio(_model(x, codes, s, b, gs, ndigits=2), y_ref, a_ref) > 1.0


# ---------------------------------------------------------------------------
# The decode kernel (one activation row, 2/4-bit codes, rows of a multiple of
# 2048 codes): each thread owns a 64-code span; one power of two per span
# (so the fixed point covers 64 activations); per group part of the span
# (one part, or two for group size 32) the digit sums are combined exactly
# (S0 + 256 S1 + 65536 S2 as two fp32 additions of exact terms), multiplied
# by the scale and added up over the parts; the bias term uses the part's
# fp32 activation sum; the span result is sr * 2^-s + bs; the spans of a row
# are added in fp32.
# ---------------------------------------------------------------------------

def _model_span(x_bits, codes, s_bits, b_bits, gs, ndigits=3, span=64):
    x = synth.bits_to_float(x_bits).astype(np.float32)[0]
    s = synth.bits_to_float(s_bits).astype(np.float32)
    b = synth.bits_to_float(b_bits).astype(np.float32)
    N, K = codes.shape
    top = 8 * ndigits - 2
    parts = 2 if gs == 32 else 1
    plen = span // parts
    y = np.zeros(N, np.float32)
    for t in range(K // span):
        xs = x[span * t:span * t + span]
        mx = float(np.max(np.abs(xs)))
        eb = int(np.frexp(np.float32(mx))[1]) + 126 if mx > 0 else 0
        sh = int(np.clip(top + 126 - eb, -126, 126))
        X = np.rint(xs.astype(np.float64) * 2.0 ** sh).astype(np.int64)
        assert np.all(np.abs(X) <= 2 ** top)
        d, rest = [], X.copy()
        for i in range(ndigits - 1):
            d.append(rest & 0xFF)
            rest = rest >> 8
        d.append(rest)
        sr = np.zeros(N, np.float32)
        bs = np.zeros(N, np.float32)
        for h in range(parts):
            lo, hi = span * t + plen * h, span * t + plen * (h + 1)
            q = codes[:, lo:hi].astype(np.int64)
            sums = [q @ di[plen * h:plen * (h + 1)] for di in d]   # exact integers
            r = (sums[0] * 1.0).astype(np.float32)
            for i in range(1, ndigits):
                r = f32(r.astype(np.float64) + sums[i].astype(np.float64) * 256.0 ** i)
            vs = f32(0.0)
            for v in x[lo:hi]:
                vs = f32(vs + v)
            g = lo // gs
            sr = f32(s[:, g].astype(np.float64) * r.astype(np.float64) + sr.astype(np.float64))
            bs = f32(b[:, g].astype(np.float64) * float(vs) + bs.astype(np.float64))
        part = f32(sr.astype(np.float64) * 2.0 ** -sh + bs.astype(np.float64))
        y = f32(y + part)
    return _bf16_round(y.astype(np.float64))[None, :]


@pytest.mark.parametrize("bits, gs", [(4, 64), (2, 32), (4, 128), (2, 64)])
def test_decode_span_roundings_meet_the_bound(bits, gs):
    N, K = 32, 2048
    x, codes, w, s, b = _inputs(N, K, bits, gs, seed=600 + bits + gs)
    y_ref, a_ref = oracle.qmv(x, w, s, b, 1, N, K, bits, gs)
    assert _ratio(_model_span(x, codes, s, b, gs), y_ref, a_ref) <= 1.0


def test_decode_span_outlier_meets_the_bound():
    x, codes, w, s, b, N, K, bits, gs = _outlier_case()
    y_ref, a_ref = oracle.qmv(x, w, s, b, 1, N, K, bits, gs)
    assert _ratio(_model_span(x, codes, s, b, gs), y_ref, a_ref) <= 1.0


def test_decode_span_two_digits_would_fail_the_outlier():
    x, codes, w, s, b, N, K, bits, gs = _outlier_case()
    y_ref, a_ref = oracle.qmv(x, w, s, b, 1, N, K, bits, gs)
    assert _ratio(_model_span(x, codes, s, b, gs, ndigits=2), y_ref, a_ref) > 1.0
