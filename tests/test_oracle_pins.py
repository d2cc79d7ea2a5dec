"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

None of these tests needs a GPU.  Each one checks the oracle against
something other than itself: hand-derived golden values, an independent
formulation of the bit layout, exact rational arithmetic on dyadic inputs, the
per-group identity, a library matmul, the odd part of silu, and the gather
routing definition.  A dropped term, a wrong sign, a swapped index or a
transposed operand in the oracle fails at least one of them.
"""
from fractions import Fraction
import os

import numpy as np
import pytest

import oracle
from tests._codes import bf16_value, digits, pack, to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
ALL_BITS = (2, 3, 4, 5, 6, 8)


def _rng(seed):
    return np.random.default_rng(seed)


def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append([c.strip() for c in line.split("|")])
    return rows


# --------------------------------------------------------------------------
# Scalars
# --------------------------------------------------------------------------

def test_bf16_widening_golden():
    for pat, val in _read_table("bf16.txt"):
        got = oracle.bf16_to_double(int(pat, 16))
        want = float(eval(val, {"__builtins__": {}}))  # "2**-133" style
        assert got == want, (pat, got, want)
        assert np.signbit(got) == np.signbit(want)


def test_silu_closed_forms():
    assert oracle.silu(0.0) == 0.0
    # silu(g) - silu(-g) = g*(sigmoid(g) + sigmoid(-g)) = g
    for g in (0.25, 1.0, 3.5, 10.0):
        assert abs((oracle.silu(g) - oracle.silu(-g)) - g) <= 1e-15 * max(1, g)
    # sigmoid(1) = e/(1+e)
    e = np.e
    assert abs(oracle.silu(1.0) - e / (1 + e)) < 1e-16
    # large positive -> identity, large negative -> 0
    assert abs(oracle.silu(40.0) - 40.0) < 1e-12
    assert abs(oracle.silu(-40.0)) < 1e-15


# --------------------------------------------------------------------------
# Layout: golden packs, exhaustive comparison with a digit-based unpacker
# --------------------------------------------------------------------------

def test_unpack_golden_fixtures():
    table = _read_table("packing.txt")
    assert {int(r[0]) for r in table} == set(ALL_BITS)
    for bits_s, hexbytes, codes_s, rep in table:
        bits = int(bits_s)
        pattern = bytes(int(h, 16) for h in hexbytes.split())
        codes = [int(c) for c in codes_s.split()]
        assert len(pattern) * 8 == bits * len(codes)
        row = pattern * int(rep)
        K = len(codes) * int(rep)
        w = np.frombuffer(row, dtype="<u4").astype(np.uint32).reshape(1, -1)
        got = oracle.unpack(w, 1, K, bits)[0]
        assert list(got) == codes * int(rep), (bits, hexbytes)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_unpack_every_byte_value(bits):
    # every byte value in every byte position of a word
    vals = np.arange(256, dtype=np.uint32)
    words = []
    for pos in range(4):
        words.append(vals << np.uint32(8 * pos))
    w = np.concatenate(words).reshape(1, -1)
    per_word = 32 // bits
    K = w.size * per_word
    got = oracle.unpack(w, 1, K, bits).reshape(-1, per_word)
    want = digits(w.reshape(-1), bits, per_word)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("bits,nbytes,ncodes", [(3, 3, 8), (6, 3, 4)])
def test_unpack_all_three_byte_packs(bits, nbytes, ncodes):
    # all 2**24 three-byte packs, laid out back to back in one row
    v = np.arange(1 << 24, dtype=np.uint32)
    by = np.stack([(v >> (8 * i)) & 0xFF for i in range(3)], axis=1).astype(np.uint8)
    row = by.reshape(-1)  # 3 * 2**24 bytes = a whole number of words
    w = row.view("<u4").reshape(1, -1)
    K = (1 << 24) * ncodes
    got = oracle.unpack(w, 1, K, bits).reshape(-1, ncodes)
    want = digits(v, bits, ncodes)
    assert np.array_equal(got, want)


def test_unpack_random_five_byte_packs():
    rng = _rng(5)
    n = 1 << 20
    v = rng.integers(0, 1 << 40, size=n, dtype=np.uint64)
    by = np.stack([(v >> np.uint64(8 * i)) & np.uint64(0xFF) for i in range(5)],
                  axis=1).astype(np.uint8)
    w = by.reshape(-1).view("<u4").reshape(1, -1)
    got = oracle.unpack(w, 1, n * 8, 5).reshape(-1, 8)
    assert np.array_equal(got, digits(v, 5, 8))


@pytest.mark.parametrize("bits", ALL_BITS)
def test_pack_unpack_roundtrip(bits):
    rng = _rng(bits)
    codes = rng.integers(0, 1 << bits, size=(7, 256), dtype=np.uint8)
    assert np.array_equal(oracle.unpack(pack(codes, bits), 7, 256, bits), codes)


def test_shape_rules():
    # K must be a positive multiple of group_size; bits and gs from the pages
    assert oracle.check_shape(8, 64, 4, 64)
    assert not oracle.check_shape(8, 96, 4, 64)
    assert not oracle.check_shape(8, 64, 7, 32)
    assert not oracle.check_shape(8, 64, 4, 16)
    assert not oracle.check_shape(8, 0, 4, 32)
    for bits in ALL_BITS:
        for gs in (32, 64, 128):
            assert oracle.check_shape(3, 2 * gs, bits, gs)


# --------------------------------------------------------------------------
# Arithmetic: exact brute force, group identity, library matmul
# --------------------------------------------------------------------------

def _dyadic(rng, shape, lo_exp, hi_exp, max_int=7):
    """Small signed integers times powers of two: exact in bf16."""
    m = rng.integers(-max_int, max_int + 1, size=shape)
    e = rng.integers(lo_exp, hi_exp + 1, size=shape)
    return m * np.power(2.0, e)


@pytest.mark.parametrize("bits", ALL_BITS)
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_qmv_exact_on_dyadic_inputs(bits, gs):
    rng = _rng(100 * bits + gs)
    for K in (gs, 2 * gs) if gs < 128 else (128,):
        M, N = 2, 5
        G = K // gs
        codes = rng.integers(0, 1 << bits, size=(N, K))
        s = _dyadic(rng, (N, G), -8, -4)
        b = _dyadic(rng, (N, G), -6, -2)
        x = _dyadic(rng, (M, K), -3, 1)
        w = pack(codes, bits)
        y, a = oracle.qmv(to_bf16_bits(x), w, to_bf16_bits(s), to_bf16_bits(b),
                          M, N, K, bits, gs)
        for m in range(M):
            for n in range(N):
                exact = Fraction(0)
                mag = Fraction(0)
                for k in range(K):
                    wh = Fraction(s[n, k // gs]) * int(codes[n, k]) + Fraction(b[n, k // gs])
                    t = Fraction(x[m, k]) * wh
                    exact += t
                    mag += abs(t)
                assert Fraction(y[m, n]) == exact
                assert Fraction(a[m, n]) == mag


def _realistic(bits, gs, M, N, K, seed, negative_scales=False):
    rng = _rng(seed)
    codes = rng.integers(0, 1 << bits, size=(N, K))
    G = K // gs
    s = rng.uniform(0.005, 0.02, size=(N, G))
    if negative_scales:
        s *= rng.choice([-1.0, 1.0], size=(N, G))
    s_bits = to_bf16_bits(bf16_value(_round_bf16(s)))
    b_bits = _round_bf16(-(2 ** bits / 2) * bf16_value(s_bits)
                         + rng.uniform(-1e-3, 1e-3, size=(N, G)))
    x_bits = _round_bf16(rng.standard_normal((M, K)))
    return codes, s_bits, b_bits, x_bits


def _round_bf16(v):
    import torch
    t = torch.from_numpy(np.asarray(v, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


@pytest.mark.parametrize("bits", ALL_BITS)
@pytest.mark.parametrize("gs", [32, 128])
def test_qmv_group_sum_identity(bits, gs):
    # y = sum_g scale_g * sum_{k in g} x_k q_k + bias_g * sum_{k in g} x_k
    M, N, K = 3, 9, 512
    codes, s_bits, b_bits, x_bits = _realistic(bits, gs, M, N, K, 7 + bits,
                                               negative_scales=True)
    y, _ = oracle.qmv(x_bits, pack(codes, bits), s_bits, b_bits, M, N, K, bits, gs)
    x = bf16_value(x_bits)
    s = bf16_value(s_bits)
    b = bf16_value(b_bits)
    G = K // gs
    xg = x.reshape(M, G, gs)
    qg = codes.reshape(N, G, gs).astype(np.float64)
    dot_xq = np.einsum("mgk,ngk->mng", xg, qg)          # sum_k x q per group
    sum_x = xg.sum(axis=2)                              # sum_k x per group
    want = (s[None] * dot_xq).sum(-1) + (b[None] * sum_x[:, None, :]).sum(-1)
    assert np.allclose(y, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


@pytest.mark.parametrize("bits", ALL_BITS)
def test_qmv_matches_library_matmul(bits):
    gs = 64
    M, N, K = 4, 33, 384
    codes, s_bits, b_bits, x_bits = _realistic(bits, gs, M, N, K, 31 + bits)
    w = pack(codes, bits)
    y, a = oracle.qmv(x_bits, w, s_bits, b_bits, M, N, K, bits, gs)
    s = np.repeat(bf16_value(s_bits), gs, axis=1)
    b = np.repeat(bf16_value(b_bits), gs, axis=1)
    w_hat = s * codes + b
    x = bf16_value(x_bits)
    want = np.matmul(x, w_hat.T)
    assert np.allclose(y, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    assert np.allclose(a, np.abs(x)[:, None, :].__mul__(np.abs(w_hat)[None]).sum(-1),
                       rtol=1e-12)
    # the dequantized matrix itself
    assert np.array_equal(oracle.dequant(w, s_bits, b_bits, N, K, bits, gs), w_hat)


def test_qmv_rows_subset_and_threads():
    bits, gs, M, N, K = 4, 64, 2, 40, 256
    codes, s_bits, b_bits, x_bits = _realistic(bits, gs, M, N, K, 3)
    w = pack(codes, bits)
    y1, a1 = oracle.qmv(x_bits, w, s_bits, b_bits, M, N, K, bits, gs)
    y4, a4 = oracle.qmv(x_bits, w, s_bits, b_bits, M, N, K, bits, gs, nthreads=4)
    assert np.array_equal(y1, y4) and np.array_equal(a1, a4)
    rows = np.array([39, 0, 17, 17, 5], dtype=np.int32)
    ys, _ = oracle.qmv(x_bits, w, s_bits, b_bits, M, N, K, bits, gs, rows=rows)
    assert np.array_equal(ys, y1[:, rows])


def test_qmv_detects_transposed_or_shifted_layout():
    # guards against reading row n+1, or group g+1, by accident
    bits, gs, M, N, K = 4, 32, 1, 6, 128
    codes, s_bits, b_bits, x_bits = _realistic(bits, gs, M, N, K, 11)
    y, _ = oracle.qmv(x_bits, pack(codes, bits), s_bits, b_bits, M, N, K, bits, gs)
    x = bf16_value(x_bits)[0]
    s = bf16_value(s_bits)
    b = bf16_value(b_bits)
    for n in range(N):
        want = sum(x[k] * (s[n, k // gs] * codes[n, k] + b[n, k // gs])
                   for k in range(K))
        assert abs(y[0, n] - want) <= 1e-12 * max(1.0, abs(want))


# --------------------------------------------------------------------------
# Fused variants
# --------------------------------------------------------------------------

def test_gate_up_is_two_matvecs():
    bits, gs, M, N, K = 8, 64, 2, 24, 256
    cg, sg, bg, x_bits = _realistic(bits, gs, M, N, K, 21)
    cu, su, bu, _ = _realistic(bits, gs, M, N, K, 22)
    (yg, ag), (yu, au) = oracle.gate_up(x_bits, pack(cg, bits), sg, bg,
                                        pack(cu, bits), su, bu, M, N, K, bits, gs)
    x = bf16_value(x_bits)
    for codes, s_bits, b_bits, y in ((cg, sg, bg, yg), (cu, su, bu, yu)):
        w_hat = (np.repeat(bf16_value(s_bits), gs, 1) * codes
                 + np.repeat(bf16_value(b_bits), gs, 1))
        want = x @ w_hat.T
        assert np.allclose(y, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    assert not np.allclose(yg, yu)


def test_silu_gate_resid_pins():
    bits, gs, M, N, K = 8, 64, 2, 20, 256
    codes, s_bits, b_bits, g_bits = _realistic(bits, gs, M, N, K, 41)
    u_bits = _round_bf16(_rng(42).standard_normal((M, K)))
    r_bits = _round_bf16(_rng(43).standard_normal((M, N)))
    w = pack(codes, bits)
    w_hat = (np.repeat(bf16_value(s_bits), gs, 1) * codes
             + np.repeat(bf16_value(b_bits), gs, 1))
    g = bf16_value(g_bits)
    u = bf16_value(u_bits)
    # odd part: y(g) - y(-g) = W_hat @ (g * u)   since silu(g) - silu(-g) = g
    neg_g_bits = g_bits ^ np.uint16(0x8000)
    y_pos, _ = oracle.silu_gate_resid(g_bits, u_bits, None, w, s_bits, b_bits,
                                      M, N, K, bits, gs)
    y_neg, _ = oracle.silu_gate_resid(neg_g_bits, u_bits, None, w, s_bits, b_bits,
                                      M, N, K, bits, gs)
    want = (g * u) @ w_hat.T
    assert np.allclose(y_pos - y_neg, want, rtol=1e-10,
                       atol=1e-12 * np.abs(want).max())
    # even part: y(g) + y(-g) = W_hat @ (|g| * (sigmoid(g) - sigmoid(-g)) ... )
    # and gate == 0 gives exactly the residual
    zeros = np.zeros((M, K), dtype=np.uint16)
    y0, a0 = oracle.silu_gate_resid(zeros, u_bits, r_bits, w, s_bits, b_bits,
                                    M, N, K, bits, gs)
    assert np.array_equal(y0, bf16_value(r_bits)) and not a0.any()
    # residual adds exactly
    y_r, _ = oracle.silu_gate_resid(g_bits, u_bits, r_bits, w, s_bits, b_bits,
                                    M, N, K, bits, gs)
    assert np.array_equal(y_r, y_pos + bf16_value(r_bits))
    # composition with a dense matmul (silu written with numpy)
    v = g / (1.0 + np.exp(-g)) * u
    want = v @ w_hat.T
    assert np.allclose(y_pos, want, rtol=1e-10, atol=1e-12 * np.abs(want).max())
    # row subset
    rows = np.array([3, 19, 0], dtype=np.int32)
    ys, _ = oracle.silu_gate_resid(g_bits, u_bits, r_bits, w, s_bits, b_bits,
                                   M, N, K, bits, gs, rows=rows)
    assert np.array_equal(ys, y_r[:, rows])


def test_gather_routing():
    bits, gs, E, N, K, T = 4, 64, 6, 16, 128, 5
    rng = _rng(77)
    codes = rng.integers(0, 1 << bits, size=(E * N, K))
    s = rng.uniform(0.005, 0.02, size=(E * N, K // gs))
    s_bits = _round_bf16(s)
    # distinct bias per expert so a mis-routed row is far off
    b = -8 * bf16_value(s_bits) + np.repeat(np.arange(E), N)[:, None] * 0.25
    b_bits = _round_bf16(b)
    x_bits = _round_bf16(rng.standard_normal((T, K)))
    w = pack(codes, bits)
    lhs = np.array([0, 0, 1, 4, 2, 3, 3, 1], dtype=np.uint32)
    rhs = np.array([5, 1, 1, 0, 2, 5, 4, 3], dtype=np.uint32)
    P = len(lhs)
    y, a, valid = oracle.gather(x_bits, w, s_bits, b_bits, lhs, rhs, P, T, E, N, K,
                                bits, gs)
    assert valid.all()
    w_hat = (np.repeat(bf16_value(s_bits), gs, 1) * codes
             + np.repeat(bf16_value(b_bits), gs, 1)).reshape(E, N, K)
    x = bf16_value(x_bits)
    for p in range(P):
        want = w_hat[rhs[p]] @ x[lhs[p]]
        assert np.allclose(y[p], want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    # permuting pairs permutes output rows exactly
    perm = rng.permutation(P)
    y2, _, _ = oracle.gather(x_bits, w, s_bits, b_bits, lhs[perm], rhs[perm], P, T,
                             E, N, K, bits, gs)
    assert np.array_equal(y2, y[perm])
    # lhs == None -> pair p reads x row p
    y3, _, _ = oracle.gather(x_bits, w, s_bits, b_bits, None, rhs[:T], T, T, E, N,
                             K, bits, gs)
    for p in range(T):
        assert np.array_equal(y3[p], oracle.qmv(x_bits[p:p + 1],
                                                w.reshape(E, N, -1)[rhs[p]],
                                                s_bits.reshape(E, N, -1)[rhs[p]],
                                                b_bits.reshape(E, N, -1)[rhs[p]],
                                                1, N, K, bits, gs)[0][0])
    # out-of-range indices are reported and not computed
    bad_rhs = rhs.copy(); bad_rhs[2] = E
    bad_lhs = lhs.copy(); bad_lhs[5] = T + 3
    y4, _, v4 = oracle.gather(x_bits, w, s_bits, b_bits, bad_lhs, bad_rhs, P, T, E,
                              N, K, bits, gs)
    assert list(v4) == [1, 1, 0, 1, 1, 0, 1, 1]
    assert not y4[2].any() and not y4[5].any()
    assert np.array_equal(y4[[0, 1, 3, 4, 6, 7]], y[[0, 1, 3, 4, 6, 7]])
