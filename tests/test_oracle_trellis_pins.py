"""Pins of the oracle's trellis mode ("Get trellis to run" compare page,
quantized.h: inst3 and qmv_trellis_impl) against things other than itself:
hand-worked state values, an independent numpy float16 evaluation of every
16-bit state, the page's printed per-value state expressions, and a dense
fp64 product of a value matrix decoded by this test."""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "trellis.txt")


def _golden():
    out = []
    for line in open(GOLDEN):
        line = line.strip()
        if line and not line.startswith("#"):
            s, v = line.split()
            out.append((int(s), float(v)))
    return out


def test_hand_worked_states():
    g = _golden()
    assert len(g) == 2
    for state, value in g:
        assert oracle.trellis_value(state) == value


def _np_values():
    # every state, with numpy's own uint32 and float16 arithmetic
    s = np.arange(1 << 16, dtype=np.uint32)
    x = (np.uint32(89226354) * s + np.uint32(64248484)) & np.uint32(0x8FFF8FFF)
    x ^= np.uint32(996162400)
    lo = (x & np.uint32(0xFFFF)).astype(np.uint16).view(np.float16)
    hi = (x >> np.uint32(16)).astype(np.uint16).view(np.float16)
    return (lo + hi).astype(np.float64)        # float16 addition, rounded to float16


def test_every_state_matches_numpy_float16():
    want = _np_values()
    got = np.array([oracle.trellis_value(int(s)) for s in range(1 << 16)])
    assert np.array_equal(got, want)
    # after the mask and XOR each half's exponent field is 011xx (12..15):
    # every half lies in [2^-3, 2), every value in (-4, 4)
    assert np.all(np.isfinite(got)) and np.max(np.abs(got)) < 4.0


def _page_states(w0, w1, bits):
    # the page's printed expressions, value by value
    wx = w0 ^ w1
    wx1 = wx ^ 1
    wf = w0 ^ (1 << bits)
    if bits == 2:
        return [w0, wf ^ (wx1 & 0x3), w0 ^ (wx & 0xf), w0 ^ (wx1 & 0x3f), w0 ^ (wx & 0xff),
                w0 ^ (wx1 & 0x3ff), w0 ^ (wx & 0xfff), w0 ^ (wx1 & 0x3fff)]
    return [w0, wf ^ (wx1 & 0xf), w0 ^ (wx & 0xff), w0 ^ (wx1 & 0xfff)]


@pytest.mark.parametrize("bits", [2, 4])
def test_states_match_the_printed_expressions(bits):
    rng = np.random.default_rng(bits)
    pairs = rng.integers(0, 1 << 16, size=(20000, 2))
    pairs[:4] = [[0, 0], [0xFFFF, 0], [0, 0xFFFF], [0xFFFF, 0xFFFF]]
    for w0, w1 in pairs:
        want = [v & 0xFFFF for v in _page_states(int(w0), int(w1), bits)]
        got = [oracle.trellis_state(int(w0), int(w1), t, bits) for t in range(16 // bits)]
        assert got == want, (w0, w1)


def _decode_matrix(w, N, K, bits):
    # value matrix V[n, k] decoded here: 16-bit words of each row, the
    # successor of the last word being the first
    vals = _np_values()
    words = np.ascontiguousarray(w).view(np.uint16).reshape(N, K * bits // 16)
    cpw = 16 // bits
    V = np.zeros((N, K))
    for n in range(N):
        u = words[n].astype(np.int64)
        nxt = np.roll(u, -1)
        for i in range(len(u)):
            st = _page_states(int(u[i]), int(nxt[i]), bits)
            for t in range(cpw):
                V[n, i * cpw + t] = vals[st[t] & 0xFFFF]
    return V


@pytest.mark.parametrize("bits, N, K", [(4, 5, 64), (2, 3, 128), (4, 7, 8), (2, 2, 16)])
def test_gemv_is_a_dense_product_of_the_values(bits, N, K):
    rng = np.random.default_rng(N * K + bits)
    M = 2
    w = rng.integers(0, 1 << 32, size=(N, K * bits // 32), dtype=np.uint64).astype(np.uint32)
    x = (rng.standard_normal((M, K)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    scales = np.array([0x3C80, 0x1234], dtype=np.uint16)   # 0.015625; the second is unused
    y, a = oracle.qmv_trellis(x, w, scales, M, N, K, bits)
    xv = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    V = _decode_matrix(w, N, K, bits)
    want = 0.015625 * (xv @ V.T)
    assert np.allclose(y, want, rtol=1e-12, atol=1e-12)
    assert np.allclose(a, 0.015625 * (np.abs(xv) @ np.abs(V).T), rtol=1e-12, atol=1e-12)


def test_gemv_exact_on_dyadic_inputs():
    # x = small integers: every product and partial sum is exact in fp64
    N, K, bits = 3, 32, 4
    rng = np.random.default_rng(3)
    w = rng.integers(0, 1 << 32, size=(N, K * bits // 32), dtype=np.uint64).astype(np.uint32)
    xi = rng.integers(-8, 9, size=(1, K))
    x = (xi.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    y, _ = oracle.qmv_trellis(x, w, np.array([0x3F80], dtype=np.uint16), 1, N, K, bits)
    V = _decode_matrix(w, N, K, bits)
    for n in range(N):
        exact = sum(int(xi[0, k]) * V[n, k] for k in range(K))   # products of dyadics
        assert y[0, n] == exact


def test_bad_arguments():
    x = np.zeros((1, 8), np.uint16)
    w = np.zeros((1, 1), np.uint32)
    with pytest.raises(ValueError):
        oracle.qmv_trellis(x, w, np.zeros(1, np.uint16), 1, 1, 8, 3)   # bits
    with pytest.raises(ValueError):
        oracle.qmv_trellis(x, w, np.zeros(1, np.uint16), 1, 1, 4, 4)   # K * bits % 32
