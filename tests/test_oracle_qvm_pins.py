"""Pins of the oracle's qvm (x @ dequant(W), the non-transposed product)
against facts fixed outside it: a dense fp64 library matmul of the
separately pinned dequantized matrix, exact rational arithmetic on dyadic
inputs, and equality with the (pinned) qmv of the transposed codes.  A
transposed operand, a scale indexed along the wrong axis or a dropped bias
fails at least one of them."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests._codes import bf16_value, pack, to_bf16_bits

ALL_BITS = (2, 3, 4, 5, 6, 8)


def _inputs(rng, M, K, N, bits, gs):
    codes = rng.integers(0, 1 << bits, size=(K, N))
    s = to_bf16_bits(np.ldexp(rng.integers(128, 256, size=(K, N // gs)).astype(float), -14))
    b = to_bf16_bits(-np.ldexp(rng.integers(128, 256, size=(K, N // gs)).astype(float), -10))
    x = to_bf16_bits(np.ldexp(rng.integers(-255, 256, size=(M, K)).astype(float), -8))
    return codes, s, b, x


@pytest.mark.parametrize("bits", ALL_BITS)
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_qvm_is_a_dense_matmul_of_the_dequantized_matrix(bits, gs):
    rng = np.random.default_rng(bits * 31 + gs)
    M, K, N = 3, 96, 2 * gs          # K != N, so a transposed operand cannot fit
    codes, s, b, x = _inputs(rng, M, K, N, bits, gs)
    w = pack(codes, bits)
    y, a = oracle.qvm(x, w, s, b, M, K, N, bits, gs)
    w_hat = oracle.dequant(w, s, b, K, N, bits, gs)            # [K, N]
    xv = bf16_value(x)
    want = xv @ w_hat
    assert np.allclose(y, want, rtol=1e-12, atol=1e-12 * np.abs(xv) @ np.abs(w_hat))
    assert np.allclose(a, np.abs(xv) @ np.abs(w_hat), rtol=1e-12)


def test_qvm_exact_on_dyadic_inputs():
    rng = np.random.default_rng(3)
    M, K, N, bits, gs = 2, 40, 64, 5, 32
    codes, s, b, x = _inputs(rng, M, K, N, bits, gs)
    y, _ = oracle.qvm(x, pack(codes, bits), s, b, M, K, N, bits, gs)
    sv, bv, xv = bf16_value(s), bf16_value(b), bf16_value(x)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(xv[m, k]) * (Fraction(sv[k, n // gs]) * int(codes[k, n]) +
                                              Fraction(bv[k, n // gs]))
                        for k in range(K))
            assert Fraction(y[m, n]) == exact, (m, n)


@pytest.mark.parametrize("bits", (2, 4, 6))
def test_qvm_equals_qmv_of_the_transposed_codes(bits):
    # with scales and biases constant over each block of gs rows of W (and
    # over its columns), W's dequantized columns are the dequantized rows of
    # the transposed codes, so qvm(x, W) == qmv(x, W^T) exactly
    rng = np.random.default_rng(40 + bits)
    M, K, N, gs = 2, 128, 96, 32
    codes = rng.integers(0, 1 << bits, size=(K, N))
    sblk = np.ldexp(rng.integers(128, 256, size=K // gs).astype(float), -12)
    bblk = -np.ldexp(rng.integers(128, 256, size=K // gs).astype(float), -9)
    s_qvm = to_bf16_bits(np.repeat(sblk, gs)[:, None].repeat(N // gs, axis=1))   # [K, N/gs]
    b_qvm = to_bf16_bits(np.repeat(bblk, gs)[:, None].repeat(N // gs, axis=1))
    s_qmv = to_bf16_bits(np.tile(sblk, (N, 1)))                                  # [N, K/gs]
    b_qmv = to_bf16_bits(np.tile(bblk, (N, 1)))
    x = to_bf16_bits(np.ldexp(rng.integers(-255, 256, size=(M, K)).astype(float), -7))
    y1, a1 = oracle.qvm(x, pack(codes, bits), s_qvm, b_qvm, M, K, N, bits, gs)
    y2, a2 = oracle.qmv(x, pack(codes.T.copy(), bits), s_qmv, b_qmv, M, N, K, bits, gs)
    assert np.array_equal(y1, y2) and np.array_equal(a1, a2)


def test_qvm_scale_runs_along_the_output_axis():
    # one nonzero scale, in group 1 of row 0: only outputs of that group see
    # the codes of row 0
    M, K, N, bits, gs = 1, 32, 64, 4, 32
    codes = np.full((K, N), 3)
    s = np.zeros((K, N // gs), dtype=np.uint16)
    s[0, 1] = to_bf16_bits([1.0])[0]
    b = np.zeros((K, N // gs), dtype=np.uint16)
    x = to_bf16_bits(np.ones((M, K)))
    y, _ = oracle.qvm(x, pack(codes, bits), s, b, M, K, N, bits, gs)
    assert (y[0, :gs] == 0).all() and (y[0, gs:] == 3.0).all()


def test_qvm_rejects_bad_shapes():
    w = np.zeros(64, dtype=np.uint32)
    s = np.zeros(8, dtype=np.uint16)
    with pytest.raises(ValueError):
        oracle.qvm(np.zeros(32, np.uint16), w, s, s, 1, 32, 48, 4, 32)   # N % gs
    with pytest.raises(ValueError):
        oracle.qvm(np.zeros(32, np.uint16), w, s, s, 1, 32, 64, 7, 32)   # bits
