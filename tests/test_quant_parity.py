"""GPU parity of affine_quantize and affine_dequantize against the CPU oracle.

Both operations are bit-exact by definition: the quantizer's codes, scales
and biases are decided by IEEE binary32 steps (the pages' precision), and
dequantization rounds the exact scale * q + bias once to bf16.  Every case
calls the CUDA path through the C ABI and compares every output bit pattern
with the oracle's; large matrices are checked on sampled rows (rows are
independent).
"""
import numpy as np
import pytest
import torch

import affine_group_quantized_b200 as agq
import oracle
from tests._codes import pack, to_bf16_bits
from tests._parity import dev_bf16, dev_u32, host_bits, sample_rows

pytestmark = pytest.mark.gpu

ALL_BITS = (2, 3, 4, 5, 6, 8)


def _weights(rng, N, K, kind):
    if kind == "normal":
        v = rng.normal(0.0, 0.02, size=(N, K))
    elif kind == "heavy":                     # heavy tails, exact zeros
        v = rng.standard_t(2.0, size=(N, K)) * 0.05
        v[rng.random(size=(N, K)) < 0.1] = 0.0
    elif kind == "positive":
        v = np.abs(rng.normal(0.5, 0.2, size=(N, K))) + 0.01
    elif kind == "negative":
        v = -np.abs(rng.normal(0.5, 0.2, size=(N, K))) - 0.01
    else:                                     # degenerate groups, row by row
        v = rng.normal(0.0, 1.0, size=(N, K))
        v[0::4] = 0.0                         # all-zero rows
        v[1::4] = 0.375                       # constant rows
        v[2::4] *= 1e-9                       # spans below n_bins * 1e-7
    bits32 = np.ascontiguousarray(v.astype(np.float32)).view(np.uint32)
    return (bits32 >> 16).astype(np.uint16)


def run_quantize(w, N, K, bits, gs):
    W = dev_bf16(w)
    Q = torch.full((N, K * bits // 32), -1, dtype=torch.int32, device="cuda")
    S = torch.full((N, K // gs), -1, dtype=torch.int16, device="cuda")
    B = torch.full((N, K // gs), -1, dtype=torch.int16, device="cuda")
    agq.affine_quantize(W, Q, S, B, N, K, bits, gs)
    torch.cuda.synchronize()
    return (Q.cpu().numpy().view(np.uint32), S.cpu().numpy().view(np.uint16),
            B.cpu().numpy().view(np.uint16))


def run_dequantize(wq, s, b, N, K, bits, gs):
    Y = torch.full((N, K), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    agq.affine_dequantize(dev_u32(wq), dev_bf16(s), dev_bf16(b), Y, N, K, bits, gs)
    torch.cuda.synchronize()
    return host_bits(Y)


def _assert_same(got, want, what):
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} of {got.size} differ; first at {i}: "
                             f"got {got[i]:#x}, want {want[i]:#x}")


@pytest.mark.parametrize("bits", ALL_BITS)
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_quantize_bit_exact(bits, gs):
    # ragged row counts: the last warp's 32 chunks run past the end
    for i, (N, K, kind) in enumerate([(37, 4 * gs, "normal"), (5, 384, "heavy"),
                                      (19, 2 * gs, "positive"), (3, gs, "negative"),
                                      (12, 512, "degenerate")]):
        if K % gs:
            continue
        w = _weights(np.random.default_rng(bits * 1000 + gs * 10 + i), N, K, kind)
        got = run_quantize(w, N, K, bits, gs)
        want = oracle.affine_quantize(w, N, K, bits, gs)
        for g, r, name in zip(got, want, ("codes", "scales", "biases")):
            _assert_same(g, r, f"quantize {name} bits={bits} gs={gs} N={N} K={K} {kind}")


def test_quantize_golden_groups_on_the_gpu():
    # the hand-derived groups of the oracle's pins, through the kernel
    import os
    rows = []
    path = os.path.join(os.path.dirname(__file__), "golden", "quantize.txt")
    for line in open(path):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append([c.strip() for c in line.split("|")])
    for c in rows:
        bits, gs = int(c[0]), int(c[1])
        lead = [float(v) for v in c[2].split()]
        vals = lead + [float(c[3])] * (gs - len(lead))
        codes = [int(v) for v in c[6].split()] + [int(c[7])] * (gs - len(lead))
        w = to_bf16_bits(np.array([vals]))
        q, s, b = run_quantize(w, 1, gs, bits, gs)
        assert s[0, 0] == int(c[4], 16) and b[0, 0] == int(c[5], 16), c
        assert np.array_equal(q, pack(np.array([codes]), bits)), c


@pytest.mark.parametrize("bits", ALL_BITS)
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_dequantize_bit_exact(bits, gs):
    rng = np.random.default_rng(bits * 7 + gs)
    for N, K in [(37, 4 * gs), (3, 384 if 384 % gs == 0 else 256), (1, gs)]:
        codes = rng.integers(0, 1 << bits, size=(N, K))
        m = rng.integers(128, 256, size=(2, N, K // gs)).astype(np.float64)
        sg = rng.choice([-1.0, 1.0], size=(2, N, K // gs))
        s = to_bf16_bits(sg[0] * np.ldexp(m[0], rng.integers(-40, 10, size=(N, K // gs)) - 7))
        b = to_bf16_bits(sg[1] * np.ldexp(m[1], rng.integers(-60, 30, size=(N, K // gs)) - 7))
        wq = pack(codes, bits)
        got = run_dequantize(wq, s, b, N, K, bits, gs)
        _assert_same(got, oracle.dequantize_bf16(wq, s, b, N, K, bits, gs),
                     f"dequantize bits={bits} gs={gs} N={N} K={K}")


def test_dequantize_ties_broken_by_the_exact_sum():
    # scale 129/128 times code 3 is halfway between two bf16 values in
    # binary32 too; a tiny bias must decide the direction
    bits, gs, K = 2, 32, 64
    codes = np.full((3, K), 3)
    s = to_bf16_bits(np.full((3, 2), 129 / 128))
    b = to_bf16_bits(np.array([[2.0 ** -60] * 2, [-(2.0 ** -60)] * 2, [0.0] * 2]))
    wq = pack(codes, bits)
    got = run_dequantize(wq, s, b, 3, K, bits, gs)
    _assert_same(got, oracle.dequantize_bf16(wq, s, b, 3, K, bits, gs), "ties")
    up, down = to_bf16_bits([3.03125])[0], to_bf16_bits([3.015625])[0]
    assert (got[0] == up).all() and (got[1] == down).all() and (got[2] == up).all()


@pytest.mark.parametrize("bits", (3, 4, 8))
def test_round_trip_matches_the_oracle(bits):
    N, K, gs = 64, 1024, 64
    w = _weights(np.random.default_rng(bits), N, K, "heavy")
    wq, s, b = run_quantize(w, N, K, bits, gs)
    got = run_dequantize(wq, s, b, N, K, bits, gs)
    owq, os_, ob = oracle.affine_quantize(w, N, K, bits, gs)
    _assert_same(got, oracle.dequantize_bf16(owq, os_, ob, N, K, bits, gs), "round trip")


@pytest.mark.parametrize("bits", (2, 4, 5, 8))
def test_full_size_matrix_sampled_rows(bits):
    # the decode weight shape (N=14336, K=4096, gs 64), one launch each way;
    # the oracle checks sampled rows
    N, K, gs = 14336, 4096, 64
    w = _weights(np.random.default_rng(50 + bits), N, K, "normal")
    wq, s, b = run_quantize(w, N, K, bits, gs)
    rows = sample_rows(N, 200, seed=bits)
    sub = np.ascontiguousarray(w[rows])
    owq, os_, ob = oracle.affine_quantize(sub, len(rows), K, bits, gs)
    _assert_same(wq[rows], owq, "full-size codes")
    _assert_same(s[rows], os_, "full-size scales")
    _assert_same(b[rows], ob, "full-size biases")
    got = run_dequantize(wq, s, b, N, K, bits, gs)
    _assert_same(got[rows], oracle.dequantize_bf16(owq, os_, ob, len(rows), K, bits, gs),
                 "full-size dequantize")


def test_empty_matrix_enqueues_nothing():
    Q = torch.full((1, 8), 7, dtype=torch.int32, device="cuda")
    S = torch.full((1, 2), 7, dtype=torch.int16, device="cuda")
    B = torch.full((1, 2), 7, dtype=torch.int16, device="cuda")
    W = torch.zeros((1, 64), dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros((1, 64), dtype=torch.bfloat16, device="cuda")
    agq.affine_quantize(W, Q, S, B, 0, 64, 4, 32)
    agq.affine_dequantize(Q, S, B, Y, 0, 64, 4, 32)
    torch.cuda.synchronize()
    assert (Q == 7).all() and (S == 7).all() and (B == 7).all() and (Y == 0).all()


@pytest.mark.parametrize("bits", (3, 4, 8))
def test_quantized_weights_feed_qmv(bits):
    # producer to consumer on the device: weights quantized by the kernel go
    # straight into qmv; the oracle quantizes the same weights and runs its
    # own qmv, and the two must agree within the GEMV tolerance
    from affine_group_quantized_b200 import synth
    from tests._parity import check, empty_bf16
    N, K, gs = 300, 1024, 64
    w = _weights(np.random.default_rng(70 + bits), N, K, "normal")
    x = synth.normal_bf16((1, K), seed=71 + bits)
    W = dev_bf16(w)
    Q = torch.empty((N, K * bits // 32), dtype=torch.int32, device="cuda")
    S = torch.empty((N, K // gs), dtype=torch.bfloat16, device="cuda")
    B = torch.empty((N, K // gs), dtype=torch.bfloat16, device="cuda")
    Y = empty_bf16(1, N)
    agq.affine_quantize(W, Q, S, B, N, K, bits, gs)
    agq.qmv(dev_bf16(x), Q, S, B, Y, 1, N, K, bits, gs)
    torch.cuda.synchronize()
    owq, os_, ob = oracle.affine_quantize(w, N, K, bits, gs)
    y_ref, a_ref = oracle.qmv(x, owq, os_, ob, 1, N, K, bits, gs)
    check(host_bits(Y), y_ref, a_ref, f"quantize -> qmv bits={bits}")
