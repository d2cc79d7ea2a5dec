"""GPU parity of qmv (y = x @ dequant(W).T) against the CPU oracle.

Every case calls the CUDA path through the C ABI (Python binding) and
compares each output with the oracle's fp64 value on the same seeded inputs.
"""
import numpy as np
import pytest
import torch

import affine_group_quantized_b200 as agq
from affine_group_quantized_b200 import synth
import oracle
from tests._parity import check, dev_bf16, dev_u32, empty_bf16, host_bits, sample_rows

pytestmark = pytest.mark.gpu

ALL_BITS = (2, 3, 4, 5, 6, 8)


def run_qmv(x, w, s, b, M, N, K, bits, gs):
    X, W, S, B = dev_bf16(x), dev_u32(w), dev_bf16(s), dev_bf16(b)
    Y = empty_bf16(M, N)
    agq.qmv(X, W, S, B, Y, M, N, K, bits, gs)
    torch.cuda.synchronize()
    return host_bits(Y)


def test_qmv_small_workload():
    # M=1, K=512, N=256, 4-bit, gs 64; b = -8 s + U[-1e-3, 1e-3]
    M, N, K, bits, gs = 1, 256, 512, 4, 64
    x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=1000, bias_jitter=1e-3)
    y = run_qmv(x, w, s, b, M, N, K, bits, gs)
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs)
    check(y, y_ref, a_ref, "qmv small")


@pytest.mark.parametrize("bits", ALL_BITS)
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_qmv_shapes(bits, gs):
    # several tiles, ragged N, K with padded unit counts
    for (M, N, K) in [(1, 301, 4 * gs), (2, 67, 1536 if gs <= 64 else 1664),
                      (1, 1, gs), (3, 45, 1024), (1, 130, 96 if gs == 32 else 2 * gs)]:
        x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=bits * 977 + gs + N)
        y = run_qmv(x, w, s, b, M, N, K, bits, gs)
        y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs)
        check(y, y_ref, a_ref, f"qmv bits={bits} gs={gs} M={M} N={N} K={K}")


@pytest.mark.parametrize("bits", ALL_BITS)
def test_qmv_decode_sweep_full_size(bits):
    # M=1, K=4096, N=14336, gs=64: full launch, oracle on sampled rows
    M, N, K, gs = 1, 14336, 4096, 64
    x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=2000 + bits)
    y = run_qmv(x, w, s, b, M, N, K, bits, gs)
    rows = sample_rows(N, 600, seed=bits)
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs, rows=rows, nthreads=8)
    check(y[:, rows], y_ref, a_ref, f"decode sweep bits={bits}")
    assert np.all(np.isfinite(y.view(np.uint16).astype(np.uint32) << 16))


def test_qmv_negative_scales_and_extreme_activations():
    bits, gs, M, N, K = 4, 32, 2, 96, 1024
    x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=7)
    s = s ^ np.where(np.arange(s.size).reshape(s.shape) % 3 == 0,
                     np.uint16(0x8000), np.uint16(0))  # flip some scale signs
    xf = synth.bits_to_float(x).astype(np.float32).copy()
    xf[0, :256] *= np.float32(2.0 ** 60)    # huge unit
    xf[0, 256:512] *= np.float32(2.0 ** -60)  # tiny unit
    xf[1, 100] = 0.0
    xf[1, 512:544] = 0.0                    # an all-zero unit
    x = synth.bf16_bits(torch.from_numpy(xf))
    y = run_qmv(x, w, s, b, M, N, K, bits, gs)
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs)
    check(y, y_ref, a_ref, "negative scales / extreme x")


@pytest.mark.parametrize("bits", [4, 8])
def test_qmv_batched_negative_scales_and_extreme_activations(bits):
    # the tensor-core path (four activation rows): sign-flipped scales, a
    # huge and a tiny unit in one row (the row's power-of-two fp16 range is
    # set by its largest value), exact zeros and an all-zero unit
    gs, M, N, K = 32, 4, 300, 1024
    x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=17 + bits)
    s = s ^ np.where(np.arange(s.size).reshape(s.shape) % 3 == 0,
                     np.uint16(0x8000), np.uint16(0))
    xf = synth.bits_to_float(x).astype(np.float32).copy()
    xf[0, :256] *= np.float32(2.0 ** 60)
    xf[0, 256:512] *= np.float32(2.0 ** -60)
    xf[1, 100] = 0.0
    xf[2, 512:544] = 0.0
    xf[3, :] *= np.float32(2.0 ** -100)   # a whole row far below 1
    x = synth.bf16_bits(torch.from_numpy(xf))
    y = run_qmv(x, w, s, b, M, N, K, bits, gs)
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs)
    check(y, y_ref, a_ref, f"batched negative scales / extreme x bits={bits}")


@pytest.mark.parametrize("gs", [32, 128])
@pytest.mark.parametrize("M", [1, 2, 4, 8])
def test_qmv_batched_full_size(M, gs):
    # K=8192, N=28672, 4-bit: full launch, oracle on sampled rows
    N, K, bits = 28672, 8192, 4
    x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=4000 + 10 * M + gs)
    y = run_qmv(x, w, s, b, M, N, K, bits, gs)
    rows = sample_rows(N, 200, seed=M + gs)
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs, rows=rows, nthreads=8)
    check(y[:, rows], y_ref, a_ref, f"batched M={M} gs={gs}")


def test_qmv_repeatable():
    bits, gs, M, N, K = 3, 64, 1, 777, 2048
    x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=99)
    y1 = run_qmv(x, w, s, b, M, N, K, bits, gs)
    y2 = run_qmv(x, w, s, b, M, N, K, bits, gs)
    assert np.array_equal(y1, y2)


def test_qmv_many_chunks_tiny_rows():
    # M = 8192 activation rows in 4096 chunks of two over N = 2 rows: each CTA
    # walks more 2-row tiles than its stage ring holds, with most consumer
    # warps idle in every tile
    M, N, K, bits, gs = 8192, 2, 128, 4, 32
    x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=4242)
    y = run_qmv(x, w, s, b, M, N, K, bits, gs)
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs, nthreads=8)
    check(y, y_ref, a_ref, "qmv many chunks")


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_qmv_batched_rows_small(bits, gs):
    # several activation rows (the tensor-core path for 2/4/8-bit codes):
    # three 128-row tiles with a ragged last one, several K stages
    for M in (3, 5, 16):
        N, K = 300, 2048
        x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=7000 + 31 * M + bits + gs)
        y = run_qmv(x, w, s, b, M, N, K, bits, gs)
        y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs)
        check(y, y_ref, a_ref, f"batched rows M={M} bits={bits} gs={gs}")


@pytest.mark.parametrize("M", [1, 2, 4, 7, 8, 12, 16])
def test_qmv_batched_rows_counts(M):
    # every activation-row count up to 16 at one shape, a single K stage
    bits, gs, N, K = 4, 32, 129, 256
    x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=7500 + M)
    y = run_qmv(x, w, s, b, M, N, K, bits, gs)
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs)
    check(y, y_ref, a_ref, f"batched rows M={M}")


def test_qmv_batched_many_tiles_per_cta():
    # more than two 128-row tiles per CTA on any current GPU (the accumulator
    # halves and the stage ring are both reused), ragged last tile; oracle on
    # sampled rows plus the last rows
    M, N, K, bits, gs = 6, 3 * 160 * 128 + 77, 2048, 4, 64
    x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=7777)
    y = run_qmv(x, w, s, b, M, N, K, bits, gs)
    rows = np.unique(np.concatenate([sample_rows(N, 300, seed=5), np.arange(N - 80, N)])).astype(np.int32)
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs, rows=rows, nthreads=8)
    check(y[:, rows], y_ref, a_ref, "batched many tiles")


def test_qmv_batched_split_tiles_repeatable():
    # a few more 128-row tiles than SMs and four K stages per tile: the
    # (tile, stage) steps are shared out evenly, so most tiles are cut into
    # parts held by two CTAs and added by the last one to finish; the sum
    # order is fixed, so repeated launches agree bit for bit, and the
    # per-tile arrival counters start from zero again after each launch
    M, N, K, bits, gs = 4, 150 * 128 - 20, 1024, 4, 32
    x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=8080)
    ys = [run_qmv(x, w, s, b, M, N, K, bits, gs) for _ in range(3)]
    assert np.array_equal(ys[0], ys[1]) and np.array_equal(ys[0], ys[2])
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs, nthreads=8)
    check(ys[0], y_ref, a_ref, "batched split tiles")
