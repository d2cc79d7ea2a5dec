"""GPU parity of the many-row tensor-core path (M > 16 activation rows, 2-,
4- and 8-bit codes; the pages' qmm_t) against the CPU oracle.

Shapes cover every column-block width (32, 64, 128 rows; M = 17 and 65 leave
most of a block empty), several column blocks, ragged weight tiles, tiles cut
between CTAs (fewer steps than SMs, and ranges that straddle tiles) and
whole tiles, the full 8192 x 28672 matrix and extreme activations.  The
qmv_noalloc form (whole tiles, no scratch) is tested with the other
qmv_noalloc tests."""
import numpy as np
import pytest
import torch

import affine_group_quantized_b200 as agq
from affine_group_quantized_b200 import synth
import oracle
from tests._parity import check, dev_bf16, dev_u32, empty_bf16, host_bits, sample_rows

pytestmark = pytest.mark.gpu


def _run(fn, x, w, s, b, M, N, K, bits, gs):
    Y = empty_bf16(M, N)
    fn(dev_bf16(x), dev_u32(w), dev_bf16(s), dev_bf16(b), Y, M, N, K, bits, gs)
    torch.cuda.synchronize()
    return host_bits(Y)


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("gs", [32, 64, 128])
@pytest.mark.parametrize("M, N, K", [
    (17, 300, 1024),    # 32-row block with 15 empty rows; three tiles, ragged
    (32, 129, 2048),    # one full 32-row block; a one-row last tile
    (64, 1000, 4096),   # 64-row block; fewer steps than SMs: every tile split
    (65, 260, 2048),    # 128-row block, mostly empty
    (128, 300, 2048),   # one full 128-row block
    (200, 500, 1024),   # two 128-row blocks, the second partial
])
def test_qmm_shapes(bits, gs, M, N, K):
    x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=8100 + 7 * M + N + bits + gs)
    y = _run(agq.qmv, x, w, s, b, M, N, K, bits, gs)
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs, nthreads=8)
    check(y, y_ref, a_ref, f"qmm M={M} N={N} K={K} bits={bits} gs={gs}")


def test_qmm_ranges_straddle_tiles():
    # 157 weight tiles of 4 steps on the SMs: ranges of about 4.2 steps, so
    # most tiles are cut between two CTAs and some CTAs hold two part tiles
    M, N, K, bits, gs = 33, 20000, 1024, 4, 32
    x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=8201)
    y = _run(agq.qmv, x, w, s, b, M, N, K, bits, gs)
    rows = np.unique(np.concatenate([sample_rows(N, 600, seed=3), np.arange(N - 40, N)]))
    rows = rows.astype(np.int32)
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs, rows=rows, nthreads=8)
    check(y[:, rows], y_ref, a_ref, "qmm straddling ranges")


@pytest.mark.parametrize("gs", [32, 128])
@pytest.mark.parametrize("M", [32, 64, 128])
def test_qmm_full_size(M, gs):
    # K=8192, N=28672, 4-bit (the batched decode matrix at prefill widths):
    # full launch, oracle on sampled rows
    N, K, bits = 28672, 8192, 4
    x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=8300 + M + gs)
    y = _run(agq.qmv, x, w, s, b, M, N, K, bits, gs)
    rows = sample_rows(N, 48, seed=M + gs)
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs, rows=rows, nthreads=8)
    check(y[:, rows], y_ref, a_ref, f"qmm full size M={M} gs={gs}")


@pytest.mark.parametrize("bits", [4, 8])
def test_qmm_negative_scales_and_extreme_activations(bits):
    # bf16 operands hold every activation exactly: a huge and a tiny span in
    # one row, exact zeros, a row far below 1, sign-flipped scales
    gs, M, N, K = 32, 40, 300, 1024
    x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=8400 + bits)
    s = s ^ np.where(np.arange(s.size).reshape(s.shape) % 3 == 0,
                     np.uint16(0x8000), np.uint16(0))
    xf = synth.bits_to_float(x).astype(np.float32).copy()
    xf[0, :256] *= np.float32(2.0 ** 40)
    xf[0, 256:512] *= np.float32(2.0 ** -40)
    xf[1, 100] = 0.0
    xf[2, 512:544] = 0.0
    xf[3, :] *= np.float32(2.0 ** -60)
    xf[39, :] = 0.0
    x = synth.bf16_bits(torch.from_numpy(xf))
    y = _run(agq.qmv, x, w, s, b, M, N, K, bits, gs)
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs)
    check(y, y_ref, a_ref, f"qmm extreme x bits={bits}")


def test_qmm_repeatable_and_side_stream():
    M, N, K, bits, gs = 96, 3000, 2048, 4, 64
    x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=8500)
    X, W, S, B = dev_bf16(x), dev_u32(w), dev_bf16(s), dev_bf16(b)
    outs = []
    st = torch.cuda.Stream()
    for i in range(3):
        Y = empty_bf16(M, N)
        if i == 1:
            with torch.cuda.stream(st):
                agq.qmv(X, W, S, B, Y, M, N, K, bits, gs)
            st.synchronize()
        else:
            agq.qmv(X, W, S, B, Y, M, N, K, bits, gs)
            torch.cuda.synchronize()
        outs.append(host_bits(Y))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_qmm_status_word_clear():
    assert agq.device_status(reset=True) == 0
