"""GPU parity of the single-row decode kernel (M = 1, 2- and 4-bit codes, K a
multiple of 2048) against the CPU oracle: every shape rule of its launch plan
(rows per CTA below, at and above one slot; warps per row 1 .. 14; row blocks
that straddle the gate/up matrices), every group size, the SiLU mode with and
without the residual, spans whose activations differ by many orders of
magnitude, and the status word after all of it."""
import numpy as np
import pytest
import torch

import affine_group_quantized_b200 as agq
from affine_group_quantized_b200 import synth
import oracle
from tests._parity import check, dev_bf16, dev_u32, empty_bf16, host_bits, sample_rows

pytestmark = pytest.mark.gpu


def _qmv(x, w, s, b, N, K, bits, gs):
    Y = empty_bf16(1, N)
    agq.qmv(dev_bf16(x), dev_u32(w), dev_bf16(s), dev_bf16(b), Y, 1, N, K, bits, gs)
    torch.cuda.synchronize()
    return host_bits(Y)


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("N, K, gs", [
    (1, 2048, 64),      # one row: one CTA, a one-row slot
    (7, 2048, 32),      # fewer rows than CTAs
    (148, 4096, 128),   # one row per CTA
    (149, 4096, 64),    # one CTA with two rows
    (1000, 6144, 32),   # three warps per row, ragged slots
    (333, 8192, 128),   # four warps per row
    (4000, 2048, 64),   # one warp per row, many slots per CTA
    (50, 28672, 64),    # fourteen warps per row, one row phase
])
def test_decode_shapes(bits, N, K, gs):
    x, w, s, b = synth.qmv_inputs(1, N, K, bits, gs, seed=31 * N + K + bits + gs)
    y = _qmv(x, w, s, b, N, K, bits, gs)
    rows = sample_rows(N, 400, seed=N + bits) if N > 400 else None
    y_ref, a_ref = oracle.qmv(x, w, s, b, 1, N, K, bits, gs, rows=rows, nthreads=8)
    check(y if rows is None else y[:, rows], y_ref, a_ref, f"decode N={N} K={K} bits={bits} gs={gs}")


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_decode_extreme_spans_and_negative_scales(bits, gs):
    # spans whose largest activation is 2^12 times the rest, all-zero spans,
    # spans of tiny values, sign-flipped scales
    N, K = 300, 4096
    x, w, s, b = synth.qmv_inputs(1, N, K, bits, gs, seed=97 + bits + gs)
    xf = synth.bits_to_float(x).astype(np.float32).copy()
    xf[0, 0:64] *= 1e-3
    xf[0, 5] = 4096.0
    xf[0, 64:128] = 0.0
    xf[0, 128:192] *= 2.0 ** -100
    xf[0, 200] = -3.0e4
    x = synth.bf16_bits(torch.from_numpy(xf))
    sf = synth.bits_to_float(s).astype(np.float32).copy()
    sf[::3] *= -1.0
    s = synth.bf16_bits(torch.from_numpy(sf))
    y = _qmv(x, w, s, b, N, K, bits, gs)
    y_ref, a_ref = oracle.qmv(x, w, s, b, 1, N, K, bits, gs)
    check(y, y_ref, a_ref, f"decode extreme bits={bits} gs={gs}")


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("N", [333, 14336])
def test_decode_gate_up(bits, N):
    # the two matrices' rows are one walk: CTA row blocks straddle them
    K, gs = 2048 if N == 333 else 4096, 64
    x, wg, sg, bg = synth.qmv_inputs(1, N, K, bits, gs, seed=41 + N)
    _, wu, su, bu = synth.qmv_inputs(1, N, K, bits, gs, seed=42 + N)
    Yg, Yu = empty_bf16(1, N), empty_bf16(1, N)
    agq.qmv_gate_up(dev_bf16(x), dev_u32(wg), dev_bf16(sg), dev_bf16(bg), dev_u32(wu),
                    dev_bf16(su), dev_bf16(bu), Yg, Yu, 1, N, K, bits, gs)
    torch.cuda.synchronize()
    yg, yu = host_bits(Yg), host_bits(Yu)
    rows = sample_rows(N, 400, seed=N) if N > 400 else None
    rg, ag = oracle.qmv(x, wg, sg, bg, 1, N, K, bits, gs, rows=rows, nthreads=8)
    ru, au = oracle.qmv(x, wu, su, bu, 1, N, K, bits, gs, rows=rows, nthreads=8)
    sel = (lambda a: a) if rows is None else (lambda a: a[:, rows])
    check(sel(yg), rg, ag, "decode gate")
    check(sel(yu), ru, au, "decode up")


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("with_resid", [True, False])
@pytest.mark.parametrize("gs", [32, 128])
def test_decode_silu_gate_resid(bits, with_resid, gs):
    N, K = 77, 4096
    g = synth.normal_bf16((1, K), seed=51)
    u = synth.normal_bf16((1, K), seed=52)
    r = synth.normal_bf16((1, N), seed=53) if with_resid else None
    _, w, s, b = synth.qmv_inputs(1, N, K, bits, gs, seed=54 + bits)
    Y = empty_bf16(1, N)
    agq.qmv_silu_gate_resid(dev_bf16(g), dev_bf16(u), None if r is None else dev_bf16(r),
                            dev_u32(w), dev_bf16(s), dev_bf16(b), Y, 1, N, K, bits, gs)
    torch.cuda.synchronize()
    y_ref, a_ref = oracle.silu_gate_resid(g, u, r, w, s, b, 1, N, K, bits, gs)
    check(host_bits(Y), y_ref, a_ref, f"decode silu bits={bits} resid={with_resid}")


def test_decode_repeatable_and_stream_ordered():
    # bit-identical results on repeated launches, also on a non-default stream
    N, K, bits, gs = 2000, 4096, 4, 64
    x, w, s, b = synth.qmv_inputs(1, N, K, bits, gs, seed=61)
    X, W, S, B = dev_bf16(x), dev_u32(w), dev_bf16(s), dev_bf16(b)
    outs = []
    st = torch.cuda.Stream()
    for i in range(4):
        Y = empty_bf16(1, N)
        if i % 2:
            with torch.cuda.stream(st):
                agq.qmv(X, W, S, B, Y, 1, N, K, bits, gs)
            st.synchronize()
        else:
            agq.qmv(X, W, S, B, Y, 1, N, K, bits, gs)
            torch.cuda.synchronize()
        outs.append(host_bits(Y))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_device_status_is_clear_after_the_kernels():
    # every kernel above ran its bounded waits to completion: the status
    # word reads 0; reading with reset leaves it 0
    assert agq.device_status(reset=True) == 0
    assert agq.device_status() == 0
