"""qmv_noalloc: the same results as qmv, with the few-row tensor-core path's
split-tile scratch taken from the library's fixed device array instead of an
allocation, and the many-row path on whole tiles (no scratch at all).
Collected last, so the allocating entry point has run first."""
import numpy as np
import pytest
import torch

import affine_group_quantized_b200 as agq
from affine_group_quantized_b200 import synth
import oracle
from tests._parity import check, dev_bf16, dev_u32, empty_bf16, host_bits, sample_rows


def _run(fn, x, w, s, b, M, N, K, bits, gs):
    Y = empty_bf16(M, N)
    fn(dev_bf16(x), dev_u32(w), dev_bf16(s), dev_bf16(b), Y, M, N, K, bits, gs)
    torch.cuda.synchronize()
    return host_bits(Y)


def test_noalloc_is_exported_and_bound():
    assert hasattr(agq.lib(), "qmv_noalloc")
    assert callable(agq.qmv_noalloc)


A = 0x10000  # a 16-byte aligned fake device address; never dereferenced


def test_noalloc_argument_checks():
    # the same host-side checks as qmv, before any device is touched
    f = agq.lib().qmv_noalloc
    ok_args = [A, A, A, A, A, 4, 64, 1024, 4, 64, None]
    names = ["x", "w", "s", "b", "y", "M", "N", "K", "bits", "gs", "stream"]

    def call(**over):
        a = list(ok_args)
        for k, v in over.items():
            a[names.index(k)] = v
        return f(*a)

    assert call(w=None) == agq.QMV_ERR_NULL
    assert "qmv_noalloc" in agq.last_error()
    assert call(bits=7) == agq.QMV_ERR_UNSUPPORTED
    assert call(K=96) == agq.QMV_ERR_SHAPE
    assert call(M=0) == agq.QMV_ERR_SHAPE
    assert call(y=A + 8) == agq.QMV_ERR_ALIGN


@pytest.mark.gpu
@pytest.mark.parametrize("M, N, K, bits, gs", [
    (4, 150 * 128 - 20, 1024, 4, 32),  # tensor cores, tiles split between CTAs
    (8, 300, 2048, 8, 64),             # tensor cores, whole tiles
    (1, 2000, 1024, 4, 64),            # one row: the streaming kernel
])
def test_noalloc_matches_qmv_twice_in_a_row(M, N, K, bits, gs):
    x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=9090 + M + bits)
    X, W, S, B = dev_bf16(x), dev_u32(w), dev_bf16(s), dev_bf16(b)
    outs = []
    for fn in (agq.qmv, agq.qmv_noalloc, agq.qmv_noalloc, agq.qmv):
        Y = empty_bf16(M, N)
        fn(X, W, S, B, Y, M, N, K, bits, gs)
        torch.cuda.synchronize()
        outs.append(host_bits(Y))
    for o in outs[1:]:
        assert np.array_equal(outs[0], o)


@pytest.mark.gpu
@pytest.mark.parametrize("M, N, K, bits, gs", [
    (48, 150 * 128 - 20, 1024, 4, 32),   # more tiles than SMs
    (130, 300, 2048, 8, 64),             # two column blocks
    (20, 700, 2048, 2, 128),
])
def test_noalloc_many_rows_whole_tiles(M, N, K, bits, gs):
    # without scratch every CTA takes whole tiles; the sums then run in
    # another order than with split tiles, so compare with the oracle, and
    # with itself
    x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=8600 + M + bits)
    y1 = _run(agq.qmv_noalloc, x, w, s, b, M, N, K, bits, gs)
    y2 = _run(agq.qmv_noalloc, x, w, s, b, M, N, K, bits, gs)
    assert np.array_equal(y1, y2)
    rows = sample_rows(N, 400, seed=M) if N > 400 else None
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs, rows=rows, nthreads=8)
    check(y1 if rows is None else y1[:, rows], y_ref, a_ref, f"qmm noalloc M={M}")
