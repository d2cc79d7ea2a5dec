"""qmv_noalloc: the same results as qmv, with the tensor-core path's
split-tile scratch taken from the library's fixed device array instead of an
allocation.  Collected last, so the allocating entry point has run first."""
import numpy as np
import pytest
import torch

import affine_group_quantized_b200 as agq
from affine_group_quantized_b200 import synth
from tests._parity import dev_bf16, dev_u32, empty_bf16, host_bits


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
