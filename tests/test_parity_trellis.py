"""GPU parity of the trellis-mode GEMV (qmv_trellis) against the CPU oracle:
both widths, rows whose words wrap within one 8-word chunk and across many,
several activation rows, the decode shape at full size."""
import numpy as np
import pytest
import torch

import affine_group_quantized_b200 as agq
from affine_group_quantized_b200 import synth
import oracle
from tests._parity import check, dev_bf16, dev_u32, empty_bf16, host_bits

pytestmark = pytest.mark.gpu


def _inputs(M, N, K, bits, seed):
    rng = np.random.default_rng(seed)
    w = rng.integers(0, 1 << 32, size=(N, K * bits // 32), dtype=np.uint64).astype(np.uint32)
    x = synth.normal_bf16((M, K), seed=seed + 1)
    scales = synth.bf16_bits(torch.tensor([0.0123, 7.0]))   # scales[0] is the matrix scale
    return x, w, scales


def _run(x, w, scales, M, N, K, bits):
    Y = empty_bf16(M, N)
    agq.qmv_trellis(dev_bf16(x), dev_u32(w), dev_bf16(scales), Y, M, N, K, bits)
    torch.cuda.synchronize()
    return host_bits(Y)


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("M, N, K", [(1, 7, 64), (1, 333, 1024), (2, 100, 2048), (3, 41, 96 * 4)])
def test_trellis_shapes(bits, M, N, K):
    if (K * bits) % 128:
        pytest.skip("K*bits must be a multiple of 128")
    x, w, s = _inputs(M, N, K, bits, seed=N + K + bits)
    y = _run(x, w, s, M, N, K, bits)
    y_ref, a_ref = oracle.qmv_trellis(x, w, s, M, N, K, bits)
    check(y, y_ref, a_ref, f"trellis bits={bits} M={M} N={N} K={K}")


@pytest.mark.parametrize("bits", [2, 4])
def test_trellis_decode_shape_full_size(bits):
    M, N, K = 1, 14336, 4096
    x, w, s = _inputs(M, N, K, bits, seed=8000 + bits)
    y = _run(x, w, s, M, N, K, bits)
    y_ref, a_ref = oracle.qmv_trellis(x, w, s, M, N, K, bits)
    check(y, y_ref, a_ref, f"trellis full bits={bits}")


def test_trellis_repeatable():
    x, w, s = _inputs(1, 500, 2048, 4, seed=3)
    a = _run(x, w, s, 1, 500, 2048, 4)
    b = _run(x, w, s, 1, 500, 2048, 4)
    assert np.array_equal(a, b)
