"""GPU parity of qvm (y = x @ dequant(W), W of K rows of N codes, groups
along N) against the CPU oracle: every width and group size, column counts
that leave a partial 256-column block, row counts that do not split evenly
between the cluster's CTAs and warps, several activation rows, sign-flipped
scales and extreme activations, the decode shape at full size."""
import numpy as np
import pytest
import torch

import affine_group_quantized_b200 as agq
from affine_group_quantized_b200 import synth
import oracle
from tests._parity import check, dev_bf16, dev_u32, empty_bf16, host_bits

pytestmark = pytest.mark.gpu


def _qvm(x, w, s, b, M, K, N, bits, gs):
    assert x.shape == (M, K) and w.shape == (K, N * bits // 32)
    Y = empty_bf16(M, N)
    agq.qvm(dev_bf16(x), dev_u32(w), dev_bf16(s), dev_bf16(b), Y, M, K, N, bits, gs)
    torch.cuda.synchronize()
    return host_bits(Y)


def _inputs(M, K, N, bits, gs, seed):
    # W: K rows of N codes (synth draws [rows, codes] weights); x: [M, K]
    _, w, s, b = synth.qmv_inputs(1, K, N, bits, gs, seed=seed)
    x = synth.normal_bf16((M, K), seed=seed + 1)
    assert x.shape == (M, K) and s.shape == (K, N // gs) and w.shape == (K, N * bits // 32)
    return x, w, s, b


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_qvm_shapes(bits, gs):
    for (M, K, N) in [(1, 100, 4 * gs), (2, 37, 1024 + gs), (1, 1, gs), (3, 513, 768)]:
        x, w, s, b = _inputs(M, K, N, bits, gs, seed=bits * 31 + gs + K)
        y = _qvm(x, w, s, b, M, K, N, bits, gs)
        y_ref, a_ref = oracle.qvm(x, w, s, b, M, K, N, bits, gs)
        check(y, y_ref, a_ref, f"qvm bits={bits} gs={gs} M={M} K={K} N={N}")


def test_qvm_negative_scales_and_extreme_activations():
    M, K, N, bits, gs = 1, 3000, 512, 4, 64
    x, w, s, b = _inputs(M, K, N, bits, gs, seed=5)
    xf = synth.bits_to_float(x).astype(np.float32).copy()
    xf[0, ::97] *= 3000.0
    xf[0, 5:40] = 0.0
    xf[0, 100:200] *= 2.0 ** -60
    x = synth.bf16_bits(torch.from_numpy(xf))
    sf = synth.bits_to_float(s).astype(np.float32).copy()
    sf[::5] *= -1.0
    s = synth.bf16_bits(torch.from_numpy(sf))
    y = _qvm(x, w, s, b, M, K, N, bits, gs)
    y_ref, a_ref = oracle.qvm(x, w, s, b, M, K, N, bits, gs)
    check(y, y_ref, a_ref, "qvm extreme")


@pytest.mark.parametrize("bits", [4, 8])
def test_qvm_decode_shape_full_size(bits):
    # the decode weight read the other way: 14336 rows of 4096 codes
    M, K, N, gs = 1, 14336, 4096, 64
    x, w, s, b = _inputs(M, K, N, bits, gs, seed=7000 + bits)
    y = _qvm(x, w, s, b, M, K, N, bits, gs)
    y_ref, a_ref = oracle.qvm(x, w, s, b, M, K, N, bits, gs)
    check(y, y_ref, a_ref, f"qvm full bits={bits}")


def test_qvm_repeatable():
    M, K, N, bits, gs = 2, 5000, 2048, 4, 32
    x, w, s, b = _inputs(M, K, N, bits, gs, seed=9)
    ys = [_qvm(x, w, s, b, M, K, N, bits, gs) for _ in range(3)]
    assert all(np.array_equal(ys[0], y) for y in ys[1:])


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_qvm_staged_shapes(bits, gs):
    # shapes whose code and scale rows are whole 16-byte units (the staged
    # kernel): rows that split unevenly between the cluster's CTAs and the
    # 64-row stages, CTAs with a single short stage, CTAs with no rows
    for (M, K, N) in [(2, 1000, 1024), (1, 70, 2048), (1, 7, 1024), (3, 4099, 3072)]:
        assert (N * bits) % 128 == 0 and (N // gs) % 8 == 0
        x, w, s, b = _inputs(M, K, N, bits, gs, seed=bits * 57 + gs + K)
        y = _qvm(x, w, s, b, M, K, N, bits, gs)
        y_ref, a_ref = oracle.qvm(x, w, s, b, M, K, N, bits, gs)
        check(y, y_ref, a_ref, f"qvm staged bits={bits} gs={gs} M={M} K={K} N={N}")
