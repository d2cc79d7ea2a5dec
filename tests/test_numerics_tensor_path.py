"""CPU model of the tensor-core path's rounding, checked against the oracle.

The batched tensor-core path (several activation rows, 2/4/8-bit codes)
computes in three roundings: each weight w_hat = s*q + b is rounded once to
fp16; each activation row is multiplied by its own power of two (largest
magnitude into [2^13, 2^14)) and rounded to fp16; the fp16 products are
summed in fp32 and the power of two is divided out before the bf16 store.
This test applies exactly those roundings with numpy (no GPU, no kernel code)
and asserts that the result meets the acceptance bound against the fp64
oracle, on the batched input distribution and on extreme activations.  It
pins the numerical reading, independently of the kernel that implements it.
"""
import numpy as np
import pytest
import torch

from affine_group_quantized_b200 import synth
import oracle
from tests import _codes
from tests._parity import ABS_COEF, REL_TOL


def _bf16_round(v: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(v, np.float32)).to(torch.bfloat16).to(
        torch.float64).numpy()


def _model(x_bits, codes, s_bits, b_bits, gs):
    """The tensor-core path's roundings on known codes."""
    x = synth.bits_to_float(x_bits).astype(np.float64)
    s = synth.bits_to_float(s_bits).astype(np.float64)
    b = synth.bits_to_float(b_bits).astype(np.float64)
    g = np.arange(codes.shape[1]) // gs
    w_hat = s[:, g] * codes + b[:, g]                     # exact in fp64
    w16 = w_hat.astype(np.float16).astype(np.float32)     # one rounding
    mx = np.abs(x).max(axis=1)
    a = np.where(mx > 0, 13 - np.floor(np.log2(np.where(mx > 0, mx, 1.0))), 0.0)
    a = np.clip(a, -126, 126)
    xs = (x * np.exp2(a)[:, None]).astype(np.float16).astype(np.float32)
    acc = xs @ w16.T                                      # fp32 products and sums
    return _bf16_round(acc.astype(np.float64) * np.exp2(-a)[:, None])


def _inputs(M, N, K, bits, gs, seed):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 1 << bits, size=(N, K), dtype=np.int64)
    w = _codes.pack(codes, bits)
    x, _, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=seed)
    return x, codes, w, s, b


def _check(y, y_ref, a_ref, what):
    err = np.abs(y - y_ref)
    bound = REL_TOL * np.abs(y_ref) + ABS_COEF * a_ref
    assert np.all(err <= bound), f"{what}: max err/bound {np.max(err / bound)}"


@pytest.mark.parametrize("bits, gs", [(4, 32), (4, 128), (8, 64), (2, 32)])
def test_tensor_path_roundings_meet_the_bound(bits, gs):
    M, N, K = 8, 48, 4096
    x, codes, w, s, b = _inputs(M, N, K, bits, gs, seed=300 + bits + gs)
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs)
    _check(_model(x, codes, s, b, gs), y_ref, a_ref, f"bits={bits} gs={gs}")


def test_tensor_path_roundings_extreme_activations():
    M, N, K, bits, gs = 4, 40, 1024, 4, 32
    x, codes, w, s, b = _inputs(M, N, K, bits, gs, seed=321)
    s = s ^ np.where(np.arange(s.size).reshape(s.shape) % 3 == 0,
                     np.uint16(0x8000), np.uint16(0))  # sign-flipped scales
    xf = synth.bits_to_float(x).astype(np.float32).copy()
    xf[0, :256] *= np.float32(2.0 ** 60)     # a huge unit ...
    xf[0, 256:512] *= np.float32(2.0 ** -60)  # ... and a tiny one in the same row
    xf[2, 512:544] = 0.0
    xf[3, :] *= np.float32(2.0 ** -100)
    x = synth.bf16_bits(torch.from_numpy(xf))
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs)
    _check(_model(x, codes, s, b, gs), y_ref, a_ref, "extreme activations")


def test_model_is_sensitive_to_a_lost_rounding_step():
    # the same model with w_hat rounded to fp8-like precision (3 mantissa
    # bits) must fail the bound: the check is not vacuous
    M, N, K, bits, gs = 4, 48, 4096, 4, 32
    x, codes, w, s, b = _inputs(M, N, K, bits, gs, seed=333)
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs)
    xv = synth.bits_to_float(x).astype(np.float64)
    sv = synth.bits_to_float(s).astype(np.float64)
    bv = synth.bits_to_float(b).astype(np.float64)
    g = np.arange(K) // gs
    w_hat = sv[:, g] * codes + bv[:, g]
    m, e = np.frexp(w_hat)
    w_coarse = np.ldexp(np.round(m * 16) / 16, e)
    y = _bf16_round((xv @ w_coarse.T).astype(np.float32).astype(np.float64))
    err = np.abs(y - y_ref)
    bound = REL_TOL * np.abs(y_ref) + ABS_COEF * a_ref
    assert np.any(err > bound)
