"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module draws random inputs and nothing else: it holds none of the
quantized product's arithmetic (no unpacking, no dequantization, no dot
products).  Packed weights are drawn as uniformly random uint32 words: when
every bit is an independent fair coin, every ``bits``-wide code of the
LSB-first bitstream is uniform on ``[0, 2**bits)``, which is exactly the
"uniform codes" recipe of the workloads, for every bit width, without ever
packing a code.

All generators run on the CPU with ``torch.Generator`` so the same seed gives
the same bytes on every machine.  bf16 tensors are returned as numpy
``uint16`` bit patterns (round-to-nearest-even from fp32).
"""
from __future__ import annotations

import numpy as np
import torch


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """fp32/bf16 tensor -> bf16 bit patterns (RNE) as numpy uint16."""
    return t.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)


def bits_to_float(h: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 values (exact widening)."""
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(shape, seed: int) -> np.ndarray:
    """x ~ N(0, 1), rounded to bf16."""
    return bf16_bits(torch.randn(shape, generator=_gen(seed), dtype=torch.float32))


def uniform_bf16(shape, lo: float, hi: float, seed: int) -> np.ndarray:
    u = torch.rand(shape, generator=_gen(seed), dtype=torch.float64)
    return bf16_bits((lo + (hi - lo) * u).to(torch.float32))


def random_words(shape, seed: int) -> np.ndarray:
    """Uniformly random uint32 words (every bit a fair coin)."""
    g = _gen(seed)
    lo = torch.randint(0, 1 << 16, shape, generator=g, dtype=torch.int64)
    hi = torch.randint(0, 1 << 16, shape, generator=g, dtype=torch.int64)
    return ((hi << 16) | lo).numpy().astype(np.uint32)


def words_per_row(K: int, bits: int) -> int:
    """uint32 words holding one packed row of K codes (layout size only)."""
    assert (K * bits) % 32 == 0
    return K * bits // 32


def affine_params(rows: int, groups: int, bits: int, seed: int,
                  scale_lo: float = 0.005, scale_hi: float = 0.02,
                  bias_jitter: float = 0.0, bias_offset_per_row_block=None):
    """scales ~ U[lo, hi] (bf16); biases = -(2**bits/2)*scale (+ U[-j, j]).

    With ``bias_jitter == 0`` the bias is an exact bf16 (a power-of-two
    multiple of a bf16).  ``bias_offset_per_row_block=(block_rows, step)``
    adds ``step * (row // block_rows)`` to every bias, which gives each
    expert of a stacked ``[E*N]`` row space a distinct bias (used to make a
    mis-routed gather row fail by far more than the tolerance).
    """
    s_bits = uniform_bf16((rows, groups), scale_lo, scale_hi, seed)
    s = torch.from_numpy(bits_to_float(s_bits).copy()).to(torch.float64)
    b = -(2.0 ** bits / 2.0) * s
    if bias_jitter:
        u = torch.rand((rows, groups), generator=_gen(seed + 7), dtype=torch.float64)
        b = b + (2.0 * u - 1.0) * bias_jitter
    if bias_offset_per_row_block is not None:
        block_rows, step = bias_offset_per_row_block
        r = torch.arange(rows, dtype=torch.float64).unsqueeze(1)
        b = b + step * torch.floor(r / block_rows)
    return s_bits, bf16_bits(b.to(torch.float32))


def qmv_inputs(M: int, N: int, K: int, bits: int, gs: int, seed: int, **kw):
    """x [M,K] bf16, w [N, K*bits/32] u32, scales/biases [N, K/gs] bf16."""
    x = normal_bf16((M, K), seed)
    w = random_words((N, words_per_row(K, bits)), seed + 1)
    s, b = affine_params(N, K // gs, bits, seed + 2, **kw)
    return x, w, s, b


def topk_routing(tokens: int, experts: int, k: int, seed: int):
    """Per token, k distinct experts drawn uniformly without replacement
    (partial Fisher-Yates).  Returns (lhs, rhs) uint32 arrays of length
    tokens*k with lhs[t*k + j] = t."""
    g = _gen(seed)
    rhs = np.zeros(tokens * k, dtype=np.uint32)
    for t in range(tokens):
        perm = list(range(experts))
        for j in range(k):
            r = int(torch.randint(j, experts, (1,), generator=g).item())
            perm[j], perm[r] = perm[r], perm[j]
            rhs[t * k + j] = perm[j]
    lhs = np.repeat(np.arange(tokens, dtype=np.uint32), k)
    return lhs, rhs


def sort_pairs_by_expert(lhs: np.ndarray, rhs: np.ndarray):
    """Stable sort of (lhs, rhs) pairs by expert; returns (lhs', rhs', perm)
    with pair i of the sorted list equal to pair perm[i] of the input."""
    perm = np.argsort(rhs, kind="stable")
    return lhs[perm].copy(), rhs[perm].copy(), perm


# Workloads (shapes and distributions only).
WORKLOADS = {
    "qmv_small": dict(M=1, K=512, N=256, bits=4, gs=64,
                      note="x~N(0,1); codes U{0..15}; s~U[.005,.02]; "
                           "b=-8s+U[-.001,.001]"),
    "decode_sweep": dict(M=1, K=4096, N=14336, gs=64, bits=(2, 3, 4, 5, 6, 8),
                         note="x~N(0,1); uniform codes; s~U[.005,.02]; "
                              "b=-(2^bits/2)s"),
    "ffn_int8": dict(K=4096, N=14336, bits=8, gs=64,
                     note="gate/up W[14336,4096], down W[4096,14336]; "
                          "s~U[.002,.01]; b=-128s; x, x_resid ~N(0,1)"),
    "batched": dict(M=(1, 2, 4, 8), K=8192, N=28672, bits=4, gs=(32, 128),
                    note="x~N(0,1)[M,8192]; s~U[.005,.02]; b=-8s"),
    "moe_gather": dict(E=64, N=1536, K=2048, bits=4, gs=64, tokens=32, topk=4,
                       note="top-4 experts per token, uniform without "
                            "replacement; sorted and unsorted"),
}
