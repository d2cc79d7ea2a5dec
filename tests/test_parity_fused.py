"""GPU parity of the fused decode variants (gate/up, silu-gate-resid) and of
gather_qmv against the CPU oracle."""
import numpy as np
import pytest
import torch

import affine_group_quantized_b200 as agq
from affine_group_quantized_b200 import synth
import oracle
from tests._parity import (check, dev_bf16, dev_u32, empty_bf16, host_bits,
                           sample_rows)

pytestmark = pytest.mark.gpu


def _gate_up(x, wg, sg, bg, wu, su, bu, M, N, K, bits, gs):
    Yg, Yu = empty_bf16(M, N), empty_bf16(M, N)
    agq.qmv_gate_up(dev_bf16(x), dev_u32(wg), dev_bf16(sg), dev_bf16(bg),
                    dev_u32(wu), dev_bf16(su), dev_bf16(bu), Yg, Yu,
                    M, N, K, bits, gs)
    torch.cuda.synchronize()
    return host_bits(Yg), host_bits(Yu)


def _silu(g, u, r, w, s, b, M, N, K, bits, gs):
    Y = empty_bf16(M, N)
    agq.qmv_silu_gate_resid(dev_bf16(g), dev_bf16(u),
                            None if r is None else dev_bf16(r),
                            dev_u32(w), dev_bf16(s), dev_bf16(b), Y,
                            M, N, K, bits, gs)
    torch.cuda.synchronize()
    return host_bits(Y)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
@pytest.mark.parametrize("M", [1, 2])
def test_gate_up_small(bits, M):
    gs, N, K = 64, 333, 1024
    x, wg, sg, bg = synth.qmv_inputs(M, N, K, bits, gs, seed=11)
    _, wu, su, bu = synth.qmv_inputs(M, N, K, bits, gs, seed=12)
    yg, yu = _gate_up(x, wg, sg, bg, wu, su, bu, M, N, K, bits, gs)
    (rg, ag), (ru, au) = oracle.gate_up(x, wg, sg, bg, wu, su, bu, M, N, K, bits, gs)
    check(yg, rg, ag, "gate")
    check(yu, ru, au, "up")


def test_ffn_int8_full_size():
    # gate/up W [14336, 4096] int8 in one launch, then down W [4096, 14336]
    # applied to silu(gate)*up with x_resid added.  The second stage's oracle
    # consumes the same bf16 gate/up buffers the GPU produced.
    bits, gs, M, N, K = 8, 64, 1, 14336, 4096
    kw = dict(scale_lo=0.002, scale_hi=0.01)
    x, wg, sg, bg = synth.qmv_inputs(M, N, K, bits, gs, seed=3000, **kw)
    _, wu, su, bu = synth.qmv_inputs(M, N, K, bits, gs, seed=3001, **kw)
    yg, yu = _gate_up(x, wg, sg, bg, wu, su, bu, M, N, K, bits, gs)
    rows = sample_rows(N, 300, seed=5)
    rg, ag = oracle.qmv(x, wg, sg, bg, M, N, K, bits, gs, rows=rows, nthreads=8)
    ru, au = oracle.qmv(x, wu, su, bu, M, N, K, bits, gs, rows=rows, nthreads=8)
    check(yg[:, rows], rg, ag, "ffn gate")
    check(yu[:, rows], ru, au, "ffn up")
    # down projection: K2 = 14336 inputs, N2 = 4096 outputs
    N2, K2 = 4096, 14336
    _, wd, sd, bd = synth.qmv_inputs(M, N2, K2, bits, gs, seed=3002, **kw)
    resid = synth.normal_bf16((M, N2), seed=3003)
    yd = _silu(yg, yu, resid, wd, sd, bd, M, N2, K2, bits, gs)
    rows2 = sample_rows(N2, 300, seed=6)
    rd, ad = oracle.silu_gate_resid(yg, yu, resid, wd, sd, bd, M, N2, K2, bits, gs,
                                    rows=rows2, nthreads=8)
    check(yd[:, rows2], rd, ad, "ffn down (silu-gate-resid)")


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
@pytest.mark.parametrize("with_resid", [True, False])
def test_silu_gate_resid_small(bits, with_resid):
    gs, M, N, K = 32, 2, 77, 2048
    g = synth.normal_bf16((M, K), seed=21)
    u = synth.normal_bf16((M, K), seed=22)
    r = synth.normal_bf16((M, N), seed=23) if with_resid else None
    _, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=24)
    y = _silu(g, u, r, w, s, b, M, N, K, bits, gs)
    y_ref, a_ref = oracle.silu_gate_resid(g, u, r, w, s, b, M, N, K, bits, gs)
    check(y, y_ref, a_ref, f"silu bits={bits} resid={with_resid}")


# --------------------------------------------------------------------------
# gather_qmv
# --------------------------------------------------------------------------

def _gather(x, w, s, b, lhs, rhs, P, T, E, N, K, bits, gs, sorted_indices):
    Y = empty_bf16(max(P, 1), N)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    agq.gather_qmv(dev_bf16(x), dev_u32(w), dev_bf16(s), dev_bf16(b),
                   None if lhs is None else dev_u32(lhs), dev_u32(rhs), Y,
                   P, T, E, N, K, bits, gs, sorted_indices=sorted_indices,
                   d_status=status)
    torch.cuda.synchronize()
    return host_bits(Y), int(status.item())


def _moe_inputs(E, N, K, bits, gs, seed, distinct_bias=True):
    x = None
    _, w, s, b = synth.qmv_inputs(1, E * N, K, bits, gs, seed=seed,
                                  bias_offset_per_row_block=(N, 0.03) if distinct_bias else None)
    return w, s, b


def test_gather_moe_workload_sorted_and_unsorted():
    # 64 experts [1536, 2048] 4-bit gs64; 32 tokens, top-4 per token
    E, N, K, bits, gs, T, k = 64, 1536, 2048, 4, 64, 32, 4
    w, s, b = _moe_inputs(E, N, K, bits, gs, seed=5000)
    x = synth.normal_bf16((T, K), seed=5001)
    lhs, rhs = synth.topk_routing(T, E, k, seed=5002)
    P = T * k
    y_u, st_u = _gather(x, w, s, b, lhs, rhs, P, T, E, N, K, bits, gs, False)
    lhs_s, rhs_s, perm = synth.sort_pairs_by_expert(lhs, rhs)
    y_s, st_s = _gather(x, w, s, b, lhs_s, rhs_s, P, T, E, N, K, bits, gs, True)
    assert st_u == 0 and st_s == 0
    # the hint changes nothing: identical bits, rows permuted
    assert np.array_equal(y_s, y_u[perm])
    rows = sample_rows(N, 48, seed=9)
    y_ref, a_ref, valid = oracle.gather(x, w, s, b, lhs, rhs, P, T, E, N, K, bits,
                                        gs, nthreads=8)
    assert valid.all()
    check(y_u[:, rows], y_ref[:, rows], a_ref[:, rows], "gather unsorted")
    # one full row set per 8th pair
    for p in range(0, P, 8):
        check(y_u[p:p + 1], y_ref[p:p + 1], a_ref[p:p + 1], f"gather pair {p}")


@pytest.mark.parametrize("bits, gs", [(2, 64), (3, 64), (4, 64), (5, 64), (6, 64), (8, 64),
                                      (4, 128), (5, 128), (3, 32)])
def test_gather_small_routing(bits, gs):
    E, N, K, T = 9, 70, 512, 6
    w, s, b = _moe_inputs(E, N, K, bits, gs, seed=bits + gs)
    x = synth.normal_bf16((T, K), seed=bits + 1)
    rng = np.random.default_rng(bits + gs)
    P = 23
    lhs = rng.integers(0, T, size=P).astype(np.uint32)
    rhs = rng.integers(0, E, size=P).astype(np.uint32)
    rhs[:5] = 3  # a long run on one expert (several x-row chunks)
    y, st = _gather(x, w, s, b, lhs, rhs, P, T, E, N, K, bits, gs, False)
    assert st == 0
    y_ref, a_ref, valid = oracle.gather(x, w, s, b, lhs, rhs, P, T, E, N, K, bits, gs)
    check(y, y_ref, a_ref, f"gather bits={bits} gs={gs}")


def test_gather_identity_lhs_and_bad_indices():
    E, N, K, bits, gs = 5, 40, 256, 4, 32
    w, s, b = _moe_inputs(E, N, K, bits, gs, seed=77)
    P = 12
    x = synth.normal_bf16((P, K), seed=78)
    rhs = (np.arange(P) * 7 % E).astype(np.uint32)
    y, st = _gather(x, w, s, b, None, rhs, P, P, E, N, K, bits, gs, False)
    y_ref, a_ref, _ = oracle.gather(x, w, s, b, None, rhs, P, P, E, N, K, bits, gs)
    assert st == 0
    check(y, y_ref, a_ref, "gather lhs=None")
    # out-of-range expert and x-row indices: flagged, rows left untouched
    lhs = np.arange(P, dtype=np.uint32)
    bad_rhs = rhs.copy(); bad_rhs[3] = E + 2
    bad_lhs = lhs.copy(); bad_lhs[7] = P + 100
    y2, st2 = _gather(x, w, s, b, bad_lhs, bad_rhs, P, P, E, N, K, bits, gs, False)
    assert st2 == 1
    sentinel = np.uint16(0x7FC1)
    assert np.all(y2[3] == sentinel) and np.all(y2[7] == sentinel)
    keep = [p for p in range(P) if p not in (3, 7)]
    assert np.array_equal(y2[keep], y[keep])


def test_gather_empty_is_a_no_op():
    E, N, K, bits, gs = 2, 16, 64, 4, 64
    w, s, b = _moe_inputs(E, N, K, bits, gs, seed=1)
    x = synth.normal_bf16((1, K), seed=2)
    agq.gather_qmv(dev_bf16(x), dev_u32(w), dev_bf16(s), dev_bf16(b), None,
                   dev_u32(np.zeros(1, np.uint32)), empty_bf16(1, N), 0, 1, E, N,
                   K, bits, gs)
    torch.cuda.synchronize()


@pytest.mark.parametrize("bits", [4, 3])
def test_gather_many_tiny_segments(bits):
    # 2-row experts and thousands of pairs: every CTA walks more tiny tiles
    # than its stage ring holds, and most consumer warps have no row in a
    # tile, so stages are reused while those warps only release them
    E, N, K, gs, T = 16, 2, 128, 64, 512
    w, s, b = _moe_inputs(E, N, K, bits, gs, seed=600 + bits)
    x = synth.normal_bf16((T, K), seed=601)
    rng = np.random.default_rng(602)
    P = 4096
    lhs = rng.integers(0, T, size=P).astype(np.uint32)
    rhs = rng.integers(0, E, size=P).astype(np.uint32)
    y, st = _gather(x, w, s, b, lhs, rhs, P, T, E, N, K, bits, gs, False)
    assert st == 0
    y_ref, a_ref, valid = oracle.gather(x, w, s, b, lhs, rhs, P, T, E, N, K, bits, gs)
    assert valid.all()
    check(y, y_ref, a_ref, f"gather tiny segments bits={bits}")
