"""CPU model of the index arithmetic of the affine_quantize and
affine_dequantize kernels (qmv_quant.cu), checked against the buffers they
touch and against the packed layout.

The model repeats each kernel's chunk arithmetic in numpy: which packed
words a dequantize chunk loads and how it shifts out its 8 codes, which
lanes share a quantize group, where the group's scale and bias go and which
bytes a quantize chunk stores.  It asserts that every access stays inside
its buffer, that the grid-stride loops visit every chunk once, and that the
codes read or written are those of the layout (built here with the
test-side packer, independently of the kernels and of the oracle).  Shapes
include matrices whose chunk count is not a multiple of a warp's 32 chunks.
"""
import numpy as np
import pytest

from tests._codes import pack

ALL_BITS = (2, 3, 4, 5, 6, 8)
SHAPES = [(1, 32), (3, 64), (37, 128), (5, 384), (64, 256), (7, 4096)]


def _gs_ok(K, gs):
    return K % gs == 0


@pytest.mark.parametrize("bits", ALL_BITS)
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_dequantize_units_read_their_codes(bits, gs):
    # a dequantize unit is 32 codes: words [u*bits, (u+1)*bits) of the packed
    # stream; code i of the unit is bits [i*bits, (i+1)*bits) of those words
    # (a funnel shift of words j, j+1 where it straddles them); its group is
    # (32u) >> gs_shift and its output is the 64 bytes of elements [32u, 32u+32)
    gs_shift = {32: 5, 64: 6, 128: 7}[gs]
    rng = np.random.default_rng(bits * 131 + gs)
    mask = (1 << bits) - 1
    for N, K in SHAPES:
        if not _gs_ok(K, gs):
            continue
        codes = rng.integers(0, 1 << bits, size=(N, K))
        words = pack(codes, bits).reshape(-1).astype(np.uint64)
        nunits = N * K // 32
        assert nunits * 32 == N * K
        u = np.arange(nunits, dtype=np.int64)
        first = u * bits
        assert (first + bits - 1).max() < words.size        # loads stay inside
        # the widest aligned loads: 16 bytes for 4/8-bit, 8 for 2/6, 4 for 3/5
        align = 16 if bits % 4 == 0 else 8 if bits % 2 == 0 else 4
        assert np.all((first * 4) % align == 0)
        got = np.zeros((nunits, 32), dtype=np.int64)
        for i in range(32):
            o = i * bits
            j, sh = o >> 5, o & 31
            lo = words[first + j] >> np.uint64(sh)
            if sh + bits > 32:
                assert j + 1 < bits                          # the next word is the unit's
                lo |= words[first + j + 1] << np.uint64(32 - sh)
            got[:, i] = (lo & np.uint64(mask)).astype(np.int64)
        assert np.array_equal(got.reshape(N, K), codes)
        g = (u * 32) >> gs_shift
        assert g.max() < N * (K // gs)
        assert np.array_equal(g, (u * 32) // gs)
        # a unit never spans two groups
        assert np.array_equal(((u * 32 + 31) >> gs_shift), g)


@pytest.mark.parametrize("units, grid, per_block", [
    (1, 1, 256), (301, 2, 256), (4097, 3, 8), (100001, 888, 8), (7, 888, 256)])
def test_dequantize_two_units_per_pass_visit_each_unit_once(units, grid, per_block):
    # thread t takes units u0 = t + 2*stride*k and u0 + stride (when below
    # the count) on pass k
    stride = grid * per_block
    seen = np.zeros(units, dtype=np.int64)
    for t in range(stride):
        u0 = t
        while u0 < units:
            seen[u0] += 1
            if u0 + stride < units:
                seen[u0 + stride] += 1
            u0 += 2 * stride
    assert (seen == 1).all()


def _grid_stride_visits(n_items, grid, per_block):
    seen = np.zeros(n_items, dtype=np.int64)
    stride = grid * per_block
    for t in range(stride):
        seen[t::stride] += 1
    return seen


@pytest.mark.parametrize("items, grid, per_block", [
    (1, 1, 256), (300, 2, 256), (4097, 3, 8), (100000, 888, 8), (7, 888, 256)])
def test_grid_stride_loops_visit_each_item_once(items, grid, per_block):
    assert (_grid_stride_visits(items, grid, per_block) == 1).all()


@pytest.mark.parametrize("bits", ALL_BITS)
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_quantize_lanes_groups_and_stores(bits, gs):
    lanes = gs // 8
    rng = np.random.default_rng(bits * 17 + gs)
    for N, K in SHAPES:
        if not _gs_ok(K, gs):
            continue
        nchunks = N * K // 8
        ngroups = N * K // gs
        nbytes = N * K * bits // 8
        codes = rng.integers(0, 1 << bits, size=(N, K)).reshape(-1)
        out = np.zeros(nbytes, dtype=np.uint8)
        written = np.zeros(nbytes, dtype=np.int64)
        sgroups = np.zeros(ngroups, dtype=np.int64)
        nwork = (nchunks + 31) // 32
        # a warp takes items wi and wi + warps per pass; every item is visited
        # once whatever the warp count
        for warps in (1, 3, 8):
            seen = np.zeros(nwork, dtype=np.int64)
            for w0 in range(warps):
                for wi in range(w0, nwork, 2 * warps):
                    seen[wi] += 1
                    if wi + warps < nwork:
                        seen[wi + warps] += 1
            assert (seen == 1).all()
        for wi in range(nwork):
            c = wi * 32 + np.arange(32)
            live = c < nchunks
            # a group's lanes are consecutive, start on a multiple of `lanes`
            # and are all live or all past the end
            grp_live = live.reshape(32 // lanes, lanes)
            assert np.all(grp_live.all(axis=1) | (~grp_live).all(axis=1))
            for lane in np.flatnonzero(live):
                cc = int(c[lane])
                # xor partners used by the reductions stay in the group
                for o in (1, 2, 4, 8)[: int(np.log2(lanes))]:
                    assert (lane ^ o) // lanes == lane // lanes
                if lane % lanes == 0:
                    g = cc // lanes
                    assert g == cc * 8 // gs and g < ngroups
                    sgroups[g] += 1
                packed = 0
                for i in range(8):
                    packed |= int(codes[cc * 8 + i]) << (bits * i)
                b0 = cc * bits
                assert b0 + bits <= nbytes
                if bits in (2, 4, 8):
                    assert b0 % bits == 0          # aligned 2/4/8-byte store
                if bits == 6:
                    assert b0 % 2 == 0             # three 2-byte stores
                for i in range(bits):
                    out[b0 + i] = (packed >> (8 * i)) & 0xFF
                    written[b0 + i] += 1
        assert (written == 1).all() and (sgroups == 1).all()
        want = pack(codes.reshape(N, K), bits).reshape(-1).view(np.uint8)
        assert np.array_equal(out, want)
