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
def test_dequantize_chunks_read_their_codes(bits, gs):
    gs_shift = {32: 5, 64: 6, 128: 7}[gs]
    rng = np.random.default_rng(bits * 131 + gs)
    for N, K in SHAPES:
        if not _gs_ok(K, gs):
            continue
        codes = rng.integers(0, 1 << bits, size=(N, K))
        words = pack(codes, bits).reshape(-1).astype(np.uint64)
        nwords = words.size
        nchunks = N * K // 8
        c = np.arange(nchunks, dtype=np.int64)
        byte0 = c * bits
        w0 = byte0 >> 2
        off = byte0 & 3
        need2 = off + bits > 4
        assert w0.max() < nwords
        assert (w0[need2] + 1).max(initial=0) < nwords
        # the chunk's bytes lie inside the words it loads
        last_byte = byte0 + bits - 1
        assert np.all((last_byte >> 2) == np.where(need2, w0 + 1, w0))
        v = words[w0].copy()
        v[need2] |= words[w0[need2] + 1] << np.uint64(32)
        v >>= (8 * off).astype(np.uint64)
        mask = np.uint64((1 << bits) - 1)
        got = np.stack([(v >> np.uint64(bits * i)) & mask for i in range(8)], axis=1)
        assert np.array_equal(got.reshape(N, K), codes)
        g = (c * 8) >> gs_shift
        assert g.max() < N * (K // gs)
        assert np.array_equal(g, (c * 8) // gs)
        # the 16-byte output vector of chunk c covers elements [8c, 8c + 8)
        assert (c.max() + 1) * 8 == N * K


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
