"""CPU model of the schedule, tensor-memory and shared-memory arithmetic of the
many-row tensor-core kernel (qmv_qmm.cu) and of the staged qvm kernel
(qmv_qvm.cuh), checked against the ranges and buffers they touch.

The model repeats each kernel's integer arithmetic in Python:
  * the stream-K ranges (qmm_start / qmm_owner): every (tile, stage) step is
    in exactly one CTA's range, owners invert starts, a CTA holds at most two
    part tiles (its first and its last segment, slots 0 and 1), and with
    whole-tile units no tile is split;
  * the split of a segment's chunks between the MMA issuers and the number of
    accumulators the epilogue adds;
  * the tensor-memory plan (A buffers below the accumulators, all inside 512
    columns) and the host's shared-memory plan for every column block;
  * the staged qvm's cluster row split, its 64-row stages and the scale
    window index of every lane.
"""
import pytest

SMEM_OPTIN = 232448        # bytes of shared memory a B200 CTA may opt into
MMA_ROWS, KC = 128, 128    # weight rows per tile, k per MMA chunk
MAX_STAGES, MAX_X, MAX_ABUFS = 16, 8, 7


# ---- the many-row kernel ----------------------------------------------------

def shape(mc):
    issuers = 1 if mc >= 128 else 2
    dcols = 2 * issuers * mc
    abufs = min(7, (512 - dcols) // 64)
    return issuers, dcols, abufs, abufs * 64


def q_start(i, nsteps, gran, grid):
    return (i * (nsteps // gran) // grid) * gran


def q_owner(v, nsteps, gran, grid):
    u, nu = v // gran, nsteps // gran
    return ((u + 1) * grid - 1) // nu


@pytest.mark.parametrize("tiles, nstage, grid, whole", [
    (3, 8, 24, False), (8, 16, 128, False), (224, 32, 148, False), (157, 4, 148, False),
    (1, 1, 1, False), (40, 3, 148, False), (224, 32, 148, True), (300, 5, 148, True),
])
def test_stream_k_ranges_cover_every_step_once(tiles, nstage, grid, whole):
    nsteps = tiles * nstage
    gran = nstage if whole else 1
    grid = min(grid, nsteps // gran)
    seen = [0] * nsteps
    for i in range(grid):
        v0, v1 = q_start(i, nsteps, gran, grid), q_start(i + 1, nsteps, gran, grid)
        assert v0 < v1                                   # every CTA has work
        for v in range(v0, v1):
            seen[v] += 1
            assert q_owner(v, nsteps, gran, grid) == i
        # segments: the CTA's steps inside one tile; part tiles (not whole)
        # only at the range's ends, slot 0 for the first, 1 for the last
        slots = []
        t = v0 // nstage
        while t * nstage < v1:
            ts = t * nstage
            lo, hi = max(v0, ts), min(v1, ts + nstage)
            if not (lo == ts and hi == ts + nstage):
                assert lo == v0 or hi == v1
                slots.append(0 if v0 >= ts else 1)
            t += 1
        assert len(slots) == len(set(slots)) <= 2
        if whole:
            assert slots == []
    assert seen == [1] * nsteps


@pytest.mark.parametrize("mc", [16, 32, 64, 128])
def test_issuers_and_accumulators(mc):
    issuers, dcols, abufs, dcol = shape(mc)
    assert abufs >= 4 and dcol + dcols <= 512 and abufs * 64 <= dcol
    # accumulator of issuer i in buffer db: inside [dcol, 512), disjoint
    cols = set()
    for db in range(2):
        for i in range(issuers):
            c0 = dcol + (db * issuers + i) * mc
            span = set(range(c0, c0 + mc))
            assert not (span & cols) and max(span) < 512
            cols |= span
    # a segment of n chunks: chunk jj goes to issuer jj % issuers; the
    # epilogue adds the first min(issuers, n) accumulators, which are exactly
    # the issuers with chunks, each of whose first chunk (jj < issuers)
    # overwrites its accumulator
    for n in range(1, 12):
        with_chunks = {jj % issuers for jj in range(n)}
        used = min(issuers, n)
        assert with_chunks == set(range(used))
        for i in with_chunks:
            assert min(jj for jj in range(n) if jj % issuers == i) < issuers


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("mc", [16, 32, 64, 128])
def test_shared_memory_plan(bits, mc):
    stage_bytes = MMA_ROWS * 128 + 2 * MMA_ROWS * 16 * 2   # codes, scale, bias windows
    xbytes = mc * 256
    room = SMEM_OPTIN - 1024 - 1024
    nxs = min(MAX_X, max(3, (room * 2 // 5) // xbytes))
    nst = min(MAX_STAGES, (room - nxs * xbytes) // stage_bytes)
    assert nst >= 2
    smem = 1024 + 1024 + nxs * xbytes + nst * stage_bytes
    assert smem <= SMEM_OPTIN
    # the rings start 1024-aligned within the first 2048 bytes, so the last
    # stage ends inside the allocation whatever the base's alignment
    for base in (0, 16, 1008, 1024):
        xring = (base + 1024 + 1023) // 1024 * 1024
        end = xring + nxs * xbytes + nst * stage_bytes
        assert end <= base + smem
        assert xring % 1024 == 0 and xbytes % 1024 == 0 and stage_bytes % 1024 == 0
    # a stage's chunks and the x slot's two 64-k boxes
    codes_per_stage = 128 * 8 // bits
    assert codes_per_stage % KC == 0
    assert (mc * 128) % 1024 == 0              # the second box stays 1024-aligned


# ---- the staged qvm ----------------------------------------------------------

@pytest.mark.parametrize("K", [1, 7, 70, 1000, 4099, 14336])
@pytest.mark.parametrize("ncl", [8, 16])
def test_qvm_rows_split_and_stages(K, ncl):
    rows = [0] * K
    xrows = (K + 8 - 1) // 8 + 1                     # activations held per CTA
    for rank in range(ncl):
        k0, k1 = K * rank // ncl, K * (rank + 1) // ncl
        assert k1 - k0 <= xrows
        nstg = (k1 - k0 + 63) // 64
        for j in range(nstg):
            kr = k0 + 64 * j
            for r in range(64):
                k = kr + r
                if k >= k1:
                    break
                rows[k] += 1
    assert rows == [1] * K


@pytest.mark.parametrize("gs", [32, 64, 128])
def test_qvm_scale_window_index(gs):
    shift = {32: 5, 64: 6, 128: 7}[gs]
    for nb in range(64):
        gwin = ((nb * 256) >> shift) & ~7
        for lane in range(32):
            c = nb * 32 + lane
            gl = ((8 * c) >> shift) - gwin
            assert 0 <= gl < 8                       # inside the 8-group window
