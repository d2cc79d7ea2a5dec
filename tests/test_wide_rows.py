"""GPU parity for rows longer than 14336 codes, up to the largest K the
library accepts (28672).

Past K = 14336 each consumer thread of the streaming kernel owns two 32-code
units of the row (four rows per thread per tile); at K = 28672 an 8-bit row
is 28 KB and a single stage of four rows fills the ring.  Every case compares
all outputs with the oracle.
"""
import pytest

from affine_group_quantized_b200 import synth
import oracle
from tests._parity import check
from tests.test_parity_fused import _silu
from tests.test_parity_qmv import run_qmv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bits, gs, K", [(4, 32, 14368), (3, 64, 28672), (4, 128, 28672),
                                         (8, 32, 28672), (2, 64, 20480)])
@pytest.mark.parametrize("M", [1, 2])
def test_qmv_wide_rows_up_to_the_maximum_K(bits, gs, K, M):
    N = 70
    x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=K + bits + M)
    y = run_qmv(x, w, s, b, M, N, K, bits, gs)
    y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs, nthreads=8)
    check(y, y_ref, a_ref, f"wide K={K} bits={bits} gs={gs} M={M}")


@pytest.mark.parametrize("bits", [4, 6])
def test_silu_gate_resid_wide_rows(bits):
    gs, M, N, K = 64, 1, 90, 20480
    g = synth.normal_bf16((M, K), seed=31)
    u = synth.normal_bf16((M, K), seed=32)
    r = synth.normal_bf16((M, N), seed=33)
    _, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=34)
    y = _silu(g, u, r, w, s, b, M, N, K, bits, gs)
    y_ref, a_ref = oracle.silu_gate_resid(g, u, r, w, s, b, M, N, K, bits, gs, nthreads=8)
    check(y, y_ref, a_ref, f"silu wide K={K} bits={bits}")
