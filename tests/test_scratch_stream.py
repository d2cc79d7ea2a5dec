"""The tensor-core path's first call in a process, made on a non-default
stream: the scratch it allocates is cleared on that stream, so the split-tile
sums of the very first launch are right.  Runs in a fresh Python process,
where no earlier call has created the scratch."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import numpy as np, torch
import affine_group_quantized_b200 as agq
from affine_group_quantized_b200 import synth
import oracle
from tests._parity import check, dev_bf16, dev_u32, empty_bf16, host_bits
torch.cuda.set_device(0)
# more 128-row tiles than SMs: the stream-K walk splits tiles between CTAs
M, N, K, bits, gs = 4, 148 * 128 + 300, 2048, 4, 64
x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=4242)
st = torch.cuda.Stream()
with torch.cuda.stream(st):
    X, W, S, B = dev_bf16(x), dev_u32(w), dev_bf16(s), dev_bf16(b)
    Y = empty_bf16(M, N)
    agq.qmv(X, W, S, B, Y, M, N, K, bits, gs)
st.synchronize()
rows = np.unique(np.r_[np.arange(0, 256), np.arange(N - 256, N),
                       np.random.default_rng(1).integers(0, N, 256)]).astype(np.int32)
y_ref, a_ref = oracle.qmv(x, w, s, b, M, N, K, bits, gs, rows=rows, nthreads=8)
check(host_bits(Y)[:, rows], y_ref, a_ref, "first split-tile call on a side stream")
print("ok")
"""


def test_first_split_tile_call_on_a_side_stream():
    env = dict(os.environ, PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr
