"""CPU-only checks of the C ABI: the library builds and loads, exports every
function include/qmv.h declares, and rejects bad arguments on the host with
the documented status codes before touching any device."""
import ctypes
import os
import re

import pytest

import affine_group_quantized_b200 as agq
from affine_group_quantized_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qmv.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return agq.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


def test_header_lists_the_entry_points():
    names = declared_functions()
    assert {"qmv", "qmv_gate_up", "qmv_silu_gate_resid", "gather_qmv",
            "qmv_last_error", "qmv_abi_version", "affine_quantize",
            "affine_dequantize", "qmv_quant_last_error"} <= set(names)
    assert set(agq.EXPORTED) <= set(names)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.qmv_abi_version() == 1


def test_library_is_sm100a_only():
    # the build targets sm_100a only (no PTX for other architectures)
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.FLAGS)


A = 0x10000  # a 16-byte aligned fake device address; never dereferenced


def _status(fn, *args):
    return fn(*args)


def test_qmv_argument_checks(lib):
    q = lib.qmv
    ok_args = [A, A, A, A, A, 1, 64, 128, 4, 64, None]

    def call(**over):
        a = list(ok_args)
        names = ["x", "w", "s", "b", "y", "M", "N", "K", "bits", "gs", "stream"]
        for k, v in over.items():
            a[names.index(k)] = v
        return q(*a)

    assert call(x=None) == agq.QMV_ERR_NULL
    assert call(y=None) == agq.QMV_ERR_NULL
    assert "NULL" in agq.last_error()
    assert call(bits=7) == agq.QMV_ERR_UNSUPPORTED
    assert call(bits=1) == agq.QMV_ERR_UNSUPPORTED
    assert call(gs=16) == agq.QMV_ERR_UNSUPPORTED
    assert call(gs=48) == agq.QMV_ERR_UNSUPPORTED
    assert call(K=96) == agq.QMV_ERR_SHAPE          # not a multiple of 64
    assert "multiple" in agq.last_error()
    assert call(K=0) == agq.QMV_ERR_SHAPE
    assert call(N=0) == agq.QMV_ERR_SHAPE
    assert call(M=0) == agq.QMV_ERR_SHAPE
    assert call(K=65536) == agq.QMV_ERR_UNSUPPORTED
    assert call(x=A + 2) == agq.QMV_ERR_ALIGN
    assert call(w=A + 4) == agq.QMV_ERR_ALIGN
    assert call(y=A + 8) == agq.QMV_ERR_ALIGN


def test_gate_up_argument_checks(lib):
    f = lib.qmv_gate_up
    base = [A] * 9 + [1, 64, 128, 8, 64, None]
    a = list(base); a[4] = None
    assert f(*a) == agq.QMV_ERR_NULL
    a = list(base); a[8] = A + 2
    assert f(*a) == agq.QMV_ERR_ALIGN
    a = list(base); a[13] = 100
    assert f(*a) == agq.QMV_ERR_UNSUPPORTED


def test_silu_argument_checks(lib):
    f = lib.qmv_silu_gate_resid
    base = [A, A, None, A, A, A, A, 1, 64, 128, 8, 64, None]
    a = list(base); a[0] = None
    assert f(*a) == agq.QMV_ERR_NULL
    a = list(base); a[2] = A + 1
    assert f(*a) == agq.QMV_ERR_ALIGN
    a = list(base); a[9] = 100
    assert f(*a) == agq.QMV_ERR_SHAPE


def test_gather_argument_checks(lib):
    f = lib.gather_qmv
    # x w s b lhs rhs y  P T E N K bits gs sorted status stream
    base = [A, A, A, A, A, A, A, 8, 4, 4, 64, 128, 4, 64, 0, None, None]

    def call(i, v):
        a = list(base); a[i] = v
        return f(*a)

    assert call(5, None) == agq.QMV_ERR_NULL          # rhs required
    assert call(7, -1) == agq.QMV_ERR_SHAPE           # num_pairs
    assert call(9, 0) == agq.QMV_ERR_SHAPE            # num_experts
    assert call(4, None) == agq.QMV_ERR_SHAPE         # lhs NULL needs T >= P
    assert call(7, 0) == agq.QMV_OK                   # empty: nothing enqueued
    assert call(5, A + 2) == agq.QMV_ERR_ALIGN
    assert call(12, 9) == agq.QMV_ERR_UNSUPPORTED
    assert call(7, 100000) == agq.QMV_ERR_UNSUPPORTED  # grouping table too big


def test_binding_raises_with_message(lib):
    with pytest.raises(agq.QmvError) as ei:
        agq.qmv(A, A, A, A, A, 1, 64, 100, 4, 64, stream=0)
    assert ei.value.status == agq.QMV_ERR_SHAPE
    assert "group_size" in str(ei.value)


def test_quantize_argument_checks(lib):
    f = lib.affine_quantize
    # w w_q scales biases N K bits gs stream
    base = [A, A, A, A, 4, 128, 4, 64, None]

    def call(i, v):
        a = list(base); a[i] = v
        return f(*a)

    for i in range(4):
        assert call(i, None) == agq.QMV_ERR_NULL
    assert call(6, 7) == agq.QMV_ERR_UNSUPPORTED      # bits
    assert call(7, 16) == agq.QMV_ERR_UNSUPPORTED     # group size
    assert call(4, -1) == agq.QMV_ERR_SHAPE
    assert call(5, 0) == agq.QMV_ERR_SHAPE
    assert call(5, 96) == agq.QMV_ERR_SHAPE           # K % group_size
    for i in range(4):
        assert call(i, A + 8) == agq.QMV_ERR_ALIGN
    assert call(4, 0) == agq.QMV_OK                   # empty: nothing enqueued
    assert "" == agq.lib().qmv_quant_last_error().decode()


def test_dequantize_argument_checks(lib):
    f = lib.affine_dequantize
    # w_q scales biases w_hat N K bits gs stream
    base = [A, A, A, A, 4, 128, 4, 64, None]

    def call(i, v):
        a = list(base); a[i] = v
        return f(*a)

    for i in range(4):
        assert call(i, None) == agq.QMV_ERR_NULL
    assert call(6, 1) == agq.QMV_ERR_UNSUPPORTED
    assert call(7, 256) == agq.QMV_ERR_UNSUPPORTED
    assert call(5, 160) == agq.QMV_ERR_SHAPE
    assert call(3, A + 2) == agq.QMV_ERR_ALIGN
    assert call(4, 0) == agq.QMV_OK


def test_quant_binding_raises_with_its_own_message(lib):
    with pytest.raises(agq.QmvError) as ei:
        agq.affine_quantize(A, A, A, A, 2, 100, 4, 64, stream=0)
    assert ei.value.status == agq.QMV_ERR_SHAPE
    assert "group_size" in str(ei.value)
    with pytest.raises(agq.QmvError) as ei:
        agq.affine_dequantize(A, A, A, A, 2, 128, 9, 64, stream=0)
    assert ei.value.status == agq.QMV_ERR_UNSUPPORTED and "bits=9" in str(ei.value)


def test_qvm_argument_checks(lib):
    q = lib.qvm
    P = ctypes.c_void_p
    q.argtypes = [P, P, P, P, P] + [ctypes.c_int] * 5 + [P]
    ok = [A, A, A, A, A, 1, 128, 256, 4, 64, None]

    def call(i=None, v=None):
        args = list(ok)
        if i is not None:
            args[i] = v
        return q(*args)

    assert call(0, None) == agq.QMV_ERR_NULL
    assert call(8, 7) == agq.QMV_ERR_UNSUPPORTED          # bits
    assert call(9, 48) == agq.QMV_ERR_UNSUPPORTED         # group size
    assert call(7, 200) == agq.QMV_ERR_SHAPE              # N % gs
    assert call(5, 0) == agq.QMV_ERR_SHAPE                # M
    assert call(6, 0) == agq.QMV_ERR_SHAPE                # K
    assert call(1, A + 4) == agq.QMV_ERR_ALIGN


def test_trellis_argument_checks(lib):
    q = lib.qmv_trellis
    P = ctypes.c_void_p
    q.argtypes = [P, P, P, P] + [ctypes.c_int] * 4 + [P]
    ok = [A, A, A, A, 1, 8, 256, 4, None]

    def call(i=None, v=None):
        args = list(ok)
        if i is not None:
            args[i] = v
        return q(*args)

    assert call(2, None) == agq.QMV_ERR_NULL
    assert call(7, 3) == agq.QMV_ERR_UNSUPPORTED          # bits
    assert call(6, 40) == agq.QMV_ERR_SHAPE               # K * bits % 128
    assert call(4, 0) == agq.QMV_ERR_SHAPE                # M
    assert call(0, A + 2) == agq.QMV_ERR_ALIGN
    assert call(2, A + 1) == agq.QMV_ERR_ALIGN             # scales need 2 bytes
