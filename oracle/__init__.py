"""ctypes wrapper around the plain-C CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this module.  The product
package never imports it and shares no code with it.

All bf16 arrays are numpy ``uint16`` bit patterns; packed weights are numpy
``uint32``.  Results are numpy ``float64``.  Each function returns
``(y, a)`` where ``a[m, n] = sum_k |v[m, k] * w_hat[n, k]|`` is the magnitude
sum that scales the acceptance tolerance.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        L.oracle_bf16_to_double.restype = ctypes.c_double
        L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_silu.restype = ctypes.c_double
        L.oracle_silu.argtypes = [ctypes.c_double]
        L.oracle_check_shape.argtypes = [I, I, I, I]
        L.oracle_row_bytes.restype = ctypes.c_longlong
        L.oracle_row_bytes.argtypes = [I, I]
        L.oracle_unpack.argtypes = [P, I, I, I, P]
        L.oracle_dequant.argtypes = [P, P, P, I, I, I, I, P]
        L.oracle_qmv.argtypes = [P, P, P, P, I, I, I, I, I, P, I, P, P, I]
        L.oracle_gate_up.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I,
                                     P, P, P, P, I]
        L.oracle_silu_gate_resid.argtypes = [P, P, P, P, P, P, I, I, I, I, I,
                                             P, I, P, P, I]
        L.oracle_gather.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I,
                                    P, P, P, I]
        L.oracle_bf16_round.restype = ctypes.c_uint16
        L.oracle_bf16_round.argtypes = [ctypes.c_double, ctypes.c_double]
        L.oracle_dequantize_bf16.argtypes = [P, P, P, I, I, I, I, P]
        L.oracle_affine_quantize.argtypes = [P, I, I, I, I, P, P, P]
        L.oracle_qvm.argtypes = [P, P, P, P, I, I, I, I, I, P, P]
        L.oracle_trellis_value.restype = ctypes.c_double
        L.oracle_trellis_value.argtypes = [ctypes.c_uint32]
        L.oracle_trellis_state.restype = ctypes.c_uint32
        L.oracle_trellis_state.argtypes = [ctypes.c_uint32, ctypes.c_uint32, I, I]
        L.oracle_qmv_trellis.argtypes = [P, P, P, I, I, I, I, P, P]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=dtype)


def _threads(nthreads):
    return int(nthreads) if nthreads else 1


def bf16_to_double(h: int) -> float:
    return lib().oracle_bf16_to_double(int(h))


def silu(g: float) -> float:
    return lib().oracle_silu(float(g))


def check_shape(N, K, bits, gs) -> bool:
    return lib().oracle_check_shape(N, K, bits, gs) == 0


def unpack(w, N, K, bits):
    w = _c(w, np.uint32)
    out = np.zeros((N, K), dtype=np.uint8)
    if lib().oracle_unpack(_p(w), N, K, bits, _p(out)):
        raise ValueError("oracle_unpack: bad arguments")
    return out


def dequant(w, scales, biases, N, K, bits, gs):
    w, s, b = _c(w, np.uint32), _c(scales, np.uint16), _c(biases, np.uint16)
    out = np.zeros((N, K), dtype=np.float64)
    if lib().oracle_dequant(_p(w), _p(s), _p(b), N, K, bits, gs, _p(out)):
        raise ValueError("oracle_dequant: bad arguments")
    return out


def qmv(x, w, scales, biases, M, N, K, bits, gs, rows=None, nthreads=1):
    x, w = _c(x, np.uint16), _c(w, np.uint32)
    s, b = _c(scales, np.uint16), _c(biases, np.uint16)
    r = _c(rows, np.int32)
    nr = N if r is None else len(r)
    y = np.zeros((M, nr), dtype=np.float64)
    a = np.zeros((M, nr), dtype=np.float64)
    if lib().oracle_qmv(_p(x), _p(w), _p(s), _p(b), M, N, K, bits, gs, _p(r),
                        nr, _p(y), _p(a), _threads(nthreads)):
        raise ValueError("oracle_qmv: bad arguments")
    return y, a


def gate_up(x, wg, sg, bg, wu, su, bu, M, N, K, bits, gs, nthreads=1):
    arrs = [_c(x, np.uint16), _c(wg, np.uint32), _c(sg, np.uint16),
            _c(bg, np.uint16), _c(wu, np.uint32), _c(su, np.uint16),
            _c(bu, np.uint16)]
    yg = np.zeros((M, N)); ag = np.zeros((M, N))
    yu = np.zeros((M, N)); au = np.zeros((M, N))
    if lib().oracle_gate_up(*[_p(t) for t in arrs], M, N, K, bits, gs,
                            _p(yg), _p(ag), _p(yu), _p(au),
                            _threads(nthreads)):
        raise ValueError("oracle_gate_up: bad arguments")
    return (yg, ag), (yu, au)


def silu_gate_resid(gate, up, x_resid, w, scales, biases, M, N, K, bits, gs,
                    rows=None, nthreads=1):
    g, u = _c(gate, np.uint16), _c(up, np.uint16)
    xr = _c(x_resid, np.uint16)
    w, s, b = _c(w, np.uint32), _c(scales, np.uint16), _c(biases, np.uint16)
    r = _c(rows, np.int32)
    nr = N if r is None else len(r)
    y = np.zeros((M, nr)); a = np.zeros((M, nr))
    if lib().oracle_silu_gate_resid(_p(g), _p(u), _p(xr), _p(w), _p(s), _p(b),
                                    M, N, K, bits, gs, _p(r), nr, _p(y), _p(a),
                                    _threads(nthreads)):
        raise ValueError("oracle_silu_gate_resid: bad arguments")
    return y, a


def gather(x, w, scales, biases, lhs, rhs, num_pairs, num_x_rows, E, N, K,
           bits, gs, nthreads=1):
    """Returns (y, a, valid): valid[p] == 0 marks a pair with an index out
    of range (its rows of y and a are left at zero)."""
    x, w = _c(x, np.uint16), _c(w, np.uint32)
    s, b = _c(scales, np.uint16), _c(biases, np.uint16)
    l, r = _c(lhs, np.uint32), _c(rhs, np.uint32)
    y = np.zeros((num_pairs, N)); a = np.zeros((num_pairs, N))
    valid = np.zeros(num_pairs, dtype=np.int32)
    rc = lib().oracle_gather(_p(x), _p(w), _p(s), _p(b), _p(l), _p(r),
                             num_pairs, num_x_rows, E, N, K, bits, gs, _p(y),
                             _p(a), _p(valid), _threads(nthreads))
    if rc < 0:
        raise ValueError("oracle_gather: bad arguments")
    return y, a, valid


def bf16_round(hi: float, lo: float = 0.0) -> int:
    """bf16 bit pattern nearest to the exact sum hi + lo (ties to even)."""
    return int(lib().oracle_bf16_round(float(hi), float(lo)))


def dequantize_bf16(w, scales, biases, N, K, bits, gs):
    """bf16 [N, K] bit patterns of scale * q + bias, rounded once."""
    w, s, b = _c(w, np.uint32), _c(scales, np.uint16), _c(biases, np.uint16)
    out = np.zeros((N, K), dtype=np.uint16)
    if lib().oracle_dequantize_bf16(_p(w), _p(s), _p(b), N, K, bits, gs,
                                    _p(out)):
        raise ValueError("oracle_dequantize_bf16: bad arguments")
    return out


def affine_quantize(w, N, K, bits, gs):
    """bf16 [N, K] weights -> (packed uint32 [N, K*bits/32], bf16 scales
    [N, K/gs], bf16 biases [N, K/gs]), computed in binary32."""
    w = _c(w, np.uint16)
    wq = np.zeros((N, K * bits // 32), dtype=np.uint32)
    s = np.zeros((N, K // gs), dtype=np.uint16)
    b = np.zeros((N, K // gs), dtype=np.uint16)
    if lib().oracle_affine_quantize(_p(w), N, K, bits, gs, _p(wq), _p(s),
                                    _p(b)):
        raise ValueError("oracle_affine_quantize: bad arguments")
    return wq, s, b


def qvm(x, w, scales, biases, M, K, N, bits, gs):
    """y[M, N] = x[M, K] @ dequant(w) for a packed w of K rows of N codes
    (scales/biases [K, N/gs]); returns (y, a) as qmv does."""
    x, w = _c(x, np.uint16), _c(w, np.uint32)
    s, b = _c(scales, np.uint16), _c(biases, np.uint16)
    y = np.zeros((M, N)); a = np.zeros((M, N))
    if lib().oracle_qvm(_p(x), _p(w), _p(s), _p(b), M, K, N, bits, gs, _p(y), _p(a)):
        raise ValueError("oracle_qvm: bad arguments")
    return y, a


def trellis_value(state: int) -> float:
    """Value of a 16-bit trellis state (the pages' inst3)."""
    return lib().oracle_trellis_value(int(state))


def trellis_state(w0: int, w1: int, t: int, bits: int) -> int:
    """State of value t of word w0 with successor word w1."""
    return int(lib().oracle_trellis_state(int(w0), int(w1), int(t), int(bits)))


def qmv_trellis(x, w, scales, M, N, K, bits):
    """Trellis-mode y[M, N] = scale * x @ V.T (scale = scales[0]); returns
    (y, a) with a = |scale| * sum_k |x * v|."""
    x, w, s = _c(x, np.uint16), _c(w, np.uint32), _c(scales, np.uint16)
    y = np.zeros((M, N)); a = np.zeros((M, N))
    if lib().oracle_qmv_trellis(_p(x), _p(w), _p(s), M, N, K, bits, _p(y), _p(a)):
        raise ValueError("oracle_qmv_trellis: bad arguments")
    return y, a
