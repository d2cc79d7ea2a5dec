"""Python binding of libqmv, the B200 (sm_100a) affine group-quantized GEMV.

Argument marshalling only: every function here forwards to the C entry point
of the same name in ``libqmv.so`` (declared in ``include/qmv.h``) and every
step of the computation runs in that library's CUDA kernels.  There is no
CPU path: if ``libqmv.so`` is missing or no CUDA device is usable, calls
raise.

Arguments may be ``torch.Tensor`` (CUDA, contiguous; the data pointer is
passed) or plain integer device addresses.  bf16 buffers are ``torch.bfloat16``
tensors (or any 2-byte dtype holding bf16 bit patterns), packed weights are
``torch.int32``/``torch.uint32`` tensors.  ``stream`` defaults to the current
torch CUDA stream.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqmv.so")

QMV_OK = 0
QMV_ERR_NULL = 1
QMV_ERR_SHAPE = 2
QMV_ERR_UNSUPPORTED = 3
QMV_ERR_ALIGN = 4
QMV_ERR_CUDA = 5

_STATUS_NAMES = {0: "QMV_OK", 1: "QMV_ERR_NULL", 2: "QMV_ERR_SHAPE",
                 3: "QMV_ERR_UNSUPPORTED", 4: "QMV_ERR_ALIGN", 5: "QMV_ERR_CUDA"}


class QmvError(RuntimeError):
    """A libqmv entry point returned a nonzero status."""

    def __init__(self, func: str, status: int, message: str):
        self.status = status
        super().__init__(f"{func}: {_STATUS_NAMES.get(status, status)}: {message}")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libqmv.so (built in-tree by ``affine_group_quantized_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m affine_group_quantized_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        P, I = ctypes.c_void_p, ctypes.c_int
        L.qmv.argtypes = [P, P, P, P, P, I, I, I, I, I, P]
        L.qmv_noalloc.argtypes = [P, P, P, P, P, I, I, I, I, I, P]
        L.qmv_gate_up.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, P]
        L.qmv_silu_gate_resid.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, P]
        L.gather_qmv.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I,
                                 P, P]
        for f in (L.qmv, L.qmv_noalloc, L.qmv_gate_up, L.qmv_silu_gate_resid, L.gather_qmv):
            f.restype = I
        L.qmv_last_error.restype = ctypes.c_char_p
        L.qmv_last_error.argtypes = []
        L.qmv_abi_version.restype = I
        L.qmv_abi_version.argtypes = []
        L.qvm.argtypes = [P, P, P, P, P, I, I, I, I, I, P]
        L.qmv_trellis.argtypes = [P, P, P, P, I, I, I, I, P]
        L.qmv_trellis.restype = I
        L.qvm.restype = I
        L.qmv_device_status.argtypes = [P, I, P]
        L.qmv_device_status.restype = I
        L.affine_quantize.argtypes = [P, P, P, P, I, I, I, I, P]
        L.affine_dequantize.argtypes = [P, P, P, P, I, I, I, I, P]
        L.affine_quantize.restype = I
        L.affine_dequantize.restype = I
        L.qmv_quant_last_error.restype = ctypes.c_char_p
        L.qmv_quant_last_error.argtypes = []
        _lib = L
    return _lib


EXPORTED = ("qmv", "qmv_noalloc", "qvm", "qmv_trellis", "qmv_gate_up", "qmv_silu_gate_resid", "gather_qmv",
            "qmv_last_error", "qmv_abi_version", "qmv_device_status", "affine_quantize",
            "affine_dequantize", "qmv_quant_last_error")


def _ptr(a):
    if a is None:
        return None
    if isinstance(a, int):
        return a
    return a.data_ptr()


def _need(name, t, nbytes):
    """A tensor argument must hold at least the bytes the call reads or
    writes (plain integer addresses are the caller's responsibility)."""
    if t is None or isinstance(t, int):
        return
    have = t.numel() * t.element_size()
    if have < nbytes:
        raise ValueError(f"{name}: {have} bytes, the call needs {nbytes}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


def _need_qmv(rows, codes, bits, gs, **arrays):
    """Sizes of a packed weight set: w [rows, codes*bits/32] uint32, scales
    and biases [rows, codes/gs] bf16."""
    _need("w", arrays.get("w"), rows * codes * bits // 8)
    for k in ("scales", "biases"):
        _need(k, arrays.get(k), 2 * rows * (codes // max(gs, 1)))


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(func: str, rc: int):
    if rc != QMV_OK:
        raise QmvError(func, rc, lib().qmv_last_error().decode())


def _check_quant(func: str, rc: int):
    if rc != QMV_OK:
        raise QmvError(func, rc, lib().qmv_quant_last_error().decode())


def last_error() -> str:
    return lib().qmv_last_error().decode()


def abi_version() -> int:
    return lib().qmv_abi_version()


def device_status(reset=False, stream=None) -> int:
    """The current device's kernel status word (0, or 2 if a bounded wait in
    some kernel gave up since the last reset); synchronizes `stream`."""
    out = ctypes.c_int(-1)
    _check("qmv_device_status", lib().qmv_device_status(ctypes.byref(out), 1 if reset else 0,
                                                        _stream(stream)))
    return out.value


def qmv(x, w, scales, biases, y, M, N, K, bits, group_size, stream=None):
    """y[M,N] = x[M,K] @ dequant(w).T  (see include/qmv.h)."""
    _need("x", x, 2 * M * K); _need("y", y, 2 * M * N)
    _need_qmv(N, K, bits, group_size, w=w, scales=scales, biases=biases)
    _check("qmv", lib().qmv(_ptr(x), _ptr(w), _ptr(scales), _ptr(biases),
                            _ptr(y), M, N, K, bits, group_size, _stream(stream)))


def qmv_noalloc(x, w, scales, biases, y, M, N, K, bits, group_size, stream=None):
    """qmv without device allocation by the library (see include/qmv.h)."""
    _need("x", x, 2 * M * K); _need("y", y, 2 * M * N)
    _need_qmv(N, K, bits, group_size, w=w, scales=scales, biases=biases)
    _check("qmv_noalloc", lib().qmv_noalloc(_ptr(x), _ptr(w), _ptr(scales), _ptr(biases),
                                            _ptr(y), M, N, K, bits, group_size,
                                            _stream(stream)))


def qvm(x, w, scales, biases, y, M, K, N, bits, group_size, stream=None):
    """y[M,N] = x[M,K] @ dequant(w) for w of K rows of N codes (see include/qmv.h)."""
    _need("x", x, 2 * M * K); _need("y", y, 2 * M * N)
    _need_qmv(K, N, bits, group_size, w=w, scales=scales, biases=biases)
    _check("qvm", lib().qvm(_ptr(x), _ptr(w), _ptr(scales), _ptr(biases), _ptr(y),
                            M, K, N, bits, group_size, _stream(stream)))


def qmv_trellis(x, w, scales, y, M, N, K, bits, stream=None):
    """Trellis-mode y[M,N] = scales[0] * x @ V.T (see include/qmv.h)."""
    _need("x", x, 2 * M * K); _need("y", y, 2 * M * N)
    _need("w", w, N * K * bits // 8); _need("scales", scales, 2)
    _check("qmv_trellis", lib().qmv_trellis(_ptr(x), _ptr(w), _ptr(scales), _ptr(y),
                                            M, N, K, bits, _stream(stream)))


def qmv_gate_up(x, w_gate, s_gate, b_gate, w_up, s_up, b_up, y_gate, y_up,
                M, N, K, bits, group_size, stream=None):
    """y_gate = x @ dequant(w_gate).T and y_up = x @ dequant(w_up).T, one launch."""
    _need("x", x, 2 * M * K); _need("y_gate", y_gate, 2 * M * N); _need("y_up", y_up, 2 * M * N)
    _need_qmv(N, K, bits, group_size, w=w_gate, scales=s_gate, biases=b_gate)
    _need_qmv(N, K, bits, group_size, w=w_up, scales=s_up, biases=b_up)
    _check("qmv_gate_up", lib().qmv_gate_up(
        _ptr(x), _ptr(w_gate), _ptr(s_gate), _ptr(b_gate), _ptr(w_up),
        _ptr(s_up), _ptr(b_up), _ptr(y_gate), _ptr(y_up), M, N, K, bits,
        group_size, _stream(stream)))


def qmv_silu_gate_resid(gate, up, x_resid, w, scales, biases, y, M, N, K,
                        bits, group_size, stream=None):
    """y = x_resid + dequant(w) @ (silu(gate) * up); x_resid may be None."""
    _need("gate", gate, 2 * M * K); _need("up", up, 2 * M * K); _need("y", y, 2 * M * N)
    _need("x_resid", x_resid, 2 * M * N)
    _need_qmv(N, K, bits, group_size, w=w, scales=scales, biases=biases)
    _check("qmv_silu_gate_resid", lib().qmv_silu_gate_resid(
        _ptr(gate), _ptr(up), _ptr(x_resid), _ptr(w), _ptr(scales),
        _ptr(biases), _ptr(y), M, N, K, bits, group_size, _stream(stream)))


def gather_qmv(x, w, scales, biases, lhs_indices, rhs_indices, y, num_pairs,
               num_x_rows, num_experts, N, K, bits, group_size,
               sorted_indices=False, d_status=None, stream=None):
    """y[p] = x[lhs[p]] @ dequant(w[rhs[p]]).T for every pair p."""
    _need("x", x, 2 * num_x_rows * K); _need("y", y, 2 * num_pairs * N)
    _need("lhs_indices", lhs_indices, 4 * num_pairs); _need("rhs_indices", rhs_indices, 4 * num_pairs)
    _need_qmv(num_experts * N, K, bits, group_size, w=w, scales=scales, biases=biases)
    _check("gather_qmv", lib().gather_qmv(
        _ptr(x), _ptr(w), _ptr(scales), _ptr(biases), _ptr(lhs_indices),
        _ptr(rhs_indices), _ptr(y), num_pairs, num_x_rows, num_experts, N, K,
        bits, group_size, 1 if sorted_indices else 0, _ptr(d_status),
        _stream(stream)))


def affine_quantize(w, w_q, scales, biases, N, K, bits, group_size, stream=None):
    """Quantize bf16 w[N,K] into packed w_q and bf16 scales/biases [N,K/gs]."""
    _need("w", w, 2 * N * K)
    _need_qmv(N, K, bits, group_size, w=w_q, scales=scales, biases=biases)
    _check_quant("affine_quantize", lib().affine_quantize(
        _ptr(w), _ptr(w_q), _ptr(scales), _ptr(biases), N, K, bits, group_size,
        _stream(stream)))


def affine_dequantize(w_q, scales, biases, w_hat, N, K, bits, group_size,
                      stream=None):
    """w_hat[N,K] = bf16(scale * q + bias) from the packed format."""
    _need("w_hat", w_hat, 2 * N * K)
    _need_qmv(N, K, bits, group_size, w=w_q, scales=scales, biases=biases)
    _check_quant("affine_dequantize", lib().affine_dequantize(
        _ptr(w_q), _ptr(scales), _ptr(biases), _ptr(w_hat), N, K, bits,
        group_size, _stream(stream)))
