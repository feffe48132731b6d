"""Python binding of libgrinqh (argument marshalling only).

Each function has the name and argument order of the C entry point in
``include/grinqh.h``.  Array arguments may be torch tensors on the GPU (their
``data_ptr()`` is passed) or raw integer device addresses; ``stream`` defaults
to torch's current CUDA stream.  A non-zero status raises ``GrinqhError``.

Every step of the decode path runs in the library's CUDA kernels; this module
never computes anything itself.  If ``libgrinqh.so`` is missing or cannot be
loaded, importing the entry points raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "GrinqhError", "lib", "lib_path", "grinqh_version", "grinqh_last_error",
    "grinqh_workspace_bytes", "grinqh_pack", "grinqh_unpack", "grinqh_assign", "grinqh_gemv",
    "grinqh_check_device_error", "grinqh_pack_dense4", "grinqh_dense4_workspace_bytes",
    "grinqh_gemv_dense4", "grinqh_decode_gemv", "grinqh_decode_gemv_noalloc",
    "grinqh_group_workspace_bytes", "grinqh_decode_gemv_group", "GrinqhLinearDesc", "MAX_GROUP",
    "grinqh_prefill_workspace_bytes", "grinqh_prefill_gemm",
    "grinqh_noalloc_check_device_error", "grinqh_noalloc_scratch",
    "grinqh_batch_workspace_bytes", "grinqh_decode_gemv_batch", "MAX_BATCH",
    "EXPORTS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libgrinqh.so")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED_SHAPE = -2
ERR_WORKSPACE_TOO_SMALL = -3
ERR_CUDA = -4
ERR_DEVICE = -5

MAX_GROUP = 4  # GRINQH_MAX_GROUP
MAX_BATCH = 8  # GRINQH_MAX_BATCH


class GrinqhLinearDesc(ctypes.Structure):
    """struct grinqh_linear: one linear of a grouped decode call (include/grinqh.h)."""
    _fields_ = [("planes", ctypes.c_void_p), ("s", ctypes.c_void_p), ("z", ctypes.c_void_p),
                ("x", ctypes.c_void_p), ("theta", ctypes.c_void_p), ("phi", ctypes.c_void_p),
                ("d_in", ctypes.c_int), ("d_out", ctypes.c_int), ("b_max", ctypes.c_int),
                ("y", ctypes.c_void_p)]


# name -> (restype, argtypes); p = pointer (passed as c_void_p), i = int, z = size_t
_P, _I, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
EXPORTS = {
    "grinqh_version": (_I, []),
    "grinqh_last_error": (ctypes.c_char_p, []),
    "grinqh_workspace_bytes": (_Z, [_I, _I, _I]),
    "grinqh_pack": (_I, [_P, _I, _I, _I, _P, _P]),
    "grinqh_unpack": (_I, [_P, _I, _I, _I, _P, _P]),
    "grinqh_assign": (_I, [_P, _P, _I, _I, _P, _P, _P, _P, _P, _P, _Z, _P]),
    "grinqh_gemv": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _P, _Z, _P]),
    "grinqh_check_device_error": (_I, [_P, _P]),
    "grinqh_pack_dense4": (_I, [_P, _I, _I, _P, _P]),
    "grinqh_dense4_workspace_bytes": (_Z, [_I, _I]),
    "grinqh_gemv_dense4": (_I, [_P, _P, _P, _P, _I, _I, _P, _P, _Z, _P]),
    "grinqh_decode_gemv": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _P, _P, _P,
                                _Z, _P]),
    "grinqh_decode_gemv_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P]),
    "grinqh_noalloc_check_device_error": (_I, [_P]),
    "grinqh_noalloc_scratch": (_I, [_P, _P]),
    "grinqh_batch_workspace_bytes": (_Z, []),
    "grinqh_decode_gemv_batch": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _Z,
                                      _P]),
    "grinqh_group_workspace_bytes": (_Z, []),
    "grinqh_decode_gemv_group": (_I, [_I, _P, _P, _Z, _P]),
    "grinqh_prefill_workspace_bytes": (_Z, []),
    "grinqh_prefill_gemm": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _Z, _P]),
}


class GrinqhError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"libgrinqh status {status}: {message}")
        self.status = status


_lib = None


def lib():
    """The loaded libgrinqh (ctypes.CDLL); raises if it is not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise ImportError(
                f"{lib_path} is missing: build it with `python -m input_adaptive_bit_b200.build` "
                "(there is no CPU fallback)")
        handle = ctypes.CDLL(lib_path)
        for name, (res, args) in EXPORTS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _ptr(a):
    if a is None:
        return None
    if isinstance(a, int):
        return a
    return a.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int):
    if status != OK:
        raise GrinqhError(status, lib().grinqh_last_error().decode())


def grinqh_version() -> int:
    return lib().grinqh_version()


def grinqh_last_error() -> str:
    return lib().grinqh_last_error().decode()


def grinqh_workspace_bytes(d_in: int, d_out: int, b_max: int) -> int:
    return lib().grinqh_workspace_bytes(d_in, d_out, b_max)


def grinqh_dense4_workspace_bytes(d_in: int, d_out: int) -> int:
    return lib().grinqh_dense4_workspace_bytes(d_in, d_out)


def grinqh_pack(q, d_in, d_out, b_max, planes, stream=None):
    _check(lib().grinqh_pack(_ptr(q), d_in, d_out, b_max, _ptr(planes), _stream(stream)))


def grinqh_unpack(planes, d_in, d_out, b_max, q_out, stream=None):
    _check(lib().grinqh_unpack(_ptr(planes), d_in, d_out, b_max, _ptr(q_out), _stream(stream)))


def grinqh_assign(x, theta, d_in, b_max, phi, b, lists, counts, grp_sums, ws, ws_bytes,
                  stream=None):
    _check(lib().grinqh_assign(_ptr(x), _ptr(theta), d_in, b_max, _ptr(phi), _ptr(b),
                               _ptr(lists), _ptr(counts), _ptr(grp_sums), _ptr(ws), ws_bytes,
                               _stream(stream)))


def grinqh_gemv(planes, s, z, grp_sums, d_in, d_out, b_max, y, ws, ws_bytes, stream=None):
    _check(lib().grinqh_gemv(_ptr(planes), _ptr(s), _ptr(z), _ptr(grp_sums), d_in, d_out,
                             b_max, _ptr(y), _ptr(ws), ws_bytes, _stream(stream)))


def grinqh_check_device_error(ws, stream=None):
    _check(lib().grinqh_check_device_error(_ptr(ws), _stream(stream)))


def grinqh_pack_dense4(q4, d_in, d_out, w4, stream=None):
    _check(lib().grinqh_pack_dense4(_ptr(q4), d_in, d_out, _ptr(w4), _stream(stream)))


def grinqh_gemv_dense4(w4, s, z, x, d_in, d_out, y, ws, ws_bytes, stream=None):
    _check(lib().grinqh_gemv_dense4(_ptr(w4), _ptr(s), _ptr(z), _ptr(x), d_in, d_out, _ptr(y),
                                    _ptr(ws), ws_bytes, _stream(stream)))


def grinqh_decode_gemv(planes, s, z, x, theta, phi, d_in, d_out, b_max, y, b, lists, counts,
                       grp_sums, ws, ws_bytes, stream=None):
    """assign + gemv fused into one kernel; b, lists, counts, grp_sums may be None."""
    _check(lib().grinqh_decode_gemv(_ptr(planes), _ptr(s), _ptr(z), _ptr(x), _ptr(theta),
                                    _ptr(phi), d_in, d_out, b_max, _ptr(y), _ptr(b), _ptr(lists),
                                    _ptr(counts), _ptr(grp_sums), _ptr(ws), ws_bytes,
                                    _stream(stream)))


def grinqh_decode_gemv_noalloc(planes, s, z, x, theta, phi, d_in, d_out, b_max, y, stream=None):
    """The fused decode kernel on the library's fixed scratch: for callers that
    cannot allocate device memory (see include/grinqh.h for limits and sharing)."""
    _check(lib().grinqh_decode_gemv_noalloc(_ptr(planes), _ptr(s), _ptr(z), _ptr(x), _ptr(theta),
                                            _ptr(phi), d_in, d_out, b_max, _ptr(y),
                                            _stream(stream)))


def grinqh_noalloc_check_device_error(stream=None):
    """Raises GrinqhError (status ERR_DEVICE) if a no-allocation call recorded a
    device error since the last check; clears it."""
    _check(lib().grinqh_noalloc_check_device_error(_stream(stream)))


def grinqh_noalloc_scratch():
    """(device address, bytes) of the no-allocation path's fixed array on the
    current device (inspection and tests)."""
    ptr, nbytes = ctypes.c_void_p(), ctypes.c_size_t()
    _check(lib().grinqh_noalloc_scratch(ctypes.byref(ptr), ctypes.byref(nbytes)))
    return int(ptr.value or 0), int(nbytes.value)


def grinqh_batch_workspace_bytes() -> int:
    return lib().grinqh_batch_workspace_bytes()


def grinqh_decode_gemv_batch(planes, s, z, x, theta, phi, B, d_in, d_out, b_max, y, u, ws,
                             ws_bytes, stream=None):
    """B <= 8 tokens (x fp16 [B][d_in]) through one linear, each with its own widths;
    y fp32 [B][d_out]; u (uint8 [d_in] union widths) may be None."""
    _check(lib().grinqh_decode_gemv_batch(_ptr(planes), _ptr(s), _ptr(z), _ptr(x), _ptr(theta),
                                          _ptr(phi), B, d_in, d_out, b_max, _ptr(y), _ptr(u),
                                          _ptr(ws), ws_bytes, _stream(stream)))


def grinqh_group_workspace_bytes() -> int:
    return lib().grinqh_group_workspace_bytes()


def grinqh_decode_gemv_group(lins, ws, ws_bytes, stream=None):
    """Several independent linears in one launch.  `lins` is a sequence of
    (planes, s, z, x, theta, phi, d_in, d_out, b_max, y) tuples (phi may be None)."""
    arr = (GrinqhLinearDesc * max(1, len(lins)))()
    for j, (planes, s, z, x, theta, phi, d_in, d_out, b_max, y) in enumerate(lins):
        arr[j] = GrinqhLinearDesc(_ptr(planes), _ptr(s), _ptr(z), _ptr(x), _ptr(theta), _ptr(phi),
                                  d_in, d_out, b_max, _ptr(y))
    _check(lib().grinqh_decode_gemv_group(len(lins), ctypes.cast(arr, ctypes.c_void_p), _ptr(ws),
                                          ws_bytes, _stream(stream)))


def grinqh_prefill_workspace_bytes() -> int:
    return lib().grinqh_prefill_workspace_bytes()


def grinqh_prefill_gemm(planes, s, z, x, phi, T, d_in, d_out, b_max, y, ws, ws_bytes, stream=None):
    """Y[T][d_out] = X[T][d_in] times the full-width w_hat (the prefill GEMM)."""
    _check(lib().grinqh_prefill_gemm(_ptr(planes), _ptr(s), _ptr(z), _ptr(x), _ptr(phi), T, d_in,
                                     d_out, b_max, _ptr(y), _ptr(ws), ws_bytes, _stream(stream)))
