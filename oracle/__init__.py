"""CPU oracle for the GRINQH decode path -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (``input_adaptive_bit_b200``) never does, and it shares no code
with it: the arithmetic lives in ``grinqh_oracle.c`` (plain C, fp64), which
this module compiles with gcc and calls through ctypes.

Every function takes numpy arrays.  fp16 inputs (x, s, z) are passed as their
raw bit patterns (``np.float16`` arrays viewed as ``uint16``); the C code
decodes them itself from the IEEE-754 binary16 definition.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "grinqh_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
# Test hook: the mutation tests point this at a deliberately broken build of the
# oracle to show that the pins catch the planted mistake.
_LIB_OVERRIDE = os.environ.get("GRINQH_ORACLE_LIB_OVERRIDE")

GROUP = 128


def compile_source(src: str, out: str) -> str:
    tmp = out + ".tmp.%d" % os.getpid()
    subprocess.check_call(
        ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-Wall", "-Wextra",
         src, "-o", tmp, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile ``grinqh_oracle.c`` into ``liboracle.so`` beside it (gcc, OpenMP)."""
    if _LIB_OVERRIDE:
        return _LIB_OVERRIDE
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_source(_SRC, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_to_f64.restype = ctypes.c_double
        lib.oracle_phi_default.argtypes = [I, P]
        lib.oracle_assign.argtypes = [P, P, I, I, P]
        lib.oracle_lists.argtypes = [P, I, I, P, P]
        lib.oracle_pack.argtypes = [P, I, I, I, P]
        lib.oracle_unpack.argtypes = [P, I, I, I, P]
        lib.oracle_reconstruct.argtypes = [P, P, P, P, I, I, I, I, I]
        lib.oracle_reconstruct.restype = ctypes.c_double
        lib.oracle_truncated_code.argtypes = [P, I, I, I, I, I]
        lib.oracle_truncated_code.restype = ctypes.c_double
        lib.oracle_gemv.argtypes = [P, P, P, P, P, P, I, I, I, P, I, P, P, I]
        lib.oracle_pack_dense4.argtypes = [P, I, I, P]
        lib.oracle_unpack_dense4.argtypes = [P, I, I, P]
        lib.oracle_gemv_dense4.argtypes = [P, P, P, P, I, I, P, I, P, P, I]
        lib.oracle_max_threads.restype = I
        _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _f16_bits(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    assert a.dtype == np.uint16, a.dtype
    return a


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def f16_to_f64(bits: int) -> float:
    return float(_load().oracle_f16_to_f64(int(bits)))


def phi_default(b_max: int) -> np.ndarray:
    """phi per level k = 0..b_max/2 (bit width 2k); phi[0] is unused."""
    out = np.zeros(b_max // 2 + 1, np.float64)
    _load().oracle_phi_default(b_max, _ptr(out))
    return out


def assign(x, theta, b_max: int) -> np.ndarray:
    x = _f16_bits(x)
    theta = np.ascontiguousarray(theta, np.float32)
    assert theta.shape == (b_max // 2,)
    b = np.zeros(x.shape[0], np.uint8)
    _load().oracle_assign(_ptr(x), _ptr(theta), x.shape[0], b_max, _ptr(b))
    return b


def lists(b, b_max: int):
    """Returns (lists [P][d_in] int32 with -1 past each count, counts [P] int32)."""
    b = np.ascontiguousarray(b, np.uint8)
    P = b_max // 2
    out = np.full((P, b.shape[0]), -1, np.int32)
    counts = np.zeros(P, np.int32)
    _load().oracle_lists(_ptr(b), b.shape[0], b_max, _ptr(out), _ptr(counts))
    return out, counts


def pack(q, b_max: int) -> np.ndarray:
    q = np.ascontiguousarray(q, np.uint8)
    d_in, d_out = q.shape
    P = b_max // 2
    planes = np.zeros((d_in, P, d_out // 16), np.uint32)
    _load().oracle_pack(_ptr(q), d_in, d_out, b_max, _ptr(planes))
    return planes


def unpack(planes, d_out: int, b_max: int) -> np.ndarray:
    planes = np.ascontiguousarray(planes, np.uint32)
    d_in = planes.shape[0]
    q = np.zeros((d_in, d_out), np.uint8)
    _load().oracle_unpack(_ptr(planes), d_in, d_out, b_max, _ptr(q))
    return q


def truncated_code(planes, d_out: int, b_max: int, i: int, o: int, b: int) -> float:
    planes = np.ascontiguousarray(planes, np.uint32)
    return float(_load().oracle_truncated_code(_ptr(planes), d_out, b_max, i, o, b))


def reconstruct(planes, s, z, phi, d_out: int, b_max: int, i: int, o: int, b: int) -> float:
    planes = np.ascontiguousarray(planes, np.uint32)
    s, z = _f16_bits(s), _f16_bits(z)
    phi = np.ascontiguousarray(phi, np.float64)
    return float(_load().oracle_reconstruct(_ptr(planes), _ptr(s), _ptr(z), _ptr(phi),
                                            d_out, b_max, i, o, b))


def gemv(planes, s, z, x, b, b_max: int, phi=None, outs=None, threads: int = 1):
    """fp64 y and its error bound sum_i |w_hat_io||x_i| (all outputs, or ``outs``)."""
    planes = np.ascontiguousarray(planes, np.uint32)
    s, z, x = _f16_bits(s), _f16_bits(z), _f16_bits(x)
    b = np.ascontiguousarray(b, np.uint8)
    d_in = x.shape[0]
    d_out = planes.shape[2] * 16
    phi = phi_default(b_max) if phi is None else np.ascontiguousarray(phi, np.float64)
    if outs is not None:
        outs = np.ascontiguousarray(outs, np.int32)
    n = d_out if outs is None else outs.shape[0]
    y = np.zeros(n, np.float64)
    bound = np.zeros(n, np.float64)
    _load().oracle_gemv(_ptr(planes), _ptr(s), _ptr(z), _ptr(x), _ptr(b), _ptr(phi),
                        d_in, d_out, b_max, _ptr(outs), n, _ptr(y), _ptr(bound), threads)
    return y, bound


def union_widths(X, theta, b_max: int) -> np.ndarray:
    """Small batch ("GRINQH: Graded Input-Based Quantization Hierarchy for
    Efficient LLM Generation", Limitations and outlook: beyond batch 1 the
    requests' active channels differ): every token t of X [B][d_in] gets its own
    widths b^(t) = assign(x_t); a step that rebuilds each weight once for the
    whole batch must read, for row i, the planes of u_i = max_t b_i^(t)."""
    return np.max(np.stack([assign(x, theta, b_max) for x in np.atleast_2d(X)]), axis=0)


def gemv_batch(planes, s, z, X, theta, b_max: int, phi=None, threads: int = 1):
    """The small-batch decode step by its definition: y_t = W_hat(b^(t))^T x_t
    for each token t, each with its own widths (same section as union_widths).
    Returns (Y [B][d_out], bounds [B][d_out], widths [B][d_in])."""
    X = np.atleast_2d(X)
    bs = np.stack([assign(x, theta, b_max) for x in X])
    ys, bounds = [], []
    for x, b in zip(X, bs):
        y, bound = gemv(planes, s, z, x, b, b_max, phi=phi, threads=threads)
        ys.append(y)
        bounds.append(bound)
    return np.stack(ys), np.stack(bounds), bs


def pack_dense4(q4) -> np.ndarray:
    q4 = np.ascontiguousarray(q4, np.uint8)
    d_in, d_out = q4.shape
    w4 = np.zeros((d_in, d_out // 8), np.uint32)
    _load().oracle_pack_dense4(_ptr(q4), d_in, d_out, _ptr(w4))
    return w4


def unpack_dense4(w4, d_out: int) -> np.ndarray:
    w4 = np.ascontiguousarray(w4, np.uint32)
    q4 = np.zeros((w4.shape[0], d_out), np.uint8)
    _load().oracle_unpack_dense4(_ptr(w4), w4.shape[0], d_out, _ptr(q4))
    return q4


def gemv_dense4(w4, s, z, x, outs=None, threads: int = 1):
    w4 = np.ascontiguousarray(w4, np.uint32)
    s, z, x = _f16_bits(s), _f16_bits(z), _f16_bits(x)
    d_in = x.shape[0]
    d_out = w4.shape[1] * 8
    if outs is not None:
        outs = np.ascontiguousarray(outs, np.int32)
    n = d_out if outs is None else outs.shape[0]
    y = np.zeros(n, np.float64)
    bound = np.zeros(n, np.float64)
    _load().oracle_gemv_dense4(_ptr(w4), _ptr(s), _ptr(z), _ptr(x), d_in, d_out,
                               _ptr(outs), n, _ptr(y), _ptr(bound), threads)
    return y, bound


def within_tolerance(y, y_ref, bound, rel: float = 1e-3, abs_: float = 1e-6) -> np.ndarray:
    """Acceptance test of the GEMV: |y - y_ref| <= rel * bound + abs_ per output.

    Where the reference is not finite (an active +-Inf input), the check asks
    only that y is not finite either.
    """
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    bound = np.asarray(bound, np.float64)
    finite = np.isfinite(y_ref) & np.isfinite(bound)
    ok = np.where(finite, np.abs(y - y_ref) <= rel * bound + abs_, ~np.isfinite(y))
    return ok


def effective_bits(b) -> float:
    """Mean assigned bit width over the input channels (s/z overhead excluded)."""
    b = np.asarray(b)
    return float(b.astype(np.float64).mean()) if b.size else 0.0
