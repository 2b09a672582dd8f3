"""FP64 CPU oracle for the block-scaled NVFP4 matmul (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The GPU library never imports it and
shares no code with it: the arithmetic lives in ``nvfp4_oracle.c`` (plain C,
FP64, decode by table, one function per output element), built here with gcc.

What each function computes follows the metrale_circuit ``hardware::exec``
module doc (bullets 1 and 2): the NVFP4 block-scaled product

    Y[m,n] = gA*gW * sum_g sA[m,g]*sW[n,g] * sum_{k in g} e2m1(A[m,k])*e2m1(W[n,k])

and its sibling paths (the exact E2M1->E4M3 FP8 path, the BF16-widen W4A16
path, and W4A8: FP8 activations under NVFP4 weights on the exact E4M3 path).  Layouts: packed codes ``uint8[rows, K/2]`` (even k in the low
nibble), E4M3 scales ``uint8[rows, K/16]``, BF16 as ``uint16`` bits.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB = os.path.join(_HERE, "libnvfp4_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
            "-ffp-contract=off", "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            D = ctypes.c_double
            lib.oracle_e2m1_value.argtypes = [ctypes.c_int]
            lib.oracle_e2m1_value.restype = D
            lib.oracle_e4m3_value.argtypes = [ctypes.c_int]
            lib.oracle_e4m3_value.restype = D
            lib.oracle_e2m1_to_e4m3_word.argtypes = [ctypes.c_uint32]
            lib.oracle_e2m1_to_e4m3_word.restype = ctypes.c_uint32
            dense = [P, P, D, P, P, D, I64, I64, I64, P, ctypes.c_int]
            at = [P, P, D, P, P, D, I64, I64, I64, P, P, I64, P, ctypes.c_int]
            for name, args in (("oracle_gemm_w4a4", dense), ("oracle_gemm_w4a4_at", at),
                               ("oracle_gemm_via_fp8", dense), ("oracle_gemm_via_fp8_at", at)):
                getattr(lib, name).argtypes = args
                getattr(lib, name).restype = ctypes.c_int
            lib.oracle_gemm_w4a8.argtypes = [P, D, P, P, D, I64, I64, I64, P, ctypes.c_int]
            lib.oracle_gemm_w4a8.restype = ctypes.c_int
            lib.oracle_gemm_w4a8_at.argtypes = [P, D, P, P, D, I64, I64, I64, P, P, I64, P,
                                                ctypes.c_int]
            lib.oracle_gemm_w4a8_at.restype = ctypes.c_int
            lib.oracle_gemm_w4a16.argtypes = [P, P, P, D, I64, I64, I64, P, ctypes.c_int]
            lib.oracle_gemm_w4a16.restype = ctypes.c_int
            lib.oracle_gemm_w4a16_at.argtypes = [P, P, P, D, I64, I64, I64, P, P, I64, P,
                                                 ctypes.c_int]
            lib.oracle_gemm_w4a16_at.restype = ctypes.c_int
            lib.oracle_gemm_grouped_w4a4.argtypes = [P, P, D, P, P, P, P, I64, I64, I64, P,
                                                     ctypes.c_int]
            lib.oracle_gemm_grouped_w4a4.restype = ctypes.c_int
            lib.oracle_gemm_grouped_w4a4_at.argtypes = [P, P, D, P, P, P, P, I64, I64, I64,
                                                        P, P, I64, P, ctypes.c_int]
            lib.oracle_gemm_grouped_w4a4_at.restype = ctypes.c_int
            _lib = lib
    return _lib


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _u8(x, shape=None) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.uint8)
    if shape is not None and x.shape != tuple(shape):
        raise ValueError(f"expected shape {tuple(shape)}, got {x.shape}")
    return x


def _ptr(x: np.ndarray):
    return x.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int):
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (code {rc})")


# --- format tables ---------------------------------------------------------------

def e2m1_value(code: int) -> float:
    return _load().oracle_e2m1_value(int(code))


def e4m3_value(byte: int) -> float:
    return _load().oracle_e4m3_value(int(byte))


def e2m1_to_e4m3_word(q: int) -> int:
    """The page-1 bit identity on a 32-bit word of four high-nibble codes."""
    return int(_load().oracle_e2m1_to_e4m3_word(int(q) & 0xFFFFFFFF))


# --- GEMMs -----------------------------------------------------------------------

def _pairs(rows, cols):
    r = np.ascontiguousarray(rows, dtype=np.int64).ravel()
    c = np.ascontiguousarray(cols, dtype=np.int64).ravel()
    if r.shape != c.shape:
        raise ValueError("rows and cols must have the same length")
    return r, c


def gemm_w4a4(A, sA, gA, W, sW, gW, M, N, K, rows=None, cols=None, threads=None):
    """FP64 W4A4 NVFP4 product.  Dense [M,N] if rows/cols are None, else Y at (rows[i], cols[i])."""
    return _dense_or_at("oracle_gemm_w4a4", A, sA, gA, W, sW, gW, M, N, K, rows, cols, threads)


def gemm_via_fp8(A, sA, gA, W, sW, gW, M, N, K, rows=None, cols=None, threads=None):
    """FP64 evaluation along the exact E2M1->E4M3 FP8 path; equals gemm_w4a4 exactly."""
    return _dense_or_at("oracle_gemm_via_fp8", A, sA, gA, W, sW, gW, M, N, K, rows, cols,
                        threads)


def _dense_or_at(name, A, sA, gA, W, sW, gW, M, N, K, rows, cols, threads):
    lib = _load()
    t = threads or default_threads()
    A = _u8(A, (M, K // 2)); W = _u8(W, (N, K // 2))
    sA = _u8(sA, (M, K // 16)); sW = _u8(sW, (N, K // 16))
    if rows is None:
        Y = np.empty((M, N), dtype=np.float64)
        _check(getattr(lib, name)(_ptr(A), _ptr(sA), float(gA), _ptr(W), _ptr(sW), float(gW),
                                  M, N, K, _ptr(Y), t))
        return Y
    r, c = _pairs(rows, cols)
    out = np.empty(r.shape, dtype=np.float64)
    _check(getattr(lib, name + "_at")(_ptr(A), _ptr(sA), float(gA), _ptr(W), _ptr(sW),
                                      float(gW), M, N, K, _ptr(r), _ptr(c), r.size, _ptr(out), t))
    return out


def gemm_w4a8(A_fp8, gA, W, sW, gW, M, N, K, rows=None, cols=None, threads=None):
    """FP64 W4A8: E4M3 activation bytes [M,K] (per-tensor scale gA) times NVFP4 W."""
    lib = _load()
    t = threads or default_threads()
    A = _u8(A_fp8, (M, K))
    W = _u8(W, (N, K // 2)); sW = _u8(sW, (N, K // 16))
    if rows is None:
        Y = np.empty((M, N), dtype=np.float64)
        _check(lib.oracle_gemm_w4a8(_ptr(A), float(gA), _ptr(W), _ptr(sW), float(gW), M, N, K,
                                    _ptr(Y), t))
        return Y
    r, c = _pairs(rows, cols)
    out = np.empty(r.shape, dtype=np.float64)
    _check(lib.oracle_gemm_w4a8_at(_ptr(A), float(gA), _ptr(W), _ptr(sW), float(gW), M, N, K,
                                   _ptr(r), _ptr(c), r.size, _ptr(out), t))
    return out


def gemm_w4a16(A_bf16_bits, W, sW, gW, M, N, K, rows=None, cols=None, threads=None):
    """FP64 W4A16: BF16 activations (given as uint16 bit patterns [M,K]) times NVFP4 W."""
    lib = _load()
    t = threads or default_threads()
    A = np.ascontiguousarray(A_bf16_bits, dtype=np.uint16)
    if A.shape != (M, K):
        raise ValueError(f"expected A shape {(M, K)}, got {A.shape}")
    W = _u8(W, (N, K // 2)); sW = _u8(sW, (N, K // 16))
    if rows is None:
        Y = np.empty((M, N), dtype=np.float64)
        _check(lib.oracle_gemm_w4a16(_ptr(A), _ptr(W), _ptr(sW), float(gW), M, N, K, _ptr(Y), t))
        return Y
    r, c = _pairs(rows, cols)
    out = np.empty(r.shape, dtype=np.float64)
    _check(lib.oracle_gemm_w4a16_at(_ptr(A), _ptr(W), _ptr(sW), float(gW), M, N, K, _ptr(r),
                                    _ptr(c), r.size, _ptr(out), t))
    return out


def gemm_grouped_w4a4(A, sA, gA, W, sW, gW, offsets, N, K, rows=None, cols=None, threads=None):
    """FP64 grouped W4A4: W is [E,N,K/2], sW [E,N,K/16], gW [E], offsets [E+1] (rows of A)."""
    lib = _load()
    t = threads or default_threads()
    off = np.ascontiguousarray(offsets, dtype=np.int64)
    E = off.size - 1
    M = int(off[-1])
    A = _u8(A, (M, K // 2)); sA = _u8(sA, (M, K // 16))
    W = _u8(W, (E, N, K // 2)); sW = _u8(sW, (E, N, K // 16))
    g = np.ascontiguousarray(gW, dtype=np.float64)
    if g.shape != (E,):
        raise ValueError("gW must hold one value per expert")
    if rows is None:
        Y = np.empty((M, N), dtype=np.float64)
        _check(lib.oracle_gemm_grouped_w4a4(_ptr(A), _ptr(sA), float(gA), _ptr(W), _ptr(sW),
                                            _ptr(g), _ptr(off), E, N, K, _ptr(Y), t))
        return Y
    r, c = _pairs(rows, cols)
    out = np.empty(r.shape, dtype=np.float64)
    _check(lib.oracle_gemm_grouped_w4a4_at(_ptr(A), _ptr(sA), float(gA), _ptr(W), _ptr(sW),
                                           _ptr(g), _ptr(off), E, N, K, _ptr(r), _ptr(c), r.size,
                                           _ptr(out), t))
    return out
