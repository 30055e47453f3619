"""Float64 CPU oracle for the NVFP4 decode GEMM -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.  The product path (the CUDA
library and its binding) never does, and shares no code with it.

The arithmetic lives in ``nvfp4_oracle.c`` (plain C, float64, explicit code
tables, sums in k order).  This module compiles it with gcc (-O2, OpenMP, no
fast-math) on first use and wraps it with ctypes.

What it computes (ignis, "Models and artifacts", section "The artifact": a
4-bit floating point body with one scale per 16 values; ignis README, "The
decode round": one pass over the weights serves every lane)::

    Y[m][n] = gscale * sum_k x[m][k] * e2m1(q[n][k]) * e4m3(s[n][k // 16])
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "liboracle.so")
_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/_build/liboracle.so``; return its path."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    lib.or_threads.restype = ctypes.c_int
    lib.or_tables.argtypes = [_P, _P]
    lib.or_count_nan_scales.argtypes = [_P, _I64, _I64]
    lib.or_count_nan_scales.restype = _I64
    lib.or_dequant.argtypes = [_P, _P, _I64, _I64, ctypes.c_float, _P]
    lib.or_gemm.argtypes = [_P, ctypes.c_int, _P, _P, ctypes.c_float, _I64, _I64, _P, _P]
    lib.or_gemm_rows.argtypes = [_P, ctypes.c_int, _P, _P, ctypes.c_float, _I64, _I64,
                                 _P, _I64, _P, _P]
    lib.or_gateup_silu.argtypes = [_P, ctypes.c_int, _P, _P, ctypes.c_float, _P, _P,
                                   ctypes.c_float, _I64, _I64, _P, _P, _P, _P, _P]
    lib.or_topk.argtypes = [_P, ctypes.c_int, _I64, _I64, ctypes.c_int, _P, _P]
    lib.or_topk.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check_planes(q, s, N, K):
    assert q.dtype == np.uint8 and q.shape == (N, K // 2) and q.flags.c_contiguous
    assert s.dtype == np.uint8 and s.shape == (N, K // 16) and s.flags.c_contiguous
    assert K % 16 == 0


def threads() -> int:
    """OpenMP threads the oracle uses."""
    return int(_load().or_threads())


def tables():
    """(E2M1[16], E4M3[256]) as float64 arrays, built from the format definitions."""
    e2 = np.zeros(16, np.float64)
    e4 = np.zeros(256, np.float64)
    _load().or_tables(_ptr(e2), _ptr(e4))
    return e2, e4


def count_nan_scales(s: np.ndarray) -> int:
    N, kb = s.shape
    return int(_load().or_count_nan_scales(_ptr(np.ascontiguousarray(s)), N, kb * 16))


def dequant(q: np.ndarray, s: np.ndarray, gscale: float) -> np.ndarray:
    """fp32 W[N][K] = fp32(e2m1 * e4m3 * gscale)."""
    N = q.shape[0]
    K = q.shape[1] * 2
    _check_planes(q, s, N, K)
    W = np.empty((N, K), np.float32)
    _load().or_dequant(_ptr(q), _ptr(s), N, K, float(gscale), _ptr(W))
    return W


def gemm(X_bits: np.ndarray, q: np.ndarray, s: np.ndarray, gscale: float):
    """(Y, A): Y[M][N] float64 result; A[M][N] = sum_k |x*w| for the tolerance."""
    M, K = X_bits.shape
    N = q.shape[0]
    _check_planes(q, s, N, K)
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    Y = np.empty((M, N), np.float64)
    A = np.empty((M, N), np.float64)
    _load().or_gemm(_ptr(X_bits), M, _ptr(q), _ptr(s), float(gscale), N, K, _ptr(Y), _ptr(A))
    return Y, A


def gemm_rows(X_bits, q, s, gscale, rows):
    """Y and A for the output rows ``rows`` only: arrays of shape [M][len(rows)]."""
    M, K = X_bits.shape
    N = q.shape[0]
    _check_planes(q, s, N, K)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    assert rows.min() >= 0 and rows.max() < N
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    Y = np.empty((M, rows.size), np.float64)
    A = np.empty((M, rows.size), np.float64)
    _load().or_gemm_rows(_ptr(X_bits), M, _ptr(q), _ptr(s), float(gscale), N, K,
                         _ptr(rows), rows.size, _ptr(Y), _ptr(A))
    return Y, A


def gateup_silu(X_bits, qg, sg, gscale_g, qu, su, gscale_u):
    """(G, U, H, AG, AU) in float64: h = silu(g) * u."""
    M, K = X_bits.shape
    Nff = qg.shape[0]
    _check_planes(qg, sg, Nff, K)
    _check_planes(qu, su, Nff, K)
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    out = [np.empty((M, Nff), np.float64) for _ in range(5)]
    _load().or_gateup_silu(_ptr(X_bits), M, _ptr(qg), _ptr(sg), float(gscale_g),
                           _ptr(qu), _ptr(su), float(gscale_u), Nff, K,
                           *[_ptr(o) for o in out])
    return tuple(out)


def gemm_tolerance(A: np.ndarray) -> np.ndarray:
    """Elementwise bound |Y_gpu - Y_oracle| <= 2e-3 * sum_k |x_k w_k| + 1e-6."""
    return 2e-3 * A + 1e-6


def silu_tolerance(G, U, AG, AU, gscale_g=None, gscale_u=None):
    """Bound on |H_gpu - h| for the fused gate/up + SiLU-multiply epilogue.

    The first term covers rounding H to bf16; the others carry the GEMM bound
    of g and u through h = silu(g) * u to first order.
    """
    sig = 1.0 / (1.0 + np.exp(-G))
    silu = G * sig
    dsilu = sig * (1.0 + G * (1.0 - sig))
    h = silu * U
    Bg = gemm_tolerance(AG)
    Bu = gemm_tolerance(AU)
    return 2.0 ** -8 * np.abs(h) + np.abs(dsilu) * np.abs(U) * Bg + np.abs(silu) * Bu + 1e-6


def topk(logits: np.ndarray, k: int, V: int | None = None):
    """Top-k of each row of an FP32 [M][ldv] array over its first V columns.

    ignis README, "What sets it apart", "Speculative decoding (DFlash2)": the
    top-k after the output head.  Returns (vals float32 [M][k], idx int32
    [M][k]), best first: IEEE totalOrder with -0 == +0, equal values by lower
    index.
    """
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    M, ldv = logits.shape
    V = ldv if V is None else int(V)
    vals = np.empty((M, k), np.float32)
    idx = np.empty((M, k), np.int32)
    rc = _load().or_topk(_ptr(logits), M, V, ldv, int(k), _ptr(vals), _ptr(idx))
    if rc != 0:
        raise ValueError(f"oracle topk: bad arguments (M={M}, V={V}, ldv={ldv}, k={k})")
    return vals, idx
