"""CPU oracle for the W4A16 group-128 linear layer -- TEST INFRASTRUCTURE.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package.  It is a plain, slow, obviously correct restatement of what the
layer computes, in fp64, on the canonical (unpacked) arrays, written from
"PerfXLLM on Snapdragon 8 Gen2":

* section 3.1 (low-precision quantisation): weight-only int4 quantisation,
  group_size 128, one scale and one zero per group.  Reading taken:
  w = fp16_RN((q - z) * s), the product exact, one rounding to fp16.
* the step before it, the group quantiser fp16 W -> (q, s, z) (section 3.1
  names int4, group 128, a scale and a zero, but no rounding rule): min-max
  asymmetric with 0 inside the range, every decision in IEEE fp32 (see
  ``quantize``).
* section 3.2, first fusion (residual addition and normalisation as one
  operator), the step that produces X: r = fp16_RN(h + d) and
  x = r * gamma / sqrt(eps + mean(r^2)) per token row (see ``add_rmsnorm``).
* the gate/up projection's epilogue, SiLU(gate) * up (an extension of the
  fusion principle of section 3.2; see ``gate_up``).
* section 3.3 item 1: C[m, n] = sum_k A[m, k] B[k, n] with A the weights and n
  the tokens; item 2: the GEMV is the n = 1 case.  Storage taken: x[n][k],
  y[n][m] (token-major), sums in fp64, ascending k.

It shares no code with the CUDA library and does not import it.  The C source
is ``w4a16_oracle.c``; this module is argument marshalling over ctypes.

Every function here is pinned by ``tests/test_oracle_pins.py`` against
brute-force exact rational arithmetic, numpy's IEEE fp16 conversion, numpy's
fp64 matmul and closed-form special cases.
"""
from __future__ import annotations

import ctypes
import threading

import numpy as np

from . import build as _build

_lib = None
_lock = threading.Lock()

_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i64 = ctypes.c_int64


def lib():
    """Load (building first if needed) the oracle shared library."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            L = ctypes.CDLL(path)
            L.w4o_fp16_to_double.argtypes = [ctypes.c_uint16]
            L.w4o_fp16_to_double.restype = ctypes.c_double
            L.w4o_fp16_from_double.argtypes = [ctypes.c_double]
            L.w4o_fp16_from_double.restype = ctypes.c_uint16
            L.w4o_fp16_from_double_array.argtypes = [_f64p, _u16p, _i64]
            L.w4o_fp16_to_double_array.argtypes = [_u16p, _f64p, _i64]
            L.w4o_set_threads.argtypes = [ctypes.c_int]
            L.w4o_get_threads.restype = ctypes.c_int
            L.w4o_dequant.argtypes = [_u8p, _u8p, _u16p, _i64, _i64, _i64, _u16p]
            L.w4o_dequant.restype = ctypes.c_int
            L.w4o_gemm.argtypes = [_u8p, _u8p, _u16p, _u16p, _i64, _i64, _i64,
                                   _i64, _f64p]
            L.w4o_gemm.restype = ctypes.c_int
            L.w4o_gemm_rows.argtypes = [_u8p, _u8p, _u16p, _u16p, _i64, _i64,
                                        _i64, _i64, _i64p, _i64, _f64p]
            L.w4o_gemm_rows.restype = ctypes.c_int
            L.w4o_quantize.argtypes = [_u16p, _i64, _i64, _i64, _u8p, _u16p, _u8p]
            L.w4o_quantize.restype = ctypes.c_int
            L.w4o_add_rmsnorm.argtypes = [_u16p, _u16p, _u16p, ctypes.c_double, _i64, _i64, _u16p, _f64p]
            L.w4o_add_rmsnorm.restype = ctypes.c_int
            _lib = L
    return _lib


def _ptr(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return a


def set_threads(n: int) -> None:
    lib().w4o_set_threads(int(n))


def get_threads() -> int:
    return int(lib().w4o_get_threads())


def fp16_to_double(bits) -> np.ndarray:
    """fp16 bit patterns -> exact float64 values."""
    b = _c(np.asarray(bits, dtype=np.uint16), np.uint16)
    out = np.empty(b.shape, dtype=np.float64)
    lib().w4o_fp16_to_double_array(_ptr(b, _u16p), _ptr(out, _f64p), b.size)
    return out


def fp16_from_double(x) -> np.ndarray:
    """float64 -> fp16 bit patterns, IEEE round-to-nearest-even."""
    a = _c(np.asarray(x, dtype=np.float64), np.float64)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().w4o_fp16_from_double_array(_ptr(a, _f64p), _ptr(out, _u16p), a.size)
    return out


def _check(q, zeros, scales, group):
    q = _c(q, np.uint8)
    zeros = _c(zeros, np.uint8)
    scales = _c(scales, np.uint16)
    M, K = q.shape
    if K % group or zeros.shape != (M, K // group) or scales.shape != zeros.shape:
        raise ValueError("inconsistent shapes")
    return q, zeros, scales, M, K


def dequant(q, zeros, scales, group: int = 128) -> np.ndarray:
    """W[m, k] as fp16 bit patterns, uint16 [M, K]."""
    q, zeros, scales, M, K = _check(q, zeros, scales, group)
    W = np.empty((M, K), dtype=np.uint16)
    rc = lib().w4o_dequant(_ptr(q, _u8p), _ptr(zeros, _u8p), _ptr(scales, _u16p),
                           M, K, group, _ptr(W, _u16p))
    if rc:
        raise RuntimeError(f"oracle dequant failed ({rc})")
    return W


def gemm(q, zeros, scales, x, group: int = 128) -> np.ndarray:
    """Y[n, m] = sum_k W[m, k] x[n, k] in fp64; float64 [N, M]."""
    q, zeros, scales, M, K = _check(q, zeros, scales, group)
    x = _c(x, np.uint16)
    N = x.shape[0]
    if x.shape != (N, K):
        raise ValueError("x must be [N, K]")
    y = np.empty((N, M), dtype=np.float64)
    rc = lib().w4o_gemm(_ptr(q, _u8p), _ptr(zeros, _u8p), _ptr(scales, _u16p),
                        _ptr(x, _u16p), M, K, N, group, _ptr(y, _f64p))
    if rc:
        raise RuntimeError(f"oracle gemm failed ({rc})")
    return y


def gemm_rows(q, zeros, scales, x, rows, group: int = 128) -> np.ndarray:
    """Only the output rows in ``rows``: float64 [N, len(rows)]."""
    q, zeros, scales, M, K = _check(q, zeros, scales, group)
    x = _c(x, np.uint16)
    N = x.shape[0]
    if x.shape != (N, K):
        raise ValueError("x must be [N, K]")
    r = _c(np.asarray(rows, dtype=np.int64), np.int64)
    y = np.empty((N, r.size), dtype=np.float64)
    rc = lib().w4o_gemm_rows(_ptr(q, _u8p), _ptr(zeros, _u8p), _ptr(scales, _u16p),
                             _ptr(x, _u16p), M, K, N, group, _ptr(r, _i64p),
                             r.size, _ptr(y, _f64p))
    if rc:
        raise RuntimeError(f"oracle gemm_rows failed ({rc})")
    return y


def quantize(W, group: int = 128):
    """Group quantiser: W fp16 bit patterns uint16 [M, K] -> (q uint8 [M, K],
    scales fp16 bits uint16 [M, K/group], zeros uint8 [M, K/group]).

    Per (row, group): lo = min(0, min w), hi = max(0, max w); r = hi - lo
    raised to 2^-14; s = fp16_RN(r / 15); f = 1 / s; z = clamp(rint(-lo f),
    0, 15); q = clamp(rint(w f) + z, 0, 15) -- each step one IEEE fp32
    operation, round to nearest even (reading of "PerfXLLM on Snapdragon 8
    Gen2", section 3.1, which fixes int4, group 128, scale and zero only)."""
    W = _c(W, np.uint16)
    if W.ndim != 2:
        raise ValueError("W must be [M, K]")
    M, K = W.shape
    if group <= 0 or K % group:
        raise ValueError("K must be a multiple of group")
    q = np.empty((M, K), dtype=np.uint8)
    scales = np.empty((M, K // group), dtype=np.uint16)
    zeros = np.empty((M, K // group), dtype=np.uint8)
    rc = lib().w4o_quantize(_ptr(W, _u16p), M, K, group, _ptr(q, _u8p), _ptr(scales, _u16p),
                            _ptr(zeros, _u8p))
    if rc:
        raise RuntimeError(f"oracle quantize failed ({rc})")
    return q, scales, zeros


def add_rmsnorm(h, gamma, eps: float, d=None):
    """Residual add and RMS normalisation per token row (reading of "PerfXLLM
    on Snapdragon 8 Gen2", section 3.2, first fusion): r = fp16_RN(h + d)
    (d None: r = h) and x = r * gamma / sqrt(eps + mean_k r^2).

    h, d: fp16 bit patterns uint16 [N, K]; gamma: uint16 [K].  Returns
    (r uint16 [N, K] fp16 bits, x float64 [N, K] unrounded)."""
    h = _c(h, np.uint16)
    if h.ndim != 2:
        raise ValueError("h must be [N, K]")
    N, K = h.shape
    gamma = _c(gamma, np.uint16).reshape(-1)
    if gamma.size != K:
        raise ValueError("gamma must hold K values")
    dp = None
    if d is not None:
        d = _c(d, np.uint16)
        if d.shape != h.shape:
            raise ValueError("d must match h")
        dp = _ptr(d, _u16p)
    r = np.empty((N, K), dtype=np.uint16)
    x = np.empty((N, K), dtype=np.float64)
    rc = lib().w4o_add_rmsnorm(_ptr(h, _u16p), dp, _ptr(gamma, _u16p), float(eps), N, K,
                               _ptr(r, _u16p), _ptr(x, _f64p))
    if rc:
        raise RuntimeError(f"oracle add_rmsnorm failed ({rc})")
    return r, x


def silu_mul(y, Mi: int) -> np.ndarray:
    """H[n][i] = silu(g) * u with g = y[n][i], u = y[n][Mi + i] and
    silu(g) = g / (1 + exp(-g)), all in fp64 (y: [N, 2 Mi] float64, e.g. the
    accumulators of ``gemm`` on a weight whose rows are the gate projection's
    Mi rows followed by the up projection's Mi rows)."""
    y = np.asarray(y, dtype=np.float64)
    if y.ndim != 2 or y.shape[1] != 2 * Mi or Mi <= 0:
        raise ValueError("y must be [N, 2 Mi]")
    g, u = y[:, :Mi], y[:, Mi:]
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g)) * u


def gate_up(q, zeros, scales, x, Mi: int, group: int = 128) -> np.ndarray:
    """The gate/up layer's output SiLU(X W_gate^T) * (X W_up^T) in fp64, for a
    canonical weight of 2 Mi rows: rows [0, Mi) the gate projection, rows
    [Mi, 2 Mi) the up projection (reading of "PerfXLLM on Snapdragon 8 Gen2",
    section 3.2: fusion removes the intermediate's round trip through global
    memory; the page names no such fusion for the feed-forward block, the
    principle is extended to it).  Returns [N, Mi]."""
    if np.asarray(q).shape[0] != 2 * Mi:
        raise ValueError("the weight must have 2 Mi rows")
    return silu_mul(gemm(q, zeros, scales, x, group), Mi)
