"""CPU oracle for the NVFP4 / fp8r quantized linear (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
path (``block_scaled_precision_act_b200``) never imports it and shares no code
with it.

The arithmetic lives in ``bsp_oracle.c`` (plain C11, explicit E2M1/E4M3 bit
tables, one IEEE binary32 operation per step, fp64 matmul).  This module only
marshals numpy arrays through ctypes.  Every function cites the passage it
follows in the C source; the readings the pages leave open are listed there.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
(closed forms from the bit definitions, an independent arithmetic encoder,
a library cast, invariants, brute-force fp64 sums).  Nothing is unpinned.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i64 = ctypes.c_int64


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e2m1_decode.restype = ctypes.c_float
        L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        L.oracle_e2m1_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_decode.restype = ctypes.c_float
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_encode_range.argtypes = [ctypes.c_int, ctypes.c_uint32, ctypes.c_int64,
                                          ctypes.c_void_p]
        L.oracle_encode_range.restype = None
        L.oracle_sf_bytes.argtypes = [_i64, _i64, ctypes.c_int]
        L.oracle_sf_bytes.restype = _i64
        L.oracle_sf_mma_offset.argtypes = [_i64, _i64, _i64]
        L.oracle_sf_mma_offset.restype = _i64
        L.oracle_sf_linear_to_mma.argtypes = [_u8p, _i64, _i64, _u8p]
        L.oracle_amax_bf16.argtypes = [_u16p, _i64]
        L.oracle_amax_bf16.restype = ctypes.c_float
        L.oracle_nvfp4_global_scale.argtypes = [_u16p, _i64]
        L.oracle_nvfp4_global_scale.restype = ctypes.c_float
        L.oracle_nvfp4_quantize.argtypes = [_u16p, _i64, _i64, ctypes.c_float, _u8p, _u8p,
                                            ctypes.c_int]
        L.oracle_nvfp4_dequant.argtypes = [_u8p, _u8p, _i64, _i64, ctypes.c_double, _f64p]
        L.oracle_nvfp4_dequant_bf16.argtypes = [_u8p, _u8p, _i64, _i64, ctypes.c_float, _u16p]
        L.oracle_fp8r_quantize.argtypes = [_u16p, _i64, _i64, _u8p, _f32p, ctypes.c_int]
        L.oracle_gemm_f64.argtypes = [_f64p, _f64p, _f64p, ctypes.c_double, _i64p, _i64,
                                      _i64, _i64, _f64p, ctypes.c_int]
        L.oracle_nvfp4_linear.argtypes = [_u8p, _u8p, ctypes.c_float, _u8p, _u8p,
                                          ctypes.c_float, _f64p, _i64p, _i64, _i64, _i64,
                                          _i64, _f64p, _f64p, _f64p, ctypes.c_int]
        L.oracle_fp8r_linear.argtypes = [_u8p, _f32p, _u8p, _f32p, _f64p, _i64p, _i64,
                                         _i64, _i64, _i64, _f64p, _f64p, _f64p,
                                         ctypes.c_int]
        L.oracle_max_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray, t):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(t)


def _as_u16(x) -> np.ndarray:
    """bf16 input as its raw uint16 bit pattern (numpy uint16 array or torch bf16 tensor)."""
    if type(x).__module__.startswith("torch"):
        import torch
        assert x.dtype == torch.bfloat16, "oracle inputs are bf16"
        return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(x)
    assert a.dtype == np.uint16, "pass bf16 as uint16 bit patterns"
    return a


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


# ---------------------------------------------------------------- codecs
def e2m1_decode(code: int) -> float:
    return float(lib().oracle_e2m1_decode(code))


def e2m1_encode(y: float) -> int:
    return int(lib().oracle_e2m1_encode(np.float32(y)))


def e4m3_decode(code: int) -> float:
    return float(lib().oracle_e4m3_decode(code))


def e4m3_encode(y: float) -> int:
    return int(lib().oracle_e4m3_encode(np.float32(y)))


def encode_range(kind: int, first: int, n: int) -> np.ndarray:
    """Codes of the fp32 values with bit patterns first .. first+n-1 (kind 0: E2M1,
    1: E4M3), the scalar encoders applied one by one."""
    out = np.empty(n, dtype=np.uint8)
    lib().oracle_encode_range(kind, first, n, out.ctypes.data)
    return out


# ---------------------------------------------------------------- scale layouts
def sf_bytes(R: int, K: int, mma: bool) -> int:
    return int(lib().oracle_sf_bytes(R, K, int(mma)))


def sf_mma_offset(r: int, c: int, K: int) -> int:
    return int(lib().oracle_sf_mma_offset(r, c, K))


def sf_linear_to_mma(sf_lin: np.ndarray, R: int, K: int) -> np.ndarray:
    sf_lin = np.ascontiguousarray(sf_lin, dtype=np.uint8)
    assert sf_lin.size == R * (K // 16)
    out = np.empty(sf_bytes(R, K, True), dtype=np.uint8)
    lib().oracle_sf_linear_to_mma(_ptr(sf_lin, _u8p), R, K, _ptr(out, _u8p))
    return out


# ---------------------------------------------------------------- quantizers
def amax(x) -> float:
    u = _as_u16(x)
    return float(lib().oracle_amax_bf16(_ptr(u, _u16p), u.size))


def nvfp4_global_scale(x) -> np.float32:
    """g = amax(X) / (448*6), one binary32 division."""
    u = _as_u16(x)
    return np.float32(lib().oracle_nvfp4_global_scale(_ptr(u, _u16p), u.size))


def nvfp4_quantize(x, g, threads: int | None = None):
    """Returns (codes uint8 [R, K/2], sf_linear uint8 [R, K/16])."""
    u = _as_u16(x)
    R, K = u.shape
    assert K % 16 == 0
    codes = np.empty((R, K // 2), dtype=np.uint8)
    sf = np.empty((R, K // 16), dtype=np.uint8)
    lib().oracle_nvfp4_quantize(_ptr(u, _u16p), R, K, ctypes.c_float(np.float32(g)),
                                _ptr(codes, _u8p), _ptr(sf, _u8p),
                                threads or default_threads())
    return codes, sf


def nvfp4_dequant(codes: np.ndarray, sf_lin: np.ndarray, g: float = 1.0) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sf_lin = np.ascontiguousarray(sf_lin, dtype=np.uint8)
    R, K2 = codes.shape
    K = 2 * K2
    if K % 16 != 0 or sf_lin.shape != (R, K // 16):
        raise ValueError(f"scales must be [R, K/16] = {(R, K // 16)}, got {sf_lin.shape}")
    out = np.empty((R, K), dtype=np.float64)
    lib().oracle_nvfp4_dequant(_ptr(codes, _u8p), _ptr(sf_lin, _u8p), R, K,
                               float(g), _ptr(out, _f64p))
    return out


def nvfp4_dequant_bf16(codes: np.ndarray, sf_lin: np.ndarray, g: float) -> np.ndarray:
    """Decode to bf16 bit patterns (uint16 [R, K]): bf16_rne(fl32(e2m1 * e4m3) * g), the
    weight decode of the dequantise-only fallback (closing paragraph of the "Kernels"
    section of "BFL (fp8r / nvfp4)")."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sf_lin = np.ascontiguousarray(sf_lin, dtype=np.uint8)
    R, K2 = codes.shape
    K = 2 * K2
    if K % 16 != 0 or sf_lin.shape != (R, K // 16):
        raise ValueError(f"scales must be [R, K/16] = {(R, K // 16)}, got {sf_lin.shape}")
    out = np.empty((R, K), dtype=np.uint16)
    lib().oracle_nvfp4_dequant_bf16(_ptr(codes, _u8p), _ptr(sf_lin, _u8p), R, K,
                                    ctypes.c_float(np.float32(g)), _ptr(out, _u16p))
    return out


def fp8r_quantize(x, threads: int | None = None):
    """Returns (q uint8 [R, K] E4M3 codes, s float32 [R])."""
    u = _as_u16(x)
    R, K = u.shape
    q = np.empty((R, K), dtype=np.uint8)
    s = np.empty((R,), dtype=np.float32)
    lib().oracle_fp8r_quantize(_ptr(u, _u16p), R, K, _ptr(q, _u8p), _ptr(s, _f32p),
                               threads or default_threads())
    return q, s


def e4m3_decode_array(q: np.ndarray) -> np.ndarray:
    table = np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)
    return table[np.asarray(q, dtype=np.uint8)]


# ---------------------------------------------------------------- GEMMs (fp64)
def gemm_f64(A: np.ndarray, W: np.ndarray, bias=None, alpha: float = 1.0,
             threads: int | None = None) -> np.ndarray:
    A = np.ascontiguousarray(A, dtype=np.float64)
    W = np.ascontiguousarray(W, dtype=np.float64)
    M, K = A.shape
    N = W.shape[0]
    Y = np.empty((M, N), dtype=np.float64)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
    lib().oracle_gemm_f64(_ptr(A, _f64p), _ptr(W, _f64p),
                          None if b is None else _ptr(b, _f64p), float(alpha), None, M,
                          N, K, _ptr(Y, _f64p), threads or default_threads())
    return Y


def nvfp4_linear(a_codes, a_sf_lin, a_global, w_codes, w_sf_lin, w_global, bias=None,
                 threads: int | None = None) -> np.ndarray:
    """Y = (gA*gW) * sum_k (e2m1*sd)_A (e2m1*sd)_W + bias, all in fp64."""
    a_codes = np.ascontiguousarray(a_codes, dtype=np.uint8)
    w_codes = np.ascontiguousarray(w_codes, dtype=np.uint8)
    a_sf_lin = np.ascontiguousarray(a_sf_lin, dtype=np.uint8)
    w_sf_lin = np.ascontiguousarray(w_sf_lin, dtype=np.uint8)
    M, K2 = a_codes.shape
    N = w_codes.shape[0]
    K = 2 * K2
    Y = np.empty((M, N), dtype=np.float64)
    sa = np.empty((M, K), dtype=np.float64)
    sw = np.empty((N, K), dtype=np.float64)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
    lib().oracle_nvfp4_linear(_ptr(a_codes, _u8p), _ptr(a_sf_lin, _u8p),
                              ctypes.c_float(np.float32(a_global)), _ptr(w_codes, _u8p),
                              _ptr(w_sf_lin, _u8p), ctypes.c_float(np.float32(w_global)),
                              None if b is None else _ptr(b, _f64p), None, M, M, N, K,
                              _ptr(Y, _f64p), _ptr(sa, _f64p), _ptr(sw, _f64p),
                              threads or default_threads())
    return Y


def fp8r_linear(a_q, a_s, w_q, w_s, bias=None, threads: int | None = None) -> np.ndarray:
    """Y = (sum_k e4m3(a) e4m3(w)) * sA[m] * sW[n] + bias, all in fp64."""
    a_q = np.ascontiguousarray(a_q, dtype=np.uint8)
    w_q = np.ascontiguousarray(w_q, dtype=np.uint8)
    a_s = np.ascontiguousarray(a_s, dtype=np.float32)
    w_s = np.ascontiguousarray(w_s, dtype=np.float32)
    M, K = a_q.shape
    N = w_q.shape[0]
    Y = np.empty((M, N), dtype=np.float64)
    sa = np.empty((M, K), dtype=np.float64)
    sw = np.empty((N, K), dtype=np.float64)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
    lib().oracle_fp8r_linear(_ptr(a_q, _u8p), _ptr(a_s, _f32p), _ptr(w_q, _u8p),
                             _ptr(w_s, _f32p), None if b is None else _ptr(b, _f64p), None,
                             M, M, N, K, _ptr(Y, _f64p), _ptr(sa, _f64p), _ptr(sw, _f64p),
                             threads or default_threads())
    return Y


def nvfp4_row_norms(codes, sf_lin, g) -> np.ndarray:
    """||xhat_row||_2 of the dequantised rows (used by the tolerance)."""
    return np.sqrt((nvfp4_dequant(codes, sf_lin, g) ** 2).sum(axis=1))


def fp8r_row_norms(q, s) -> np.ndarray:
    d = e4m3_decode_array(q) * np.asarray(s, dtype=np.float64)[:, None]
    return np.sqrt((d ** 2).sum(axis=1))
