"""fp64 CPU oracle for paged decode attention, page append and state merge.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg may import this package; the CUDA library and its Python
binding never do.  The arithmetic lives in oracle.c (plain C, double
precision, OpenMP over independent rows); this module only marshals numpy
arrays into it.

16-bit tensors (q, the KV pool, new K/V rows) are passed as their raw bit
patterns (numpy uint16), so the oracle sees exactly the bytes the GPU sees.
"""
import ctypes
import os

import numpy as np

from . import build as _build

F16 = 0
BF16 = 1
FP8_E4M3 = 3
FP8_E5M2 = 4

_STATUS = {
    0: "ok",
    1: "bad argument",
    2: "page_indptr not monotone / negative",
    3: "last_page_len outside [1, page_size]",
    4: "page id outside the pool",
    5: "append count larger than the request or malformed append_indptr",
    6: "out of host memory",
}

_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_build.build())
        p = ctypes.c_void_p
        i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_decode.argtypes = [p, p, i32, i64, i32, i32, i32, i32, i32,
                                      p, p, p, dbl, p, p]
        lib.oracle_decode.restype = i32
        lib.oracle_append.argtypes = [p, i64, i32, i32, i32, i32, p, p, p, p, p, p]
        lib.oracle_append.restype = i32
        lib.oracle_merge.argtypes = [p, p, i64, i32, i32, i32, p, p]
        lib.oracle_merge.restype = None
        f32 = ctypes.c_float
        lib.oracle_decode_fp8.argtypes = [p, i32, p, i32, f32, f32, i64, i32, i32, i32, i32,
                                          i32, p, p, p, dbl, p, p]
        lib.oracle_decode_fp8.restype = i32
        lib.oracle_append_fp8.argtypes = [p, i32, f32, f32, i64, i32, i32, i32, i32, p, p, p,
                                          p, p, i32, p]
        lib.oracle_append_fp8.restype = i32
        lib.oracle_append_attention.argtypes = [p, p, i32, i64, i32, i32, i32, i32, i32,
                                                p, p, p, p, i32, i32, dbl, p, p]
        lib.oracle_append_attention.restype = i32
        lib.oracle_e4m3_decode.argtypes = [p, i64, p]
        lib.oracle_e4m3_decode.restype = i32
        lib.oracle_e4m3_encode.argtypes = [p, i64, f32, p]
        lib.oracle_e4m3_encode.restype = i32
        lib.oracle_e5m2_decode.argtypes = [p, i64, p]
        lib.oracle_e5m2_decode.restype = i32
        lib.oracle_e5m2_encode.argtypes = [p, i64, f32, p]
        lib.oracle_e5m2_encode.restype = i32
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = i32
        _lib = lib
    return _lib


class OracleError(RuntimeError):
    pass


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use (OMP_NUM_THREADS or all cores)."""
    return int(_load().oracle_num_threads())


def decode(q_bits, pool_bits, dtype, page_indptr, page_indices, last_page_len,
           scale, num_qo_heads=None):
    """Exact decode attention.

    q_bits    uint16 [B, Hq, D]       stored fp16/bf16 bit patterns
    pool_bits uint16 [P, 2, Hkv, ps, D]
    dtype     F16 or BF16
    Returns (out float64 [B, Hq, D], lse float64 [B, Hq]) with lse in natural log.
    """
    q_bits, qp = _c(q_bits, np.uint16)
    pool_bits, pp = _c(pool_bits, np.uint16)
    if pool_bits.ndim != 5 or pool_bits.shape[1] != 2:
        raise ValueError("pool must be [P, 2, Hkv, ps, D]")
    P, _, hkv, ps, d = pool_bits.shape
    B, hq, dq = q_bits.shape
    if dq != d:
        raise ValueError("q head_dim does not match pool head_dim")
    indptr, ip = _c(page_indptr, np.int32)
    indices, xp = _c(page_indices if len(page_indices) else np.zeros(1, np.int32), np.int32)
    last, lp = _c(last_page_len if len(last_page_len) else np.zeros(1, np.int32), np.int32)
    out = np.zeros((B, hq, d), np.float64)
    lse = np.zeros((B, hq), np.float64)
    rc = _load().oracle_decode(qp, pp, int(dtype), P, ps, hkv, d, B, hq, ip, xp, lp,
                               float(scale), out.ctypes.data_as(ctypes.c_void_p),
                               lse.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise OracleError(f"oracle_decode: {_STATUS.get(rc, rc)}")
    return out, lse


def append(pool_bits, page_indptr, page_indices, last_page_len, k_new_bits,
           v_new_bits, append_indptr):
    """Return a copy of the pool with the new rows scattered in.

    pool_bits  uint16 [P, 2, Hkv, ps, D]  (not modified)
    k/v_new    uint16 [nnz, Hkv, D]
    The table is the table after the append (pages already allocated).
    """
    pool = np.array(pool_bits, dtype=np.uint16, copy=True, order="C")
    P, _, hkv, ps, d = pool.shape
    B = len(page_indptr) - 1
    indptr, ip = _c(page_indptr, np.int32)
    indices, xp = _c(page_indices if len(page_indices) else np.zeros(1, np.int32), np.int32)
    last, lp = _c(last_page_len if len(last_page_len) else np.zeros(1, np.int32), np.int32)
    kn, kp = _c(k_new_bits if np.size(k_new_bits) else np.zeros(1, np.uint16), np.uint16)
    vn, vp = _c(v_new_bits if np.size(v_new_bits) else np.zeros(1, np.uint16), np.uint16)
    ap, app = _c(append_indptr, np.int32)
    rc = _load().oracle_append(pool.ctypes.data_as(ctypes.c_void_p), P, ps, hkv, d, B,
                               ip, xp, lp, kp, vp, app)
    if rc != 0:
        raise OracleError(f"oracle_append: {_STATUS.get(rc, rc)}")
    return pool


def merge(v, s):
    """Merge attention states.

    v float [N, S, H, D] normalised partial outputs, s float [N, S, H] natural-log lse.
    Returns (v_out float64 [N, H, D], s_out float64 [N, H]).
    """
    v, vp = _c(v, np.float64)
    s, sp = _c(s, np.float64)
    N, S, H, D = v.shape
    if s.shape != (N, S, H):
        raise ValueError("s must be [N, S, H]")
    vo = np.zeros((N, H, D), np.float64)
    so = np.zeros((N, H), np.float64)
    _load().oracle_merge(vp, sp, N, S, H, D, vo.ctypes.data_as(ctypes.c_void_p),
                         so.ctypes.data_as(ctypes.c_void_p))
    return vo, so


def _fmt(fmt):
    return {"e4m3": "e4m3", FP8_E4M3: "e4m3", "e5m2": "e5m2", FP8_E5M2: "e5m2"}[fmt]


def fp8_values(codes, fmt="e4m3"):
    """Exact value of every code of the format, float64 (NaN / inf where the format has them)."""
    codes, cp = _c(codes, np.uint8)
    out = np.zeros(codes.shape, np.float64)
    getattr(_load(), f"oracle_{_fmt(fmt)}_decode")(cp, codes.size,
                                                   out.ctypes.data_as(ctypes.c_void_p))
    return out


def fp8_encode(x, scale=1.0, fmt="e4m3"):
    """Codes of float32(x) / float32(scale): nearest, ties to even, saturating."""
    x, xp = _c(x, np.float32)
    codes = np.zeros(x.shape, np.uint8)
    rc = getattr(_load(), f"oracle_{_fmt(fmt)}_encode")(xp, x.size, float(scale),
                                                        codes.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise OracleError(f"oracle_{_fmt(fmt)}_encode: {_STATUS.get(rc, rc)}")
    return codes


def e4m3_values(codes):
    """Exact value of every E4M3 code (NaN for 0x7f / 0xff), float64."""
    return fp8_values(codes, "e4m3")


def e4m3_encode(x, scale=1.0):
    """E4M3 codes of float32(x) / float32(scale): nearest, ties to even, saturating."""
    return fp8_encode(x, scale, "e4m3")


def decode_fp8(q_bits, q_dtype, pool_codes, k_scale, v_scale, page_indptr, page_indices,
               last_page_len, scale, fmt="e4m3"):
    """Exact decode attention over an E4M3 pool.

    q_bits     uint16 [B, Hq, D]  fp16/bf16 bits (q_dtype)
    pool_codes uint8 [P, 2, Hkv, ps, D]; K = code value * k_scale, V = * v_scale
    Returns (out float64 [B, Hq, D], lse float64 [B, Hq]).
    """
    q_bits, qp = _c(q_bits, np.uint16)
    pool_codes, pp = _c(pool_codes, np.uint8)
    if pool_codes.ndim != 5 or pool_codes.shape[1] != 2:
        raise ValueError("pool must be [P, 2, Hkv, ps, D]")
    P, _, hkv, ps, d = pool_codes.shape
    B, hq, dq = q_bits.shape
    if dq != d:
        raise ValueError("q head_dim does not match pool head_dim")
    indptr, ip = _c(page_indptr, np.int32)
    indices, xp = _c(page_indices if len(page_indices) else np.zeros(1, np.int32), np.int32)
    last, lp = _c(last_page_len if len(last_page_len) else np.zeros(1, np.int32), np.int32)
    out = np.zeros((B, hq, d), np.float64)
    lse = np.zeros((B, hq), np.float64)
    fp8 = FP8_E4M3 if _fmt(fmt) == "e4m3" else FP8_E5M2
    rc = _load().oracle_decode_fp8(qp, int(q_dtype), pp, fp8, float(k_scale), float(v_scale), P, ps,
                                   hkv, d, B, hq, ip, xp, lp, float(scale),
                                   out.ctypes.data_as(ctypes.c_void_p),
                                   lse.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise OracleError(f"oracle_decode_fp8: {_STATUS.get(rc, rc)}")
    return out, lse


def append_fp8(pool_codes, k_scale, v_scale, page_indptr, page_indices, last_page_len,
               k_new_bits, v_new_bits, new_dtype, append_indptr, fmt="e4m3"):
    """Return a copy of an E4M3 pool with the new 16-bit rows quantised in.

    pool_codes uint8 [P, 2, Hkv, ps, D] (not modified); k/v_new uint16 [nnz, Hkv, D]
    of type new_dtype; element x is stored as e4m3(float32(x) / scale).
    """
    pool = np.array(pool_codes, dtype=np.uint8, copy=True, order="C")
    P, _, hkv, ps, d = pool.shape
    B = len(page_indptr) - 1
    indptr, ip = _c(page_indptr, np.int32)
    indices, xp = _c(page_indices if len(page_indices) else np.zeros(1, np.int32), np.int32)
    last, lp = _c(last_page_len if len(last_page_len) else np.zeros(1, np.int32), np.int32)
    kn, kp = _c(k_new_bits if np.size(k_new_bits) else np.zeros(1, np.uint16), np.uint16)
    vn, vp = _c(v_new_bits if np.size(v_new_bits) else np.zeros(1, np.uint16), np.uint16)
    ap, app = _c(append_indptr, np.int32)
    fp8 = FP8_E4M3 if _fmt(fmt) == "e4m3" else FP8_E5M2
    rc = _load().oracle_append_fp8(pool.ctypes.data_as(ctypes.c_void_p), fp8, float(k_scale),
                                   float(v_scale), P, ps, hkv, d, B, ip, xp, lp, kp, vp,
                                   int(new_dtype), app)
    if rc != 0:
        raise OracleError(f"oracle_append_fp8: {_STATUS.get(rc, rc)}")
    return pool


def append_attention(q_bits, pool_bits, dtype, page_indptr, page_indices, last_page_len,
                     qo_indptr, scale, window_left=-1, sink_tokens=0):
    """Exact attention of each request's chunk of new query tokens over its cache.

    q_bits    uint16 [nnz_q, Hq, D]; request b's tokens are rows qo_indptr[b]:qo_indptr[b+1]
    pool_bits uint16 [P, 2, Hkv, ps, D]; the table is the table after the append
    Query i of request b sits at position L_b - q_len_b + i and sees keys t <= pos
    (and, with window_left >= 0, t >= pos - window_left unless t < sink_tokens).
    Returns (out float64 [nnz_q, Hq, D], lse float64 [nnz_q, Hq]).
    """
    q_bits, qp = _c(q_bits, np.uint16)
    pool_bits, pp = _c(pool_bits, np.uint16)
    P, _, hkv, ps, d = pool_bits.shape
    nnz, hq, dq = q_bits.shape
    if dq != d:
        raise ValueError("q head_dim does not match pool head_dim")
    B = len(page_indptr) - 1
    indptr, ip = _c(page_indptr, np.int32)
    indices, xp = _c(page_indices if len(page_indices) else np.zeros(1, np.int32), np.int32)
    last, lp = _c(last_page_len if len(last_page_len) else np.zeros(1, np.int32), np.int32)
    qo, qop = _c(qo_indptr, np.int32)
    if len(qo) != B + 1 or (B and qo[-1] != nnz):
        raise ValueError("qo_indptr must have batch + 1 entries ending at nnz_q")
    out = np.zeros((nnz, hq, d), np.float64)
    lse = np.zeros((nnz, hq), np.float64)
    rc = _load().oracle_append_attention(qp, pp, int(dtype), P, ps, hkv, d, B, hq, ip, xp, lp,
                                         qop, int(window_left), int(sink_tokens), float(scale),
                                         out.ctypes.data_as(ctypes.c_void_p),
                                         lse.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise OracleError(f"oracle_append_attention: {_STATUS.get(rc, rc)}")
    return out, lse
