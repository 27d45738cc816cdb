"""ctypes binding of libpkv.so: argument marshalling only."""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

F16, BF16, F32, FP8_E4M3, FP8_E5M2 = 0, 1, 2, 3, 4
DEVERR_PAGE_ID = 0x01
DEVERR_INDPTR = 0x02
DEVERR_LAST_LEN = 0x04
DEVERR_APPEND = 0x08
DEVERR_TIMEOUT = 0x10
DEVERR_CONTEXT_LEN = 0x20
LAYOUT_HND, LAYOUT_NHD = 0, 1
TABLE_CSR, TABLE_BLOCK = 0, 1
TABLE_READY_AT_LAUNCH = 0x1

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpkv.so")

_P = ctypes.c_void_p
_I32 = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_F32 = ctypes.c_float

_SIGNATURES = {
    "pkv_status_string": ([_I32], ctypes.c_char_p),
    "pkv_last_error": ([], ctypes.c_char_p),
    "pkv_default_partitions": ([_I32], _I32),
    "pkv_decode_workspace_bytes": ([_I32, _I32, _I32, _I32, _I32], _SZ),
    "pkv_append": ([_P, _I64, _I32, _I32, _I32, _I32, _P, _P, _P, _I32, _P, _P, _P, _I64, _P, _P], _I32),
    "pkv_decode": ([_P, _I32, _P, _I64, _I32, _I32, _I32, _I32, _P, _P, _P, _I32, _F32, _I32,
                    _P, _SZ, _P, _P, _P, _P], _I32),
    "pkv_merge_states": ([_P, _P, _I64, _I32, _I32, _I32, _P, _I32, _P, _P], _I32),
    "pkv_read_error_word": ([_P, _P, _I32, _P], _I32),
    "pkv_check_table": ([_P, _P, _P, _I32, _I64, _I32], _I32),
    "pkv_plan_segments": ([_P, _P, _I32, _I32, _I32, _I32, _P, _I64], _I64),
    "pkv_set_wait_limit_ns": ([ctypes.c_uint64], ctypes.c_uint64),
}
_SIGNATURES["pkv_decode_static_workspace"] = (
    [_P, _I32, _P, _I64, _I32, _I32, _I32, _I32, _P, _P, _P, _I32, _F32, _I32, _P, _P, _P, _P], _I32)
_SIGNATURES["pkv_cascade_workspace_bytes"] = ([_I32, _I32, _I32, _I32, _I64, _I32], _SZ)
_SIGNATURES["pkv_cascade_decode"] = (
    [_P, _I32, _P, _I64, _I32, _I32, _I32, _I32, _P, _I64, _P, _P, _P, _I32, _F32, _I32, _P, _SZ,
     _P, _P, _P, _P], _I32)
class PoolDesc(ctypes.Structure):
    """pkv_pool_desc"""
    _fields_ = [("data", ctypes.c_void_p), ("num_pages", ctypes.c_int64),
                ("page_size", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("layout", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class TableDesc(ctypes.Structure):
    """pkv_table_desc"""
    _fields_ = [("kind", ctypes.c_int32), ("batch", ctypes.c_int32),
                ("page_indptr", ctypes.c_void_p), ("page_indices", ctypes.c_void_p),
                ("last_page_len", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("context_lens", ctypes.c_void_p), ("max_blocks_per_seq", ctypes.c_int32),
                ("flags", ctypes.c_int32)]


_PP = ctypes.POINTER(PoolDesc)
_TP = ctypes.POINTER(TableDesc)
_SIGNATURES["pkv_decode_ex"] = ([_P, _I32, _PP, _TP, _F32, _I32, _P, _SZ, _P, _P, _P, _P], _I32)
_SIGNATURES["pkv_append_ex"] = ([_PP, _TP, _P, _P, _P, _I64, _P, _P], _I32)
_SIGNATURES["pkv_decode_fp8"] = (
    [_P, _I32, _I32, _PP, _F32, _F32, _TP, _F32, _I32, _P, _SZ, _P, _P, _P, _P], _I32)
_SIGNATURES["pkv_append_fp8"] = ([_PP, _F32, _F32, _TP, _P, _P, _I32, _P, _I64, _P, _P], _I32)
_SIGNATURES["pkv_append_attention_plan"] = (
    [_P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _P, _I64, _P], _I64)
_SIGNATURES["pkv_append_attention_workspace_bytes"] = ([_I64, _I32, _I32], _SZ)
_SIGNATURES["pkv_append_attention"] = (
    [_P, _P, _I64, _I32, _PP, _TP, _P, _I64, _I32, _I32, _I32, _F32, _P, _SZ, _P, _P, _P, _P], _I32)
_SIGNATURES["pkv_append_attention_short_workspace_bytes"] = ([_I32, _I32, _I32, _I32], _SZ)
_SIGNATURES["pkv_append_attention_short"] = (
    [_P, _P, _I64, _I32, _I32, _PP, _TP, _P, _P, _P, _I64, _F32, _I32, _P, _SZ, _P, _P, _P, _P], _I32)
_SIGNATURES["pkv_decode_append"] = (
    [_P, _I32, _PP, _TP, _P, _P, _P, _I64, _F32, _I32, _P, _SZ, _P, _P, _P, _P], _I32)
_SIGNATURES["paged_kv_append"] = _SIGNATURES["pkv_append"]
_SIGNATURES["paged_decode_attention"] = _SIGNATURES["pkv_decode"]
_SIGNATURES["merge_states"] = _SIGNATURES["pkv_merge_states"]

_lib = None


class PkvError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(what)


def lib():
    """The loaded libpkv.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_479_b200.build` "
                "(there is no CPU fallback)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.argtypes = args
            fn.restype = res
        _lib = handle
    return _lib


def _check(status: int, what: str):
    if status != 0:
        L = lib()
        raise PkvError(status, f"{what}: {L.pkv_status_string(status).decode()}: "
                               f"{L.pkv_last_error().decode()}")


_DTYPES = {torch.float16: F16, torch.bfloat16: BF16, torch.float32: F32,
           torch.uint8: FP8_E4M3, torch.float8_e4m3fn: FP8_E4M3, torch.float8_e5m2: FP8_E5M2}


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev_tensor(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")
    return t


def _stream(stream, device) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def set_wait_limit_ns(nanoseconds: int) -> int:
    """Time limit of the decode kernel's internal waits for later launches
    (0 = the default, one second); returns the previous limit."""
    return int(lib().pkv_set_wait_limit_ns(int(nanoseconds)))


def default_partitions(device=None) -> int:
    dev = torch.cuda.current_device() if device is None else torch.device(device).index or 0
    n = lib().pkv_default_partitions(dev)
    if n <= 0:
        raise PkvError(4, "pkv_default_partitions failed")
    return n


def decode_workspace_bytes(batch: int, num_qo_heads: int, num_kv_heads: int,
                           head_dim: int = 128, num_partitions: int = 0) -> int:
    n = lib().pkv_decode_workspace_bytes(batch, num_qo_heads, num_kv_heads, head_dim,
                                          num_partitions)
    if n == 0:
        raise PkvError(1, "pkv_decode_workspace_bytes: invalid shapes")
    return int(n)


def paged_kv_append(pool, page_indptr, page_indices, last_page_len, k_new, v_new,
                    append_indptr, error_word=None, stream=None) -> None:
    """Scatter k_new / v_new [nnz, Hkv, D] into `pool` [P, 2, Hkv, ps, D] (C: pkv_append).
    The page table is the table after the append."""
    _dev_tensor(pool, "pool")
    P, two, hkv, ps, d = pool.shape
    if two != 2:
        raise ValueError("pool must be [P, 2, Hkv, ps, D]")
    for name, t in (("page_indptr", page_indptr), ("page_indices", page_indices),
                    ("last_page_len", last_page_len), ("append_indptr", append_indptr)):
        _dev_tensor(t, name, torch.int32)
    _dev_tensor(k_new, "k_new", pool.dtype)
    _dev_tensor(v_new, "v_new", pool.dtype)
    batch = last_page_len.numel()
    st = lib().pkv_append(_ptr(pool), P, ps, hkv, d, _DTYPES[pool.dtype], _ptr(page_indptr),
                          _ptr(page_indices), _ptr(last_page_len), batch, _ptr(k_new),
                          _ptr(v_new), _ptr(append_indptr), k_new.shape[0], _ptr(error_word),
                          _stream(stream, pool.device))
    _check(st, "pkv_append")


def paged_decode_attention(q, pool, page_indptr, page_indices, last_page_len, workspace,
                           out=None, lse=None, sm_scale=None, num_partitions: int = 0,
                           error_word=None, stream=None, return_lse: bool = True):
    """Decode attention of q [B, Hq, D] over the paged pool (C: pkv_decode).
    Returns (out [B, Hq, D] in q's dtype, lse [B, Hq] float32 or None)."""
    _dev_tensor(q, "q", pool.dtype)
    _dev_tensor(pool, "pool")
    _dev_tensor(workspace, "workspace")
    for name, t in (("page_indptr", page_indptr), ("page_indices", page_indices),
                    ("last_page_len", last_page_len)):
        _dev_tensor(t, name, torch.int32)
    B, hq, d = q.shape
    P, _, hkv, ps, dp = pool.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, hq), dtype=torch.float32, device=q.device)
    scale = float(sm_scale) if sm_scale is not None else 1.0 / float(d) ** 0.5
    st = lib().pkv_decode(_ptr(q), hq, _ptr(pool), P, ps, hkv, dp, _DTYPES[pool.dtype],
                          _ptr(page_indptr), _ptr(page_indices), _ptr(last_page_len), B, scale,
                          num_partitions, _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _ptr(out), _ptr(lse),
                          _ptr(error_word), _stream(stream, q.device))
    _check(st, "pkv_decode")
    return out, lse


def decode_static_workspace(q, pool, page_indptr, page_indices, last_page_len, out, lse=None,
                            sm_scale=None, num_partitions: int = 0, error_word=None,
                            stream=None):
    """Decode attention like paged_decode_attention, for callers that cannot
    allocate device memory: the library's own static scratch replaces the
    workspace, and the caller passes the output buffers (nothing is allocated
    here).  Calls sharing that scratch must not overlap on the GPU
    (C: pkv_decode_static_workspace)."""
    _dev_tensor(q, "q", pool.dtype)
    _dev_tensor(pool, "pool")
    _dev_tensor(out, "out", pool.dtype)
    for name, t in (("page_indptr", page_indptr), ("page_indices", page_indices),
                    ("last_page_len", last_page_len)):
        _dev_tensor(t, name, torch.int32)
    B, hq, d = q.shape
    P, _, hkv, ps, dp = pool.shape
    scale = float(sm_scale) if sm_scale is not None else 1.0 / float(d) ** 0.5
    st = lib().pkv_decode_static_workspace(_ptr(q), hq, _ptr(pool), P, ps, hkv, dp,
                                           _DTYPES[pool.dtype], _ptr(page_indptr),
                                           _ptr(page_indices), _ptr(last_page_len), B, scale,
                                           num_partitions, _ptr(out), _ptr(lse),
                                           _ptr(error_word), _stream(stream, q.device))
    _check(st, "pkv_decode_static_workspace")
    return out, lse


def cascade_workspace_bytes(batch: int, num_qo_heads: int, num_kv_heads: int, prefix_len: int,
                            head_dim: int = 128, num_partitions: int = 0) -> int:
    n = lib().pkv_cascade_workspace_bytes(batch, num_qo_heads, num_kv_heads, head_dim,
                                           int(prefix_len), num_partitions)
    if n == 0:
        raise PkvError(1, "pkv_cascade_workspace_bytes: invalid shapes")
    return int(n)


def cascade_decode(q, pool, prefix_pages, prefix_len, page_indptr, page_indices, last_page_len,
                   workspace, out=None, lse=None, sm_scale=None, num_partitions: int = 0,
                   error_word=None, stream=None, return_lse: bool = True):
    """Decode attention for requests that all start with one shared prefix
    (C: pkv_cascade_decode).  The page table holds each request's own pages."""
    _dev_tensor(q, "q", pool.dtype)
    _dev_tensor(pool, "pool")
    _dev_tensor(workspace, "workspace")
    for name, t in (("prefix_pages", prefix_pages), ("page_indptr", page_indptr),
                    ("page_indices", page_indices), ("last_page_len", last_page_len)):
        _dev_tensor(t, name, torch.int32)
    B, hq, d = q.shape
    P, _, hkv, ps, dp = pool.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, hq), dtype=torch.float32, device=q.device)
    scale = float(sm_scale) if sm_scale is not None else 1.0 / float(d) ** 0.5
    st = lib().pkv_cascade_decode(_ptr(q), hq, _ptr(pool), P, ps, hkv, dp, _DTYPES[pool.dtype],
                                  _ptr(prefix_pages), int(prefix_len), _ptr(page_indptr),
                                  _ptr(page_indices), _ptr(last_page_len), B, scale,
                                  num_partitions, _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _ptr(out),
                                  _ptr(lse), _ptr(error_word), _stream(stream, q.device))
    _check(st, "pkv_cascade_decode")
    return out, lse


def pool_desc(pool, layout: str = "HND") -> PoolDesc:
    """Descriptor of a pool tensor: HND [P, 2, Hkv, ps, D] or NHD [P, 2, ps, Hkv, D]."""
    _dev_tensor(pool, "pool")
    if layout == "HND":
        P, two, hkv, ps, d = pool.shape
    elif layout == "NHD":
        P, two, ps, hkv, d = pool.shape
    else:
        raise ValueError("layout must be 'HND' or 'NHD'")
    if two != 2:
        raise ValueError("the second pool axis must be (K, V)")
    return PoolDesc(pool.data_ptr(), P, ps, hkv, d, _DTYPES[pool.dtype],
                    LAYOUT_HND if layout == "HND" else LAYOUT_NHD, 0)


def csr_table(page_indptr, page_indices, last_page_len, ready_at_launch: bool = False) -> TableDesc:
    """CSR page table.  ready_at_launch: no kernel right before the call in the
    stream writes the table (PKV_TABLE_READY_AT_LAUNCH), so the decode may read
    it while that kernel finishes."""
    for name, t in (("page_indptr", page_indptr), ("page_indices", page_indices),
                    ("last_page_len", last_page_len)):
        _dev_tensor(t, name, torch.int32)
    t = TableDesc(TABLE_CSR, last_page_len.numel(), page_indptr.data_ptr(),
                  page_indices.data_ptr(), last_page_len.data_ptr(), None, None, 0,
                  TABLE_READY_AT_LAUNCH if ready_at_launch else 0)
    t._keep = (page_indptr, page_indices, last_page_len)  # the descriptor holds raw pointers
    return t


def block_table(table, context_lens, ready_at_launch: bool = False) -> TableDesc:
    """Dense [batch, max_blocks_per_seq] block table + context lengths (tokens);
    ready_at_launch as for csr_table."""
    _dev_tensor(table, "block_table", torch.int32)
    _dev_tensor(context_lens, "context_lens", torch.int32)
    if table.dim() != 2 or table.shape[0] != context_lens.numel():
        raise ValueError("block_table must be [batch, max_blocks_per_seq]")
    t = TableDesc(TABLE_BLOCK, table.shape[0], None, None, None, table.data_ptr(),
                  context_lens.data_ptr(), table.shape[1],
                  TABLE_READY_AT_LAUNCH if ready_at_launch else 0)
    t._keep = (table, context_lens)
    return t


def paged_decode_attention_ex(q, pool, table: TableDesc, workspace, layout: str = "HND",
                              out=None, lse=None, sm_scale=None, num_partitions: int = 0,
                              error_word=None, stream=None, return_lse: bool = True):
    """pkv_decode_ex: decode on an HND/NHD pool with a CSR or dense block table."""
    _dev_tensor(q, "q", pool.dtype)
    _dev_tensor(workspace, "workspace")
    pd = pool_desc(pool, layout)
    B, hq, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, hq), dtype=torch.float32, device=q.device)
    scale = float(sm_scale) if sm_scale is not None else 1.0 / float(d) ** 0.5
    st = lib().pkv_decode_ex(_ptr(q), hq, ctypes.byref(pd), ctypes.byref(table), scale,
                             num_partitions, _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _ptr(out), _ptr(lse),
                             _ptr(error_word), _stream(stream, q.device))
    _check(st, "pkv_decode_ex")
    return out, lse


def paged_kv_append_ex(pool, table: TableDesc, k_new, v_new, append_indptr, layout: str = "HND",
                       error_word=None, stream=None) -> None:
    """pkv_append_ex: append on an HND/NHD pool with a CSR or dense block table."""
    pd = pool_desc(pool, layout)
    _dev_tensor(k_new, "k_new", pool.dtype)
    _dev_tensor(v_new, "v_new", pool.dtype)
    _dev_tensor(append_indptr, "append_indptr", torch.int32)
    st = lib().pkv_append_ex(ctypes.byref(pd), ctypes.byref(table), _ptr(k_new), _ptr(v_new),
                             _ptr(append_indptr), k_new.shape[0], _ptr(error_word),
                             _stream(stream, pool.device))
    _check(st, "pkv_append_ex")


def paged_decode_append(q, pool, table: TableDesc, k_new, v_new, append_indptr, workspace,
                        layout: str = "HND", out=None, lse=None, sm_scale=None,
                        num_partitions: int = 0, error_word=None, stream=None,
                        return_lse: bool = True):
    """pkv_decode_append: the step's append (k_new / v_new rows by the int32
    append_indptr) and the decode in one launch; table = the table after the append."""
    _dev_tensor(q, "q", pool.dtype)
    _dev_tensor(workspace, "workspace")
    _dev_tensor(k_new, "k_new", pool.dtype)
    _dev_tensor(v_new, "v_new", pool.dtype)
    _dev_tensor(append_indptr, "append_indptr", torch.int32)
    pd = pool_desc(pool, layout)
    B, hq, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, hq), dtype=torch.float32, device=q.device)
    scale = float(sm_scale) if sm_scale is not None else 1.0 / float(d) ** 0.5
    st = lib().pkv_decode_append(_ptr(q), hq, ctypes.byref(pd), ctypes.byref(table), _ptr(k_new),
                                 _ptr(v_new), _ptr(append_indptr), k_new.shape[0], scale,
                                 num_partitions, _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _ptr(out),
                                 _ptr(lse), _ptr(error_word), _stream(stream, q.device))
    _check(st, "pkv_decode_append")
    return out, lse


def _fp8_pool(pool, layout, fmt):
    """Descriptor of an 8-bit pool: a float8_e4m3fn / float8_e5m2 tensor, or uint8
    codes of the format `fmt` ("e4m3" or "e5m2")."""
    if pool.dtype not in (torch.uint8, torch.float8_e4m3fn, torch.float8_e5m2):
        raise ValueError("an 8-bit pool must be a uint8, float8_e4m3fn or float8_e5m2 tensor")
    pd = pool_desc(pool, layout)
    if pool.dtype == torch.uint8:
        if fmt not in ("e4m3", "e5m2"):
            raise ValueError("fp8_format must be 'e4m3' or 'e5m2'")
        pd.dtype = FP8_E4M3 if fmt == "e4m3" else FP8_E5M2
    return pd


def paged_decode_attention_fp8(q, pool, table: TableDesc, workspace, k_scale: float,
                               v_scale: float, layout: str = "HND", out=None, lse=None,
                               sm_scale=None, num_partitions: int = 0, error_word=None,
                               stream=None, return_lse: bool = True, fp8_format: str = "e4m3"):
    """pkv_decode_fp8: decode over an 8-bit pool (key = code * k_scale, value = code * v_scale);
    q and out are fp16 or bf16."""
    _dev_tensor(q, "q")
    if q.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("q must be fp16 or bf16")
    _dev_tensor(workspace, "workspace")
    pd = _fp8_pool(pool, layout, fp8_format)
    B, hq, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, hq), dtype=torch.float32, device=q.device)
    scale = float(sm_scale) if sm_scale is not None else 1.0 / float(d) ** 0.5
    st = lib().pkv_decode_fp8(_ptr(q), _DTYPES[q.dtype], hq, ctypes.byref(pd), float(k_scale),
                              float(v_scale), ctypes.byref(table), scale, num_partitions,
                              _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _ptr(out), _ptr(lse), _ptr(error_word), _stream(stream, q.device))
    _check(st, "pkv_decode_fp8")
    return out, lse


def paged_kv_append_fp8(pool, table: TableDesc, k_new, v_new, append_indptr, k_scale: float,
                        v_scale: float, layout: str = "HND", error_word=None,
                        stream=None, fp8_format: str = "e4m3") -> None:
    """pkv_append_fp8: quantise fp16/bf16 rows into an 8-bit pool (x -> fp8(x / scale))."""
    pd = _fp8_pool(pool, layout, fp8_format)
    _dev_tensor(k_new, "k_new")
    _dev_tensor(v_new, "v_new", k_new.dtype)
    if k_new.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("k_new / v_new must be fp16 or bf16")
    _dev_tensor(append_indptr, "append_indptr", torch.int32)
    st = lib().pkv_append_fp8(ctypes.byref(pd), float(k_scale), float(v_scale),
                              ctypes.byref(table), _ptr(k_new), _ptr(v_new), _DTYPES[k_new.dtype],
                              _ptr(append_indptr), k_new.shape[0], _ptr(error_word),
                              _stream(stream, pool.device))
    _check(st, "pkv_append_fp8")


def append_attention_plan(qo_indptr_h, kv_len_h, num_qo_heads: int, num_kv_heads: int,
                          window_left: int = -1, sink_tokens: int = 0, num_sms: int = 0):
    """pkv_append_attention_plan on host arrays: (plan int32 [n, 4], suggested splits)."""
    qo = np.ascontiguousarray(qo_indptr_h, np.int32)
    kl = None if kv_len_h is None else np.ascontiguousarray(kv_len_h, np.int32)
    B = len(qo) - 1
    if num_sms == 0 and torch.cuda.is_available():
        num_sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    splits = ctypes.c_int32(1)
    kp = None if kl is None else kl.ctypes.data_as(_P)
    n = lib().pkv_append_attention_plan(qo.ctypes.data_as(_P), kp, B, num_qo_heads, num_kv_heads,
                                        window_left, sink_tokens, num_sms, None, 0, None)
    if n < 0:
        raise ValueError("pkv_append_attention_plan rejected the arguments")
    plan = np.zeros((max(n, 1), 4), np.int32)
    n2 = lib().pkv_append_attention_plan(qo.ctypes.data_as(_P), kp, B, num_qo_heads, num_kv_heads,
                                         window_left, sink_tokens, num_sms,
                                         plan.ctypes.data_as(_P), n, ctypes.byref(splits))
    assert n2 == n
    return plan[:n], int(splits.value)


def append_attention_workspace_bytes(nnz_q: int, num_qo_heads: int, num_splits: int) -> int:
    return int(lib().pkv_append_attention_workspace_bytes(nnz_q, num_qo_heads, num_splits))


def append_attention(q, qo_indptr, pool, table: TableDesc, plan, num_splits: int = 1,
                     layout: str = "HND", window_left: int = -1, sink_tokens: int = 0,
                     workspace=None, out=None, lse=None, sm_scale=None, error_word=None,
                     stream=None, return_lse: bool = True):
    """pkv_append_attention: every request's chunk of query tokens (rows of q,
    split by the device int32 qo_indptr) over its cache, causal, optional window.
    plan: device int32 [n, 4] from append_attention_plan."""
    _dev_tensor(q, "q", pool.dtype)
    _dev_tensor(qo_indptr, "qo_indptr", torch.int32)
    _dev_tensor(plan, "plan", torch.int32)
    pd = pool_desc(pool, layout)
    nnz, hq, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((nnz, hq), dtype=torch.float32, device=q.device)
    need = append_attention_workspace_bytes(nnz, hq, num_splits)
    if workspace is None and need:
        workspace = torch.empty(need // 4 + 64, dtype=torch.int32, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    scale = float(sm_scale) if sm_scale is not None else 1.0 / float(d) ** 0.5
    st = lib().pkv_append_attention(_ptr(q), _ptr(qo_indptr), nnz, hq, ctypes.byref(pd),
                                    ctypes.byref(table), _ptr(plan), plan.shape[0], num_splits,
                                    window_left, sink_tokens, scale, _ptr(workspace), ws_bytes,
                                    _ptr(out), _ptr(lse), _ptr(error_word),
                                    _stream(stream, q.device))
    _check(st, "pkv_append_attention")
    return out, lse


def append_attention_short_workspace_bytes(num_qo_heads: int, num_kv_heads: int, max_q_len: int,
                                           num_partitions: int = 0) -> int:
    return int(lib().pkv_append_attention_short_workspace_bytes(num_qo_heads, num_kv_heads,
                                                               max_q_len, num_partitions))


def append_attention_short(q, qo_indptr, pool, table: TableDesc, max_q_len: int, workspace,
                           layout: str = "HND", num_partitions: int = 0, out=None, lse=None,
                           sm_scale=None, error_word=None, stream=None, return_lse: bool = True,
                           k_new=None, v_new=None, append_indptr=None):
    """pkv_append_attention_short: append attention (no window) for chunks of at
    most max_q_len tokens, max_q_len * (Hq / Hkv) <= 16, on the decode kernel's
    schedule.  workspace: zero-filled device buffer of
    append_attention_short_workspace_bytes bytes.  With k_new / v_new /
    append_indptr the chunk's K/V rows are appended by the same launch."""
    _dev_tensor(q, "q", pool.dtype)
    _dev_tensor(qo_indptr, "qo_indptr", torch.int32)
    nnz_new = 0
    if k_new is not None:
        _dev_tensor(k_new, "k_new", pool.dtype)
        _dev_tensor(v_new, "v_new", pool.dtype)
        _dev_tensor(append_indptr, "append_indptr", torch.int32)
        nnz_new = k_new.shape[0]
    pd = pool_desc(pool, layout)
    nnz, hq, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((nnz, hq), dtype=torch.float32, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    scale = float(sm_scale) if sm_scale is not None else 1.0 / float(d) ** 0.5
    st = lib().pkv_append_attention_short(_ptr(q), _ptr(qo_indptr), nnz, max_q_len, hq,
                                          ctypes.byref(pd), ctypes.byref(table), _ptr(k_new),
                                          _ptr(v_new), _ptr(append_indptr), nnz_new, scale,
                                          num_partitions, _ptr(workspace), ws_bytes, _ptr(out),
                                          _ptr(lse), _ptr(error_word), _stream(stream, q.device))
    _check(st, "pkv_append_attention_short")
    return out, lse


def merge_states(v, s, out_dtype=torch.float32, v_out=None, s_out=None, stream=None,
                 return_lse: bool = True):
    """Merge states v [N, S, H, D] float32 with lse s [N, S, H] (C: pkv_merge_states)."""
    _dev_tensor(v, "v", torch.float32)
    _dev_tensor(s, "s", torch.float32)
    N, S, H, D = v.shape
    if v_out is None:
        v_out = torch.empty((N, H, D), dtype=out_dtype, device=v.device)
    if s_out is None and return_lse:
        s_out = torch.empty((N, H), dtype=torch.float32, device=v.device)
    st = lib().pkv_merge_states(_ptr(v), _ptr(s), N, S, H, D, _ptr(v_out), _DTYPES[v_out.dtype],
                                _ptr(s_out), _stream(stream, v.device))
    _check(st, "pkv_merge_states")
    return v_out, s_out


def read_error_word(error_word, clear: bool = True, stream=None) -> int:
    """Synchronise and return the device error word (PKV_DEVERR_* bits)."""
    val = ctypes.c_int32(0)
    st = lib().pkv_read_error_word(_ptr(error_word), ctypes.byref(val), int(clear),
                                   _stream(stream, error_word.device))
    if st not in (0, 5):
        _check(st, "pkv_read_error_word")
    return int(val.value)


def check_table(page_indptr, page_indices, last_page_len, num_pages: int, page_size: int) -> None:
    """Host-side table check (C: pkv_check_table); raises PkvError when invalid."""
    ip = np.ascontiguousarray(page_indptr, np.int32)
    ix = np.ascontiguousarray(page_indices, np.int32)
    ll = np.ascontiguousarray(last_page_len, np.int32)
    st = lib().pkv_check_table(ip.ctypes.data_as(_P), ix.ctypes.data_as(_P) if ix.size else None,
                               ll.ctypes.data_as(_P), len(ll), int(num_pages), int(page_size))
    _check(st, "pkv_check_table")


def plan_segments(page_indptr, last_page_len, page_size: int, num_kv_heads: int,
                  num_partitions: int) -> np.ndarray:
    """Host mirror of the decode kernel's split-KV partition (C: pkv_plan_segments).
    Rows: partition, request, kv head, first tile, end tile, state slot (-1 =
    direct output), partitions covering the pair."""
    ip = np.ascontiguousarray(page_indptr, np.int32)
    ll = np.ascontiguousarray(last_page_len, np.int32)
    L = lib()
    n = L.pkv_plan_segments(ip.ctypes.data_as(_P), ll.ctypes.data_as(_P), len(ll), page_size,
                            num_kv_heads, num_partitions, None, 0)
    if n < 0:
        raise PkvError(1, "pkv_plan_segments: invalid arguments")
    out = np.zeros((max(n, 1), 7), np.int64)
    L.pkv_plan_segments(ip.ctypes.data_as(_P), ll.ctypes.data_as(_P), len(ll), page_size,
                        num_kv_heads, num_partitions, out.ctypes.data_as(_P), n)
    return out[:n]
