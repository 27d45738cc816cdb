"""The decode entry point that allocates nothing (pkv_decode_static_workspace).

Some users of this library cannot allocate device memory where they decode
and have no spare buffer to lend as a workspace (an engine that reserved all
free HBM for its KV pool, a plugin without access to its host's allocator, a
latency-critical loop where cudaMalloc's device synchronisation is not
allowed).  For them pkv_decode_static_workspace runs the decode kernel on
scratch that lives inside libpkv.  These tests call it through the C ABI and
check it against pkv_decode with a caller-owned workspace, on two calls in a
row (the second call reuses the scratch the first one left behind).

The file is named to be collected last, so a run that stops at the first
failure has already run every other test; it passes on its own in a fresh
process as well as after the others.
"""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_479_b200 as pkv
from paged_kv_cache_479_b200 import workloads as wl

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
REL_L2 = 2e-3
LSE_ABS = 1e-3


def _device_case():
    w = wl.make_workload("no-alloc", [1000, 17, 300, 4096, 1, 2049], num_qo_heads=32,
                         num_kv_heads=8, page_size=16, dtype="bf16", seed=77, pool_factor=1.3)
    q, pool, _, _ = wl.make_tensors(w, "cpu")
    dev = torch.device("cuda")
    t = lambda a: torch.as_tensor(a, device=dev)
    return (w, q.to(dev), pool.to(dev), t(w.page_indptr), t(w.page_indices),
            t(w.last_page_len))


def _call_c_abi(w, q, pool, indptr, indices, last, out, lse, err, num_partitions=0):
    p = lambda x: ctypes.c_void_p(x.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return pkv.lib().pkv_decode_static_workspace(
        p(q), w.num_qo_heads, p(pool), w.num_pages, w.page_size, w.num_kv_heads, 128, pkv.BF16,
        p(indptr), p(indices), p(last), w.batch, w.sm_scale, num_partitions, p(out), p(lse),
        p(err), stream)


def test_static_workspace_matches_caller_workspace_twice():
    w, q, pool, indptr, indices, last = _device_case()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.zeros(pkv.decode_workspace_bytes(w.batch, 32, 8) // 4 + 64, dtype=torch.int32,
                     device="cuda")
    ref_o, ref_l = pkv.paged_decode_attention(q, pool, indptr, indices, last, ws,
                                              sm_scale=w.sm_scale, error_word=err)
    torch.cuda.synchronize()
    ref_o = ref_o.double().cpu().numpy()
    ref_l = ref_l.double().cpu().numpy()
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.full((w.batch, 32), float("nan"), device="cuda")
        st = _call_c_abi(w, q, pool, indptr, indices, last, out, lse, err)
        assert st == 0, pkv.lib().pkv_last_error()
        torch.cuda.synchronize()
        o = out.double().cpu().numpy()
        l = lse.double().cpu().numpy()
        assert np.isfinite(o).all() and np.isfinite(l).all(), f"call {call}"
        diff = o - ref_o
        assert np.abs(diff).max() <= MAX_ABS, f"call {call}"
        assert np.linalg.norm(diff) / np.linalg.norm(ref_o) <= REL_L2, f"call {call}"
        assert np.abs(l - ref_l).max() <= LSE_ABS, f"call {call}"
    assert pkv.read_error_word(err) == 0


def test_static_workspace_rejects_oversize_request():
    w, q, pool, indptr, indices, last = _device_case()
    out = torch.empty_like(q)
    lse = torch.empty((w.batch, 32), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    # 100000 partitions would need far more than the static scratch holds
    st = _call_c_abi(w, q, pool, indptr, indices, last, out, lse, err, num_partitions=100000)
    assert st == 3   # PKV_ERR_WORKSPACE, nothing launched
    assert b"static scratch" in pkv.lib().pkv_last_error()
