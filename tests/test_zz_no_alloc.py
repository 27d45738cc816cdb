"""The decode entry point that allocates nothing (pkv_decode_static_workspace).

Some users of this library cannot allocate device memory where they decode
and have no spare buffer to lend as a workspace (an engine that reserved all
free HBM for its KV pool, a plugin without access to its host's allocator, a
latency-critical loop where cudaMalloc's device synchronisation is not
allowed).  For them pkv_decode_static_workspace runs the decode kernel on
scratch that lives inside libpkv.  These tests call it through the C ABI and
check it against pkv_decode with a caller-owned workspace at the same
partition count -- bitwise, since for a fixed partition count the kernel's
results are reproducible -- on calls in a row that reuse what the previous
call left in the shared scratch, with partition counts that reshape the
scratch's counter and state regions between calls, and against the fp64
oracle once.

The file is named to be collected last, so a run that stops at the first
failure has already run every other test; it passes on its own in a fresh
process as well as after the others.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_479_b200 as pkv
from paged_kv_cache_479_b200 import workloads as wl

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
REL_L2 = 2e-3
LSE_ABS = 1e-3


def _case(hq, hkv, seed):
    w = wl.make_workload("no-alloc", [1000, 17, 300, 4096, 1, 2049, 0, 513], num_qo_heads=hq,
                         num_kv_heads=hkv, page_size=16, dtype="bf16", seed=seed,
                         pool_factor=1.3)
    q, pool, _, _ = wl.make_tensors(w, "cpu")
    dev = torch.device("cuda")
    t = lambda a: torch.as_tensor(a, device=dev)
    return (w, q, pool, q.to(dev), pool.to(dev), t(w.page_indptr), t(w.page_indices),
            t(w.last_page_len))


def _call_c_abi(w, q, pool, indptr, indices, last, out, lse, err, num_partitions=0):
    p = lambda x: ctypes.c_void_p(x.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return pkv.lib().pkv_decode_static_workspace(
        p(q), w.num_qo_heads, p(pool), w.num_pages, w.page_size, w.num_kv_heads, 128, pkv.BF16,
        p(indptr), p(indices), p(last), w.batch, w.sm_scale, num_partitions, p(out), p(lse),
        p(err), stream)


def _caller_ws(w, q, pool, indptr, indices, last, n, err):
    ws = torch.zeros(pkv.decode_workspace_bytes(w.batch, w.num_qo_heads, w.num_kv_heads, 128, n)
                     // 4 + 64, dtype=torch.int32, device="cuda")
    o, l = pkv.paged_decode_attention(q, pool, indptr, indices, last, ws, sm_scale=w.sm_scale,
                                      num_partitions=n, error_word=err)
    torch.cuda.synchronize()
    return o, l


@pytest.mark.parametrize("hq,hkv", [(32, 8), (64, 8)])
def test_static_workspace_bitwise_equal_across_partition_counts(hq, hkv):
    """Calls in a row on the shared scratch -- 148, 7, 148 partitions, then
    the default -- each bitwise equal to pkv_decode with its own zeroed
    workspace at the same partition count; the first is checked against the
    fp64 oracle."""
    w, q_h, pool_h, q, pool, indptr, indices, last = _case(hq, hkv, seed=77 + hq)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call, n in enumerate([148, 7, 148, 0]):
        ref_o, ref_l = _caller_ws(w, q, pool, indptr, indices, last, n, err)
        out = torch.full_like(q, float("nan"))
        lse = torch.full((w.batch, hq), float("nan"), device="cuda")
        st = _call_c_abi(w, q, pool, indptr, indices, last, out, lse, err, num_partitions=n)
        assert st == 0, pkv.lib().pkv_last_error()
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref_o.view(torch.int16)), f"call {call}, N={n}"
        assert torch.equal(lse.view(torch.int32), ref_l.view(torch.int32)), f"call {call}, N={n}"
        if call == 0:
            exp_o, exp_l = oracle.decode(wl.bits(q_h), wl.bits(pool_h), oracle.BF16,
                                         w.page_indptr, w.page_indices, w.last_page_len,
                                         w.sm_scale)
            o = out.double().cpu().numpy()
            l = lse.double().cpu().numpy()
            assert np.isfinite(o).all()
            diff = o - exp_o
            assert np.abs(diff).max() <= MAX_ABS
            assert np.linalg.norm(diff) / np.linalg.norm(exp_o) <= REL_L2
            with np.errstate(invalid="ignore"):
                dl = np.where(np.isneginf(l) & np.isneginf(exp_l), 0.0, l - exp_l)
            assert np.abs(dl).max() <= LSE_ABS
    assert pkv.read_error_word(err) == 0


def test_static_workspace_rejects_oversize_request():
    w, _, _, q, pool, indptr, indices, last = _case(32, 8, seed=77)
    out = torch.empty_like(q)
    lse = torch.empty((w.batch, 32), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    # 100000 partitions would need far more than the static scratch holds
    st = _call_c_abi(w, q, pool, indptr, indices, last, out, lse, err, num_partitions=100000)
    assert st == 3   # PKV_ERR_WORKSPACE, nothing launched
    assert b"static scratch" in pkv.lib().pkv_last_error()
