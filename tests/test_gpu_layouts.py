"""GPU parity of the descriptor calls: NHD pools and dense (vLLM-style) block
tables give the same results as the HND / CSR path, and match the oracle."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_479_b200 as pkv
from paged_kv_cache_479_b200 import workloads as wl
from _util import assert_parity, oracle_decode

pytestmark = pytest.mark.gpu


def dense_block_table(w, pad=-1):
    """CSR table -> [B, max_blocks] block table (unused entries = pad) + context lengths."""
    nps = np.diff(w.page_indptr)
    mb = int(max(1, nps.max()))
    bt = np.full((w.batch, mb), pad, np.int32)
    for b in range(w.batch):
        bt[b, :nps[b]] = w.pages_of(b)
    return bt, w.kv_lens.astype(np.int32)


def workspace(w):
    return torch.zeros(pkv.decode_workspace_bytes(w.batch, w.num_qo_heads, w.num_kv_heads) // 4 + 64,
                       dtype=torch.int32, device="cuda")


@pytest.mark.parametrize("layout,kind", [("HND", "block"), ("NHD", "csr"), ("NHD", "block")])
@pytest.mark.parametrize("cfg", [0, 1])
def test_decode_layouts_and_tables(layout, kind, cfg):
    if cfg == 0:
        w = wl.make_workload("lt", [1000, 17, 0, 300, 4097], num_qo_heads=32, num_kv_heads=8,
                             page_size=16, dtype="bf16", seed=80, pool_factor=1.3)
    else:
        w = wl.make_workload("lt", [513, 2000, 1], num_qo_heads=16, num_kv_heads=2,
                             page_size=64, dtype="f16", seed=81, pool_factor=1.2)
    q, pool, _, _ = wl.make_tensors(w, "cpu")
    q, pool = q.cuda(), pool.cuda()
    t = lambda a: torch.as_tensor(np.ascontiguousarray(a, np.int32), device="cuda")
    ip, ix, ll = t(w.page_indptr), t(w.page_indices), t(w.last_page_len)
    ref_out, ref_lse = pkv.paged_decode_attention(q, pool, ip, ix, ll, workspace(w),
                                                  sm_scale=w.sm_scale)
    p = pool.permute(0, 1, 3, 2, 4).contiguous() if layout == "NHD" else pool
    if kind == "csr":
        table = pkv.csr_table(ip, ix, ll)
        keep = (ip, ix, ll)
    else:
        bt, ctx = dense_block_table(w)
        keep = (t(bt), t(ctx))
        table = pkv.block_table(*keep)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = pkv.paged_decode_attention_ex(q, p, table, workspace(w), layout=layout,
                                             sm_scale=w.sm_scale, error_word=err)
    torch.cuda.synchronize()
    assert pkv.read_error_word(err) == 0
    # same tiles in shared memory, same partition: bitwise the same as HND / CSR
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    ro, rl = oracle_decode(w, wl.bits(q), wl.bits(pool))
    assert_parity(out, lse, ro, rl, what=f"{layout}/{kind}")


@pytest.mark.parametrize("layout,kind", [("HND", "block"), ("NHD", "csr"), ("NHD", "block")])
def test_append_layouts_and_tables(layout, kind):
    w = wl.make_workload("lta", [1, 15, 16, 17, 33, 300], num_qo_heads=8, num_kv_heads=4,
                         page_size=16, dtype="bf16", seed=82, pool_factor=1.5,
                         append_counts=[1, 15, 1, 17, 2, 40])
    q, pool, k_new, v_new = wl.make_tensors(w, "cpu")
    expect = oracle.append(wl.bits(pool), w.page_indptr, w.page_indices, w.last_page_len,
                           wl.bits(k_new), wl.bits(v_new), w.append_indptr)
    t = lambda a: torch.as_tensor(np.ascontiguousarray(a, np.int32), device="cuda")
    p = pool.permute(0, 1, 3, 2, 4).contiguous().cuda() if layout == "NHD" else pool.cuda()
    if kind == "csr":
        keep = (t(w.page_indptr), t(w.page_indices), t(w.last_page_len))
        table = pkv.csr_table(*keep)
    else:
        bt, ctx = dense_block_table(w)
        keep = (t(bt), t(ctx))
        table = pkv.block_table(*keep)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.paged_kv_append_ex(p, table, k_new.cuda(), v_new.cuda(), t(w.append_indptr),
                           layout=layout, error_word=err)
    torch.cuda.synchronize()
    assert pkv.read_error_word(err) == 0
    got = p.permute(0, 1, 3, 2, 4) if layout == "NHD" else p
    assert np.array_equal(wl.bits(got.contiguous()), expect)


def test_block_table_context_len_beyond_row_sets_error():
    w = wl.make_workload("ctx", [40, 20], num_qo_heads=8, num_kv_heads=2, page_size=16,
                         dtype="bf16", seed=83)
    q, pool, _, _ = wl.make_tensors(w, "cuda")
    bt, ctx = dense_block_table(w)
    ctx[1] = bt.shape[1] * 16 + 1          # more tokens than the row can hold
    t = lambda a: torch.as_tensor(np.ascontiguousarray(a, np.int32), device="cuda")
    keep = (t(bt), t(ctx))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = pkv.paged_decode_attention_ex(q, pool, pkv.block_table(*keep), workspace(w),
                                             sm_scale=w.sm_scale, error_word=err)
    torch.cuda.synchronize()
    assert pkv.read_error_word(err) & pkv.DEVERR_CONTEXT_LEN
    assert torch.all(out[1] == 0)


@pytest.mark.parametrize("kind", ["csr", "block"])
def test_table_ready_at_launch(kind):
    """PKV_TABLE_READY_AT_LAUNCH lets the decode read the table before the
    preceding kernel finishes.  That kernel may still write q and the pool:
    here each decode runs right after a kernel that rewrites q (and one that
    rewrites a page), and must see the new values -- bitwise the result of
    the same decode without the flag, and within the oracle's bounds."""
    w = wl.make_workload("early", [3000, 17, 0, 900, 1, 4096], num_qo_heads=32, num_kv_heads=8,
                         page_size=16, dtype="bf16", seed=82, pool_factor=1.3)
    q, pool, _, _ = wl.make_tensors(w, "cpu")
    q, pool = q.cuda(), pool.cuda()
    t = lambda a: torch.as_tensor(np.ascontiguousarray(a, np.int32), device="cuda")
    ip, ix, ll = t(w.page_indptr), t(w.page_indices), t(w.last_page_len)
    if kind == "csr":
        keep = (ip, ix, ll)
        table_f = pkv.csr_table(ip, ix, ll, ready_at_launch=True)
        table_0 = pkv.csr_table(ip, ix, ll)
    else:
        bt, ctx = dense_block_table(w)
        keep = (t(bt), t(ctx))
        table_f = pkv.block_table(*keep, ready_at_launch=True)
        table_0 = pkv.block_table(*keep)
    gen = torch.Generator(device="cuda").manual_seed(5)
    qs = [torch.randn(q.shape, generator=gen, device="cuda").to(q.dtype) for _ in range(4)]
    page = int(w.pages_of(0)[3])
    vals = [torch.randn(pool[page].shape, generator=gen, device="cuda").to(pool.dtype) for _ in range(4)]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws_f, ws_0 = workspace(w), workspace(w)
    outs = []
    for i in range(4):
        q.copy_(qs[i])            # a kernel right before the decode writes q ...
        pool[page].copy_(vals[i])  # ... and a page the decode reads
        outs.append(pkv.paged_decode_attention_ex(q, pool, table_f, ws_f, sm_scale=w.sm_scale,
                                                  error_word=err))
    torch.cuda.synchronize()
    assert pkv.read_error_word(err) == 0
    for i in range(4):
        q.copy_(qs[i])
        pool[page].copy_(vals[i])
        ref = pkv.paged_decode_attention_ex(q, pool, table_0, ws_0, sm_scale=w.sm_scale)
        torch.cuda.synchronize()
        assert torch.equal(outs[i][0], ref[0]) and torch.equal(outs[i][1], ref[1]), i
    ro, rl = oracle_decode(w, wl.bits(q), wl.bits(pool))
    assert_parity(outs[3][0], outs[3][1], ro, rl, what=f"ready at launch, {kind}")
