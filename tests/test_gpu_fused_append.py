"""GPU parity of the fused step (pkv_decode_append): the pool it leaves is
bitwise what pkv_append_ex writes, and its out / lse are bitwise what
pkv_decode_ex computes on that pool -- and match the oracle's append and
decode."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_479_b200 as pkv
from paged_kv_cache_479_b200 import workloads as wl
from _util import assert_parity, oracle_decode

pytestmark = pytest.mark.gpu


def i32(a):
    return torch.as_tensor(np.ascontiguousarray(a, np.int32), device="cuda")


def dense_block_table(w):
    nps = np.diff(w.page_indptr)
    bt = np.full((w.batch, int(max(1, nps.max()))), -1, np.int32)
    for b in range(w.batch):
        bt[b, :nps[b]] = w.pages_of(b)
    return bt, w.kv_lens.astype(np.int32)


def workspace(w, parts=0):
    nb = pkv.decode_workspace_bytes(w.batch, w.num_qo_heads, w.num_kv_heads, 128, parts)
    return torch.zeros(nb // 4 + 64, dtype=torch.int32, device="cuda")


CASES = [
    # lens (after the append), appended tokens, hq, hkv, ps, dtype
    ([1000, 17, 300, 4097, 1], [1, 1, 1, 1, 1], 32, 8, 16, "bf16"),          # decode step
    ([1, 15, 16, 17, 33, 300, 700], [1, 15, 1, 17, 2, 40, 600], 8, 4, 16, "bf16"),  # many rows
    ([513, 2000, 64], [3, 64, 64], 16, 2, 64, "f16"),
    ([129, 0, 260], [129, 0, 5], 8, 1, 32, "bf16"),                        # whole request new
]


@pytest.mark.parametrize("layout,kind", [("HND", "csr"), ("NHD", "block")])
@pytest.mark.parametrize("parts", [0, 7])
@pytest.mark.parametrize("i", range(len(CASES)))
def test_fused_step_matches_append_then_decode(i, parts, layout, kind):
    lens, counts, hq, hkv, ps, dt = CASES[i]
    w = wl.make_workload("fused", lens, num_qo_heads=hq, num_kv_heads=hkv, page_size=ps,
                         dtype=dt, seed=900 + i, pool_factor=1.3, append_counts=counts)
    q, pool, k_new, v_new = wl.make_tensors(w, "cpu")
    pool_after = oracle.append(wl.bits(pool), w.page_indptr, w.page_indices, w.last_page_len,
                               wl.bits(k_new), wl.bits(v_new), w.append_indptr)
    q, k_new, v_new = q.cuda(), k_new.cuda(), v_new.cuda()
    base = pool.permute(0, 1, 3, 2, 4).contiguous() if layout == "NHD" else pool
    if kind == "csr":
        keep = (i32(w.page_indptr), i32(w.page_indices), i32(w.last_page_len))
        table = pkv.csr_table(*keep)
    else:
        bt, ctx = dense_block_table(w)
        keep = (i32(bt), i32(ctx))
        table = pkv.block_table(*keep)
    app = i32(w.append_indptr)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    # separate calls
    p_sep = base.cuda()
    pkv.paged_kv_append_ex(p_sep, table, k_new, v_new, app, layout=layout, error_word=err)
    o_sep, l_sep = pkv.paged_decode_attention_ex(q, p_sep, table, workspace(w, parts),
                                                 layout=layout, sm_scale=w.sm_scale,
                                                 num_partitions=parts, error_word=err)
    # fused
    p_fus = base.cuda()
    o_fus, l_fus = pkv.paged_decode_append(q, p_fus, table, k_new, v_new, app, workspace(w, parts),
                                           layout=layout, sm_scale=w.sm_scale,
                                           num_partitions=parts, error_word=err)
    torch.cuda.synchronize()
    assert pkv.read_error_word(err) == 0
    # bitwise (unused slots hold NaN canaries, which compare unequal as values)
    assert torch.equal(p_fus.view(torch.int16), p_sep.view(torch.int16))
    assert torch.equal(o_fus, o_sep) and torch.equal(l_fus, l_sep)
    hnd = p_fus.permute(0, 1, 3, 2, 4).contiguous() if layout == "NHD" else p_fus
    assert np.array_equal(wl.bits(hnd), pool_after)
    ro, rl = oracle_decode(w, wl.bits(q), pool_after)
    assert_parity(o_fus, l_fus, ro, rl, what=f"fused case {i}")


def test_fused_step_bad_append_indptr_sets_error_bit():
    w = wl.make_workload("fused-bad", [100, 50], num_qo_heads=8, num_kv_heads=2, page_size=16,
                         dtype="bf16", seed=950, pool_factor=1.3, append_counts=[1, 1])
    q, pool, k_new, v_new = wl.make_tensors(w, "cuda")
    keep = (i32(w.page_indptr), i32(w.page_indices), i32(w.last_page_len))
    table = pkv.csr_table(*keep)
    bad = i32([0, 1, 5])                            # request 1 claims rows past nnz_new
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.paged_decode_append(q, pool, table, k_new, v_new, bad, workspace(w), sm_scale=w.sm_scale,
                            error_word=err)
    torch.cuda.synchronize()
    assert pkv.read_error_word(err) & pkv.DEVERR_APPEND
