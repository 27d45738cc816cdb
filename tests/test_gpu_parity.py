"""GPU parity: the CUDA library (through the C ABI) against the fp64 CPU oracle
on identical seeded inputs.

Bar: page-append bit-exact (the whole pool, canaries included); 16-bit
attention output with max |err| <= 1e-2 and relative L2 error <= 2e-3, lse
within 1e-3, and every output finite (NaN canaries sit in every slot that
holds no token, so any stray read shows up)."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_479_b200 as pkv
from paged_kv_cache_479_b200 import workloads as wl
from _util import DeviceCase, assert_parity, errors, oracle_decode, oracle_decode_from_device

pytestmark = pytest.mark.gpu


def host_case(w, num_partitions=0):
    q, pool, k_new, v_new = wl.make_tensors(w, "cpu")
    return DeviceCase(w, q, pool, k_new, v_new, num_partitions), q, pool, k_new, v_new


# ------------------------------------------------------------------ append

@pytest.mark.parametrize("cfg", ["ragged", "named2"])
def test_append_bit_exact(cfg):
    if cfg == "named2":
        w = wl.named(2)
    else:
        w = wl.make_workload("append", [1, 15, 16, 17, 33, 300, 64, 5], num_qo_heads=8,
                             num_kv_heads=4, page_size=16, dtype="f16", seed=31, pool_factor=1.5,
                             append_counts=[1, 15, 1, 17, 2, 40, 16, 0])
    dc, q, pool, k_new, v_new = host_case(w)
    expect = oracle.append(wl.bits(pool), w.page_indptr, w.page_indices, w.last_page_len,
                           wl.bits(k_new), wl.bits(v_new), w.append_indptr)
    dc.append()
    torch.cuda.synchronize()
    got = wl.bits(dc.pool)
    assert np.array_equal(got, expect)
    assert dc.error_bits() == 0


@pytest.mark.parametrize("ps", [32, 256])
def test_append_large_pages(ps):
    w = wl.make_workload("append", [700, 3, 256], num_qo_heads=4, num_kv_heads=2, page_size=ps,
                         dtype="bf16", seed=32, pool_factor=1.3, append_counts=[300, 3, 1])
    dc, q, pool, k_new, v_new = host_case(w)
    expect = oracle.append(wl.bits(pool), w.page_indptr, w.page_indices, w.last_page_len,
                           wl.bits(k_new), wl.bits(v_new), w.append_indptr)
    dc.append()
    torch.cuda.synchronize()
    assert np.array_equal(wl.bits(dc.pool), expect)


# ------------------------------------------------------------------ decode, small shapes

SMALL = [
    # lens, hq, hkv, ps, dtype
    ([17, 64, 100, 255], 8, 2, 16, "f16"),
    ([1, 2, 15, 16, 17, 31, 32, 33], 32, 8, 16, "bf16"),
    ([1000, 1, 513], 64, 8, 16, "bf16"),
    ([300, 7, 0, 45], 8, 8, 32, "bf16"),
    ([777, 1, 64], 16, 4, 64, "f16"),
    ([2000, 129], 8, 8, 128, "bf16"),
    ([5000, 256, 257], 32, 8, 256, "bf16"),
    ([100, 37], 4, 4, 16, "f16"),
    ([129, 3000], 16, 8, 16, "bf16"),
]


@pytest.mark.parametrize("i", range(len(SMALL)))
@pytest.mark.parametrize("N", [0, 1, 5])
def test_decode_small_shapes(i, N):
    lens, hq, hkv, ps, dt = SMALL[i]
    w = wl.make_workload("small", lens, num_qo_heads=hq, num_kv_heads=hkv, page_size=ps,
                         dtype=dt, seed=40 + i, pool_factor=1.4)
    dc, q, pool, _, _ = host_case(w, N)
    out, lse = dc.decode()
    ref_o, ref_l = oracle_decode(w, wl.bits(q), wl.bits(pool))
    assert_parity(out, lse, ref_o, ref_l, what=f"case {i} N={N}")
    assert dc.error_bits() == 0
    empty = np.flatnonzero(w.kv_lens == 0)
    if len(empty):
        assert torch.all(out[empty] == 0) and torch.all(torch.isneginf(lse[empty]))


def test_many_tiny_requests():
    rng = np.random.default_rng(5)
    lens = rng.integers(0, 40, size=700)
    w = wl.make_workload("tiny-many", lens, num_qo_heads=16, num_kv_heads=4, page_size=16,
                         dtype="bf16", seed=41, pool_factor=1.2)
    for N in (0, 3, 64):
        dc, q, pool, _, _ = host_case(w, N)
        out, lse = dc.decode()
        ref_o, ref_l = oracle_decode(w, wl.bits(q), wl.bits(pool))
        assert_parity(out, lse, ref_o, ref_l, what=f"N={N}")


def test_large_logits_and_peaked_softmax():
    w = wl.make_workload("peaked", [3000, 40], num_qo_heads=16, num_kv_heads=2, page_size=32,
                         dtype="bf16", seed=42, q_std=3.0, key_offset_std=8.0)
    dc, q, pool, _, _ = host_case(w)
    out, lse = dc.decode()
    ref_o, ref_l = oracle_decode(w, wl.bits(q), wl.bits(pool))
    assert np.abs(ref_l).max() > 50
    assert_parity(out, lse, ref_o, ref_l)


def test_single_token_returns_value():
    # one cached token: the weight is exactly 1, so the output is V_0 rounded once
    w = wl.make_workload("one", [1, 1, 1], num_qo_heads=8, num_kv_heads=2, page_size=16,
                         dtype="bf16", seed=43)
    dc, q, pool, _, _ = host_case(w)
    out, lse = dc.decode()
    for b in range(3):
        page = w.pages_of(b)[0]
        for h in range(8):
            assert torch.equal(out[b, h].cpu(), pool[page, 1, h // 4, 0])


# ------------------------------------------------------------------ invariances

def test_page_permutation_bitwise_and_determinism():
    w = wl.make_workload("perm", [900, 33, 2500, 16], num_qo_heads=32, num_kv_heads=8,
                         page_size=16, dtype="bf16", seed=44, pool_factor=1.3)
    dc, q, pool, _, _ = host_case(w)
    out1, lse1 = dc.decode()
    out2, lse2 = dc.decode()
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)
    perm = np.random.default_rng(3).permutation(w.num_pages)
    pool_p = torch.empty_like(pool)
    pool_p[torch.as_tensor(perm)] = pool
    wp = wl.Workload(**{**w.__dict__, "page_indices": perm[w.page_indices].astype(np.int32)})
    dcp = DeviceCase(wp, q, pool_p)
    out3, lse3 = dcp.decode()
    assert torch.equal(out1, out3) and torch.equal(lse1, lse3)


def test_partition_count_only_changes_rounding():
    w = wl.make_workload("split", [4000, 100, 2049], num_qo_heads=64, num_kv_heads=8,
                         page_size=16, dtype="bf16", seed=45)
    dc, q, pool, _, _ = host_case(w)
    ref_o, ref_l = oracle_decode(w, wl.bits(q), wl.bits(pool))
    lses = []
    for N in (1, 2, 7, 0, 300):
        out, lse = dc.decode(num_partitions=N)
        assert_parity(out, lse, ref_o, ref_l, what=f"N={N}")
        lses.append(lse.cpu().numpy())
    for l in lses[1:]:
        np.testing.assert_allclose(l, lses[0], rtol=0, atol=1e-4)


# ------------------------------------------------------------------ device-side table errors

def test_bad_page_id_sets_error_bit_and_completes():
    w = wl.make_workload("bad", [100, 50], num_qo_heads=8, num_kv_heads=2, page_size=16,
                         dtype="f16", seed=46)
    q, pool, _, _ = wl.make_tensors(w)
    bad = w.page_indices.copy()
    bad[2] = w.num_pages + 5
    wb = wl.Workload(**{**w.__dict__, "page_indices": bad})
    dc = DeviceCase(wb, q, pool)
    dc.decode()
    assert dc.error_bits() & pkv.DEVERR_PAGE_ID
    assert dc.error_bits() == 0   # read_error_word cleared it
    # the same word after a clean call stays clear
    DeviceCase(w, q, pool).decode()


def test_bad_last_page_len_sets_error_bit():
    w = wl.make_workload("bad", [100, 50], num_qo_heads=8, num_kv_heads=2, page_size=16,
                         dtype="f16", seed=47)
    q, pool, _, _ = wl.make_tensors(w)
    last = w.last_page_len.copy()
    last[1] = 17
    dc = DeviceCase(wl.Workload(**{**w.__dict__, "last_page_len": last}), q, pool)
    out, lse = dc.decode()
    assert dc.error_bits() & pkv.DEVERR_LAST_LEN
    assert torch.all(out[1] == 0)


def test_append_overflow_sets_error_bit():
    w = wl.make_workload("bad", [3], num_qo_heads=2, num_kv_heads=1, page_size=16, dtype="f16",
                         seed=48, append_counts=[2])
    dc, q, pool, k_new, v_new = host_case(w)
    dc.append_indptr = torch.tensor([0, 4], dtype=torch.int32, device="cuda")
    dc.k_new = torch.zeros((4, 1, 128), dtype=torch.float16, device="cuda")
    dc.v_new = dc.k_new.clone()
    before = dc.pool.clone()
    dc.append()
    assert dc.error_bits() & pkv.DEVERR_APPEND
    # rows that fit were written, the overflowing ones were skipped
    assert not torch.equal(before, dc.pool)


# ------------------------------------------------------------------ merge

# whole rows through shared memory (S * H a multiple of 4, rows up to 112 KiB:
# 5 and 20 states of 8 heads), one warp per (row, head) with 16-byte loads (40
# states: five batches of 8; 3 x 3 heads), per-dim loads (head_dim 64, 200)
@pytest.mark.parametrize("out_dtype,S,D,H", [(torch.float32, 5, 128, 8), (torch.bfloat16, 5, 128, 8),
                                             (torch.float16, 5, 128, 8), (torch.float32, 20, 128, 8),
                                             (torch.float32, 40, 128, 8),
                                             (torch.bfloat16, 3, 128, 3), (torch.float32, 3, 64, 8),
                                             (torch.float32, 7, 200, 8)])
def test_merge_states_matches_oracle(out_dtype, S, D, H):
    g = torch.Generator().manual_seed(9)
    N = 37
    v = torch.randn((N, S, H, D), generator=g)
    s = torch.randn((N, S, H), generator=g) * 4
    s[3, 2] = -float("inf")
    v[3, 2] = float("nan")        # no weight, so its values never matter
    s[5] = -float("inf")          # a row with no keys at all
    ref_o, ref_s = oracle.merge(v.double().numpy(), s.double().numpy())
    vo, so = pkv.merge_states(v.cuda(), s.cuda(), out_dtype=out_dtype)
    torch.cuda.synchronize()
    vo = vo.float().cpu().numpy()
    tol = 1e-5 if out_dtype == torch.float32 else (1e-2 if out_dtype == torch.bfloat16 else 2e-3)
    np.testing.assert_allclose(vo, ref_o, rtol=0, atol=tol * max(1.0, np.abs(ref_o).max()))
    so = so.cpu().numpy()
    assert np.all(np.isneginf(so[5])) and np.all(vo[5] == 0)
    fin = np.isfinite(ref_s)
    np.testing.assert_allclose(so[fin], ref_s[fin], rtol=0, atol=1e-5)


def test_merge_paths_bitwise_equal():
    """Up to 8 states the shared-memory row path and the per-warp path take the
    same maximum and add in the same order: bitwise equal results.  A lse array
    one float off 16-byte alignment sends the call down the per-warp path."""
    g = torch.Generator().manual_seed(11)
    N, S, H, D = 29, 5, 8, 128
    v = torch.randn((N, S, H, D), generator=g).cuda()
    s = torch.randn((N, S, H), generator=g) * 4
    s[2, 1] = -float("inf")
    s[4] = -float("inf")
    s_aligned = s.cuda()
    buf = torch.empty(N * S * H + 1, device="cuda")
    s_offset = buf[1:].view(N, S, H)
    s_offset.copy_(s_aligned)
    assert s_aligned.data_ptr() % 16 == 0 and s_offset.data_ptr() % 16 != 0
    for dt, iv in ((torch.bfloat16, torch.int16), (torch.float16, torch.int16),
                   (torch.float32, torch.int32)):
        o1, l1 = pkv.merge_states(v, s_aligned, out_dtype=dt)
        o2, l2 = pkv.merge_states(v, s_offset, out_dtype=dt)
        torch.cuda.synchronize()
        assert torch.equal(o1.view(iv), o2.view(iv)), dt
        assert torch.equal(l1.view(torch.int32), l2.view(torch.int32)), dt


def test_merge_of_gpu_splits_equals_whole():
    # decode two halves of each request separately, merge with the library's
    # merge kernel, compare with decoding the whole request
    lens = [1000, 700]
    w = wl.make_workload("whole", lens, num_qo_heads=32, num_kv_heads=8, page_size=16,
                         dtype="bf16", seed=49)
    dc, q, pool, _, _ = host_case(w)
    whole_o, whole_l = dc.decode()
    cut = 512
    # halves as separate requests over the same pages: [0, cut) and [cut, L)
    ip, ix, ll = [0], [], []
    for b in range(2):
        pages = list(w.pages_of(b))
        ix += pages[:cut // 16]; ip.append(len(ix)); ll.append(16)
        rest = pages[cut // 16:]; ix += rest; ip.append(len(ix)); ll.append(int(w.last_page_len[b]))
    # the second half of each request starts at token `cut` (page aligned)
    wh = wl.Workload(**{**w.__dict__, "batch": 4, "page_indptr": np.array(ip, np.int32),
                        "page_indices": np.array(ix, np.int32), "last_page_len": np.array(ll, np.int32),
                        "kv_lens": np.array([cut, lens[0] - cut, cut, lens[1] - cut]),
                        "append_counts": np.zeros(4, np.int64)})
    qh = q.repeat_interleave(2, dim=0)
    dh = DeviceCase(wh, qh, pool)
    ho, hl = dh.decode()
    # the halves' bf16 outputs, widened, are the partial states to merge
    v = ho.float().view(2, 2, 32, 128).contiguous()
    s = hl.view(2, 2, 32).contiguous()
    mo, ml = pkv.merge_states(v, s, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle_decode(w, wl.bits(q), wl.bits(pool))
    e = errors(mo, ml, ref_o, ref_l)
    assert e["max_abs"] <= 1e-2 and e["rel_l2"] <= 4e-3 and e["lse_abs"] <= 1e-3, e


# ------------------------------------------------------------------ the named workloads

def test_named_1_tiny():
    w = wl.named(1)
    dc, q, pool, _, _ = host_case(w)
    out, lse = dc.decode()
    ref_o, ref_l = oracle_decode(w, wl.bits(q), wl.bits(pool))
    assert_parity(out, lse, ref_o, ref_l, what="named 1")


def test_named_2_append_then_decode():
    w = wl.named(2)
    dc, q, pool, k_new, v_new = host_case(w)
    dc.append()
    out, lse = dc.decode()
    pool_after = oracle.append(wl.bits(pool), w.page_indptr, w.page_indices, w.last_page_len,
                               wl.bits(k_new), wl.bits(v_new), w.append_indptr)
    ref_o, ref_l = oracle_decode(w, wl.bits(q), pool_after)
    assert_parity(out, lse, ref_o, ref_l, what="named 2")
    assert dc.error_bits() == 0


def _device_named(cfg, sample):
    w = wl.named(cfg)
    q, pool, _, _ = wl.make_tensors(w, "cuda")
    dc = DeviceCase(w, q, pool)
    out, lse = dc.decode()
    ref_o, ref_l = oracle_decode_from_device(w, q, pool, sample)
    e = assert_parity(out, lse, ref_o, ref_l, rows=sample, what=f"named {cfg}")
    assert torch.isfinite(out.float()).all()
    assert dc.error_bits() == 0
    return e


def test_named_3_long_context_every_request():
    """The 128K workload in full: all 8 requests against the oracle, each
    request's pages copied to the host on its own (537 MB at a time); the
    bar applies to the whole output."""
    w = wl.named(3)
    q, pool, _, _ = wl.make_tensors(w, "cuda")
    dc = DeviceCase(w, q, pool)
    out, lse = dc.decode()
    assert dc.error_bits() == 0
    ref_o = np.zeros((w.batch, w.num_qo_heads, w.head_dim))
    ref_l = np.zeros((w.batch, w.num_qo_heads))
    for b in range(w.batch):
        o_b, l_b = oracle_decode_from_device(w, q, pool, [b])
        ref_o[b], ref_l[b] = o_b[0], l_b[0]
    assert_parity(out, lse, ref_o, ref_l, what="named 3, all requests")


def test_named_4_single_200k_sequence():
    _device_named(4, [0])


def test_named_5_shared_prefix_sampled():
    _device_named(5, [0, 17, 101, 255])
