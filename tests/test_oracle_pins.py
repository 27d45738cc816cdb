"""Pins for the fp64 CPU oracle, checked against things other than itself.

Each test fixes the oracle to an independent fact: a library routine on the
same data (torch's scaled_dot_product_attention / logsumexp in float64 on
dense, unpaged K/V), a closed form, an invariance that the definition of
attention implies, a hand-derived tiny case, or a number the pages print.
A plausible slip in the oracle (swapped K/V, wrong head mapping, wrong
page/slot index, ignoring last_page_len, a missing max-subtraction, a wrong
merge weight) fails at least one of them; test_oracle_mutants.py plants such
slips in a copy of the oracle and checks that these pins catch them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_479_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# test-side helpers: write dense K/V INTO pages (the oracle reads them back)
# ---------------------------------------------------------------------------

def to_bits(x: torch.Tensor, dtype: str) -> np.ndarray:
    t = x.to(torch.float16 if dtype == "f16" else torch.bfloat16)
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def widen(bits: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.float16 if dtype == "f16" else torch.bfloat16).to(torch.float64)


def scatter_dense(w, k_dense, v_dense, fill=wl.CANARY):
    """Place per-request dense K/V ([L_b, Hkv, D] uint16 lists) into a pool
    following w's page table; every other slot keeps `fill`."""
    pool = np.full(w.pool_shape, fill, np.uint16)
    for b in range(w.batch):
        pages = w.pages_of(b)
        for t in range(int(w.kv_lens[b])):
            page, slot = pages[t // w.page_size], t % w.page_size
            pool[page, 0, :, slot, :] = k_dense[b][t]
            pool[page, 1, :, slot, :] = v_dense[b][t]
    return pool


def random_dense(w, gen, k_scale=1.0):
    ks, vs = [], []
    for b in range(w.batch):
        L = int(w.kv_lens[b])
        ks.append(to_bits(torch.randn((L, w.num_kv_heads, w.head_dim), generator=gen) * k_scale, w.dtype))
        vs.append(to_bits(torch.randn((L, w.num_kv_heads, w.head_dim), generator=gen), w.dtype))
    return ks, vs


def sdpa_reference(w, q_bits, k_dense, v_dense, scale):
    """torch SDPA (float64, CPU) on dense unpaged K/V; GQA via enable_gqa,
    which maps query head h to KV head h // (Hq/Hkv)."""
    outs, lses = [], []
    q = widen(q_bits, w.dtype)
    for b in range(w.batch):
        k = widen(k_dense[b], w.dtype).permute(1, 0, 2)[None]   # [1,Hkv,L,D]
        v = widen(v_dense[b], w.dtype).permute(1, 0, 2)[None]
        qb = q[b][None, :, None, :]                             # [1,Hq,1,D]
        o = torch.nn.functional.scaled_dot_product_attention(qb, k, v, scale=scale, enable_gqa=True)
        outs.append(o[0, :, 0, :])
        kk = k[0].repeat_interleave(w.group, dim=0)             # [Hq,L,D]
        s = torch.einsum("hd,hld->hl", q[b], kk) * scale
        lses.append(torch.logsumexp(s, dim=-1))
    return torch.stack(outs).numpy(), torch.stack(lses).numpy()


CASES = [
    # (lens, hq, hkv, ps, dtype, pool_factor)
    ([17, 64, 100, 255], 8, 2, 16, "f16", 2.2),
    ([1, 5, 33, 48, 200], 32, 8, 16, "bf16", 1.25),
    ([300, 7], 8, 8, 32, "bf16", 1.0),
    ([513], 8, 1, 256, "f16", 3.0),
    ([40, 16, 15, 17], 16, 2, 64, "bf16", 1.5),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_oracle_matches_dense_sdpa(case):
    lens, hq, hkv, ps, dtype, pf = CASES[case]
    w = wl.make_workload("pin", lens, num_qo_heads=hq, num_kv_heads=hkv, page_size=ps,
                         dtype=dtype, seed=100 + case, pool_factor=pf, head_dim=128)
    gen = torch.Generator().manual_seed(7 + case)
    k_dense, v_dense = random_dense(w, gen)
    q_bits = to_bits(torch.randn((w.batch, hq, 128), generator=gen), dtype)
    pool = scatter_dense(w, k_dense, v_dense)
    out, lse = oracle.decode(q_bits, pool, oracle.BF16 if dtype == "bf16" else oracle.F16,
                             w.page_indptr, w.page_indices, w.last_page_len, w.sm_scale)
    ref_o, ref_l = sdpa_reference(w, q_bits, k_dense, v_dense, w.sm_scale)
    assert np.isfinite(out).all()                 # canaries (NaN) never read
    np.testing.assert_allclose(out, ref_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_l, rtol=0, atol=1e-12)


def test_large_logits_need_max_subtraction():
    # scores of order 1e3: exp() overflows unless the max is subtracted first
    w = wl.make_workload("pin", [50, 9], num_qo_heads=4, num_kv_heads=2, page_size=16,
                         dtype="bf16", seed=3, pool_factor=1.0)
    gen = torch.Generator().manual_seed(11)
    k_dense, v_dense = random_dense(w, gen)
    q_bits = to_bits(torch.randn((2, 4, 128), generator=gen), "bf16")
    pool = scatter_dense(w, k_dense, v_dense)
    scale = 100.0
    out, lse = oracle.decode(q_bits, pool, oracle.BF16, w.page_indptr, w.page_indices,
                             w.last_page_len, scale)
    ref_o, ref_l = sdpa_reference(w, q_bits, k_dense, v_dense, scale)
    assert np.abs(lse).max() > 700
    np.testing.assert_allclose(out, ref_o, rtol=0, atol=1e-10)
    np.testing.assert_allclose(lse, ref_l, rtol=1e-14, atol=1e-9)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_single_token_returns_its_value_exactly(dtype):
    # one cached token: weight exactly 1, so o = V_0 and lse = s_0.  Spread every
    # finite 16-bit pattern over the V rows: this also pins the exact widening
    # of stored values (against numpy's float16 and torch's bfloat16 casts).
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = widen(allbits, dtype).numpy()
    finite = allbits[np.isfinite(vals)]
    D = 128
    nreq = -(-len(finite) // D)
    padded = np.zeros(nreq * D, np.uint16)
    padded[:len(finite)] = finite
    w = wl.make_workload("pin", [1] * nreq, num_qo_heads=2, num_kv_heads=1, page_size=16,
                         dtype=dtype, seed=5)
    gen = torch.Generator().manual_seed(1)
    k_dense = [to_bits(torch.randn((1, 1, D), generator=gen), dtype) for _ in range(nreq)]
    v_dense = [padded[i * D:(i + 1) * D].reshape(1, 1, D) for i in range(nreq)]
    q_bits = to_bits(torch.randn((nreq, 2, D), generator=gen), dtype)
    pool = scatter_dense(w, k_dense, v_dense)
    out, lse = oracle.decode(q_bits, pool, oracle.BF16 if dtype == "bf16" else oracle.F16,
                             w.page_indptr, w.page_indices, w.last_page_len, 0.25)
    expect_v = widen(np.stack([v[0, 0] for v in v_dense]), dtype).numpy()
    assert np.array_equal(out[:, 0, :], expect_v) and np.array_equal(out[:, 1, :], expect_v)
    q = widen(q_bits, dtype).numpy()
    k0 = widen(np.stack([k[0, 0] for k in k_dense]), dtype).numpy()
    s0 = 0.25 * np.einsum("nhd,nd->nh", q, k0)
    np.testing.assert_allclose(lse, s0, rtol=0, atol=1e-12)


def test_identical_keys_give_mean_of_values():
    # all keys equal: every score equals s, weights 1/L, o = mean V, lse = s + ln L
    L = 77
    w = wl.make_workload("pin", [L], num_qo_heads=4, num_kv_heads=1, page_size=16,
                         dtype="bf16", seed=9, pool_factor=2.0)
    gen = torch.Generator().manual_seed(2)
    key = to_bits(torch.randn((1, 1, 128), generator=gen), "bf16")
    k_dense = [np.repeat(key, L, axis=0)]
    v_dense = [to_bits(torch.randn((L, 1, 128), generator=gen), "bf16")]
    q_bits = to_bits(torch.randn((1, 4, 128), generator=gen), "bf16")
    pool = scatter_dense(w, k_dense, v_dense)
    out, lse = oracle.decode(q_bits, pool, oracle.BF16, w.page_indptr, w.page_indices,
                             w.last_page_len, w.sm_scale)
    mean_v = widen(v_dense[0], "bf16").numpy()[:, 0, :].mean(axis=0)
    s = w.sm_scale * widen(q_bits, "bf16").numpy()[0] @ widen(key, "bf16").numpy()[0, 0]
    for h in range(4):
        np.testing.assert_allclose(out[0, h], mean_v, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0], s + math.log(L), rtol=0, atol=1e-12)


def test_zero_query_gives_mean_of_values_and_value_shift():
    w = wl.make_workload("pin", [37, 3], num_qo_heads=2, num_kv_heads=2, page_size=16,
                         dtype="f16", seed=4, pool_factor=1.0)
    gen = torch.Generator().manual_seed(8)
    k_dense, v_dense = random_dense(w, gen)
    pool = scatter_dense(w, k_dense, v_dense)
    q0 = np.zeros((2, 2, 128), np.uint16)                  # +0.0 in fp16
    out, lse = oracle.decode(q0, pool, oracle.F16, w.page_indptr, w.page_indices,
                             w.last_page_len, w.sm_scale)
    for b in range(2):
        mv = widen(v_dense[b], "f16").numpy().mean(axis=0)   # [Hkv, D]
        np.testing.assert_allclose(out[b], mv, rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[b], math.log(w.kv_lens[b]), atol=1e-14)
    # V -> V + c shifts o by exactly c (weights sum to one).  V on a 1/64 grid
    # in [-4, 4] keeps V and V + 0.5 exact in fp16.
    v_dense = [to_bits(torch.randint(-256, 257, v.shape, generator=gen).double() / 64, "f16")
               for v in v_dense]
    pool = scatter_dense(w, k_dense, v_dense)
    q_bits = to_bits(torch.randn((2, 2, 128), generator=gen), "f16")
    base, _ = oracle.decode(q_bits, pool, oracle.F16, w.page_indptr, w.page_indices,
                            w.last_page_len, w.sm_scale)
    shifted_v = [to_bits(widen(v, "f16") + 0.5, "f16") for v in v_dense]
    assert all(np.array_equal(widen(s, "f16").numpy(), widen(v, "f16").numpy() + 0.5)
               for s, v in zip(shifted_v, v_dense))
    pool2 = scatter_dense(w, k_dense, shifted_v)
    shifted, _ = oracle.decode(q_bits, pool2, oracle.F16, w.page_indptr, w.page_indices,
                               w.last_page_len, w.sm_scale)
    np.testing.assert_allclose(shifted, base + 0.5, rtol=0, atol=1e-12)


def test_page_permutation_invariance_is_exact():
    w = wl.make_workload("pin", [130, 16, 61], num_qo_heads=8, num_kv_heads=2, page_size=16,
                         dtype="bf16", seed=12, pool_factor=1.5)
    gen = torch.Generator().manual_seed(3)
    k_dense, v_dense = random_dense(w, gen)
    q_bits = to_bits(torch.randn((3, 8, 128), generator=gen), "bf16")
    pool = scatter_dense(w, k_dense, v_dense)
    perm = np.random.default_rng(0).permutation(w.num_pages)
    pool_p = np.empty_like(pool)
    pool_p[perm] = pool                                    # physical page i -> perm[i]
    idx_p = perm[w.page_indices].astype(np.int32)
    a = oracle.decode(q_bits, pool, oracle.BF16, w.page_indptr, w.page_indices, w.last_page_len, w.sm_scale)
    b = oracle.decode(q_bits, pool_p, oracle.BF16, w.page_indptr, idx_p, w.last_page_len, w.sm_scale)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_token_permutation_invariance():
    # decode attention is a function of the SET of (k, v) pairs
    w = wl.make_workload("pin", [90], num_qo_heads=4, num_kv_heads=1, page_size=16,
                         dtype="bf16", seed=13)
    gen = torch.Generator().manual_seed(4)
    k_dense, v_dense = random_dense(w, gen)
    q_bits = to_bits(torch.randn((1, 4, 128), generator=gen), "bf16")
    perm = np.random.default_rng(1).permutation(90)
    a = oracle.decode(q_bits, scatter_dense(w, k_dense, v_dense), oracle.BF16,
                      w.page_indptr, w.page_indices, w.last_page_len, w.sm_scale)
    b = oracle.decode(q_bits, scatter_dense(w, [k_dense[0][perm]], [v_dense[0][perm]]), oracle.BF16,
                      w.page_indptr, w.page_indices, w.last_page_len, w.sm_scale)
    np.testing.assert_allclose(a[0], b[0], rtol=0, atol=1e-13)
    np.testing.assert_allclose(a[1], b[1], rtol=0, atol=1e-12)


def test_hand_derived_tiny_cases():
    # D = 4, page_size 2, dyadic values.  scale = ln 3 and q.k = (0, 1) give
    # weights (1, 3)/4: o = (V0 + 3 V1)/4, lse = ln 4.  A second request with
    # q.k = (0, 1, 2) and scale ln 2 gives weights (1, 2, 4)/7, lse = ln 7.
    # The second request's 3rd token sits on the first slot of its 2nd page.
    f16 = np.float16
    P, ps, D = 4, 2, 4
    pool = np.full((P, 2, 1, ps, D), wl.CANARY, np.uint16)
    def put(page, slot, k, v):
        pool[page, 0, 0, slot] = np.array(k, f16).view(np.uint16)
        pool[page, 1, 0, slot] = np.array(v, f16).view(np.uint16)
    # request 0: pages [3], tokens: k0=(0,0,0,0), k1=(1,0,0,0)
    put(3, 0, [0, 0, 0, 0], [1, 2, 3, 4])
    put(3, 1, [1, 0, 0, 0], [-1, 0.5, 8, 0.25])
    # request 1: pages [0, 2]: k=(0,..),(0,1,..),(0,2,..)
    put(0, 0, [0, 0, 0, 0], [7, 0, 0, 0])
    put(0, 1, [0, 1, 0, 0], [0, 7, 0, 0])
    put(2, 0, [0, 2, 0, 0], [0, 0, 7, 0])
    indptr = np.array([0, 1, 3], np.int32)
    indices = np.array([3, 0, 2], np.int32)
    last = np.array([2, 1], np.int32)
    q = np.array([[[1, 0, 0, 0]], [[0, 1, 0, 0]]], f16).view(np.uint16)
    o0, l0 = oracle.decode(q[:1], pool, oracle.F16, indptr[:2], indices, last[:1], math.log(3))
    np.testing.assert_allclose(o0[0, 0], [(1 - 3) / 4, (2 + 1.5) / 4, (3 + 24) / 4, (4 + 0.75) / 4], atol=1e-15)
    np.testing.assert_allclose(l0[0, 0], math.log(4), atol=1e-15)
    o1, l1 = oracle.decode(q[1:], pool, oracle.F16, np.array([0, 2], np.int32), indices[1:],
                           last[1:], math.log(2))
    np.testing.assert_allclose(o1[0, 0], [7 / 7, 14 / 7, 28 / 7, 0], atol=1e-14)
    np.testing.assert_allclose(l1[0, 0], math.log(7), atol=1e-15)


def test_empty_request_and_canaries():
    w = wl.make_workload("pin", [0, 20, 0, 3], num_qo_heads=4, num_kv_heads=2, page_size=16,
                         dtype="f16", seed=14, pool_factor=3.0)
    gen = torch.Generator().manual_seed(5)
    k_dense, v_dense = random_dense(w, gen)
    q_bits = to_bits(torch.randn((4, 4, 128), generator=gen), "f16")
    with_nan = scatter_dense(w, k_dense, v_dense, fill=wl.CANARY)
    with_junk = scatter_dense(w, k_dense, v_dense, fill=0x3C00)   # 1.0 everywhere else
    a = oracle.decode(q_bits, with_nan, oracle.F16, w.page_indptr, w.page_indices, w.last_page_len, w.sm_scale)
    b = oracle.decode(q_bits, with_junk, oracle.F16, w.page_indptr, w.page_indices, w.last_page_len, w.sm_scale)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    for r in (0, 2):
        assert np.all(a[0][r] == 0.0) and np.all(a[1][r] == -np.inf)
    assert np.isfinite(a[0][[1, 3]]).all()


def test_invalid_tables_are_rejected():
    w = wl.make_workload("pin", [20, 5], num_qo_heads=2, num_kv_heads=1, page_size=16,
                         dtype="f16", seed=15)
    q = np.zeros((2, 2, 128), np.uint16)
    pool = np.zeros(w.pool_shape, np.uint16)
    bad_last = w.last_page_len.copy(); bad_last[1] = 17
    with pytest.raises(oracle.OracleError):
        oracle.decode(q, pool, oracle.F16, w.page_indptr, w.page_indices, bad_last, 1.0)
    bad_last[1] = 0
    with pytest.raises(oracle.OracleError):
        oracle.decode(q, pool, oracle.F16, w.page_indptr, w.page_indices, bad_last, 1.0)
    bad_idx = w.page_indices.copy(); bad_idx[0] = w.num_pages
    with pytest.raises(oracle.OracleError):
        oracle.decode(q, pool, oracle.F16, w.page_indptr, bad_idx, w.last_page_len, 1.0)
    bad_ptr = np.array([0, 2, 1], np.int32)
    with pytest.raises(oracle.OracleError):
        oracle.decode(q, pool, oracle.F16, bad_ptr, w.page_indices, w.last_page_len, 1.0)


# ---------------------------------------------------------------------------
# merge
# ---------------------------------------------------------------------------

def test_merge_of_split_sequence_equals_whole():
    # attention over a sequence equals the LSE-merge of attention over any
    # partition of its tokens into consecutive parts
    L = 211
    cuts = [0, 1, 50, 51, 160, L]
    w = wl.make_workload("pin", [L], num_qo_heads=8, num_kv_heads=2, page_size=16,
                         dtype="bf16", seed=16)
    gen = torch.Generator().manual_seed(6)
    k_dense, v_dense = random_dense(w, gen)
    q_bits = to_bits(torch.randn((1, 8, 128), generator=gen), "bf16")
    whole = oracle.decode(q_bits, scatter_dense(w, k_dense, v_dense), oracle.BF16,
                          w.page_indptr, w.page_indices, w.last_page_len, w.sm_scale)
    parts = [(cuts[i], cuts[i + 1]) for i in range(len(cuts) - 1)]
    wp = wl.make_workload("pin", [e - s for s, e in parts], num_qo_heads=8, num_kv_heads=2,
                          page_size=16, dtype="bf16", seed=17)
    po, pl = oracle.decode(np.repeat(q_bits, len(parts), axis=0),
                           scatter_dense(wp, [k_dense[0][s:e] for s, e in parts],
                                         [v_dense[0][s:e] for s, e in parts]),
                           oracle.BF16, wp.page_indptr, wp.page_indices, wp.last_page_len, w.sm_scale)
    mo, ml = oracle.merge(po[None], pl[None])
    np.testing.assert_allclose(mo[0], whole[0][0], rtol=0, atol=1e-13)
    np.testing.assert_allclose(ml[0], whole[1][0], rtol=0, atol=1e-12)


def test_merge_closed_forms():
    rng = np.random.default_rng(0)
    v = rng.normal(size=(3, 4, 2, 8))
    s = rng.normal(size=(3, 4, 2))
    # one state: identity
    o1, l1 = oracle.merge(v[:, :1], s[:, :1])
    assert np.array_equal(o1, v[:, 0]) and np.array_equal(l1, s[:, 0])
    # two states with equal lse: plain average, lse + ln 2
    s2 = np.repeat(s[:, :1], 2, axis=1)
    o2, l2 = oracle.merge(v[:, :2], s2)
    np.testing.assert_allclose(o2, (v[:, 0] + v[:, 1]) / 2, atol=1e-15)
    np.testing.assert_allclose(l2, s[:, 0] + math.log(2), atol=1e-15)
    # lse differing by ln 3: weights 1:3
    s3 = s[:, :2].copy(); s3[:, 1] = s3[:, 0] + math.log(3)
    o3, _ = oracle.merge(v[:, :2], s3)
    np.testing.assert_allclose(o3, (v[:, 0] + 3 * v[:, 1]) / 4, atol=1e-14)
    # a -inf state (attention over no keys) carries no weight, even with NaN values
    vn = v[:, :2].copy(); vn[:, 1] = np.nan
    sn = s[:, :2].copy(); sn[:, 1] = -np.inf
    o4, l4 = oracle.merge(vn, sn)
    assert np.array_equal(o4, v[:, 0]) and np.array_equal(l4, s[:, 0])
    # all -inf: zero output, -inf lse
    o5, l5 = oracle.merge(v, np.full_like(s, -np.inf))
    assert np.all(o5 == 0) and np.all(l5 == -np.inf)


# ---------------------------------------------------------------------------
# append
# ---------------------------------------------------------------------------

def test_append_hand_derived_positions():
    # page_size 4.  Request 0 owns pages [5, 2] and holds 7 tokens after
    # appending 2 -> the new tokens are positions 5 and 6 = page 2, slots 1, 2.
    # Request 1 owns page [0] and holds 1 token after appending 1 -> page 0 slot 0.
    P, ps, hkv, D = 6, 4, 2, 8
    pool = np.arange(P * 2 * hkv * ps * D, dtype=np.uint16).reshape(P, 2, hkv, ps, D)
    indptr = np.array([0, 2, 3], np.int32)
    indices = np.array([5, 2, 0], np.int32)
    last = np.array([3, 1], np.int32)
    app = np.array([0, 2, 3], np.int32)
    k_new = (50000 + np.arange(3 * hkv * D)).astype(np.uint16).reshape(3, hkv, D)
    v_new = (60000 + np.arange(3 * hkv * D)).astype(np.uint16).reshape(3, hkv, D)
    out = oracle.append(pool, indptr, indices, last, k_new, v_new, app)
    expect = pool.copy()
    for row, (page, slot) in enumerate([(2, 1), (2, 2), (0, 0)]):
        expect[page, 0, :, slot, :] = k_new[row]
        expect[page, 1, :, slot, :] = v_new[row]
    assert np.array_equal(out, expect)


def test_append_extends_the_logical_sequence():
    # after appending, the sequence read through the table is the old
    # sequence followed by the new rows; every byte outside them is unchanged
    lens = np.array([31, 32, 1, 100, 16], np.int64)
    counts = np.array([1, 3, 1, 0, 16], np.int64)
    w = wl.make_workload("pin", lens, num_qo_heads=4, num_kv_heads=2, page_size=16,
                         dtype="bf16", seed=18, pool_factor=1.6, append_counts=counts)
    q, pool, k_new, v_new = wl.make_tensors(w)
    before = wl.bits(pool)
    after = oracle.append(before, w.page_indptr, w.page_indices, w.last_page_len,
                          wl.bits(k_new), wl.bits(v_new), w.append_indptr)
    kb, vb = wl.bits(k_new), wl.bits(v_new)
    touched = np.zeros(before.shape, bool)
    for b in range(w.batch):
        pages = w.pages_of(b)
        L, n = int(lens[b]), int(counts[b])
        for t in range(L):
            page, slot = pages[t // 16], t % 16
            if t < L - n:
                assert np.array_equal(after[page, :, :, slot], before[page, :, :, slot])
            else:
                row = w.append_indptr[b] + t - (L - n)
                assert np.array_equal(after[page, 0, :, slot], kb[row])
                assert np.array_equal(after[page, 1, :, slot], vb[row])
                touched[page, :, :, slot] = True
    assert np.array_equal(after[~touched], before[~touched])


def test_append_rejects_overflow():
    w = wl.make_workload("pin", [3], num_qo_heads=2, num_kv_heads=1, page_size=16,
                         dtype="f16", seed=19)
    pool = np.zeros(w.pool_shape, np.uint16)
    kn = np.zeros((4, 1, 128), np.uint16)
    with pytest.raises(oracle.OracleError):
        oracle.append(pool, w.page_indptr, w.page_indices, w.last_page_len, kn, kn,
                      np.array([0, 4], np.int32))


# ---------------------------------------------------------------------------
# the benchmark's byte counter against the numbers the pages print
# ---------------------------------------------------------------------------

def test_kv_byte_counter_matches_printed_values():
    with open(os.path.join(GOLDEN, "kv_cache_memory.json")) as f:
        g = json.load(f)
    for c in g["cases"]:
        nbytes = wl.kv_cache_bytes(c["num_layers"], c["num_kv_heads"], c["head_dim"],
                                   c["seq_len"], c["dtype_bytes"])
        assert f"{nbytes / 1024 ** 3:.1f}" == c["printed_gb"]
    # the workloads use the page's GQA ratios
    assert (wl.named(2).num_qo_heads, wl.named(2).num_kv_heads) == tuple(g["gqa_ratios"]["Llama-3-8B"])
    assert (wl.named(3).num_qo_heads, wl.named(3).num_kv_heads) == tuple(g["gqa_ratios"]["Llama-3-70B"])
    # 128K x 8 requests of one 70B-shaped layer = 4 GiB of K/V
    w3 = wl.named(3)
    assert wl.kv_cache_bytes(1, 8, 128, int(w3.kv_lens.sum())) == 4 * 1024 ** 3
