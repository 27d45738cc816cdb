"""GPU parity of the multi-token append attention (pkv_append_attention):
each request's chunk of query tokens attends causally over its paged cache,
optionally through a window with sink tokens; compared with the oracle."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_479_b200 as pkv
from paged_kv_cache_479_b200 import workloads as wl
from _util import assert_parity, odtype

pytestmark = pytest.mark.gpu


def i32(a):
    return torch.as_tensor(np.ascontiguousarray(a, np.int32), device="cuda")


def dense_block_table(w):
    nps = np.diff(w.page_indptr)
    bt = np.full((w.batch, int(max(1, nps.max()))), -1, np.int32)
    for b in range(w.batch):
        bt[b, :nps[b]] = w.pages_of(b)
    return bt, w.kv_lens.astype(np.int32)


class ChunkCase:
    def __init__(self, lens, q_lens, hq, hkv, ps, dtype, seed, pool_factor=1.3, device_gen=False):
        self.w = wl.make_workload("chunk", lens, num_qo_heads=hq, num_kv_heads=hkv, page_size=ps,
                                  dtype=dtype, seed=seed, pool_factor=pool_factor)
        dev = "cuda" if device_gen else "cpu"
        _, self.pool, _, _ = wl.make_tensors(self.w, dev)
        self.q_lens = np.asarray(q_lens, np.int64)
        self.qo = wl.chunk_indptr(self.q_lens)
        self.q = wl.make_chunk_queries(self.w, self.q_lens, dev)

    def run(self, splits=None, window_left=-1, sink=0, layout="HND", kind="csr"):
        w = self.w
        plan, auto = pkv.append_attention_plan(self.qo, w.kv_lens, w.num_qo_heads, w.num_kv_heads,
                                               window_left, sink)
        S = auto if splits is None else splits
        pool = self.pool.cuda()
        if layout == "NHD":
            pool = pool.permute(0, 1, 3, 2, 4).contiguous()
        if kind == "csr":
            keep = (i32(w.page_indptr), i32(w.page_indices), i32(w.last_page_len))
            table = pkv.csr_table(*keep)
        else:
            bt, ctx = dense_block_table(w)
            keep = (i32(bt), i32(ctx))
            table = pkv.block_table(*keep)
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        out, lse = pkv.append_attention(self.q.cuda(), i32(self.qo), pool, table, i32(plan), S,
                                        layout=layout, window_left=window_left, sink_tokens=sink,
                                        sm_scale=w.sm_scale, error_word=err)
        torch.cuda.synchronize()
        assert pkv.read_error_word(err) == 0
        return out, lse

    def run_short(self, max_q_len, layout="HND", kind="csr", parts=0, out=None):
        w = self.w
        pool = self.pool.cuda()
        if layout == "NHD":
            pool = pool.permute(0, 1, 3, 2, 4).contiguous()
        if kind == "csr":
            keep = (i32(w.page_indptr), i32(w.page_indices), i32(w.last_page_len))
            table = pkv.csr_table(*keep)
        else:
            bt, ctx = dense_block_table(w)
            keep = (i32(bt), i32(ctx))
            table = pkv.block_table(*keep)
        nb = pkv.append_attention_short_workspace_bytes(w.num_qo_heads, w.num_kv_heads, max_q_len,
                                                        parts)
        assert nb > 0
        ws = torch.zeros(nb // 4 + 64, dtype=torch.int32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        out, lse = pkv.append_attention_short(self.q.cuda(), i32(self.qo), pool, table, max_q_len,
                                              ws, layout=layout, num_partitions=parts, out=out,
                                              sm_scale=w.sm_scale, error_word=err)
        torch.cuda.synchronize()
        self.err = pkv.read_error_word(err)
        return out, lse

    def oracle(self, window_left=-1, sink=0):
        w = self.w
        return oracle.append_attention(wl.bits(self.q), wl.bits(self.pool), odtype(w),
                                       w.page_indptr, w.page_indices, w.last_page_len, self.qo,
                                       w.sm_scale, window_left, sink)


CASES = [
    # lens, q_lens, hq, hkv, ps, dtype, window_left, sink
    ([40, 100, 17, 64, 300], [5, 100, 1, 16, 0], 32, 8, 16, "bf16", -1, 0),
    ([300, 33, 700], [37, 33, 129], 16, 2, 32, "f16", -1, 0),
    ([129, 70, 260], [64, 1, 200], 8, 8, 16, "bf16", 31, 0),
    ([260, 90, 513], [120, 90, 3], 8, 1, 64, "f16", 50, 7),
    ([1000, 600], [300, 600], 32, 8, 256, "bf16", 100, 4),
    ([77], [77], 8, 2, 16, "bf16", 0, 0),
    ([300, 45, 129], [70, 45, 100], 12, 4, 16, "bf16", -1, 0),   # G = 3: Q staged per thread
]


@pytest.mark.parametrize("i", range(len(CASES)))
def test_append_attention_matches_oracle(i):
    lens, q_lens, hq, hkv, ps, dt, wlft, sink = CASES[i]
    c = ChunkCase(lens, q_lens, hq, hkv, ps, dt, 700 + i)
    out, lse = c.run(splits=1, window_left=wlft, sink=sink)
    ro, rl = c.oracle(wlft, sink)
    assert_parity(out, lse, ro, rl, what=f"chunk case {i}")


@pytest.mark.parametrize("S", [2, 5, 33])
def test_append_attention_key_splits(S):
    c = ChunkCase([2000, 90, 1500], [40, 90, 5], 32, 8, 16, "bf16", 720)
    out, lse = c.run(splits=S)
    ro, rl = c.oracle()
    assert_parity(out, lse, ro, rl, what=f"splits={S}")
    out, lse = c.run(splits=S, window_left=300, sink=16)
    ro, rl = c.oracle(300, 16)
    assert_parity(out, lse, ro, rl, what=f"splits={S} window")


@pytest.mark.parametrize("hq,hkv", [(12, 4), (8, 8)])
def test_append_attention_key_splits_other_groups(hq, hkv):
    """Key splits write fp32 states: by bulk-tensor stores for whole 128-row
    tiles when G divides 128 (G = 1 here), per thread otherwise (G = 3) and
    for the partial tiles of every block."""
    c = ChunkCase([1500, 700, 90], [100, 43, 90], hq, hkv, 16, "bf16", 725)
    out, lse = c.run(splits=3)
    ro, rl = c.oracle()
    assert_parity(out, lse, ro, rl, what=f"G={hq // hkv} splits=3")


def test_append_attention_planner_splits():
    c = ChunkCase([4000, 3000], [4, 4], 32, 8, 16, "f16", 721)
    _, S = pkv.append_attention_plan(c.qo, c.w.kv_lens, 32, 8)
    assert S > 1                                  # 2 row blocks x 8 heads: split the keys
    out, lse = c.run()
    ro, rl = c.oracle()
    assert_parity(out, lse, ro, rl, what=f"auto splits {S}")


@pytest.mark.parametrize("layout,kind", [("HND", "block"), ("NHD", "csr"), ("NHD", "block")])
def test_append_attention_layouts_and_tables_bitwise(layout, kind):
    c = ChunkCase([400, 17, 1000], [100, 17, 9], 32, 8, 16, "bf16", 722)
    ref = c.run(splits=2)
    out, lse = c.run(splits=2, layout=layout, kind=kind)
    assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1])


def test_single_token_chunks_match_the_decode():
    c = ChunkCase([40, 100, 17, 256, 3000], [1] * 5, 32, 8, 16, "bf16", 723)
    out, lse = c.run()
    w = c.w
    ws = torch.zeros(pkv.decode_workspace_bytes(w.batch, 32, 8) // 4 + 64, dtype=torch.int32,
                     device="cuda")
    do, dl = pkv.paged_decode_attention(c.q.cuda(), c.pool.cuda(), i32(w.page_indptr),
                                        i32(w.page_indices), i32(w.last_page_len), ws,
                                        sm_scale=w.sm_scale)
    ro, rl = c.oracle()
    assert_parity(out, lse, ro, rl, what="q_len 1")
    assert_parity(do, dl, ro, rl, what="decode")


def truncated_request(w, b, pos):
    """Table of request b's first pos + 1 tokens (for the decode oracle)."""
    pages = w.pages_of(b)[: pos // w.page_size + 1].astype(np.int32)
    return (np.array([0, len(pages)], np.int32), pages,
            np.array([pos % w.page_size + 1], np.int32))


def test_chunked_prefill_shape_sampled():
    # the chunked-prefill workload at full size, checked on sampled query rows:
    # query i of a chunk is the decode of a request truncated at its position
    w, q_lens = wl.named_chunk("prefill")
    _, pool, k_new, v_new = wl.make_tensors(w, "cuda")   # the chunk's K/V: appended rows
    qo = wl.chunk_indptr(q_lens)
    q = wl.make_chunk_queries(w, q_lens, "cuda")
    plan, S = pkv.append_attention_plan(qo, w.kv_lens, w.num_qo_heads, w.num_kv_heads)
    ip, ix, ll = i32(w.page_indptr), i32(w.page_indices), i32(w.last_page_len)
    table = pkv.csr_table(ip, ix, ll)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.paged_kv_append(pool, ip, ix, ll, k_new, v_new, i32(w.append_indptr), error_word=err)
    out, lse = pkv.append_attention(q, i32(qo), pool, table, i32(plan), S,
                                    sm_scale=w.sm_scale, error_word=err)
    torch.cuda.synchronize()
    assert pkv.read_error_word(err) == 0
    rng = np.random.default_rng(3)
    for b in range(w.batch):
        L, n = int(w.kv_lens[b]), int(q_lens[b])
        for i in sorted(set(rng.integers(0, n, size=3).tolist()) | {0, n - 1}):
            pos = L - n + i
            ip, ix, ll = truncated_request(w, b, pos)
            uniq, inv = np.unique(ix, return_inverse=True)
            sub = wl.bits(pool[torch.as_tensor(uniq, device="cuda", dtype=torch.long)])
            row = int(qo[b]) + i
            ro, rl = oracle.decode(wl.bits(q[row:row + 1]), sub, odtype(w), ip,
                                   inv.astype(np.int32), ll, w.sm_scale)
            assert_parity(out[row:row + 1], lse[row:row + 1], ro, rl, what=f"b{b} i{i}")


@pytest.mark.parametrize("big", [65280.0, 65536.0, 1e30, 2e-6])
def test_bf16_values_outside_fp16_range(big):
    # V entries at and beyond fp16's range (65280 is the largest bf16 value
    # fp16 holds) and below its normal range: the bf16 P.V must stay exact
    c = ChunkCase([300, 130, 70], [70, 130, 1], 16, 4, 16, "bf16", 725)
    w = c.w
    rng = np.random.default_rng(9)
    for b in range(w.batch):
        pages = w.pages_of(b)
        for tok in rng.choice(int(w.kv_lens[b]), size=4, replace=False):
            pg, slot = int(pages[tok // w.page_size]), int(tok % w.page_size)
            dims = torch.as_tensor(rng.choice(128, size=3, replace=False))
            signs = torch.as_tensor(rng.choice([-1.0, 1.0], size=3), dtype=torch.float32)
            c.pool[pg, 1, :, slot, dims] = (signs * big).to(c.pool.dtype)
    out, lse = c.run(splits=1)
    ro, rl = c.oracle()
    o = out.float().cpu().numpy().reshape(ro.shape)
    assert np.isfinite(o).all()
    # large outputs: the bf16 store rounds by up to 2^-8 relative (half an ulp
    # at the bottom of a binade)
    assert np.all(np.abs(o - ro) <= 1e-2 + 6e-3 * np.abs(ro))
    assert np.abs(lse.cpu().numpy().reshape(rl.shape) - rl).max() <= 1e-3


SHORT_CASES = [
    # lens, q_lens, hq, hkv, ps, dtype, max_q_len  (columns = max_q_len * hq / hkv)
    ([40, 100, 17, 64, 300, 1000], [4, 3, 1, 4, 2, 4], 32, 8, 16, "bf16", 4),   # 16 columns
    ([33, 700, 16, 129], [2, 2, 1, 2], 16, 2, 32, "f16", 2),                    # G = 8
    ([300, 18, 65], [16, 16, 5], 8, 8, 16, "bf16", 16),                         # G = 1
    ([90, 513, 2000], [1, 2, 2], 16, 4, 64, "bf16", 2),                         # 8 columns
    ([1, 5, 3000], [1, 0, 3], 8, 2, 16, "f16", 4),                              # q_len 0
    ([33, 20], [4, 4], 16, 4, 16, "bf16", 4),                                   # chunk across tiles
]


@pytest.mark.parametrize("parts", [0, 3, 148])
@pytest.mark.parametrize("i", range(len(SHORT_CASES)))
def test_short_chunks_match_oracle(i, parts):
    lens, q_lens, hq, hkv, ps, dt, mq = SHORT_CASES[i]
    c = ChunkCase(lens, q_lens, hq, hkv, ps, dt, 740 + i)
    out, lse = c.run_short(mq, parts=parts)
    assert c.err == 0
    ro, rl = c.oracle()
    assert_parity(out, lse, ro, rl, what=f"short case {i} parts {parts}")


@pytest.mark.parametrize("layout,kind", [("HND", "block"), ("NHD", "csr")])
def test_short_chunks_layouts_and_tables_bitwise(layout, kind):
    c = ChunkCase([400, 17, 1000], [4, 2, 3], 32, 8, 16, "bf16", 746)
    ref = c.run_short(4)
    out, lse = c.run_short(4, layout=layout, kind=kind)
    assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1])


@pytest.mark.parametrize("parts", [0, 5])
def test_short_chunks_fused_append_matches_separate(parts):
    # the chunk's K/V rows appended by the attention launch itself: the pool and
    # the outputs are bitwise those of the separate append and attention
    q_lens = np.array([4, 3, 1, 4, 2, 4], np.int64)
    w = wl.make_workload("short-fused", [40, 100, 17, 300, 33, 2000], num_qo_heads=32,
                         num_kv_heads=8, page_size=16, dtype="bf16", seed=760, pool_factor=1.3,
                         append_counts=q_lens)
    _, pool, k_new, v_new = wl.make_tensors(w, "cuda")
    qo = wl.chunk_indptr(q_lens)
    q = wl.make_chunk_queries(w, q_lens, "cuda")
    ip, ix, ll = i32(w.page_indptr), i32(w.page_indices), i32(w.last_page_len)
    table = pkv.csr_table(ip, ix, ll)
    app, qoi = i32(w.append_indptr), i32(qo)
    nb = pkv.append_attention_short_workspace_bytes(w.num_qo_heads, w.num_kv_heads, 4, parts)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    p_sep = pool.clone()
    pkv.paged_kv_append(p_sep, ip, ix, ll, k_new, v_new, app, error_word=err)
    ws = torch.zeros(nb // 4 + 64, dtype=torch.int32, device="cuda")
    o_sep, l_sep = pkv.append_attention_short(q, qoi, p_sep, table, 4, ws, num_partitions=parts,
                                              sm_scale=w.sm_scale, error_word=err)
    p_fus = pool.clone()
    ws = torch.zeros(nb // 4 + 64, dtype=torch.int32, device="cuda")
    o_fus, l_fus = pkv.append_attention_short(q, qoi, p_fus, table, 4, ws, num_partitions=parts,
                                              sm_scale=w.sm_scale, error_word=err,
                                              k_new=k_new, v_new=v_new, append_indptr=app)
    torch.cuda.synchronize()
    assert pkv.read_error_word(err) == 0
    assert torch.equal(p_fus.view(torch.int16), p_sep.view(torch.int16))
    assert torch.equal(o_fus, o_sep) and torch.equal(l_fus, l_sep)
    ro, rl = oracle.append_attention(wl.bits(q), wl.bits(p_fus), odtype(w), w.page_indptr,
                                     w.page_indices, w.last_page_len, qo, w.sm_scale)
    assert_parity(o_fus, l_fus, ro, rl, what="fused short")


def test_short_chunk_longer_than_bound_sets_error_bit():
    c = ChunkCase([100, 100, 60], [2, 5, 3], 32, 8, 16, "bf16", 747)
    sentinel = torch.full_like(c.q, 7.0, device="cuda")
    out, lse = c.run_short(4, out=sentinel)
    assert c.err & pkv.DEVERR_APPEND
    ro, rl = c.oracle()
    qo = c.qo
    keep = np.r_[qo[0]:qo[1], qo[2]:qo[3]]
    assert_parity(out[keep], lse[keep], ro[keep], rl[keep], what="in-bound requests")
    assert bool((out[qo[1]:qo[2]] == 7.0).all())    # the long chunk's rows are left alone


def test_speculative_verification_shape_sampled():
    # the speculative-verification workload at full size through the short
    # path, checked on sampled query rows against the truncated-request decode
    w, q_lens = wl.named_chunk("spec")
    _, pool, k_new, v_new = wl.make_tensors(w, "cuda")
    qo = wl.chunk_indptr(q_lens)
    q = wl.make_chunk_queries(w, q_lens, "cuda")
    ip, ix, ll = i32(w.page_indptr), i32(w.page_indices), i32(w.last_page_len)
    table = pkv.csr_table(ip, ix, ll)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.paged_kv_append(pool, ip, ix, ll, k_new, v_new, i32(w.append_indptr), error_word=err)
    mq = int(q_lens.max())
    nb = pkv.append_attention_short_workspace_bytes(w.num_qo_heads, w.num_kv_heads, mq)
    ws = torch.zeros(nb // 4 + 64, dtype=torch.int32, device="cuda")
    out, lse = pkv.append_attention_short(q, i32(qo), pool, table, mq, ws, sm_scale=w.sm_scale,
                                          error_word=err)
    torch.cuda.synchronize()
    assert pkv.read_error_word(err) == 0
    rng = np.random.default_rng(5)
    for b in sorted(rng.choice(w.batch, size=12, replace=False).tolist()):
        L, n = int(w.kv_lens[b]), int(q_lens[b])
        for i in range(n):
            pos = L - n + i
            ip_, ix_, ll_ = truncated_request(w, b, pos)
            uniq, inv = np.unique(ix_, return_inverse=True)
            sub = wl.bits(pool[torch.as_tensor(uniq, device="cuda", dtype=torch.long)])
            row = int(qo[b]) + i
            ro, rl = oracle.decode(wl.bits(q[row:row + 1]), sub, odtype(w), ip_,
                                   inv.astype(np.int32), ll_, w.sm_scale)
            assert_parity(out[row:row + 1], lse[row:row + 1], ro, rl, what=f"b{b} i{i}")


def test_bad_plan_entry_sets_error_bit():
    c = ChunkCase([100, 50], [10, 5], 8, 2, 16, "bf16", 724)
    w = c.w
    plan, _ = pkv.append_attention_plan(c.qo, w.kv_lens, 8, 2)
    bad = plan.copy()
    k = int(np.flatnonzero(plan[:, 0] == 0)[0])     # request 0's (only) block
    bad[k, 2] = 10 * 4 + 1                          # more rows than the chunk has
    keep = (i32(w.page_indptr), i32(w.page_indices), i32(w.last_page_len))
    table = pkv.csr_table(*keep)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.append_attention(c.q.cuda(), i32(c.qo), c.pool.cuda(), table, i32(bad), 1,
                         sm_scale=w.sm_scale, error_word=err)
    torch.cuda.synchronize()
    assert pkv.read_error_word(err) & pkv.DEVERR_APPEND
