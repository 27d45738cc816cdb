"""Host-only checks of the C ABI (no GPU): the library loads and exports every
symbol include/pkv.h declares, host helpers behave, arguments are rejected
before any launch, and the split-KV partition mirror covers the work
exactly once with balanced shares."""
import ctypes
import os
import re

import numpy as np
import pytest

import paged_kv_cache_479_b200 as pkv
from paged_kv_cache_479_b200 import workloads as wl

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "pkv.h")


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"^PKV_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, flags=re.M)


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 13
    L = ctypes.CDLL(pkv._binding.LIB_PATH)
    for n in names:
        assert hasattr(L, n), f"libpkv.so does not export {n}"
    assert {"pkv_append", "pkv_decode", "pkv_merge_states",
            "paged_kv_append", "paged_decode_attention", "merge_states"} <= set(names)


def test_wait_limit_setting_round_trips():
    """pkv_set_wait_limit_ns returns the previous limit; 0 selects the
    default of one second (host-only state, no launch)."""
    prev = pkv.set_wait_limit_ns(0)
    try:
        assert pkv.set_wait_limit_ns(5000) == 1_000_000_000
        assert pkv.set_wait_limit_ns(0) == 5000
        assert pkv.set_wait_limit_ns(0) == 1_000_000_000
    finally:
        pkv.set_wait_limit_ns(prev)


def test_unknown_table_flags_rejected():
    L = pkv.lib()
    p = ctypes.c_void_p(4096)
    pool = pkv.PoolDesc(4096, 64, 16, 2, 128, pkv.BF16, 0, 0)
    for flags, status in ((2, 1), (0x80000000, 1)):
        table = pkv.TableDesc(0, 4, 4096, 4096, 4096, None, None, 0, flags)
        assert L.pkv_decode_ex(p, 8, ctypes.byref(pool), ctypes.byref(table), 0.1, 8, p, 1 << 30,
                               ctypes.c_void_p(8192), None, None, None) == status
    assert b"table flags" in L.pkv_last_error()


def test_status_strings():
    L = pkv.lib()
    assert L.pkv_status_string(0) == b"PKV_OK"
    assert L.pkv_status_string(3) == b"PKV_ERR_WORKSPACE"
    assert L.pkv_status_string(99) == b"PKV_ERR_UNKNOWN"


def test_workspace_bytes():
    L = pkv.lib()
    assert L.pkv_decode_workspace_bytes(8, 64, 8, 128, 148) > 0
    assert L.pkv_decode_workspace_bytes(8, 64, 8, 64, 148) == 0     # head_dim 128 only
    assert L.pkv_decode_workspace_bytes(8, 128, 8, 128, 148) == 0    # group 16 > 8
    assert L.pkv_decode_workspace_bytes(8, 30, 8, 128, 148) == 0     # Hq % Hkv != 0
    a = L.pkv_decode_workspace_bytes(8, 64, 8, 128, 100)
    b = L.pkv_decode_workspace_bytes(8, 64, 8, 128, 200)
    assert b > a and a % 256 == 0


def _decode_args(**over):
    args = dict(q=ctypes.c_void_p(4096), hq=8, pool=ctypes.c_void_p(4096), P=64, ps=16, hkv=2,
                d=128, dtype=pkv.F16, ip=ctypes.c_void_p(4096), ix=ctypes.c_void_p(4096),
                ll=ctypes.c_void_p(4096), B=4, scale=0.1, N=8, ws=ctypes.c_void_p(4096),
                wsb=1 << 30, out=ctypes.c_void_p(8192), lse=None, err=None, stream=None)
    args.update(over)
    return list(args.values())


@pytest.mark.parametrize("over,status", [
    (dict(d=64), 2), (dict(hq=32, hkv=2), 2), (dict(ps=24), 2), (dict(hq=9), 1),
    (dict(dtype=7), 1), (dict(scale=float("inf")), 1), (dict(N=-1), 1),
    (dict(q=ctypes.c_void_p(4097)), 1), (dict(out=None), 1), (dict(ws=ctypes.c_void_p(4100)), 3),
    (dict(wsb=100), 3), (dict(out=ctypes.c_void_p(4096)), 1),
])
def test_decode_rejects_bad_arguments_before_launch(over, status):
    L = pkv.lib()
    assert L.pkv_decode(*_decode_args(**over)) == status
    assert L.pkv_last_error() != b""


def test_append_and_merge_reject_bad_arguments():
    L = pkv.lib()
    p = ctypes.c_void_p(4096)
    assert L.pkv_append(p, 8, 16, 2, 12, pkv.F16, p, p, p, 2, p, p, p, 3, None, None) == 2
    assert L.pkv_append(p, 8, 16, 2, 128, 5, p, p, p, 2, p, p, p, 3, None, None) == 1
    assert L.pkv_append(ctypes.c_void_p(4098), 8, 16, 2, 128, pkv.F16, p, p, p, 2, p, p, p, 3,
                        None, None) == 1
    # nothing to append is a no-op, not an error
    assert L.pkv_append(None, 8, 16, 2, 128, pkv.F16, None, None, None, 2, None, None, None, 0,
                        None, None) == 0
    assert L.pkv_merge_states(p, p, 4, 0, 2, 128, p, pkv.F32, None, None) == 1
    assert L.pkv_merge_states(p, p, 4, 2, 2, 128, p, 9, None, None) == 1
    assert L.pkv_merge_states(None, None, 0, 2, 2, 128, None, pkv.F32, None, None) == 0


def test_check_table():
    w = wl.named(2)
    pkv.check_table(w.page_indptr, w.page_indices, w.last_page_len, w.num_pages, 16)
    bad = w.last_page_len.copy(); bad[3] = 17
    with pytest.raises(pkv.PkvError, match="last_page_len"):
        pkv.check_table(w.page_indptr, w.page_indices, bad, w.num_pages, 16)
    bad = w.page_indices.copy(); bad[5] = w.num_pages
    with pytest.raises(pkv.PkvError, match="page_indices"):
        pkv.check_table(w.page_indptr, bad, w.last_page_len, w.num_pages, 16)
    bad = w.page_indptr.copy(); bad[4] = bad[3] - 1
    with pytest.raises(pkv.PkvError, match="decreases"):
        pkv.check_table(bad, w.page_indices, w.last_page_len, w.num_pages, 16)


def _tiles(w):
    return [int(-(-int(L) // 16)) for L in w.kv_lens]


def reference_plan(w, N, cost):
    """The split-KV partition written out from its definition: pair (b, g)
    occupies `cost` fixed units followed by its tiles in the flattened (b, g)
    order; partition c takes units [floor(cW/N), floor((c+1)W/N)); a pair's
    partial-state slot is 2c + 1 in its first covering partition, 2c in the
    others, and -1 when one partition holds all its tiles."""
    tiles = _tiles(w)
    units = [t + cost if t else 0 for t in tiles]
    W = w.num_kv_heads * sum(units)
    if W == 0:
        return []
    N = min(N, W)
    bounds = [c * W // N for c in range(N + 1)]
    rows = []
    start = 0
    for b in range(w.batch):
        for g in range(w.num_kv_heads):
            lo_real, hi_real = start + cost, start + units[b]
            parts = []
            for c in range(N):
                lo, hi = max(bounds[c], lo_real), min(bounds[c + 1], hi_real)
                if lo < hi:
                    parts.append((c, lo - lo_real, hi - lo_real))
            for j, (c, t0, t1) in enumerate(parts):
                slot = -1 if len(parts) == 1 else 2 * c + (1 if j == 0 else 0)
                rows.append((c, b, g, t0, t1, slot, len(parts)))
            start += units[b]
    return sorted(rows)


def library_cost():
    """The fixed per-pair cost the library charges, recovered from probe plans: the
    one value in 0..64 for which the definition reproduces every probe."""
    w = wl.make_workload("probe", [16, 1, 40, 300, 17, 5, 90, 33, 2, 160], num_qo_heads=4,
                         num_kv_heads=2, page_size=16, dtype="f16", seed=2)
    costs = set(range(0, 65))
    for N in (7, 13, 29, 61, 97):
        got = sorted(map(tuple, pkv.plan_segments(w.page_indptr, w.last_page_len, 16, 2,
                                                  N).tolist()))
        costs &= {k for k in costs if reference_plan(w, N, k) == got}
    assert len(costs) == 1, sorted(costs)
    return costs.pop()


def check_plan(w, N):
    seg = pkv.plan_segments(w.page_indptr, w.last_page_len, w.page_size, w.num_kv_heads, N)
    got = sorted(map(tuple, seg.tolist()))
    assert got == reference_plan(w, N, library_cost())
    tiles = _tiles(w)
    # every (request, kv head, tile) exactly once
    cover = set()
    for c, b, g, t0, t1, slot, ncov in got:
        for t in range(t0, t1):
            assert (b, g, t) not in cover
            cover.add((b, g, t))
    assert len(cover) == w.num_kv_heads * sum(tiles)
    # state slots unique and below 2N
    slots = [r[5] for r in got if r[5] >= 0]
    assert len(slots) == len(set(slots)) and all(0 <= x < 2 * N for x in slots)
    return seg


@pytest.mark.parametrize("cfg", [1, 2, 4, 5])
@pytest.mark.parametrize("N", [1, 2, 7, 148, 1000])
def test_partition_covers_work_exactly_once(cfg, N):
    check_plan(wl.named(cfg), N)


def test_partition_with_empty_and_tiny_requests():
    w = wl.make_workload("t", [0, 1, 0, 0, 17, 300, 0, 16, 2], num_qo_heads=4, num_kv_heads=2,
                         page_size=16, dtype="f16", seed=1)
    for N in (1, 3, 5, 8, 40, 148, 500):
        check_plan(w, N)
    w = wl.make_workload("t", [0, 0], num_qo_heads=4, num_kv_heads=2, page_size=16,
                         dtype="f16", seed=1)
    assert len(pkv.plan_segments(w.page_indptr, w.last_page_len, 16, 2, 4)) == 0


def test_partition_long_single_sequence_fills_all_partitions():
    w = wl.named(4)
    seg = check_plan(w, 148)
    assert set(seg[:, 0].tolist()) == set(range(148))
    assert (seg[:, 6] > 1).all()   # every pair is split, so every segment merges
    per = np.bincount(seg[:, 0], weights=seg[:, 4] - seg[:, 3])
    assert per.max() - per.min() <= library_cost() + 1


def test_partition_balances_time_weighted_work():
    # each partition's tiles plus the fixed cost of the pairs it starts is the
    # same up to one pair's fixed cost and rounding
    w = wl.named(5)
    N = 148
    seg = check_plan(w, N)
    cost = library_cost()
    work = np.zeros(N)
    for c, b, g, t0, t1, slot, ncov in seg:
        work[c] += (t1 - t0) + (cost if t0 == 0 else 0)
    assert work.max() - work.min() <= 2 * cost + 2


def test_descriptor_calls_reject_bad_arguments():
    L = pkv.lib()
    p = ctypes.c_void_p(4096)
    pool = pkv.PoolDesc(4096, 64, 16, 2, 128, pkv.BF16, 0, 0)
    csr = pkv.TableDesc(pkv.TABLE_CSR if hasattr(pkv, "TABLE_CSR") else 0, 4, 4096, 4096, 4096,
                        None, None, 0, 0)
    args = lambda pool, table: [p, 8, ctypes.byref(pool) if pool is not None else None,
                                ctypes.byref(table) if table is not None else None, 0.1, 8, p,
                                1 << 30, ctypes.c_void_p(8192), None, None, None]
    assert L.pkv_decode_ex(*args(None, csr)) == 1
    assert L.pkv_decode_ex(*args(pool, None)) == 1
    bad_layout = pkv.PoolDesc(4096, 64, 16, 2, 128, pkv.BF16, 7, 0)
    assert L.pkv_decode_ex(*args(bad_layout, csr)) == 1
    bad_kind = pkv.TableDesc(5, 4, 4096, 4096, 4096, None, None, 0, 0)
    assert L.pkv_decode_ex(*args(pool, bad_kind)) == 1
    empty_block = pkv.TableDesc(1, 4, None, None, None, 4096, 4096, 0, 0)
    assert L.pkv_decode_ex(*args(pool, empty_block)) == 1   # max_blocks_per_seq 0
    hd64 = pkv.PoolDesc(4096, 64, 16, 2, 64, pkv.BF16, 1, 0)
    assert L.pkv_decode_ex(*args(hd64, csr)) == 2
    assert L.pkv_append_ex(None, ctypes.byref(csr), p, p, p, 3, None, None) == 1
    assert L.pkv_append_ex(ctypes.byref(bad_layout), ctypes.byref(csr), p, p, p, 3, None, None) == 1


def test_fp8_calls_reject_bad_arguments():
    L = pkv.lib()
    p = ctypes.c_void_p(4096)
    fp8 = pkv.PoolDesc(4096, 64, 16, 2, 128, pkv.FP8_E4M3, 0, 0)
    bf16 = pkv.PoolDesc(4096, 64, 16, 2, 128, pkv.BF16, 0, 0)
    csr = pkv.TableDesc(0, 4, 4096, 4096, 4096, None, None, 0, 0)

    def dec(pool, q_dtype=pkv.BF16, ks=0.5, vs=0.5):
        return L.pkv_decode_fp8(p, q_dtype, 8, ctypes.byref(pool), ks, vs, ctypes.byref(csr), 0.1,
                                8, p, 1 << 30, ctypes.c_void_p(8192), None, None, None)

    def app(pool, new_dtype=pkv.BF16, ks=0.5, vs=0.5):
        return L.pkv_append_fp8(ctypes.byref(pool), ks, vs, ctypes.byref(csr), p, p, new_dtype, p,
                                3, None, None)

    for ks, vs in ((0.0, 1.0), (1.0, -1.0), (float("inf"), 1.0), (1.0, float("nan"))):
        assert dec(fp8, ks=ks, vs=vs) == 1
        assert app(fp8, ks=ks, vs=vs) == 1
    assert dec(bf16) == 1                       # the fp8 calls need an E4M3 pool
    assert app(bf16) == 1
    assert dec(fp8, q_dtype=pkv.F32) == 1       # q is fp16 or bf16
    assert dec(fp8, q_dtype=pkv.FP8_E4M3) == 1
    assert app(fp8, new_dtype=pkv.FP8_E4M3) == 1
    # the descriptor calls without scales refuse an E4M3 pool
    assert L.pkv_decode_ex(p, 8, ctypes.byref(fp8), ctypes.byref(csr), 0.1, 8, p, 1 << 30,
                           ctypes.c_void_p(8192), None, None, None) == 1
    assert L.pkv_append_ex(ctypes.byref(fp8), ctypes.byref(csr), p, p, p, 3, None, None) == 1
    assert b"pkv_append_fp8" in L.pkv_last_error()


def test_append_attention_plan_covers_rows_once():
    rng = np.random.default_rng(9)
    q_lens = rng.integers(0, 400, size=37)
    qo = wl.chunk_indptr(q_lens)
    kv = (q_lens + rng.integers(0, 3000, size=37)).astype(np.int32)
    for hq, hkv in ((32, 8), (8, 8), (64, 8)):
        G = hq // hkv
        plan, S = pkv.append_attention_plan(qo, kv, hq, hkv, num_sms=148)
        seen = [np.zeros(int(n) * G, int) for n in q_lens]
        for b, r0, n, pad in plan:
            assert 1 <= n <= 256 and pad == 0
            seen[b][r0:r0 + n] += 1
        assert all((s == 1).all() for s in seen)
        # longest first: key tiles of 64 up to the block's last row (no window),
        # non-increasing, ties in request and row order
        base = kv.astype(np.int64) - q_lens
        tiles = [(int(base[b]) + (int(r0) + int(n) - 1) // G + 1 + 63) // 64 for b, r0, n, _ in plan]
        assert all(x >= y for x, y in zip(tiles, tiles[1:]))
        for i in range(len(plan) - 1):
            if tiles[i] == tiles[i + 1]:
                assert tuple(plan[i, :2]) < tuple(plan[i + 1, :2])
        assert 1 <= S <= 32


def test_append_attention_plan_splits_and_rejects():
    L = pkv.lib()
    qo = np.array([0, 4, 8], np.int32)
    kv = np.array([4000, 3000], np.int32)
    _, S = pkv.append_attention_plan(qo, kv, 32, 8, num_sms=148)
    assert S > 1                                   # 2 blocks x 8 heads on 148 SMs
    _, S1 = pkv.append_attention_plan(qo, None, 32, 8, num_sms=148)
    assert S1 == 1                                 # no lengths: no split suggested
    big = wl.chunk_indptr([2048] * 8)
    _, S2 = pkv.append_attention_plan(big, np.full(8, 8192, np.int32), 32, 8, num_sms=148)
    assert S2 == 1                                 # 8 x 64 blocks x 8 heads fill the GPU
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    bad_start = np.array([1, 4, 8], np.int32)
    assert L.pkv_append_attention_plan(p(bad_start), None, 2, 32, 8, -1, 0, 148, None, 0, None) == -1
    dec = np.array([0, 4, 2], np.int32)
    assert L.pkv_append_attention_plan(p(dec), None, 2, 32, 8, -1, 0, 148, None, 0, None) == -1
    short = np.array([3, 3000], np.int32)           # 4 queries but 3 tokens
    assert L.pkv_append_attention_plan(p(qo), p(short), 2, 32, 8, -1, 0, 148, None, 0, None) == -1
    assert L.pkv_append_attention_plan(p(qo), None, 2, 30, 8, -1, 0, 148, None, 0, None) == -1
    assert pkv.append_attention_workspace_bytes(100, 32, 1) == 0
    assert pkv.append_attention_workspace_bytes(100, 32, 3) >= 100 * 3 * 32 * 129 * 4


def test_append_attention_rejects_bad_arguments():
    L = pkv.lib()
    P = ctypes.c_void_p(4096)
    pool = pkv.PoolDesc(4096, 64, 16, 2, 128, pkv.BF16, 0, 0)
    csr = pkv.TableDesc(0, 4, 4096, 4096, 4096, None, None, 0, 0)

    def call(pool=pool, splits=1, ws_bytes=0, plan=P):
        return L.pkv_append_attention(P, P, 16, 8, ctypes.byref(pool), ctypes.byref(csr), plan, 3,
                                      splits, -1, 0, 0.1, None, ws_bytes, ctypes.c_void_p(8192),
                                      None, None, None)

    assert call(splits=0) == 1
    assert call(pkv.PoolDesc(4096, 64, 16, 2, 128, pkv.FP8_E4M3, 0, 0)) == 1
    assert call(pkv.PoolDesc(4096, 64, 16, 2, 64, pkv.BF16, 0, 0)) == 2
    assert call(pkv.PoolDesc(4096, 64, 8, 2, 128, pkv.BF16, 0, 0)) == 2
    assert call(splits=4) == 3                       # no workspace for the split states
    assert call(plan=ctypes.c_void_p(4100)) == 1     # misaligned plan


def test_append_attention_short_rejects_bad_arguments():
    L = pkv.lib()
    P = ctypes.c_void_p(4096)
    WS = ctypes.c_void_p(1 << 20)
    pool = pkv.PoolDesc(4096, 64, 16, 2, 128, pkv.BF16, 0, 0)      # 2 kv heads: G = 4 with hq 8
    csr = pkv.TableDesc(0, 4, 4096, 4096, 4096, None, None, 0, 0)
    need = pkv.append_attention_short_workspace_bytes(8, 2, 4, 4)

    def call(pool=pool, max_q_len=4, hq=8, ws_bytes=need, qo=P):
        return L.pkv_append_attention_short(P, qo, 16, max_q_len, hq, ctypes.byref(pool),
                                            ctypes.byref(csr), None, None, None, 0, 0.1, 4, WS,
                                            ws_bytes, ctypes.c_void_p(8192), None, None, None)

    assert call(max_q_len=5) == 2                     # 5 tokens x 4 heads > 16 columns
    assert call(max_q_len=0) == 2
    assert call(hq=7) == 1                            # not a multiple of the kv heads
    assert call(pkv.PoolDesc(4096, 64, 16, 2, 128, pkv.FP8_E4M3, 0, 0)) == 1
    assert call(pkv.PoolDesc(4096, 64, 16, 2, 64, pkv.BF16, 0, 0)) == 2
    assert call(ws_bytes=need - 1) == 3
    assert call(qo=None) == 1
    # the optional fused append: negative count, rows aliasing the pool
    assert L.pkv_append_attention_short(P, P, 16, 4, 8, ctypes.byref(pool), ctypes.byref(csr),
                                        None, None, None, -1, 0.1, 4, WS, need,
                                        ctypes.c_void_p(8192), None, None, None) == 1
    assert L.pkv_append_attention_short(P, P, 16, 4, 8, ctypes.byref(pool), ctypes.byref(csr),
                                        ctypes.c_void_p(4096), ctypes.c_void_p(12288), P, 4, 0.1,
                                        4, WS, need, ctypes.c_void_p(8192), None, None, None) == 1
    # 8 or 16 state columns per slot
    assert pkv.append_attention_short_workspace_bytes(32, 8, 5, 4) == 0
    assert pkv.append_attention_short_workspace_bytes(32, 8, 0, 4) == 0
    w2 = pkv.append_attention_short_workspace_bytes(32, 8, 2, 148)
    w4 = pkv.append_attention_short_workspace_bytes(32, 8, 4, 148)
    assert w2 >= 2 * 148 * 8 * 129 * 4 and w4 >= 2 * 148 * 16 * 129 * 4 and w4 > w2


def test_decode_append_rejects_bad_arguments():
    L = pkv.lib()
    P = ctypes.c_void_p(4096)
    K, V = ctypes.c_void_p(12288), ctypes.c_void_p(16384)
    WS = ctypes.c_void_p(1 << 20)
    pool = pkv.PoolDesc(4096, 64, 16, 2, 128, pkv.BF16, 0, 0)
    csr = pkv.TableDesc(0, 4, 4096, 4096, 4096, None, None, 0, 0)

    def call(pool=pool, k=K, v=V, nnz=4):
        return L.pkv_decode_append(P, 8, ctypes.byref(pool), ctypes.byref(csr), k, v, P, nnz, 0.1,
                                   4, WS, 1 << 20, ctypes.c_void_p(8192), None, None, None)

    assert call(pkv.PoolDesc(4096, 64, 16, 2, 128, pkv.FP8_E4M3, 0, 0)) == 1  # 8-bit pool
    assert call(k=None) == 1
    assert call(v=ctypes.c_void_p(16388)) == 1        # misaligned
    assert call(nnz=-1) == 1
    assert call(k=ctypes.c_void_p(4096)) == 1         # k_new aliases the pool


@pytest.mark.parametrize("N", [1, 3, 7, 148, 600])
def test_fused_append_writes_every_new_row_once(N):
    # the fused append writes a new row from the segment that owns its tile, in
    # the 32-tile batch that holds it; over the host mirror of the partition
    # every (request, kv head, new position) comes out exactly once
    lens = [1, 15, 16, 17, 33, 300, 700, 0, 4097, 2]
    counts = [1, 15, 1, 17, 2, 40, 600, 0, 513, 2]
    w = wl.make_workload("fa", lens, num_qo_heads=8, num_kv_heads=4, page_size=16,
                         dtype="bf16", seed=5, append_counts=counts)
    seg = pkv.plan_segments(w.page_indptr, w.last_page_len, 16, 4, N)
    written = []
    for c, b, g, t0, t1, slot, ncov in seg.tolist():
        L, n_new = int(w.kv_lens[b]), int(counts[b])
        n = t1 - t0
        for k0 in range(0, max(n, 0), 32):
            lo = max((t0 + k0) * 16, L - n_new)
            hi = min((t0 + min(k0 + 32, n)) * 16, L)
            written += [(b, g, p) for p in range(lo, hi)]
    expect = [(b, g, p) for b in range(w.batch) for g in range(4)
              for p in range(int(w.kv_lens[b]) - counts[b], int(w.kv_lens[b]))]
    assert sorted(written) == sorted(expect)


def _shared_pairs_by_first_and_last_unit(lens, ps, hkv, N, seg_cost=16):
    """For every partition, the (request, kv head) pairs holding its first and
    its last flat unit, kept when the partition holds a tile of the pair and
    the pair's tiles span several partitions -- written from the partition's
    definition (fixed cost first, then the pair's 16-token tiles)."""
    units = [(-(-L // 16) + seg_cost) if L > 0 else 0 for L in lens]
    W = hkv * sum(units)
    Np = min(N, W)
    part_of = lambda f: ((f + 1) * Np - 1) // W
    starts = np.concatenate([[0], np.cumsum(units)])

    def pair_at(f):
        b = int(np.searchsorted(starts, f // hkv, side="right")) - 1
        while units[b] == 0 or not (hkv * starts[b] <= f < hkv * (starts[b] + units[b])):
            b += 1 if f >= hkv * (starts[b] + units[b]) else -1
        kvh = (f - hkv * starts[b]) // units[b]
        ps0 = hkv * starts[b] + kvh * units[b]
        return b, kvh, part_of(ps0 + seg_cost), part_of(ps0 + units[b] - 1)

    out = {}
    for c in range(Np):
        f0, f1 = W * c // Np, W * (c + 1) // Np
        got = set()
        for f in (f0, f1 - 1):
            b, kvh, c_first, c_last = pair_at(f)
            if c_last > c_first and c_first <= c <= c_last:
                got.add((b, kvh))
        out[c] = got
    return out


@pytest.mark.parametrize("lens,ps,hkv,N", [
    ([3000, 500, 17, 8000, 1, 2049], 16, 8, 148),
    ([3000, 500, 17, 8000, 1, 2049], 16, 8, 7),
    ([1, 2, 3, 0, 4, 5], 16, 2, 300),
    ([200000], 256, 8, 148),
    ([131072] * 8, 16, 8, 148),
    ([100, 4096, 0, 33, 77, 5000, 1, 16], 32, 4, 37),
])
def test_shared_pairs_are_those_of_the_first_and_last_unit(lens, ps, hkv, N):
    """The decode kernel counts each partition in on the pairs holding its
    first and last unit (also when it gives up part-way); that must be exactly
    the set of split pairs whose partial states the partition writes, as the
    host mirror of the partition lists them."""
    w = wl.make_workload("pairs", lens, num_qo_heads=hkv, num_kv_heads=hkv, page_size=ps,
                         dtype="bf16", seed=3)
    seg = pkv.plan_segments(w.page_indptr, w.last_page_len, ps, hkv, N)
    expect = _shared_pairs_by_first_and_last_unit(list(w.kv_lens), ps, hkv, N)
    for c, pairs in expect.items():
        rows = seg[(seg[:, 0] == c) & (seg[:, 6] > 1)]
        assert {(int(r[1]), int(r[2])) for r in rows} == pairs, f"partition {c}"
        assert len(pairs) <= 2
