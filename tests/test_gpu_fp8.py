"""GPU parity of the 8-bit (FP8 E4M3 and E5M2) KV cache: pkv_decode_fp8
against the oracle's decode over the same codes and scales, and
pkv_append_fp8 bit for bit against the oracle's quantising scatter."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_479_b200 as pkv
from paged_kv_cache_479_b200 import workloads as wl
from _util import assert_parity, odtype

pytestmark = pytest.mark.gpu

K_SCALE = 1.0 / 16          # typical codes (magnitude ~16) -> keys of magnitude ~1
V_SCALE = 0.0071            # not a power of two; the largest code (448) -> 3.2


def i32(a):
    return torch.as_tensor(np.ascontiguousarray(a, np.int32), device="cuda")


def dense_block_table(w):
    nps = np.diff(w.page_indptr)
    bt = np.full((w.batch, int(max(1, nps.max()))), -1, np.int32)
    for b in range(w.batch):
        bt[b, :nps[b]] = w.pages_of(b)
    return bt, w.kv_lens.astype(np.int32)


def workspace(w, n=0):
    nb = pkv.decode_workspace_bytes(w.batch, w.num_qo_heads, w.num_kv_heads, 128, n)
    return torch.zeros(nb // 4 + 64, dtype=torch.int32, device="cuda")


def table_of(w, kind):
    if kind == "csr":
        keep = (i32(w.page_indptr), i32(w.page_indices if len(w.page_indices) else [0]),
                i32(w.last_page_len))
        return pkv.csr_table(*keep), keep
    bt, ctx = dense_block_table(w)
    keep = (i32(bt), i32(ctx))
    return pkv.block_table(*keep), keep


def to_layout(pool, layout):
    return pool.permute(0, 1, 3, 2, 4).contiguous() if layout == "NHD" else pool


def fp8_decode(w, q, pool, layout="HND", kind="csr", ks=K_SCALE, vs=V_SCALE, n=0, fmt="e4m3"):
    table, keep = table_of(w, kind)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = pkv.paged_decode_attention_fp8(q, to_layout(pool, layout), table, workspace(w, n),
                                              ks, vs, layout=layout, sm_scale=w.sm_scale,
                                              num_partitions=n, error_word=err, fp8_format=fmt)
    torch.cuda.synchronize()
    assert pkv.read_error_word(err) == 0
    return out, lse


def oracle_fp8(w, q, pool, ks=K_SCALE, vs=V_SCALE, fmt="e4m3"):
    return oracle.decode_fp8(wl.bits(q), odtype(w), pool.cpu().numpy(), ks, vs, w.page_indptr,
                             w.page_indices, w.last_page_len, w.sm_scale, fmt)


CASES = [
    # lens, hq, hkv, ps, dtype
    ([1000, 17, 0, 300, 4097], 32, 8, 16, "bf16"),
    ([513, 2000, 1, 64], 16, 2, 64, "f16"),
    ([5, 16, 33, 100, 15], 8, 8, 16, "bf16"),     # group 1
    ([2500, 31], 8, 1, 32, "f16"),                # group 8
    ([700, 129], 32, 8, 256, "bf16"),
]


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("i", range(len(CASES)))
def test_fp8_decode_matches_oracle(i, fmt):
    lens, hq, hkv, ps, dt = CASES[i]
    w = wl.make_workload("fp8", lens, num_qo_heads=hq, num_kv_heads=hkv, page_size=ps, dtype=dt,
                         seed=900 + i, pool_factor=1.3)
    q, pool, _, _ = wl.make_fp8_tensors(w, "cpu", fmt)
    out, lse = fp8_decode(w, q.cuda(), pool.cuda(), fmt=fmt)
    ro, rl = oracle_fp8(w, q, pool, fmt=fmt)
    assert_parity(out, lse, ro, rl, what=f"{fmt} case {i}")


@pytest.mark.parametrize("layout,kind", [("HND", "block"), ("NHD", "csr"), ("NHD", "block")])
def test_fp8_layouts_and_tables_are_bitwise_equal(layout, kind):
    w = wl.make_workload("fp8l", [1000, 17, 0, 300, 4097], num_qo_heads=32, num_kv_heads=8,
                         page_size=16, dtype="bf16", seed=910, pool_factor=1.3)
    q, pool, _, _ = wl.make_fp8_tensors(w, "cuda")
    ref = fp8_decode(w, q, pool)
    out, lse = fp8_decode(w, q, pool, layout, kind)
    assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1])


@pytest.mark.parametrize("n", [1, 7, 148, 300])
def test_fp8_partition_counts(n):
    w = wl.make_workload("fp8n", [3000, 1, 255, 4096], num_qo_heads=32, num_kv_heads=8,
                         page_size=16, dtype="bf16", seed=911, pool_factor=1.2)
    q, pool, _, _ = wl.make_fp8_tensors(w, "cpu")
    out, lse = fp8_decode(w, q.cuda(), pool.cuda(), n=n)
    ro, rl = oracle_fp8(w, q, pool)
    assert_parity(out, lse, ro, rl, what=f"fp8 N={n}")


@pytest.mark.parametrize("n", [1, 3, 64])
def test_fp8_many_short_segments(n):
    fmt = "e5m2" if n == 3 else "e4m3"
    # hundreds of one-tile (request, kv head) segments per partition: the
    # producer runs many segments ahead of the consumers through the 32-slot
    # ring, so every staged query block and segment record is reused often
    rng = np.random.default_rng(6)
    lens = rng.integers(0, 40, size=700)
    w = wl.make_workload("fp8tiny", lens, num_qo_heads=16, num_kv_heads=4, page_size=16,
                         dtype="bf16", seed=914, pool_factor=1.2)
    q, pool, _, _ = wl.make_fp8_tensors(w, "cpu", fmt)
    out, lse = fp8_decode(w, q.cuda(), pool.cuda(), n=n, fmt=fmt)
    ro, rl = oracle_fp8(w, q, pool, fmt=fmt)
    assert_parity(out, lse, ro, rl, what=f"{fmt} tiny N={n}")


def test_fp8_query_scaling_extremes():
    # bf16 queries far outside fp16's range (both ways) and an all-zero row
    w = wl.make_workload("fp8q", [200, 77], num_qo_heads=16, num_kv_heads=2, page_size=16,
                         dtype="bf16", seed=912)
    q, pool, _, _ = wl.make_fp8_tensors(w, "cpu")
    q = q.float()
    q[0, :4] *= 2.0 ** 20 / 64      # scores stay moderate: k_scale below shrinks keys
    q[0, 4:8] *= 2.0 ** -30
    q[1, 0] = 0
    q = q.to(torch.bfloat16)
    ks = 2.0 ** -20
    out, lse = fp8_decode(w, q.cuda(), pool.cuda(), ks=ks)
    ro, rl = oracle_fp8(w, q, pool, ks=ks)
    assert_parity(out, lse, ro, rl, what="fp8 q scaling")


def test_fp8_scales_are_exact_factors_on_the_gpu():
    # powers of two: doubling v_scale doubles out exactly; k_scale * c == sm_scale * c
    w = wl.make_workload("fp8s", [300, 40], num_qo_heads=16, num_kv_heads=4, page_size=16,
                         dtype="f16", seed=913)
    q, pool, _, _ = wl.make_fp8_tensors(w, "cuda")
    o1, l1 = fp8_decode(w, q, pool, ks=0.25, vs=0.5)
    o2, l2 = fp8_decode(w, q, pool, ks=0.25, vs=1.0)
    torch.testing.assert_close(o2.float(), 2 * o1.float(), rtol=0, atol=0)
    assert torch.equal(l1, l2)


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("layout,kind", [("HND", "csr"), ("HND", "block"), ("NHD", "csr"),
                                         ("NHD", "block")])
@pytest.mark.parametrize("dt", ["bf16", "f16"])
def test_fp8_append_bit_exact(layout, kind, dt, fmt):
    w = wl.make_workload("fp8a", [1, 15, 16, 17, 33, 300], num_qo_heads=8, num_kv_heads=4,
                         page_size=16, dtype=dt, seed=920, pool_factor=1.5,
                         append_counts=[1, 15, 1, 17, 2, 40])
    _, pool, k_new, v_new = wl.make_fp8_tensors(w, "cpu", fmt)
    # spread the inputs so the scales reach saturation (K) and subnormals (V)
    k_new = (k_new.float() * 8).to(k_new.dtype)
    v_new = (v_new.float() * 0.002).to(v_new.dtype)
    ks, vs = (0.015, 0.5) if fmt == "e4m3" else (2e-4, 64.0)
    sat = 0x7E if fmt == "e4m3" else 0x7B
    expect = oracle.append_fp8(pool.numpy(), ks, vs, w.page_indptr, w.page_indices,
                               w.last_page_len, wl.bits(k_new), wl.bits(v_new), odtype(w),
                               w.append_indptr, fmt)
    assert (expect == sat).any() and (expect == 0x80 | sat).any()   # saturated codes occur
    p = to_layout(pool.cuda(), layout)
    table, keep = table_of(w, kind)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.paged_kv_append_fp8(p, table, k_new.cuda(), v_new.cuda(), i32(w.append_indptr), ks, vs,
                            layout=layout, error_word=err, fp8_format=fmt)
    torch.cuda.synchronize()
    assert pkv.read_error_word(err) == 0
    got = (p.permute(0, 1, 3, 2, 4) if layout == "NHD" else p).contiguous().cpu().numpy()
    assert np.array_equal(got, expect)


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_fp8_append_then_decode_step(fmt):
    w = wl.named(2)
    q, pool, k_new, v_new = wl.make_fp8_tensors(w, "cpu", fmt)
    ks, vs = K_SCALE, V_SCALE
    after = oracle.append_fp8(pool.numpy(), ks, vs, w.page_indptr, w.page_indices,
                              w.last_page_len, wl.bits(k_new), wl.bits(v_new), odtype(w),
                              w.append_indptr, fmt)
    p = pool.cuda()
    table, keep = table_of(w, "csr")
    pkv.paged_kv_append_fp8(p, table, k_new.cuda(), v_new.cuda(), i32(w.append_indptr), ks, vs,
                            fp8_format=fmt)
    out, lse = fp8_decode(w, q.cuda(), p, fmt=fmt)
    assert np.array_equal(p.cpu().numpy(), after)
    ro, rl = oracle.decode_fp8(wl.bits(q), odtype(w), after, ks, vs, w.page_indptr,
                               w.page_indices, w.last_page_len, w.sm_scale, fmt)
    assert_parity(out, lse, ro, rl, what="fp8 append+decode")


def test_fp8_long_context_sampled():
    # the 8 x 128K-token long-context shape on an 8-bit pool; two requests checked
    w = wl.named(3)
    q, pool, _, _ = wl.make_fp8_tensors(w, "cuda")
    out, lse = fp8_decode(w, q, pool)
    for b in (0, 5):
        sub_pool, ip, ix, ll = wl.subset(
            w, [b], lambda ids: pool[torch.as_tensor(ids, device="cuda", dtype=torch.long)].cpu().numpy())
        ro, rl = oracle.decode_fp8(wl.bits(q[b:b + 1]), odtype(w), sub_pool, K_SCALE, V_SCALE, ip,
                                   ix, ll, w.sm_scale)
        assert_parity(out[b:b + 1], lse[b:b + 1], ro, rl, what=f"fp8 128K request {b}")
