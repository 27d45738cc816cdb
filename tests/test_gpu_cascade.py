"""GPU parity of the shared-prefix cascade (pkv_cascade_decode) against the oracle.

The cascade computes the same attention as a plain decode over the prefix
followed by each request's own tokens, so the oracle is oracle.decode on that
concatenation.  When the prefix ends inside a page (not representable as one
CSR table), the test repacks every request's tokens into fresh pages itself
before calling the oracle."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_479_b200 as pkv
from paged_kv_cache_479_b200 import workloads as wl
from _util import assert_parity, errors, oracle_decode_from_device

pytestmark = pytest.mark.gpu


def cascade_inputs(w, prefix, prefix_len, indptr, indices, last, dev="cuda"):
    t = lambda a: torch.as_tensor(np.ascontiguousarray(a, np.int32), device=dev)
    return t(prefix if len(prefix) else np.zeros(1, np.int32)), t(indptr), \
        t(indices if len(indices) else np.zeros(1, np.int32)), t(last)


def run_cascade(w, q, pool, prefix, prefix_len, indptr, indices, last, num_partitions=0):
    pp, ip, ix, ll = cascade_inputs(w, prefix, prefix_len, indptr, indices, last)
    nb = pkv.cascade_workspace_bytes(w.batch, w.num_qo_heads, w.num_kv_heads, prefix_len,
                                     num_partitions=num_partitions)
    ws = torch.zeros(nb // 4 + 64, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = pkv.cascade_decode(q, pool, pp, prefix_len, ip, ix, ll, ws, sm_scale=w.sm_scale,
                                  num_partitions=num_partitions, error_word=err)
    torch.cuda.synchronize()
    assert pkv.read_error_word(err) == 0
    return out, lse


def repacked_oracle(w, q_bits, pool_bits, prefix, prefix_len, indptr, indices, last):
    """Oracle on every request's tokens (prefix, then its own) copied into fresh pages."""
    ps, hkv, D = w.page_size, w.num_kv_heads, w.head_dim
    seqs = []
    pre = [(prefix[t // ps], t % ps) for t in range(prefix_len)]
    for b in range(w.batch):
        own_pages = indices[indptr[b]:indptr[b + 1]]
        n_own = (len(own_pages) - 1) * ps + last[b] if len(own_pages) else 0
        own = [(own_pages[t // ps], t % ps) for t in range(n_own)]
        seqs.append(pre + own)
    lens = [len(x) for x in seqs]
    npages = [-(-L // ps) for L in lens]
    P = sum(npages)
    new = np.full((P, 2, hkv, ps, D), wl.CANARY, np.uint16)
    ip2 = np.zeros(w.batch + 1, np.int32)
    last2 = np.zeros(w.batch, np.int32)
    cur = 0
    for b, seq in enumerate(seqs):
        for t, (page, slot) in enumerate(seq):
            new[cur + t // ps, :, :, t % ps, :] = pool_bits[page, :, :, slot, :]
        ip2[b + 1] = ip2[b] + npages[b]
        last2[b] = lens[b] - (npages[b] - 1) * ps if lens[b] else 0
        cur += npages[b]
    ix2 = np.arange(P, dtype=np.int32)
    return oracle.decode(q_bits, new, oracle.BF16 if w.dtype == "bf16" else oracle.F16,
                         ip2, ix2, last2, w.sm_scale)


@pytest.mark.parametrize("case", [
    # batch, own lengths, hq, hkv, ps, dtype, prefix_pages, prefix_cut (tokens dropped from the prefix end)
    (9, "rand", 32, 8, 16, "bf16", 19, 4),
    (37, "rand", 64, 8, 16, "bf16", 8, 0),
    (5, "rand", 16, 2, 32, "f16", 5, 31),
    (3, "zero", 32, 8, 16, "bf16", 4, 7),
    (70, "rand", 8, 1, 256, "bf16", 2, 200),
    (50, "rand", 24, 8, 16, "bf16", 6, 3),    # G = 3: Q staged and states written per thread
])
def test_cascade_matches_oracle_small(case):
    batch, mode, hq, hkv, ps, dt, prefix_pages, cut = case
    rng = np.random.default_rng(batch)
    own = rng.integers(1, 300, size=batch) if mode == "rand" else np.zeros(batch, np.int64)
    own[0] = 0  # one request with no tokens of its own
    full = prefix_pages * ps
    w = wl.make_workload("cascade", full + own, num_qo_heads=hq, num_kv_heads=hkv, page_size=ps,
                         dtype=dt, seed=60 + batch, shared_prefix_len=full, pool_factor=1.2)
    prefix, _, ip, ix, ll = wl.cascade_view(w)
    prefix_len = full - cut
    q, pool, _, _ = wl.make_tensors(w, "cpu")
    out, lse = run_cascade(w, q.cuda(), pool.cuda(), prefix, prefix_len, ip, ix, ll)
    ref_o, ref_l = repacked_oracle(w, wl.bits(q), wl.bits(pool), prefix, prefix_len, ip, ix, ll)
    assert_parity(out, lse, ref_o, ref_l, what=str(case))


@pytest.mark.parametrize("N", [1, 3])
def test_cascade_requests_without_own_tokens(N):
    """Requests that hold only the prefix get the prefix's attention alone; with
    one or three partitions a CTA finalises more of them than it lists, so both
    the warps' path and the per-thread path run."""
    batch = 45
    own = np.zeros(batch, np.int64)
    own[[3, 20, 44]] = [17, 300, 1]
    full = 6 * 16
    w = wl.make_workload("cascade-empty", full + own, num_qo_heads=32, num_kv_heads=8,
                         page_size=16, dtype="bf16", seed=61, shared_prefix_len=full,
                         pool_factor=1.2)
    prefix, _, ip, ix, ll = wl.cascade_view(w)
    q, pool, _, _ = wl.make_tensors(w, "cpu")
    out, lse = run_cascade(w, q.cuda(), pool.cuda(), prefix, full, ip, ix, ll, num_partitions=N)
    ref_o, ref_l = repacked_oracle(w, wl.bits(q), wl.bits(pool), prefix, full, ip, ix, ll)
    assert_parity(out, lse, ref_o, ref_l, what=f"empty own, N={N}")


@pytest.mark.parametrize("N", [0, 3])
def test_cascade_with_no_own_tokens_at_all(N):
    """Every request holds only the prefix: the own-page decode has no work, and
    its CTAs (which read their table before the dependency wait) must still not
    let the launch complete before the prefix step, whose states the merge
    reads right after.  A long prefix keeps the prefix step running."""
    batch = 16
    full = 128 * 16
    w = wl.make_workload("cascade-prefix-only", np.full(batch, full), num_qo_heads=32,
                         num_kv_heads=8, page_size=16, dtype="bf16", seed=62,
                         shared_prefix_len=full, pool_factor=1.2)
    prefix, _, ip, ix, ll = wl.cascade_view(w)
    q, pool, _, _ = wl.make_tensors(w, "cpu")
    qd, pd = q.cuda(), pool.cuda()
    ref_o, ref_l = repacked_oracle(w, wl.bits(q), wl.bits(pool), prefix, full, ip, ix, ll)
    for _ in range(3):
        out, lse = run_cascade(w, qd, pd, prefix, full, ip, ix, ll, num_partitions=N)
        assert_parity(out, lse, ref_o, ref_l, what=f"prefix only, N={N}")


def test_cascade_equals_decode_on_shared_prefix_workload():
    w = wl.named(5)
    q, pool, _, _ = wl.make_tensors(w, "cuda")
    prefix, prefix_len, ip, ix, ll = wl.cascade_view(w)
    out, lse = run_cascade(w, q, pool, prefix, prefix_len, ip, ix, ll)
    sample = [0, 17, 101, 255]
    ref_o, ref_l = oracle_decode_from_device(w, q, pool, sample)
    assert_parity(out, lse, ref_o, ref_l, rows=sample, what="named 5 cascade")
    assert torch.isfinite(out.float()).all()
    # and agrees with the plain decode of the full table on every row
    t = lambda a: torch.as_tensor(a, device="cuda")
    ws = torch.zeros(pkv.decode_workspace_bytes(w.batch, 32, 8) // 4 + 64, dtype=torch.int32,
                     device="cuda")
    out_d, lse_d = pkv.paged_decode_attention(q, pool, t(w.page_indptr), t(w.page_indices),
                                              t(w.last_page_len), ws, sm_scale=w.sm_scale)
    torch.cuda.synchronize()
    diff = (out.float() - out_d.float()).abs().max().item()
    assert diff <= 2e-2
    assert (lse - lse_d).abs().max().item() <= 1e-3


def test_cascade_without_prefix_is_plain_decode():
    w = wl.make_workload("noprefix", [40, 300, 1], num_qo_heads=32, num_kv_heads=8,
                         page_size=16, dtype="bf16", seed=70)
    q, pool, _, _ = wl.make_tensors(w, "cuda")
    out, lse = run_cascade(w, q, pool, np.zeros(0, np.int32), 0, w.page_indptr, w.page_indices,
                           w.last_page_len)
    ref_o, ref_l = oracle.decode(wl.bits(q), wl.bits(pool), oracle.BF16, w.page_indptr,
                                 w.page_indices, w.last_page_len, w.sm_scale)
    assert_parity(out, lse, ref_o, ref_l)
