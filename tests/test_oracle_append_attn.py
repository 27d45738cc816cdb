"""Pins of the oracle's multi-token append attention (a chunk of new query
tokens per request, causal over the paged cache, optional window with sink
tokens) against torch SDPA with an explicit mask (a library routine),
hand-derived cases, the single-token decode it reduces to, and the
chunking invariance that chunked prefill relies on."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_479_b200 import workloads as wl

from test_oracle_pins import scatter_dense, to_bits, widen


def visible_mask(q_len, L, window_left=-1, sink=0):
    """[q_len, L] bool: query i (position L - q_len + i) sees key t."""
    pos = np.arange(L - q_len, L)[:, None]
    t = np.arange(L)[None, :]
    m = t <= pos
    if window_left >= 0:
        m &= (t >= pos - window_left) | (t < sink)
    return m


def case(lens, q_lens, hq, hkv, ps, dtype, seed, pool_factor=1.3):
    w = wl.make_workload("aa", lens, num_qo_heads=hq, num_kv_heads=hkv, page_size=ps,
                         dtype=dtype, seed=seed, pool_factor=pool_factor)
    gen = torch.Generator().manual_seed(seed)
    k_dense = [to_bits(torch.randn((L, hkv, 128), generator=gen), dtype) for L in w.kv_lens]
    v_dense = [to_bits(torch.randn((L, hkv, 128), generator=gen), dtype) for L in w.kv_lens]
    pool = scatter_dense(w, k_dense, v_dense)
    qo = np.zeros(len(lens) + 1, np.int32)
    qo[1:] = np.cumsum(q_lens)
    q_bits = to_bits(torch.randn((int(qo[-1]), hq, 128), generator=gen), dtype)
    return w, q_bits, pool, k_dense, v_dense, qo


def sdpa_masked(w, q_bits, qo, k_dense, v_dense, window_left=-1, sink=0):
    outs, lses = [], []
    q = widen(q_bits, w.dtype)
    for b in range(w.batch):
        n = int(qo[b + 1] - qo[b])
        if n == 0:
            continue
        L = int(w.kv_lens[b])
        k = widen(k_dense[b], w.dtype).permute(1, 0, 2)[None]         # [1,Hkv,L,D]
        v = widen(v_dense[b], w.dtype).permute(1, 0, 2)[None]
        qb = q[qo[b]:qo[b + 1]].permute(1, 0, 2)[None]                 # [1,Hq,n,D]
        mask = torch.from_numpy(visible_mask(n, L, window_left, sink))
        o = torch.nn.functional.scaled_dot_product_attention(qb, k, v, attn_mask=mask,
                                                             scale=w.sm_scale, enable_gqa=True)
        outs.append(o[0].permute(1, 0, 2))                             # [n,Hq,D]
        kk = k[0].repeat_interleave(w.group, dim=0)                    # [Hq,L,D]
        s = torch.einsum("hnd,hld->hnl", qb[0], kk) * w.sm_scale
        s = s.masked_fill(~mask[None], float("-inf"))
        lses.append(torch.logsumexp(s, dim=-1).permute(1, 0))         # [n,Hq]
    return torch.cat(outs).numpy(), torch.cat(lses).numpy()


CASES = [
    # lens, q_lens, hq, hkv, ps, dtype, window_left, sink
    ([40, 100, 17, 64], [5, 100, 1, 16], 8, 2, 16, "bf16", -1, 0),
    ([300, 33], [37, 33], 16, 2, 32, "f16", -1, 0),
    ([129, 70, 200], [64, 0, 9], 8, 8, 16, "bf16", 31, 0),
    ([260, 90], [120, 90], 8, 1, 64, "f16", 50, 7),
]


def run_oracle(w, q_bits, pool, qo, window_left=-1, sink=0):
    return oracle.append_attention(q_bits, pool, oracle.BF16 if w.dtype == "bf16" else oracle.F16,
                                   w.page_indptr, w.page_indices, w.last_page_len, qo,
                                   w.sm_scale, window_left, sink)


@pytest.mark.parametrize("i", range(len(CASES)))
def test_append_attention_matches_masked_sdpa(i):
    lens, q_lens, hq, hkv, ps, dt, wlft, sink = CASES[i]
    w, q_bits, pool, kd, vd, qo = case(lens, q_lens, hq, hkv, ps, dt, 500 + i)
    out, lse = run_oracle(w, q_bits, pool, qo, wlft, sink)
    ro, rl = sdpa_masked(w, q_bits, qo, kd, vd, wlft, sink)
    assert np.isfinite(out).all()                 # canaries (NaN) never read
    np.testing.assert_allclose(out, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)


def test_single_token_chunks_are_the_decode():
    w, q_bits, pool, _, _, qo = case([40, 100, 17, 256], [1, 1, 1, 1], 8, 2, 16, "bf16", 510)
    out, lse = run_oracle(w, q_bits, pool, qo)
    do, dl = oracle.decode(q_bits, pool, oracle.BF16, w.page_indptr, w.page_indices,
                           w.last_page_len, w.sm_scale)
    np.testing.assert_array_equal(out, do)
    np.testing.assert_array_equal(lse, dl)


def test_chunking_invariance():
    # a prompt processed as one chunk, or as its last chunk against a cache that
    # already holds the earlier tokens, gives the same rows for that last chunk
    w, q_bits, pool, _, _, qo = case([150], [150], 8, 2, 16, "f16", 511)
    whole, whole_l = run_oracle(w, q_bits, pool, qo)
    tail = np.array([0, 40], np.int32)
    part, part_l = run_oracle(w, q_bits[110:], pool, tail)
    np.testing.assert_array_equal(part, whole[110:])
    np.testing.assert_array_equal(part_l, whole_l[110:])


def test_hand_derived_identical_keys_and_windows():
    # identical keys: every visible key has the same score, so each query's
    # output is the plain mean of the values it may see
    w = wl.make_workload("aa", [6], num_qo_heads=2, num_kv_heads=1, page_size=16, dtype="f16",
                         seed=512)
    gen = torch.Generator().manual_seed(3)
    key = to_bits(torch.randn((1, 1, 128), generator=gen), "f16")
    kd = [np.repeat(key, 6, axis=0)]
    vals = (torch.arange(6, dtype=torch.float64)[:, None, None] * 0.25
            + torch.arange(128, dtype=torch.float64)[None, None, :] / 64)
    vd = [to_bits(vals, "f16")]                  # exact in fp16
    pool = scatter_dense(w, kd, vd)
    qo = np.array([0, 3], np.int32)              # queries at positions 3, 4, 5
    q_bits = to_bits(torch.randn((3, 2, 128), generator=gen), "f16")
    v = widen(vd[0], "f16")[:, 0].numpy()        # [6, 128]
    out, _ = run_oracle(w, q_bits, pool, qo)
    for i, pos in enumerate((3, 4, 5)):
        np.testing.assert_allclose(out[i, 0], v[:pos + 1].mean(0), rtol=0, atol=1e-14)
    # window_left 0: a query sees only itself
    out, lse = run_oracle(w, q_bits, pool, qo, window_left=0)
    for i, pos in enumerate((3, 4, 5)):
        np.testing.assert_array_equal(out[i, 1], v[pos])
    # window_left 1 with 2 sink tokens: keys {0, 1} plus {pos - 1, pos}
    out, _ = run_oracle(w, q_bits, pool, qo, window_left=1, sink=2)
    for i, pos in enumerate((3, 4, 5)):
        seen = sorted({0, 1, pos - 1, pos})
        np.testing.assert_allclose(out[i, 0], v[seen].mean(0), rtol=0, atol=1e-14)


def test_rejects_bad_chunks():
    w, q_bits, pool, _, _, qo = case([10, 5], [3, 2], 4, 2, 16, "f16", 513)
    with pytest.raises(oracle.OracleError):          # more queries than tokens
        run_oracle(w, np.zeros((9, 4, 128), np.uint16), pool, np.array([0, 3, 9], np.int32))
    with pytest.raises(oracle.OracleError):          # qo_indptr must start at 0
        run_oracle(w, q_bits, pool, np.array([1, 3, 5], np.int32))
