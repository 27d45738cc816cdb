"""Seeded synthetic workloads for paged decode attention.

This module holds the input recipe shared by the tests, the benchmark and
the smoke check: request lengths, the page table (a tiny host-side page
allocator), and the random q / K / V values.  It contains none of the
attention arithmetic: the CUDA library and the CPU oracle each compute on
the arrays produced here.

Recipe (one seed per workload; lengths are drawn first, then the page
placement, then q, K, V, then the new K/V rows of an append):
  * values: fp32 draws from N(0, 1) (q optionally scaled, K optionally
    offset per KV head), rounded to the stored 16-bit type by torch (RNE);
  * pages: a seeded random permutation of the pool; request b takes the
    next ceil(len_b / page_size) entries, in logical order (the "page table
    maps logical positions to scattered physical pages" picture of
    "上下文窗口优化实战：如何用PagedAttention+FlashInfer将Llama3-70B的128K上下文吞吐提升3.8倍？",
    section 2.3);
  * a shared prefix is stored once: its pages head every request's list
    (physical page sharing between requests with a common prefix,
    "大模型推理极致优化：FlashAttention+PageAttention联合调优", section 3.2);
  * canaries: every slot that holds no token -- unused pages, slots past
    last_page_len in a last page, and the slots an append is about to
    fill -- carries the 16-bit pattern 0x7FFF, a NaN in both fp16 and
    bf16, so a kernel that reads a slot it must skip returns NaN.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

CANARY = 0x7FFF          # NaN in fp16 and in bf16
SEED_BASE = 479000       # seed of named workload i is SEED_BASE + i
TILE_TOKENS = 16


@dataclasses.dataclass
class Workload:
    """A decode step's shapes, page table and value distribution."""
    name: str
    batch: int
    num_qo_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    dtype: str                       # "f16" or "bf16"
    kv_lens: np.ndarray              # int64 [B], tokens per request AFTER the append
    num_pages: int                   # pages in the pool
    page_indptr: np.ndarray          # int32 [B+1]
    page_indices: np.ndarray         # int32 [page_indptr[B]]
    last_page_len: np.ndarray        # int32 [B]
    append_counts: np.ndarray        # int64 [B], new tokens appended this step (0 = none)
    shared_prefix_pages: int = 0     # leading pages shared by every request
    q_std: float = 1.0
    key_offset_std: float = 0.0
    seed: int = 0
    note: str = ""

    @property
    def group(self) -> int:
        return self.num_qo_heads // self.num_kv_heads

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def elem_bytes(self) -> int:
        return 2

    @property
    def append_indptr(self) -> np.ndarray:
        out = np.zeros(self.batch + 1, np.int32)
        np.cumsum(self.append_counts, out=out[1:])
        return out

    @property
    def nnz_new(self) -> int:
        return int(self.append_counts.sum())

    @property
    def pool_shape(self):
        return (self.num_pages, 2, self.num_kv_heads, self.page_size, self.head_dim)

    @property
    def torch_dtype(self):
        return torch.float16 if self.dtype == "f16" else torch.bfloat16

    def pages_of(self, b: int) -> np.ndarray:
        return self.page_indices[self.page_indptr[b]:self.page_indptr[b + 1]]


# --------------------------------------------------------------------------
# byte counters (the benchmark's metric)
# --------------------------------------------------------------------------

def kv_cache_bytes(num_layers: int, num_kv_heads: int, head_dim: int, seq_len: int,
                   dtype_bytes: int = 2) -> int:
    """K and V bytes cached for seq_len tokens: 2 * Hkv * D * bytes per token and
    layer ("大模型长上下文窗口工程化实战：从RoPE扩展到百万Token推理的生产级部署",
    section 2.1, which prints 16.0 GB for Llama-3-8B and 40.0 GB for Llama-3-70B
    at 128K; the printed unit is 1024**3 bytes)."""
    return 2 * num_kv_heads * head_dim * dtype_bytes * num_layers * seq_len


def unique_kv_tokens(w: Workload) -> int:
    """Tokens whose K/V must come from HBM once: a shared prefix counts once."""
    prefix = w.shared_prefix_pages * w.page_size
    return int(w.kv_lens.sum() - prefix * max(w.batch - 1, 0)) if prefix else int(w.kv_lens.sum())


def decode_bytes(w: Workload, kv_elem_bytes: Optional[int] = None) -> int:
    """Algorithmic HBM bytes of one decode launch: unique K/V once, q in, out,
    the page table, and the fp32 lse.  kv_elem_bytes: bytes of a cached
    element (1 for an E4M3 pool; default the workload's 16-bit type)."""
    kvb = w.elem_bytes if kv_elem_bytes is None else kv_elem_bytes
    kv = kv_cache_bytes(1, w.num_kv_heads, w.head_dim, unique_kv_tokens(w), kvb)
    qo = 2 * w.batch * w.num_qo_heads * w.head_dim * w.elem_bytes
    table = 4 * (w.batch + 1 + len(w.page_indices) + w.batch)
    lse = 4 * w.batch * w.num_qo_heads
    return kv + qo + table + lse


def append_bytes(w: Workload, kv_elem_bytes: Optional[int] = None) -> int:
    """Algorithmic bytes of one append launch: new 16-bit rows read, then
    written into the pool (kv_elem_bytes each)."""
    kvb = w.elem_bytes if kv_elem_bytes is None else kv_elem_bytes
    elems = 2 * w.nnz_new * w.num_kv_heads * w.head_dim
    return elems * (w.elem_bytes + kvb) + 4 * (w.batch + 1) if w.nnz_new else 0


def logical_kv_bytes(w: Workload, kv_elem_bytes: Optional[int] = None) -> int:
    kvb = w.elem_bytes if kv_elem_bytes is None else kv_elem_bytes
    return kv_cache_bytes(1, w.num_kv_heads, w.head_dim, int(w.kv_lens.sum()), kvb)


# --------------------------------------------------------------------------
# page tables
# --------------------------------------------------------------------------

def build_table(kv_lens, page_size: int, rng: np.random.Generator, *,
                pool_pages: Optional[int] = None, pool_factor: float = 1.0,
                shared_prefix_len: int = 0):
    """Host page allocator: returns (num_pages, indptr, indices, last_page_len, prefix_pages).

    num_pages(b) = ceil(len_b / page_size) ("上下文窗口优化实战：如何用PagedAttention+FlashInfer
    将Llama3-70B的128K上下文吞吐提升3.8倍？", section 2.3, allocate_pages); the pool is
    either pool_pages, or ceil(pool_factor * pages needed); physical ids are the
    leading entries of a seeded permutation of the pool.
    """
    kv_lens = np.asarray(kv_lens, np.int64)
    if shared_prefix_len % page_size:
        raise ValueError("a shared prefix must fill whole pages")
    prefix_pages = shared_prefix_len // page_size
    if prefix_pages and np.any(kv_lens < shared_prefix_len):
        raise ValueError("every request must contain the shared prefix")
    own = [(-(-(int(L) - shared_prefix_len) // page_size)) if L > 0 else 0 for L in kv_lens]
    needed = prefix_pages + int(sum(own))
    P = pool_pages if pool_pages is not None else int(math.ceil(pool_factor * needed))
    if P < needed:
        raise ValueError("pool too small")
    perm = rng.permutation(P).astype(np.int32)
    prefix_ids = perm[:prefix_pages]
    cursor = prefix_pages
    indptr = np.zeros(len(kv_lens) + 1, np.int32)
    chunks = []
    last = np.zeros(len(kv_lens), np.int32)
    for b, L in enumerate(kv_lens):
        ids = perm[cursor:cursor + own[b]]
        cursor += own[b]
        ids = np.concatenate([prefix_ids, ids]) if (prefix_pages and L > 0) else ids
        chunks.append(ids)
        indptr[b + 1] = indptr[b] + len(ids)
        last[b] = (int(L) - (len(ids) - 1) * page_size) if L > 0 else 0
    indices = np.concatenate(chunks).astype(np.int32) if chunks else np.zeros(0, np.int32)
    return P, indptr, indices, last, prefix_pages


def make_workload(name, kv_lens, *, num_qo_heads, num_kv_heads, head_dim=128,
                  page_size=16, dtype="bf16", seed=0, pool_pages=None, pool_factor=1.0,
                  shared_prefix_len=0, append_counts=None, q_std=1.0,
                  key_offset_std=0.0, note="") -> Workload:
    rng = np.random.default_rng(seed)
    kv_lens = np.asarray(kv_lens, np.int64)
    P, indptr, indices, last, prefix_pages = build_table(
        kv_lens, page_size, rng, pool_pages=pool_pages, pool_factor=pool_factor,
        shared_prefix_len=shared_prefix_len)
    if append_counts is None:
        append_counts = np.zeros(len(kv_lens), np.int64)
    append_counts = np.asarray(append_counts, np.int64)
    if np.any(append_counts > kv_lens):
        raise ValueError("cannot append more tokens than the request holds")
    return Workload(name=name, batch=len(kv_lens), num_qo_heads=num_qo_heads,
                    num_kv_heads=num_kv_heads, head_dim=head_dim, page_size=page_size,
                    dtype=dtype, kv_lens=kv_lens, num_pages=P, page_indptr=indptr,
                    page_indices=indices, last_page_len=last, append_counts=append_counts,
                    shared_prefix_pages=prefix_pages, q_std=q_std,
                    key_offset_std=key_offset_std, seed=seed, note=note)


def named(config_id: int) -> Workload:
    """The five named workloads (seed 479000 + id)."""
    seed = SEED_BASE + config_id
    rng = np.random.default_rng(seed + 10_000)  # length draws
    if config_id == 1:
        return make_workload("tiny paged decode: 4 requests, KV {17,64,100,255}, 8q/2kv, D128, ps16, fp16",
                             [17, 64, 100, 255], num_qo_heads=8, num_kv_heads=2,
                             page_size=16, dtype="f16", seed=seed, pool_pages=64)
    if config_id == 2:
        lens = rng.integers(512, 4096, size=64, endpoint=True) + 1   # +1 = the appended token
        return make_workload("Llama-3-8B-shaped decode layer: batch 64, KV U[512,4096]+1 appended, 32q/8kv, D128, ps16, bf16",
                             lens, num_qo_heads=32, num_kv_heads=8, page_size=16,
                             dtype="bf16", seed=seed, pool_factor=1.25,
                             append_counts=np.ones(64, np.int64))
    if config_id == 3:
        return make_workload("Llama3-70B-shaped long context: batch 8, KV 131072, 64q/8kv, D128, ps16, bf16",
                             [131072] * 8, num_qo_heads=64, num_kv_heads=8, page_size=16,
                             dtype="bf16", seed=seed)
    if config_id == 4:
        return make_workload("single very long sequence: batch 1, KV 200000, 32q/8kv, D128, ps256, bf16, per-head key offset",
                             [200000], num_qo_heads=32, num_kv_heads=8, page_size=256,
                             dtype="bf16", seed=seed, q_std=3.0, key_offset_std=8.0,
                             note="keys + per-KV-head offset ~N(0,8^2) per element; q ~ N(0,3^2)")
    if config_id == 5:
        suffix = np.rint(np.exp(rng.normal(math.log(256.0), 1.0, size=256))).astype(np.int64)
        suffix = np.clip(suffix, 1, 8192)
        return make_workload("shared-prefix mixed batch: 256 requests, 4096-token shared prefix + lognormal suffix (median 256, sigma 1, [1,8192]), 32q/8kv, D128, ps16, bf16",
                             4096 + suffix, num_qo_heads=32, num_kv_heads=8, page_size=16,
                             dtype="bf16", seed=seed, shared_prefix_len=4096)
    raise ValueError(f"no named workload {config_id}")


# --------------------------------------------------------------------------
# values
# --------------------------------------------------------------------------

def _canary_mask_slots(w: Workload):
    """(page, slot) pairs that hold no token before the append runs."""
    used = np.zeros(w.num_pages, bool)
    used[w.page_indices] = True
    pairs = []
    for b in range(w.batch):
        pages = w.pages_of(b)
        if len(pages) == 0:
            continue
        lp = int(w.last_page_len[b])
        for s in range(lp, w.page_size):
            pairs.append((int(pages[-1]), s))
        n_new = int(w.append_counts[b])
        L = int(w.kv_lens[b])
        for pos in range(L - n_new, L):
            pairs.append((int(pages[pos // w.page_size]), pos % w.page_size))
    return np.flatnonzero(~used), np.array(pairs, np.int64).reshape(-1, 2)


def _fill(pool, q, k_new, v_new, w: Workload, gen, device):
    """Draw q, the pool and the new rows in a fixed order from one generator."""
    dt = w.torch_dtype
    q.copy_((torch.randn(q.shape, generator=gen, device=device) * w.q_std).to(dt))
    offs = None
    if w.key_offset_std:
        offs = torch.randn((w.num_kv_heads, w.head_dim), generator=gen, device=device) * w.key_offset_std
    chunk = max(1, (1 << 26) // (2 * w.num_kv_heads * w.page_size * w.head_dim))
    for p0 in range(0, w.num_pages, chunk):
        p1 = min(w.num_pages, p0 + chunk)
        x = torch.randn((p1 - p0,) + tuple(w.pool_shape[1:]), generator=gen, device=device)
        if offs is not None:
            x[:, 0] += offs[None, :, None, :]
        pool[p0:p1].copy_(x.to(dt))
        del x
    if w.nnz_new:
        kn = torch.randn(k_new.shape, generator=gen, device=device)
        if offs is not None:
            kn += offs[None]
        k_new.copy_(kn.to(dt))
        v_new.copy_(torch.randn(v_new.shape, generator=gen, device=device).to(dt))
    unused, pairs = _canary_mask_slots(w)
    bits = pool.view(torch.int16)
    if len(unused):
        bits[torch.as_tensor(unused, device=device)] = CANARY
    if len(pairs):
        pg = torch.as_tensor(pairs[:, 0], device=device)
        sl = torch.as_tensor(pairs[:, 1], device=device)
        bits[pg, :, :, sl, :] = CANARY


def make_tensors(w: Workload, device="cpu"):
    """q [B,Hq,D], pool [P,2,Hkv,ps,D] (state BEFORE the append), k_new / v_new
    [nnz,Hkv,D], all in the workload's 16-bit dtype on `device`.

    The same seed gives the same bytes on the same kind of device; a CPU and a
    CUDA generator give different streams, so a parity test draws on one side
    and copies the bytes to the other.
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(w.seed))
    dt = w.torch_dtype
    q = torch.empty((w.batch, w.num_qo_heads, w.head_dim), dtype=dt, device=device)
    pool = torch.empty(w.pool_shape, dtype=dt, device=device)
    k_new = torch.empty((w.nnz_new, w.num_kv_heads, w.head_dim), dtype=dt, device=device)
    v_new = torch.empty_like(k_new)
    _fill(pool, q, k_new, v_new, w, gen, device)
    return q, pool, k_new, v_new


# --------------------------------------------------------------------------
# 8-bit (E4M3) pools
# --------------------------------------------------------------------------

FP8_CANARY = 0x7F  # NaN in E4M3 and in E5M2: fills every slot that holds no token
FP8_EXP_MEAN = 11  # exponent field of a typical code: magnitude 2^(11-7) = 16
FP8_E5M2_EXP_MEAN = 19  # the same magnitude in E5M2: 2^(19-15) = 16


def e4m3_codes(shape, gen, device, exp_mean=FP8_EXP_MEAN, exp_std=1.25):
    """Random E4M3 codes assembled field by field (no conversion arithmetic):
    sign uniform, exponent field round(N(exp_mean, exp_std)) clipped to
    [0, 15] (0 gives subnormals), fraction uniform; the NaN codes S.1111.111
    are never drawn (they become S.1111.110 = +-448)."""
    sign = torch.randint(0, 2, shape, generator=gen, device=device, dtype=torch.int32)
    e = torch.randn(shape, generator=gen, device=device) * exp_std + exp_mean
    e = e.round().clamp(0, 15).to(torch.int32)
    m = torch.randint(0, 8, shape, generator=gen, device=device, dtype=torch.int32)
    code = (sign << 7) | (e << 3) | m
    code = torch.where((code & 0x7F) == 0x7F, code - 1, code)
    return code.to(torch.uint8)


def e5m2_codes(shape, gen, device, exp_mean=FP8_E5M2_EXP_MEAN, exp_std=1.25):
    """Random E5M2 codes assembled field by field: sign uniform, exponent field
    round(N(exp_mean, exp_std)) clipped to [0, 23] (0 gives subnormals; the
    largest magnitude is 448, the E4M3 range, so both formats give values of
    the same spread -- the far exponents up to 30 stay reachable through the
    append's quantisation), fraction uniform."""
    sign = torch.randint(0, 2, shape, generator=gen, device=device, dtype=torch.int32)
    e = torch.randn(shape, generator=gen, device=device) * exp_std + exp_mean
    e = e.round().clamp(0, 23).to(torch.int32)
    m = torch.randint(0, 4, shape, generator=gen, device=device, dtype=torch.int32)
    return ((sign << 7) | (e << 2) | m).to(torch.uint8)


def make_fp8_tensors(w: Workload, device="cpu", fmt="e4m3"):
    """q [B,Hq,D] and new rows [nnz,Hkv,D] in the workload's 16-bit dtype, and
    an 8-bit pool [P,2,Hkv,ps,D] (uint8 codes of the format; state before the
    append) whose slots that hold no token carry FP8_CANARY (a NaN code of both
    formats)."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(w.seed) + 8)
    dt = w.torch_dtype
    q = (torch.randn((w.batch, w.num_qo_heads, w.head_dim), generator=gen, device=device)
         * w.q_std).to(dt)
    pool = torch.empty(w.pool_shape, dtype=torch.uint8, device=device)
    chunk = max(1, (1 << 26) // (2 * w.num_kv_heads * w.page_size * w.head_dim))
    for p0 in range(0, w.num_pages, chunk):
        p1 = min(w.num_pages, p0 + chunk)
        draw = e4m3_codes if fmt == "e4m3" else e5m2_codes
        pool[p0:p1] = draw((p1 - p0,) + tuple(w.pool_shape[1:]), gen, device)
    k_new = torch.randn((w.nnz_new, w.num_kv_heads, w.head_dim), generator=gen,
                        device=device).to(dt)
    v_new = torch.randn((w.nnz_new, w.num_kv_heads, w.head_dim), generator=gen,
                        device=device).to(dt)
    unused, pairs = _canary_mask_slots(w)
    if len(unused):
        pool[torch.as_tensor(unused, device=device)] = FP8_CANARY
    if len(pairs):
        pg = torch.as_tensor(pairs[:, 0], device=device)
        sl = torch.as_tensor(pairs[:, 1], device=device)
        pool[pg, :, :, sl, :] = FP8_CANARY
    return q, pool, k_new, v_new


# --------------------------------------------------------------------------
# multi-token chunks (append attention)
# --------------------------------------------------------------------------

def chunk_indptr(q_lens) -> np.ndarray:
    qo = np.zeros(len(q_lens) + 1, np.int32)
    qo[1:] = np.cumsum(np.asarray(q_lens, np.int64))
    return qo


def make_chunk_queries(w: Workload, q_lens, device="cpu", seed_offset=17):
    """Query rows [sum(q_lens), Hq, D] of the workload's dtype for chunks of
    q_lens tokens per request (the last q_lens[b] of request b's tokens)."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(w.seed) + seed_offset)
    n = int(np.sum(q_lens))
    return (torch.randn((n, w.num_qo_heads, w.head_dim), generator=gen, device=device)
            * w.q_std).to(w.torch_dtype)


def named_chunk(kind: str):
    """Append-attention workloads: (workload, q_lens); the chunk's K/V rows are
    the workload's appended tokens (append_counts = q_lens).

    "prefill": chunked prefill of a Llama-3-8B-shaped layer -- 4 prompts whose
      2048-token chunk lands on 6144 cached tokens (8192 after the append),
      32q/8kv, D128, ps16, bf16.
    "spec": verification of 4 speculative tokens for the decode batch of the
      Llama-3-8B-shaped workload -- batch 64, KV U[512,4096] + 4, 32q/8kv, bf16.
    """
    seed = SEED_BASE + 100
    if kind == "prefill":
        q_lens = np.full(4, 2048, np.int64)
        w = make_workload("chunked prefill: 4 x (6144 cached + 2048-token chunk), 32q/8kv, D128, ps16, bf16",
                          [8192] * 4, num_qo_heads=32, num_kv_heads=8, page_size=16,
                          dtype="bf16", seed=seed, pool_factor=1.1, append_counts=q_lens)
        return w, q_lens
    if kind == "spec":
        rng = np.random.default_rng(seed + 10_000)
        lens = rng.integers(512, 4096, size=64, endpoint=True) + 4
        q_lens = np.full(64, 4, np.int64)
        w = make_workload("speculative verification: batch 64, KV U[512,4096] + 4 draft tokens, 32q/8kv, D128, ps16, bf16",
                          lens, num_qo_heads=32, num_kv_heads=8, page_size=16, dtype="bf16",
                          seed=seed + 1, pool_factor=1.25, append_counts=q_lens)
        return w, q_lens
    raise ValueError(f"no chunk workload {kind!r}")


def chunk_flops(w: Workload, q_lens, window_left: int = -1, sink: int = 0) -> int:
    """Algorithmic FLOPs of append attention: 2 * D per (query head, visible
    key) for the scores and as many for P.V."""
    total = 0
    for b in range(w.batch):
        L, n = int(w.kv_lens[b]), int(q_lens[b])
        pos = np.arange(L - n, L, dtype=np.int64)
        vis = pos + 1
        if window_left >= 0:
            vis = np.minimum(vis, window_left + 1 + np.minimum(sink, np.maximum(pos - window_left, 0)))
        total += int(vis.sum())
    return 4 * w.head_dim * w.num_qo_heads * total


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 bit patterns of a 16-bit tensor, on the host."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def from_bits(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, np.uint16).view(np.int16))
    return t.view(torch.float16 if dtype == "f16" else torch.bfloat16)


def cascade_view(w: Workload):
    """Split w's table into its shared prefix and each request's own pages:
    (prefix page ids, prefix tokens, own indptr, own indices, own last_page_len)."""
    k = w.shared_prefix_pages
    prefix = w.pages_of(0)[:k].astype(np.int32) if w.batch else np.zeros(0, np.int32)
    indptr = np.zeros(w.batch + 1, np.int32)
    chunks = []
    last = np.zeros(w.batch, np.int32)
    for b in range(w.batch):
        own = w.pages_of(b)[k:]
        chunks.append(own)
        indptr[b + 1] = indptr[b] + len(own)
        last[b] = w.last_page_len[b] if len(own) else 0
    indices = np.concatenate(chunks).astype(np.int32) if chunks else np.zeros(0, np.int32)
    return prefix, k * w.page_size, indptr, indices, last


def subset(w: Workload, requests, pool_bits_of_pages):
    """A compact copy of requests `requests` of workload w: the returned table
    renumbers their pages 0..n-1 in order of first use; `pool_bits_of_pages(ids)`
    must return the uint16 pool rows of those physical ids.  Used to run the
    oracle on sampled requests of a full-size workload."""
    requests = list(requests)
    ids = np.concatenate([w.pages_of(b) for b in requests]) if requests else np.zeros(0, np.int32)
    uniq, inv = np.unique(ids, return_inverse=True)
    indptr = np.zeros(len(requests) + 1, np.int32)
    for i, b in enumerate(requests):
        indptr[i + 1] = indptr[i] + len(w.pages_of(b))
    last = w.last_page_len[requests].astype(np.int32)
    return pool_bits_of_pages(uniq), indptr, inv.astype(np.int32), last
