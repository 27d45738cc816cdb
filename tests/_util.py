"""Shared helpers of the GPU parity tests: move a workload to the device, run
the library, run the oracle on the same bytes, and compare."""
import numpy as np
import torch

import oracle
import paged_kv_cache_479_b200 as pkv
from paged_kv_cache_479_b200 import workloads as wl

# acceptance bar for 16-bit outputs against the fp64 oracle
MAX_ABS = 1e-2
REL_L2 = 2e-3
LSE_ABS = 1e-3


def odtype(w):
    return oracle.BF16 if w.dtype == "bf16" else oracle.F16


class DeviceCase:
    """A workload's tensors and page table on the GPU, plus scratch buffers."""

    def __init__(self, w, q, pool, k_new=None, v_new=None, num_partitions=0):
        dev = torch.device("cuda")
        self.w = w
        self.q = q.to(dev)
        self.pool = pool.to(dev)
        self.k_new = None if k_new is None else k_new.to(dev)
        self.v_new = None if v_new is None else v_new.to(dev)
        self.indptr = torch.as_tensor(w.page_indptr, device=dev)
        self.indices = torch.as_tensor(w.page_indices if len(w.page_indices) else np.zeros(1, np.int32), device=dev)
        self.last = torch.as_tensor(w.last_page_len, device=dev)
        self.append_indptr = torch.as_tensor(w.append_indptr, device=dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.num_partitions = num_partitions
        self.ws = self.workspace(num_partitions)

    def workspace(self, n):
        nb = pkv.decode_workspace_bytes(self.w.batch, self.w.num_qo_heads, self.w.num_kv_heads,
                                        128, n)
        return torch.zeros(nb // 4 + 64, dtype=torch.int32, device="cuda")

    def append(self):
        pkv.paged_kv_append(self.pool, self.indptr, self.indices, self.last, self.k_new,
                            self.v_new, self.append_indptr, error_word=self.err)

    def decode(self, num_partitions=None, ws=None):
        n = self.num_partitions if num_partitions is None else num_partitions
        if ws is None:
            ws = self.ws if n == self.num_partitions else self.workspace(n)
        out, lse = pkv.paged_decode_attention(self.q, self.pool, self.indptr, self.indices,
                                              self.last, ws, sm_scale=self.w.sm_scale,
                                              num_partitions=n, error_word=self.err)
        torch.cuda.synchronize()
        return out, lse

    def error_bits(self):
        return pkv.read_error_word(self.err)


def oracle_decode(w, q_bits, pool_bits, requests=None):
    """Oracle on all requests, or on the listed ones (compacted sub-table)."""
    if requests is None:
        return oracle.decode(q_bits, pool_bits, odtype(w), w.page_indptr, w.page_indices,
                             w.last_page_len, w.sm_scale)
    sub_pool, ip, ix, ll = wl.subset(w, requests, lambda ids: pool_bits[ids])
    return oracle.decode(q_bits[requests], sub_pool, odtype(w), ip, ix, ll, w.sm_scale)


def oracle_decode_from_device(w, q, pool, requests):
    """Oracle on sampled requests of a workload that lives on the device: only
    those requests' pages are copied to the host."""
    def pages(ids):
        return wl.bits(pool[torch.as_tensor(ids, device=pool.device, dtype=torch.long)])
    sub_pool, ip, ix, ll = wl.subset(w, requests, pages)
    qb = wl.bits(q[torch.as_tensor(requests, device=q.device, dtype=torch.long)])
    return oracle.decode(qb, sub_pool, odtype(w), ip, ix, ll, w.sm_scale)


def errors(out, lse, ref_o, ref_l, rows=None):
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.cpu().numpy().astype(np.float64) if lse is not None else None
    if rows is not None:
        o = o[rows]
        l = l[rows] if l is not None else None
    finite = np.isfinite(o).all()
    diff = o - ref_o
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    denom = float(np.linalg.norm(ref_o))
    rel = float(np.linalg.norm(diff) / denom) if denom > 0 else float(np.linalg.norm(diff))
    lse_err = 0.0
    if l is not None and l.size:
        both_inf = np.isneginf(l) & np.isneginf(ref_l)
        with np.errstate(invalid="ignore"):
            d = np.where(both_inf, 0.0, l - ref_l)
        lse_err = float(np.abs(d).max())
    return dict(finite=bool(finite), max_abs=max_abs, rel_l2=rel, lse_abs=lse_err)


def assert_parity(out, lse, ref_o, ref_l, rows=None, what=""):
    e = errors(out, lse, ref_o, ref_l, rows)
    assert e["finite"], f"{what}: non-finite output {e}"
    assert e["max_abs"] <= MAX_ABS, f"{what}: {e}"
    assert e["rel_l2"] <= REL_L2, f"{what}: {e}"
    assert e["lse_abs"] <= LSE_ABS, f"{what}: {e}"
    return e
