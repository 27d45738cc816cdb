"""Failure detection on the GPU without a fault: decode launches whose
internal waits run out.

Every wait inside the decode kernel has a time limit (one second by default).
pkv_set_wait_limit_ns shortens it to 1 ns here, so the consumer warps give up
on their first tile that has not landed yet.  The launch must still complete
(the CTA lets its own copies in flight land first), report
PKV_DEVERR_TIMEOUT through the error word, leave the CUDA context usable,
and leave the workspace's arrival counters at zero: the next call with the
default limit, on the same workspace and without clearing it, matches the
fp64 oracle and is bitwise equal to a call on a fresh workspace."""
import numpy as np
import pytest
import torch

import paged_kv_cache_479_b200 as pkv
from paged_kv_cache_479_b200 import workloads as wl
from _util import DeviceCase, assert_parity, oracle_decode

pytestmark = pytest.mark.gpu


def _fresh_ws(dc, n):
    return dc.workspace(n)


@pytest.mark.parametrize("N", [0, 7])
def test_timed_out_launch_reports_and_leaves_workspace_reusable(N):
    w = wl.make_workload("wait-limit", [3000, 500, 17, 8000, 1, 2049], num_qo_heads=32,
                         num_kv_heads=8, page_size=16, dtype="bf16", seed=91, pool_factor=1.3)
    q, pool, _, _ = wl.make_tensors(w, "cpu")
    dc = DeviceCase(w, q, pool, num_partitions=N)
    ref_o, ref_l = oracle_decode(w, wl.bits(q), wl.bits(pool))

    prev = pkv.set_wait_limit_ns(1)
    try:
        for _ in range(2):
            dc.decode()   # synchronises: the launch completed without a CUDA error
            err = int(dc.err.item())
            assert err & pkv.DEVERR_TIMEOUT, hex(err)
            dc.err.zero_()
    finally:
        assert pkv.set_wait_limit_ns(prev) == 1
    assert pkv.set_wait_limit_ns(0) == prev   # 0 selects the default again

    out, lse = dc.decode()   # same workspace, not cleared
    assert dc.error_bits() == 0
    assert_parity(out, lse, ref_o, ref_l, what=f"after timeouts, N={N}")
    fresh_o, fresh_l = dc.decode(ws=_fresh_ws(dc, N))
    assert torch.equal(out.view(torch.int16), fresh_o.view(torch.int16))
    assert torch.equal(lse.view(torch.int32), fresh_l.view(torch.int32))
