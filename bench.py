#!/usr/bin/env python
"""Benchmark: batched decode attention over a paged KV cache on B200.

One step = one pass of the whole decode hot path over one batch: append the
step's new K/V token(s) into their pages (when the workload appends), then
decode attention for every request with the split-KV partition and the
in-kernel merge.  On 16-bit pools the append runs inside the decode launch
(pkv_decode_append; --separate-append launches it on its own).  Default
workload: the Llama3-70B-shaped 128K long context (batch 8, every KV length
131072, 64 q / 8 kv heads, head_dim 128, page size 16, bf16, 4 GiB of K/V,
random page placement, split-KV on).  Its line also carries `per_config`:
the same measurement, same steps, for the tiny case, the Llama-3-8B-shaped
decode layer (with its append), the single 200K sequence and the shared-
prefix batch (plain decode and the cascade), each with its own oracle
cpu_baseline.

Metric: KV HBM GB/s (algorithmic bytes: unique K/V once + q + out + page
table + lse, plus the append's rows), with us/step and decoded tokens/s.

Timing: W untimed steps, then the K steps captured back to back in one CUDA
graph and replayed once between two CUDA events on the launching stream
(barrier and synchronize on both sides, max over ranks).  Nothing sits
between two launches, so each may start while the previous one drains
(programmatic dependent launch), as in a serving loop; the per-launch time
in `roofline` is the timed region divided by its launches.

  python bench.py [--gpus N --steps K --warmup W] [--workload 1..5] [--impl reference]

N > 1 (launched by torch.distributed.run, one rank per GPU): every rank runs
its own independent batch of the same shape (weak scaling; no collective on
the data path; the barrier and the max-over-ranks timing use NCCL).
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_479_b200 import workloads as wl  # noqa: E402

METRIC = "paged decode attn: KV HBM GB/s (% of B200 peak), µs/step, tokens/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
DECODE_SOURCES = ["csrc/decode.cu", "csrc/common.cuh", "csrc/partition.cuh"]


def parse():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=300)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["pkv", "reference"], default="pkv")
    p.add_argument("--workload", type=int, default=3, choices=[1, 2, 3, 4, 5])
    p.add_argument("--partitions", type=int, default=0, help="split-KV partitions (0 = one per SM)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--separate-append", action="store_true",
                   help="launch the append on its own instead of fusing it into the decode "
                        "(pkv_decode_append; 16-bit pools, plain decode)")
    p.add_argument("--fused-chunk-append", action="store_true",
                   help="--chunk spec: append the chunk's K/V inside the short-chunk launch "
                        "(slower than a separate append at 4 rows per request)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-early-table", action="store_true",
                   help="do not mark the page table ready at launch (the decode then waits for "
                        "the previous kernel before it reads the table)")
    p.add_argument("--no-per-config", action="store_true",
                   help="headline workload only (by default the 128K headline line also "
                        "carries per_config numbers of workloads 1, 2, 4, 5 and the 5 cascade)")
    p.add_argument("--per-config-cpu-seconds", type=float, default=4.0,
                   help="oracle time budget of each per_config cpu_baseline")
    p.add_argument("--cascade", action="store_true",
                   help="decode a shared-prefix workload with pkv_cascade_decode")
    p.add_argument("--no-graph", action="store_true",
                   help="launch every call from Python instead of replaying one CUDA graph")
    p.add_argument("--kv", choices=["16bit", "e4m3", "e5m2"], default="16bit",
                   help="KV pool type: the workload's 16-bit type, or FP8 (E4M3 / E5M2) codes "
                        "with per-tensor K/V scales (q and out stay 16-bit)")
    p.add_argument("--chunk", choices=["prefill", "spec"], default=None,
                   help="time multi-token append attention instead of the decode: chunked "
                        "prefill (TFLOP/s) or speculative verification (GB/s)")
    p.add_argument("--chunk-path", choices=["auto", "tc", "short"], default="auto",
                   help="append attention kernel: tcgen05 row blocks, the short-chunk decode "
                        "schedule (q_len * G <= 16), or auto (short when it applies)")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle time budget for cpu_baseline")
    p.add_argument("--ref-seconds", type=float, default=150.0, help="oracle time budget of the reference arm")
    return p.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def rank_value_seed(base_seed, rank, copy):
    """Seed of the values of batch copy `copy` on `rank`: every rank decodes its own
    independent batch of the same shape (weak scaling)."""
    return base_seed + 1000 * rank + copy


def max_over_ranks(x, world, device):
    """Max of a float over all ranks (the slowest rank times the job)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_step_per_rank, world, ms_total, steps):
    """Whole-job GB/s: every rank's bytes over the slowest rank's time."""
    return bytes_per_step_per_rank * world / (ms_total / 1e3 / steps) / 1e9


def measured_tensor():
    """Measured bf16 dense GEMM throughput (burst, TFLOP/s)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def measured_hbm():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def decode_source_hash():
    h = hashlib.sha256()
    for rel in DECODE_SOURCES:
        with open(os.path.join(ROOT, "paged_kv_cache_479_b200", rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload_id):
    """DRAM bytes per decode launch from a committed ncu summary, only while the
    kernel sources are the ones that summary was taken on."""
    path = os.path.join(ROOT, "profiles", "decode_dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("source_hash") != decode_source_hash():
        return None
    entry = rec.get("workloads", {}).get(str(workload_id))
    return None if entry is None else int(entry["dram_bytes_per_launch"])


class ClockSampler:
    """SM clock, power and throttle reasons of one GPU, read through NVML
    every 2 ms from a background thread (read-only queries; no setting is
    touched), so that even a timed region of a few milliseconds holds
    samples.  Falls back to `nvidia-smi -lms 100` when NVML is unavailable."""
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    PERIOD_S = 0.002

    def __init__(self, device_index):
        self.samples = []
        self.source = None
        self._stop = threading.Event()
        self.proc = None
        uuid = str(torch.cuda.get_device_properties(device_index).uuid)
        self.ident = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(self.ident)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
            self.bits = [pynvml.nvmlClocksEventReasonHwSlowdown,
                         pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                         pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                         pynvml.nvmlClocksEventReasonSwPowerCap]
            self.source = f"NVML every {self.PERIOD_S * 1e3:.0f} ms"
            self.thread = threading.Thread(target=self._poll_nvml, daemon=True)
            self.thread.start()
        except Exception:
            self._start_smi()

    def _poll_nvml(self):
        nv, h = self.nvml, self.handle
        while not self._stop.is_set():
            try:
                mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                r = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                self.samples.append((time.time(), mhz, self.max_mhz, pw,
                                     [bool(r & b) for b in self.bits]))
            except Exception:
                pass
            self._stop.wait(self.PERIOD_S)

    def _start_smi(self):
        fields = ["clocks.sm", "clocks.max.sm", "power.draw",
                  "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
                  "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.ident, f"--query-gpu={','.join(fields)}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True, bufsize=1)
            self.source = "nvidia-smi every 100 ms"
            self.thread = threading.Thread(target=self._read_smi, args=(len(fields),), daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read_smi(self, nf):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) != nf:
                continue
            try:
                self.samples.append((time.time(), float(parts[0]), float(parts[1]),
                                     float(parts[2]) if parts[2] not in ("[N/A]", "N/A") else 0.0,
                                     [p == "Active" for p in parts[3:]]))
            except ValueError:
                continue

    def stop(self):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed region"
        if not inside:
            inside = self.samples
            window = "whole run (timed region shorter than the sampling period)"
        if not inside:
            return None
        mhz = [s[1] for s in inside]
        reasons = sorted({self.REASONS[i] for s in inside for i, a in enumerate(s[4]) if a})
        return {"sm_mhz": statistics.median(mhz), "sm_mhz_min": min(mhz),
                "sm_max_mhz": max(s[2] for s in inside), "reasons": reasons,
                "samples": len(inside), "window": window, "source": self.source,
                "power_w_max": round(max(s[3] for s in inside), 1)}


# scales of the E4M3 pools (typical codes have magnitude ~16: keys ~1, values ~0.1)
FP8_K_SCALE = 1.0 / 16
FP8_V_SCALE = 0.0071


def kv_elem_bytes(args):
    return 1 if getattr(args, "kv", "16bit") != "16bit" else None


def algorithmic_bytes(w, args=None):
    kvb = kv_elem_bytes(args)
    return wl.decode_bytes(w, kvb) + wl.append_bytes(w, kvb)


def workload_config(w, args, rotation, partitions):
    cfg = {"workload": w.name, "batch": w.batch, "kv_tokens": int(w.kv_lens.sum()),
           "num_qo_heads": w.num_qo_heads, "num_kv_heads": w.num_kv_heads,
           "head_dim": w.head_dim, "page_size": w.page_size, "pool_pages": w.num_pages,
           "appended_tokens": w.nnz_new, "partitions": partitions,
           "algorithmic_bytes_per_step": algorithmic_bytes(w, args),
           "unique_kv_bytes": wl.kv_cache_bytes(1, w.num_kv_heads, w.head_dim, wl.unique_kv_tokens(w),
                                                kv_elem_bytes(args) or w.elem_bytes),
           "logical_kv_bytes": wl.logical_kv_bytes(w, kv_elem_bytes(args)),
           "l2": (f"inputs larger than L2: {rotation} rotating batch copies of "
                  f"{wl.logical_kv_bytes(w, kv_elem_bytes(args)) / 1e6:.0f} MB K/V each"),
           "parallelism": f"dp{args.gpus} (independent batches per GPU)"}
    if w.note:
        cfg["values"] = w.note
    if getattr(args, "kv", "16bit") != "16bit":
        cfg["kv_cache"] = (f"FP8 {args.kv.upper()} codes, k_scale {FP8_K_SCALE}, v_scale {FP8_V_SCALE}; "
                           f"q / out {w.dtype}; append quantises the new {w.dtype} rows")
    if getattr(args, "cascade", False):
        cfg["method"] = "shared-prefix cascade: prefix attention once per 256 query rows (tcgen05), own pages by the decode kernel, states merged"
    return cfg


# --------------------------------------------------------------------------
# CPU oracle timing (the reported baseline; never tuned)
# --------------------------------------------------------------------------

def head_workload(w, n):
    """The first n requests of a workload (same shapes and value recipe)."""
    prefix = w.shared_prefix_pages * w.page_size
    return wl.make_workload(f"{w.name} [first {n} requests]", w.kv_lens[:n],
                            num_qo_heads=w.num_qo_heads, num_kv_heads=w.num_kv_heads,
                            head_dim=w.head_dim, page_size=w.page_size, dtype=w.dtype,
                            seed=w.seed, pool_factor=1.0, shared_prefix_len=prefix,
                            append_counts=w.append_counts[:n], q_std=w.q_std,
                            key_offset_std=w.key_offset_std, note=w.note)


def time_oracle(w, q_bits, pool_bits):
    import oracle
    t0 = time.perf_counter()
    oracle.decode(q_bits, pool_bits, oracle.BF16 if w.dtype == "bf16" else oracle.F16,
                  w.page_indptr, w.page_indices, w.last_page_len, w.sm_scale)
    return time.perf_counter() - t0


def oracle_sample(w, budget_s):
    """Pick the first n requests so the oracle runs about budget_s; returns
    (workload, q_bits, pool_bits, seconds of one run)."""
    n = 1
    while True:
        ws = head_workload(w, n)
        q, pool, _, _ = wl.make_tensors(ws, "cpu")
        qb, pb = wl.bits(q), wl.bits(pool)
        t = time_oracle(ws, qb, pb)
        if n >= w.batch or t * 1.5 >= budget_s:
            return ws, qb, pb, t
        n = min(w.batch, max(n + 1, int(n * budget_s / max(t, 1e-3) * 0.8)))


def cpu_baseline(w, budget_s):
    import oracle
    ws, qb, pb, t = oracle_sample(w, budget_s)
    kv = wl.kv_cache_bytes(1, ws.num_kv_heads, ws.head_dim, wl.unique_kv_tokens(ws))
    return {"value": round(kv / t / 1e9, 4), "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": (f"fp64 C oracle (OpenMP) on the first {ws.batch} of {w.batch} requests "
                       f"({int(ws.kv_lens.sum())} KV tokens, {kv / 1e6:.1f} MB K/V), {t:.2f} s"),
            "seconds": round(t, 3)}


def run_reference(args):
    """The reference arm: the fp64 CPU oracle, as it stands, on the machine's host
    cores, on a bounded sample of the same workload per step."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    w = wl.named(args.workload)
    per_step = max(0.05, args.ref_seconds / max(1, args.steps + args.warmup))
    ws, qb, pb, _ = oracle_sample(w, per_step)
    for _ in range(args.warmup):
        time_oracle(ws, qb, pb)
    times = [time_oracle(ws, qb, pb) for _ in range(args.steps)]
    total = sum(times)
    kv = wl.kv_cache_bytes(1, ws.num_kv_heads, ws.head_dim, wl.unique_kv_tokens(ws))
    value = kv * args.steps / total / 1e9
    sample = (f"first {ws.batch} of {w.batch} requests per step "
              f"({int(ws.kv_lens.sum())} KV tokens, {kv / 1e6:.1f} MB K/V)")
    cfg = workload_config(w, args, 1, 0)
    cfg["reference_sample"] = sample
    line = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": cfg, "impl": "reference",
            "us_per_step": round(total / args.steps * 1e6, 1),
            "tokens_per_s": round(ws.batch * args.steps / total, 2),
            "cpu_baseline": {"kind": "oracle", "cores": oracle.num_threads(), "sample": sample,
                             "value": round(value, 4), "unit": "GB/s"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
# the GPU arm
# --------------------------------------------------------------------------

def pack(tensors, dev):
    """One pinned host buffer and one device buffer holding `tensors` back to back
    (256-byte aligned); returns ((host_bytes, device_bytes), device views)."""
    offs, total = [], 0
    for t in tensors:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    host = torch.empty(total, dtype=torch.uint8).pin_memory()
    devbuf = torch.empty(total, dtype=torch.uint8, device=dev)
    views = []
    for t, o in zip(tensors, offs):
        n = t.numel() * t.element_size()
        host[o:o + n].copy_(t.contiguous().view(-1).view(torch.uint8))
        views.append(devbuf[o:o + n].view(t.dtype).view(t.shape))
    return (host, devbuf), views


class Batch:
    """One copy of the workload's tensors on the device."""

    def __init__(self, w, dev, value_seed, fp8=None):
        wv = wl.Workload(**{**w.__dict__, "seed": value_seed})
        if fp8:
            self.q, self.pool, self.k_new, self.v_new = wl.make_fp8_tensors(wv, dev, fp8)
        else:
            self.q, self.pool, self.k_new, self.v_new = wl.make_tensors(wv, dev)


def measure_decode(w, args, dev, rank, world, *, cascade=False, fp8=None, e2e=False,
                   clocks=None):
    """Time args.steps decode steps of workload w (after args.warmup untimed
    ones); returns a dict of the measurement.  A step is the append (fused into
    the decode launch on 16-bit pools) and the decode, or the three launches of
    the shared-prefix cascade."""
    import paged_kv_cache_479_b200 as pkv

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    N = args.partitions or pkv.default_partitions(dev.index)
    kvb = 1 if fp8 else None
    kv_bytes = wl.logical_kv_bytes(w, kvb)
    rotation = 2 if kv_bytes < (2 << 30) else 1
    batches = [Batch(w, dev, rank_value_seed(w.seed, rank, r), fp8) for r in range(rotation)]
    t = lambda a: torch.as_tensor(a, device=dev)
    indptr, indices, last = t(w.page_indptr), t(w.page_indices), t(w.last_page_len)
    app = t(w.append_indptr)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    if cascade:
        c_prefix, c_len, c_ip, c_ix, c_ll = wl.cascade_view(w)
        c_prefix, c_ip, c_ix, c_ll = (t(np.ascontiguousarray(x, np.int32)) for x in
                                      (c_prefix, c_ip, c_ix, c_ll))
        ws_bytes = pkv.cascade_workspace_bytes(w.batch, w.num_qo_heads, w.num_kv_heads, c_len,
                                               num_partitions=N)
    else:
        ws_bytes = pkv.decode_workspace_bytes(w.batch, w.num_qo_heads, w.num_kv_heads, 128, N)
    ws = torch.zeros(ws_bytes // 4 + 64, dtype=torch.int32, device=dev)
    out = torch.empty_like(batches[0].q)
    lse = torch.empty((w.batch, w.num_qo_heads), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    # the step's append runs inside the decode launch (pkv_decode_append) unless
    # it cannot (8-bit pool, cascade) or --separate-append asks otherwise
    fused = bool(w.nnz_new) and not fp8 and not cascade and not args.separate_append
    launches_per_step = (3 if cascade else 1) + (1 if w.nnz_new and not fused else 0)
    # nothing in a step writes the page table, so the decode may read it while
    # the previous step's kernel drains (PKV_TABLE_READY_AT_LAUNCH)
    early = not getattr(args, "no_early_table", False)
    table = pkv.csr_table(indptr, indices, last, ready_at_launch=early)

    def append_call(bt):
        if fused:
            return
        if w.nnz_new and fp8:
            pkv.paged_kv_append_fp8(bt.pool, table, bt.k_new, bt.v_new, app, FP8_K_SCALE,
                                    FP8_V_SCALE, error_word=err,
                                    stream=torch.cuda.current_stream(dev), fp8_format=fp8)
        elif w.nnz_new:
            pkv.paged_kv_append(bt.pool, indptr, indices, last, bt.k_new, bt.v_new, app,
                                error_word=err, stream=torch.cuda.current_stream(dev))

    def decode_call(bt):
        cur = torch.cuda.current_stream(dev)
        if fp8:
            pkv.paged_decode_attention_fp8(bt.q, bt.pool, table, ws, FP8_K_SCALE, FP8_V_SCALE,
                                           out=out, lse=lse, sm_scale=w.sm_scale,
                                           num_partitions=N, error_word=err, stream=cur,
                                           fp8_format=fp8)
        elif cascade:
            pkv.cascade_decode(bt.q, bt.pool, c_prefix, c_len, c_ip, c_ix, c_ll, ws, out=out,
                               lse=lse, sm_scale=w.sm_scale, num_partitions=N, error_word=err,
                               stream=cur)
        elif fused:
            pkv.paged_decode_append(bt.q, bt.pool, table, bt.k_new, bt.v_new, app, ws, out=out,
                                    lse=lse, sm_scale=w.sm_scale, num_partitions=N,
                                    error_word=err, stream=cur)
        else:
            pkv.paged_decode_attention_ex(bt.q, bt.pool, table, ws, out=out, lse=lse,
                                          sm_scale=w.sm_scale, num_partitions=N, error_word=err,
                                          stream=cur)

    for i in range(args.warmup):
        append_call(batches[i % rotation])
        decode_call(batches[i % rotation])
    torch.cuda.synchronize()
    if pkv.read_error_word(err) != 0:
        raise RuntimeError("device error bits set during warm-up")

    # The K timed steps go back to back into one CUDA graph (each library call
    # is capturable: no allocation, no sync) replayed once between two events:
    # no event or host work sits between launches, so each launch may start
    # (programmatic dependent launch) while the previous one drains, as in a
    # serving loop.  Per-launch time = the timed region / its launches.
    graphs = []
    K = args.steps

    def steps_fn(n, with_append=True):
        def run():
            for i in range(n):
                if with_append:
                    append_call(batches[i % rotation])
                decode_call(batches[i % rotation])
        if args.no_graph:
            return run
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run()
        graphs.append(g)
        return g.replay

    def timed(fn):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        h0 = time.time()
        start.record(stream)
        fn()
        end.record(stream)
        torch.cuda.synchronize()
        h1 = time.time()
        barrier()
        return max_over_ranks(start.elapsed_time(end), world, dev), h0, h1

    steps_g = steps_fn(K)
    ms, t_host0, t_host1 = timed(steps_g)
    if launches_per_step == 1 or cascade:
        decode_ms = ms / K   # the decode launch (with the fused append), or the cascade's step
    else:
        # the append runs as its own launch: time the decode launches alone too
        decode_ms = timed(steps_fn(K, with_append=False))[0] / K
    if pkv.read_error_word(err) != 0:
        raise RuntimeError("device error bits set during the timed steps")

    step_bytes = algorithmic_bytes(w, args if fp8 else None)
    # the timed launch's algorithmic bytes (with the append when it is fused in)
    dec_bytes = wl.decode_bytes(w, kvb) + (wl.append_bytes(w) if fused else 0)
    res = {"ms": ms, "K": K, "decode_ms": decode_ms, "step_bytes": step_bytes,
           "dec_bytes": dec_bytes, "fused": fused, "launches_per_step": launches_per_step,
           "rotation": rotation, "N": N, "t_host0": t_host0, "t_host1": t_host1, "e2e": None,
           "early_table": early}

    # ---- end to end through the public API with host buffers: every step copies
    # its inputs (q, new K/V rows, the page table) from pinned host memory in one
    # transfer, runs append + decode, and reads out + lse back in one transfer
    if e2e:
        src = batches[0]
        inputs = [src.q.cpu(), src.k_new.cpu(), src.v_new.cpu()] + [
            torch.from_numpy(np.ascontiguousarray(x)) for x in
            (w.page_indptr, w.page_indices, w.last_page_len, w.append_indptr)]
        h_in, d_in = pack(inputs, dev)
        q_d, k_d, v_d, ip_d, ix_d, ll_d, ap_d = d_in
        h_out, d_out = pack([out.cpu(), lse.cpu()], dev)
        out_d, lse_d = d_out
        h2d, d2h = h_in[0].numel(), h_out[0].numel()
        e2e_table = pkv.csr_table(ip_d, ix_d, ll_d, ready_at_launch=early)

        def e2e_calls(_):
            cur = torch.cuda.current_stream(dev)
            h_in[1].copy_(h_in[0], non_blocking=True)
            if fp8:
                if w.nnz_new:
                    pkv.paged_kv_append_fp8(src.pool, e2e_table, k_d, v_d, ap_d, FP8_K_SCALE,
                                            FP8_V_SCALE, error_word=err, stream=cur,
                                            fp8_format=fp8)
                pkv.paged_decode_attention_fp8(q_d, src.pool, e2e_table, ws, FP8_K_SCALE,
                                               FP8_V_SCALE, out=out_d, lse=lse_d,
                                               sm_scale=w.sm_scale, num_partitions=N,
                                               error_word=err, stream=cur, fp8_format=fp8)
            elif fused:
                pkv.paged_decode_append(q_d, src.pool, e2e_table, k_d, v_d, ap_d, ws, out=out_d,
                                        lse=lse_d, sm_scale=w.sm_scale, num_partitions=N,
                                        error_word=err, stream=cur)
            else:
                if w.nnz_new:
                    pkv.paged_kv_append(src.pool, ip_d, ix_d, ll_d, k_d, v_d, ap_d,
                                        error_word=err, stream=cur)
                if cascade:
                    pkv.cascade_decode(q_d, src.pool, c_prefix, c_len, c_ip, c_ix, c_ll, ws,
                                       out=out_d, lse=lse_d, sm_scale=w.sm_scale,
                                       num_partitions=N, error_word=err, stream=cur)
                else:
                    pkv.paged_decode_attention_ex(q_d, src.pool, e2e_table, ws, out=out_d,
                                                  lse=lse_d, sm_scale=w.sm_scale,
                                                  num_partitions=N, error_word=err, stream=cur)
            h_out[0].copy_(h_out[1], non_blocking=True)

        e2e_calls(None)
        torch.cuda.synchronize()
        if args.no_graph:
            e2e_replay = lambda: e2e_calls(None)
        else:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                e2e_calls(None)
            graphs.append(g)
            e2e_replay = g.replay

        def e2e_step():
            e2e_replay()
            stream.synchronize()   # the caller needs the result before the next step

        for _ in range(args.warmup):
            e2e_step()
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        if pkv.read_error_word(err) != 0:
            raise RuntimeError("device error bits set during the end-to-end steps")
        res["e2e"] = {"value": round(job_throughput(step_bytes, world, e_ms, K), 2), "unit": "GB/s",
                      "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                      "us_per_step": round(e_ms / K * 1e3, 2),
                      "path": "pinned host -> device (1 copy), " +
                              ("append fused into the decode launch" if fused else
                               ("append + " if w.nnz_new else "") +
                               ("cascade decode" if cascade else "decode")) +
                              ", device -> pinned host (1 copy), stream sync every step" +
                              ("" if args.no_graph else "; the step's calls replayed as one CUDA graph")}
    del graphs
    return res


def kernel_name(fused, cascade, fp8):
    if cascade:
        return "pkv_cascade_decode (prefix + own-page decode + merge launches)"
    if fp8:
        return f"decode_kernel ({fp8} pool)"
    return "decode_kernel (append fused)" if fused else "decode_kernel"


def per_config_entry(w, args, r, world, peak, cascade, with_cpu):
    """One workload's numbers for the line's per_config object."""
    us = r["ms"] / r["K"] * 1e3
    value = job_throughput(r["step_bytes"], world, r["ms"], r["K"])
    achieved = r["dec_bytes"] / (r["decode_ms"] / 1e3) / 1e9
    e = {"workload": w.name, "method": ("shared-prefix cascade (pkv_cascade_decode)" if cascade
                                        else ("fused append + decode" if r["fused"] else "decode")),
         "us_per_step": round(us, 2), "decode_us": round(r["decode_ms"] * 1e3, 2),
         "kv_gb_s": round(value, 2), "tokens_per_s": round(w.batch * world / (us / 1e6), 1),
         "pct_of_8tbs": round(100 * value / world / NOMINAL_HBM_GBS, 2),
         "frac_of_measured_hbm": round(value / world / peak, 4),
         "decode_launch_gb_s": round(achieved, 1),
         "decode_launch_frac_of_measured_hbm": round(achieved / peak, 4),
         "algorithmic_bytes_per_step": r["step_bytes"],
         "unique_kv_bytes": wl.kv_cache_bytes(1, w.num_kv_heads, w.head_dim,
                                              wl.unique_kv_tokens(w), w.elem_bytes),
         "gpu_launches_per_step": r["launches_per_step"]}
    if with_cpu:
        e["cpu_baseline"] = cpu_baseline(w, args.per_config_cpu_seconds)
    return e


def run_pkv(args):
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                             device_id=dev)

    w = wl.named(args.workload)
    if args.cascade and not w.shared_prefix_pages:
        raise SystemExit("--cascade needs a workload with a shared prefix (workload 5)")
    fp8 = None if args.kv == "16bit" else args.kv
    if fp8 and args.cascade:
        raise SystemExit("--cascade runs on 16-bit pools only")
    peak, peak_kind = measured_hbm()

    clocks = ClockSampler(local)
    r = measure_decode(w, args, dev, rank, world, cascade=args.cascade, fp8=fp8,
                       e2e=not args.no_e2e)
    clock_summary = clocks.summary(r["t_host0"], r["t_host1"])
    K, ms = r["K"], r["ms"]
    value = job_throughput(r["step_bytes"], world, ms, K)
    achieved = r["dec_bytes"] / (r["decode_ms"] / 1e3) / 1e9
    fused = r["fused"]

    # the other named workloads, each the same number of steps, one at a time
    per_config = None
    if not args.no_per_config and not fp8 and not args.cascade and args.workload == 3:
        per_config = {}
        plan = [(1, False), (2, False), (4, False), (5, False), (5, True)]
        for wid, casc in plan:
            wk = wl.named(wid)
            torch.cuda.empty_cache()
            rk = measure_decode(wk, args, dev, rank, world, cascade=casc)
            key = f"{wid}{'_cascade' if casc else ''}"
            per_config[key] = per_config_entry(
                wk, args, rk, world, peak, casc,
                with_cpu=(world == 1 and not args.no_cpu_baseline and not casc))
        torch.cuda.empty_cache()
    clocks.stop()

    if rank == 0:
        traffic = None if (args.cascade or fp8) else recorded_traffic(args.workload)
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": round(ms / K, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": (f"{fp8} KV widened to f16, f32 accumulate" if fp8 else
                      ("bf16" if w.dtype == "bf16" else "f16")), "data": "synthetic",
            "config": {**workload_config(w, args, r["rotation"], r["N"]),
                       "launch": (("the fused append + decode launch (pkv_decode_append)" if fused
                                   else ("the cascade's launches" if args.cascade else
                                         ("append and decode" if w.nnz_new else "decode"))) +
                                  (" of the K steps called back to back" if args.no_graph else
                                   " of the K steps captured back to back in one CUDA graph, "
                                   "replayed once") +
                                  " between two events (nothing between launches: each may "
                                  "start while the previous drains); per launch = the region / "
                                  "its launches" +
                                  ("; page table marked ready at launch (read while the previous "
                                   "step's kernel drains)" if r["early_table"] and not args.cascade
                                   else ""))},
            "us_per_step": round(ms / K * 1e3, 2),
            "tokens_per_s": round(w.batch * world / (ms / 1e3 / K), 1),
            "pct_of_8tbs": round(100 * value / world / NOMINAL_HBM_GBS, 2),
            "pct_of_measured_hbm": round(100 * value / world / peak, 2),
            "roofline": {"bound": "hbm",
                         "kernel": kernel_name(fused, args.cascade, fp8),
                         "achieved": round(achieved, 1),
                         "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "peak_kind": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                         if peak_kind == "measured" else "fallback 6650 GB/s",
                         "traffic": traffic, "algorithmic_bytes_per_launch": r["dec_bytes"],
                         "avg_launch_us": round(r["decode_ms"] * 1e3, 2)},
            "gpu_launches": K * r["launches_per_step"],
            "e2e": r["e2e"],
            "clocks": clock_summary,
        }
        if world == 1 and not args.no_cpu_baseline and not fp8:
            line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
        if per_config is not None:
            line["per_config"] = per_config
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def run_chunk(args):
    """Append K/V of every request's chunk, then the chunk's causal attention."""
    import paged_kv_cache_479_b200 as pkv

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                             device_id=dev)
    w, q_lens = wl.named_chunk(args.chunk)
    qo = wl.chunk_indptr(q_lens)
    rotation = 2
    batches = []
    for r in range(rotation):
        wv = wl.Workload(**{**w.__dict__, "seed": rank_value_seed(w.seed, rank, r)})
        _, pool, k_new, v_new = wl.make_tensors(wv, dev)
        batches.append((wl.make_chunk_queries(wv, q_lens, dev), pool, k_new, v_new))
    t = lambda a: torch.as_tensor(np.ascontiguousarray(a, np.int32), device=dev)
    indptr, indices, last = t(w.page_indptr), t(w.page_indices), t(w.last_page_len)
    app, qo_d = t(w.append_indptr), t(qo)
    table = pkv.csr_table(indptr, indices, last)
    plan_h, S = pkv.append_attention_plan(qo, w.kv_lens, w.num_qo_heads, w.num_kv_heads)
    plan = t(plan_h)
    need = pkv.append_attention_workspace_bytes(int(qo[-1]), w.num_qo_heads, S)
    ws = torch.zeros(need // 4 + 64, dtype=torch.int32, device=dev)
    # chunks of at most 16 / G tokens run on the decode schedule (short path)
    G = w.num_qo_heads // w.num_kv_heads
    mq = int(q_lens.max())
    short = args.chunk_path == "short" or (args.chunk_path == "auto" and mq * G <= 16)
    if short:
        need_s = pkv.append_attention_short_workspace_bytes(w.num_qo_heads, w.num_kv_heads, mq)
        ws_s = torch.zeros(need_s // 4 + 64, dtype=torch.int32, device=dev)
    out = torch.empty_like(batches[0][0])
    lse = torch.empty(out.shape[:2], dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    # the short path can append the chunk's K/V inside its own launch; with 4 rows
    # per (request, kv head) the producer-side writes delay the loads more than a
    # separate append costs, so it is opt-in
    fuse_short = short and args.fused_chunk_append

    def append_call(bt):
        if fuse_short:
            return
        pkv.paged_kv_append(bt[1], indptr, indices, last, bt[2], bt[3], app, error_word=err,
                            stream=torch.cuda.current_stream(dev))

    def attn_call(bt):
        if short:
            fused_rows = dict(k_new=bt[2], v_new=bt[3], append_indptr=app) if fuse_short else {}
            pkv.append_attention_short(bt[0], qo_d, bt[1], table, mq, ws_s, out=out, lse=lse,
                                       sm_scale=w.sm_scale, error_word=err,
                                       stream=torch.cuda.current_stream(dev), **fused_rows)
        else:
            pkv.append_attention(bt[0], qo_d, bt[1], table, plan, S, workspace=ws, out=out,
                                 lse=lse, sm_scale=w.sm_scale, error_word=err,
                                 stream=torch.cuda.current_stream(dev))

    for i in range(args.warmup):
        append_call(batches[i % rotation])
        attn_call(batches[i % rotation])
    torch.cuda.synchronize()
    if pkv.read_error_word(err) != 0:
        raise RuntimeError("device error bits set during warm-up")
    K = args.steps
    graphs = []

    # the K steps back to back in one CUDA graph, replayed once between two
    # events (as in the decode bench); the attention launches alone are timed
    # the same way when the append is a launch of its own
    def steps_fn(n, with_append=True):
        def run():
            for i in range(n):
                if with_append:
                    append_call(batches[i % rotation])
                attn_call(batches[i % rotation])
        if args.no_graph:
            return run
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run()
        graphs.append(g)
        return g.replay

    def timed(fn):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        h0 = time.time()
        start.record(stream)
        fn()
        end.record(stream)
        torch.cuda.synchronize()
        h1 = time.time()
        if world > 1:
            torch.distributed.barrier()
        return max_over_ranks(start.elapsed_time(end), world, dev), h0, h1

    clocks = ClockSampler(local)
    ms, t_host0, t_host1 = timed(steps_fn(K))
    attn_ms = ms / K if fuse_short else timed(steps_fn(K, with_append=False))[0] / K
    clocks.stop()
    del graphs
    if pkv.read_error_word(err) != 0:
        raise RuntimeError("device error bits set during the timed steps")
    flops = wl.chunk_flops(w, q_lens)
    nnz = int(qo[-1])
    kv = wl.kv_cache_bytes(1, w.num_kv_heads, w.head_dim, int(w.kv_lens.sum()))
    attn_bytes = kv + 2 * nnz * w.num_qo_heads * w.head_dim * 2 + 4 * nnz * w.num_qo_heads
    step_bytes = attn_bytes + wl.append_bytes(w)
    if args.chunk == "prefill":
        peak, kind = measured_tensor()
        achieved = flops / (attn_ms / 1e3) / 1e12
        value = flops * world * K / (ms / 1e3) / 1e12
        metric, unit, bound, runit = ("append attention, chunked prefill: causal attention TFLOP/s",
                                      "TFLOP/s", "tensor", "TFLOP/s")
    else:
        peak, kind = measured_hbm()
        launch_bytes = attn_bytes + (wl.append_bytes(w) if fuse_short else 0)
        achieved = launch_bytes / (attn_ms / 1e3) / 1e9
        value = job_throughput(step_bytes, world, ms, K)
        metric, unit, bound, runit = ("append attention, speculative verification: KV HBM GB/s",
                                      "GB/s", "hbm", "GB/s")
    if rank == 0:
        line = {
            "metric": metric, "value": round(value, 2), "unit": unit, "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": round(ms / K, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "query_tokens": nnz,
                       "kv_tokens_after_append": int(w.kv_lens.sum()),
                       "path": ("short chunks on the decode schedule (pkv_append_attention_short)"
                                if short else "tcgen05 row blocks (pkv_append_attention)"),
                       "splits": None if short else S,
                       "row_blocks": None if short else int(plan_h.shape[0]),
                       "flops_per_step": flops,
                       "attention_bytes_per_step": attn_bytes,
                       "l2": f"2 rotating batch copies of {kv / 1e6:.0f} MB K/V",
                       "launch": ("append fused into the attention launch" if fuse_short else
                                  "append and append attention") +
                                 " of the K steps captured back to back in one CUDA graph, "
                                 "replayed once between two events; the attention launches "
                                 "alone timed the same way",
                       "parallelism": f"dp{world} (independent batches per GPU)"},
            "us_per_step": round(ms / K * 1e3, 2),
            "tokens_per_s": round(nnz * world / (ms / K / 1e3), 1),
            "roofline": {"bound": bound,
                         "kernel": ("decode_kernel (short chunks" + (", append fused)" if fuse_short else ")") if short
                                    else "chunk_kernel" + (" + merge" if S > 1 else "")),
                         "achieved": round(achieved, 1), "peak": peak, "unit": runit,
                         "frac": round(achieved / peak, 4),
                         "peak_kind": f"{kind} (MEASURED_PEAKS.json "
                                      f"{'bf16_tflops, burst' if bound == 'tensor' else 'hbm_gbs'})",
                         "traffic": None, "avg_launch_us": round(attn_ms * 1e3, 2)},
            "gpu_launches": K * ((1 if fuse_short else 2) + (1 if S > 1 and not short else 0)),
            "e2e": None,
            "clocks": clocks.summary(t_host0, t_host1),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def main():
    args = parse()
    if args.chunk and args.impl != "reference":
        run_chunk(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_pkv(args)


if __name__ == "__main__":
    main()
