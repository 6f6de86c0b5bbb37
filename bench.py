#!/usr/bin/env python3
"""Paged decode attention benchmark: effective KV HBM GB/s, % of peak, µs/step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 4] [--impl ours|reference]

One step = one decode step of the workload through the run stage (plan made
beforehand, as a serving engine does once per step and reuses across
layers): for the plain workloads one ``pa_run`` launch, for the cascade
``pa_cascade_run``.  Inputs are resident in HBM; L2 is flushed (a 256 MB
write, then a 256 MB read) before every timed step, outside the CUDA events.
``value`` is the algorithmic K/V bytes of all ranks' steps divided by the
max-over-ranks device time.  ``e2e`` repeats the step through the public API
from host buffers: plan on the host, upload of the work list, copies of q
and kv_indices from pinned memory, the run, and the copy of o and lse back.

The default workload is 4 (vector-sparse decode: B 256, GQA 64/8, page size
1, bf16, 4.59 GB of K/V per step), the largest configuration on one GPU.  On
one GPU its run also times, each with the same flush-and-events protocol:
its contiguous page-size-16 twin (``vector_sparse_vs_contiguous``: the
bandwidth ratio), and workloads 1, 2, 3, 5 (decode; for the cascade also its
prefix level), 2f8 and 3f8 (workloads 2 and 3 with 8-bit E4M3 caches), 2rope
(workload 2 with rotary positions applied on the fly) and 6 (prefill /
append) under ``per_config``.

With N > 1 (torchrun) every rank runs its own replica of the workload on
its own GPU (no collective on the data path; the requests of a batch are
independent), so scaling is weak; the extra workloads are skipped.

``--impl reference``: the fp64 CPU oracle timed on the host cores on a
bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode: effective KV HBM GB/s and % of B200 peak; µs per decode step"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_FLUSH_BYTES = 256 << 20
EXTRA_SOAK_S = 0.3          # run-in before each extra workload's timed steps
CPU_BASELINE_SECONDS = 10.0  # target CPU time of the oracle's bounded sample


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="4",
                    help="1 2 3 4 4c 4s 5 (decode), 6 (prefill / append); default: 4, the "
                         "largest single-GPU configuration, whose run also times 4c and "
                         "workloads 1, 2, 3, 5 and 6 as extra keys")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--soak-seconds", type=float, default=1.0,
                    help="untimed run-in after warm-up so clocks settle and get sampled")
    ap.add_argument("--min-chunk-tokens", type=int, default=0,
                    help="split-KV minimum chunk (tokens); 0 = library default")
    ap.add_argument("--ctas-per-sm", type=int, default=0,
                    help="CTA budget per SM for the plan; 0 = occupancy of the kernel")
    ap.add_argument("--kernel", default="auto", choices=["auto", "cuda_cores", "tensor_cores"],
                    help="decode kernel: auto (tensor cores for GQA group 8, CUDA cores for "
                         "1, 2 and 4), cuda_cores or tensor_cores")
    ap.add_argument("--piece-cost-tokens", type=int, default=0,
                    help="plan cost of a piece boundary in tokens; 0 = the kernel's default, "
                         "< 0 = none")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="time only the chosen workload (no contiguous twin, no per_config)")
    return ap.parse_args()


def workload(name):
    from serving_attention_paged_b200 import workloads as W
    key = int(name) if name.isdigit() else name
    return W.WORKLOADS[key]()


def workload_config(w):
    lens = w.kv_lens()
    cfg = {"workload": w.name, "batch": w.batch, "num_qo_heads": w.num_qo_heads,
           "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "page_size": w.page_size,
           "q_dtype": w.dtype, "kv_dtype": w.kv_dtype or w.dtype, "accumulate": "f32",
           "kv_len": (int(lens[0]) if len(set(lens.tolist())) == 1 else
                      {"min": int(lens.min()), "max": int(lens.max()), "sum": int(lens.sum())}),
           "pool_pages": w.num_pages, "kv_bytes_per_step": w.kv_bytes(),
           "l2": "flushed before every timed step: 256 MB write, then a 256 MB read of another "
                 "buffer so the dirty lines are written back before the events (both untimed)"}
    if w.prefix_len:
        cfg["shared_prefix_tokens"] = w.prefix_len
    return cfg


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# the sources each kernel is compiled from (a capture in profiles/ holds only
# while their digest matches)
_CSRC = "serving_attention_paged_b200/csrc/"
KERNEL_SOURCES = {
    "decode_tc": [_CSRC + f for f in ("decode_tc.cu", "common.cuh", "tcgen05.cuh", "launch.cuh")],
    "decode": [_CSRC + f for f in ("decode.cu", "decode_kernel.cuh", "common.cuh", "launch.cuh")],
    "cascade": [_CSRC + f for f in ("cascade.cu", "attn_tile.cuh", "tcgen05.cuh")],
    "prefill": [_CSRC + f for f in ("prefill.cu", "attn_tile.cuh", "tcgen05.cuh", "common.cuh",
                                    "plan.cpp")],
}


def source_digest(files):
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_sources, workload_name):
    """DRAM bytes per launch recorded by an ncu capture in profiles/, if the
    capture's source digest still matches the kernel sources (else None)."""
    digest = source_digest(kernel_sources)
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    for f in sorted(os.listdir(pdir)):
        if not f.endswith(".md"):
            continue
        txt = open(os.path.join(pdir, f)).read()
        m_w = re.search(r"^workload:\s*(\S+)", txt, re.M)
        m_d = re.search(r"^source_digest:\s*(\S+)", txt, re.M)
        m_t = re.search(r"^dram_bytes_per_full_launch:\s*([0-9.eE+]+)", txt, re.M)
        if m_w and m_d and m_t and m_w.group(1) == workload_name and m_d.group(1) == digest:
            return float(m_t.group(1))
    return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid):
        self.uuid = gpu_uuid
        self.proc = None
        self.out = tempfile.TemporaryFile(mode="w+")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.uuid}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.seek(0)
        rows = [r.split(", ") for r in self.out.read().strip().splitlines() if r.strip()]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 8:
                continue
            try:
                sm.append(float(r[0]))
                mx = float(r[1])
            except ValueError:
                continue
            for n, v in zip(names, r[4:8]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(x: float, device) -> float:
    """The largest value of x over all ranks (x itself without a process group)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbs(world: int, bytes_per_rank: int, max_seconds: float) -> float:
    """Whole-job GB/s: every rank processed bytes_per_rank; the slowest rank sets the time."""
    return world * bytes_per_rank / max_seconds / 1e9


def cpu_baseline(w, dev, seconds):
    """The oracle as it stands, on the host cores, over a bounded sample of the
    same workload: whole requests (every q head), in request order, as many as
    fit about ``seconds`` of CPU time (estimated from the first request)."""
    import oracle
    lens = w.kv_lens()
    threads = os.cpu_count() or 1
    indptr, indices, last = w.flat_tables()
    kw = dict(num_qo_heads=w.num_qo_heads, num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
              page_size=w.page_size, dtype=w.dtype, sm_scale=w.sm_scale, threads=threads,
              kv_dtype=w.kv_dtype, k_scale=w.k_scale, v_scale=w.v_scale)

    def run(reqs):
        t0 = time.perf_counter()
        oracle.paged_decode_requests(dev["q"], dev["k_pool"], dev["v_pool"], indptr, indices,
                                     last, reqs, **kw)
        return time.perf_counter() - t0

    t1 = run([0])
    per_token = t1 / max(1, int(lens[0]) + w.prefix_len)
    n, toks = 0, 0
    while n < w.batch and (toks + int(lens[n]) + w.prefix_len) * per_token <= seconds:
        toks += int(lens[n]) + w.prefix_len
        n += 1
    reqs = list(range(max(1, n)))
    dt = run(reqs)
    toks = sum(int(lens[b]) + w.prefix_len for b in reqs)
    nbytes = 2 * toks * w.num_kv_heads * w.head_dim * (1 if w.kv_dtype else 2)
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"the first {len(reqs)} of {w.batch} requests (all {w.num_qo_heads} q "
                      f"heads each), {toks} tokens, {nbytes} KV bytes, {dt:.2f} s, fp64"}


def run_reference(args):
    """Reference arm: the fp64 oracle, timed on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    w = workload(args.workload)
    if w.qo_lens is not None:
        run_reference_prefill(args, w)
        return
    # a bounded sample: the first request(s), drawn on the host
    n_req = 1
    lens = w.kv_lens()
    from serving_attention_paged_b200 import workloads as W
    sub = W.make_workload(w.name, lens[:n_req], num_qo_heads=w.num_qo_heads,
                          num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                          page_size=w.page_size, dtype=w.dtype, seed=w.seed,
                          prefix_len=w.prefix_len, kv_dtype=w.kv_dtype, k_scale=w.k_scale,
                          v_scale=w.v_scale)
    t = sub.materialize()
    indptr, indices, last = sub.flat_tables()
    threads = os.cpu_count() or 1
    kw = dict(num_qo_heads=sub.num_qo_heads, num_kv_heads=sub.num_kv_heads,
              head_dim=sub.head_dim, page_size=sub.page_size, dtype=sub.dtype,
              sm_scale=sub.sm_scale, threads=threads, kv_dtype=sub.kv_dtype,
              k_scale=sub.k_scale, v_scale=sub.v_scale)

    def step():
        oracle.paged_decode(t["q"], t["k_pool"], t["v_pool"], indptr, indices, last, **kw)

    for _ in range(args.warmup):
        step()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        step()
        times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    nbytes = sub.kv_bytes()
    value = nbytes / sec / 1e9
    sample = (f"{n_req} of {w.batch} requests per step (all {w.num_qo_heads} q heads), "
              f"{sub.total_tokens()} tokens, {nbytes} KV bytes, fp64")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}))



def run_reference_prefill(args, w):
    """Reference arm for prefill: the oracle on every 16th new token of the
    first request, drawn on the host."""
    import oracle
    from serving_attention_paged_b200 import workloads as W
    lens = w.kv_lens()
    sub = W.make_workload(w.name, lens[:1], num_qo_heads=w.num_qo_heads,
                          num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                          page_size=w.page_size, dtype=w.dtype, seed=w.seed,
                          qo_lens=w.qo_lens[:1])
    t = sub.materialize()
    sel = np.arange(0, sub.query_rows(), 16)
    threads = os.cpu_count() or 1

    def step():
        oracle.paged_prefill(t["q"], t["k_pool"], t["v_pool"], sub.qo_indptr, sub.kv_indptr,
                             sub.kv_indices, sub.last_page_len, num_qo_heads=sub.num_qo_heads,
                             num_kv_heads=sub.num_kv_heads, head_dim=sub.head_dim,
                             page_size=sub.page_size, dtype=sub.dtype, sm_scale=sub.sm_scale,
                             queries=sel, threads=threads)

    for _ in range(args.warmup):
        step()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        step()
        times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    flops = prefill_query_flops(sub, sel)
    value = flops / sec / 1e12
    sample = (f"every 16th new token of request 0 ({len(sel)} of {w.query_rows()} tokens, all "
              f"{w.num_qo_heads} q heads), {flops / 1e9:.2f} GFLOP per step, fp64")
    print(json.dumps({
        "impl": "reference", "metric": PREFILL_METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name, "batch": w.batch,
                                        "num_qo_heads": w.num_qo_heads,
                                        "num_kv_heads": w.num_kv_heads, "causal": True},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}))

def make_l2_flush(dev_t):
    """A 256 MB write, then a 256 MB read of another buffer so the dirty lines
    of that write are written back too (both outside the timed events)."""
    import torch
    flush_w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev_t)
    flush_r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev_t)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev_t)

    def flush_l2():
        flush_w.fill_(1.0)                       # evicts the inputs ...
        torch.sum(flush_r, dim=0, out=flush_sink)  # ... and the dirty lines of that write

    return flush_l2


def timed_steps(step, flush_l2, args, stream, dev_t, world, soak_seconds):
    """W warm-up steps, an untimed soak while the clocks are sampled, then K
    steps each bracketed by CUDA events on the launching stream (L2 flushed
    before each, outside the events).  Returns the max-over-ranks mean step
    time (ms), this rank's step times and the clock record."""
    import torch
    import torch.distributed as dist
    for _ in range(max(args.warmup, 3)):
        flush_l2()
        step()
    torch.cuda.synchronize()

    uuid = str(torch.cuda.get_device_properties(dev_t).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    sampler.start()
    t_end = time.perf_counter() + soak_seconds
    while time.perf_counter() < t_end:
        for _ in range(20):
            flush_l2()
            step()
        torch.cuda.synchronize()

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed")
    for i in range(args.steps):
        flush_l2()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    step_ms = [st.elapsed_time(en) for st, en in zip(starts, ends)]
    ms = max_over_ranks(sum(step_ms) / len(step_ms), dev_t)
    return ms, step_ms, clocks


PREFILL_METRIC = ("paged prefill / append (causal): attention TFLOP/s and % of B200 dense "
                  "tensor peak; µs per step")


def measured_tensor_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        return float(json.load(open(path))["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def prefill_cpu_baseline(w, dev, stride):
    """The oracle as it stands, on the host cores, over every ``stride``-th new
    token of the workload (all q heads)."""
    import oracle
    threads = os.cpu_count() or 1
    sel = np.arange(0, w.query_rows(), stride)
    t0 = time.perf_counter()
    oracle.paged_prefill(dev["q"], dev["k_pool"], dev["v_pool"], w.qo_indptr, w.kv_indptr,
                         w.kv_indices, w.last_page_len, num_qo_heads=w.num_qo_heads,
                         num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                         page_size=w.page_size, dtype=w.dtype, sm_scale=w.sm_scale,
                         queries=sel, threads=threads)
    dt = time.perf_counter() - t0
    flops = prefill_query_flops(w, sel)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"every {stride}th new token ({len(sel)} of {w.query_rows()}, all "
                      f"{w.num_qo_heads} q heads), {flops / 1e9:.2f} GFLOP, {dt:.2f} s, fp64"}


def prefill_query_flops(w, queries):
    """Attention flops of the listed new tokens (4 per visible key and element)."""
    qo, lens = w.qo_indptr, w.kv_lens()
    b = np.searchsorted(qo, queries, side="right") - 1
    i = queries - qo[b]
    visible = lens[b] - (qo[b + 1] - qo[b]) + i + 1
    return int(4 * visible.sum() * w.num_qo_heads * w.head_dim)


def prefill_timing(args, w, dev, stream, dev_t, world, flush_l2):
    """The prefill / append workload as a per-config entry: µs per step and
    causal attention TFLOP/s against the measured dense tensor peak."""
    from serving_attention_paged_b200.wrapper import PagedPrefill
    pf = PagedPrefill(w.qo_indptr, w.kv_indptr, w.last_page_len, num_qo_heads=w.num_qo_heads,
                      num_kv_heads=w.num_kv_heads, page_size=w.page_size, dtype=w.dtype,
                      sm_scale=w.sm_scale, num_pages=w.num_pages, causal=True, device=dev_t)
    o, lse = pf.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"])

    def step():
        pf.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"], o, lse, stream=stream)

    ms, step_ms, clocks = timed_steps(step, flush_l2, args, stream, dev_t, world,
                                      soak_seconds=EXTRA_SOAK_S)
    flops = w.prefill_flops()
    tf = flops / (ms * 1e-3) / 1e12
    peak, peak_kind = measured_tensor_peak()
    return {"workload": w.name, **step_stats(step_ms), "flops_per_step": flops,
            "tflop_s": round(tf, 1), "pct_of_tensor_peak": round(100.0 * tf / peak, 2),
            "tensor_peak_kind": peak_kind, "kernel": "paged_prefill_kernel",
            "sm_mhz": clocks["sm_mhz"], "clock_reasons": clocks["reasons"]}, ms


def run_prefill(args, w, dev, stream, dev_t, world, rank):
    """Prefill / append step: one pa_prefill_run launch over all new tokens."""
    import torch
    from serving_attention_paged_b200 import pagedattn as C
    from serving_attention_paged_b200.wrapper import PagedPrefill
    t0 = time.perf_counter()
    pf = PagedPrefill(w.qo_indptr, w.kv_indptr, w.last_page_len, num_qo_heads=w.num_qo_heads,
                      num_kv_heads=w.num_kv_heads, page_size=w.page_size, dtype=w.dtype,
                      sm_scale=w.sm_scale, num_pages=w.num_pages, causal=True, device=dev_t)
    setup_us = (time.perf_counter() - t0) * 1e6
    reps = 20
    t0 = time.perf_counter()
    for _ in range(reps):
        C.pa_prefill_plan_create(pf.problem, True, w.qo_indptr, w.kv_indptr, w.last_page_len)
    plan_us = (time.perf_counter() - t0) * 1e6 / reps
    o, lse = pf.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"])

    def step():
        pf.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"], o, lse, stream=stream)

    flush_l2 = make_l2_flush(dev_t)
    ms, step_ms, clocks = timed_steps(step, flush_l2, args, stream, dev_t, world,
                                      soak_seconds=args.soak_seconds)
    flops = w.prefill_flops()
    value = world * flops / (ms * 1e-3) / 1e12
    achieved = flops / (ms * 1e-3) / 1e12
    peak, peak_kind = measured_tensor_peak()
    traffic = profiled_traffic(KERNEL_SOURCES["prefill"], w.name)

    e2e = None
    if not args.no_e2e:
        q_h = dev["q"].cpu().pin_memory()
        idx_h = dev["kv_indices"].cpu().pin_memory()
        o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        lse_h = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        q_d = torch.empty_like(dev["q"])
        idx_d = torch.empty_like(dev["kv_indices"])
        e2e_s = []
        for i in range(max(args.warmup, 3) + args.steps):
            flush_l2()
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            plan = C.pa_prefill_plan_create(pf.problem, True, w.qo_indptr, w.kv_indptr,
                                            w.last_page_len)
            C.pa_plan_upload(plan, pf.workspace, pf.workspace.numel(), stream)
            q_d.copy_(q_h, non_blocking=True)
            idx_d.copy_(idx_h, non_blocking=True)
            C.pa_prefill_run(plan, q_d, dev["k_pool"], dev["v_pool"], idx_d, o, lse,
                             pf.workspace, pf.workspace.numel(), stream)
            o_h.copy_(o, non_blocking=True)
            lse_h.copy_(lse, non_blocking=True)
            torch.cuda.synchronize()
            if i >= max(args.warmup, 3):
                e2e_s.append(time.perf_counter() - t0)
        e2e_max = max_over_ranks(sum(e2e_s) / len(e2e_s), dev_t)
        h2d = q_h.numel() * q_h.element_size() + idx_h.numel() * 4 + len(pf.tiles()) * 24
        e2e = {"value": world * flops / e2e_max / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(o_h.numel() * o_h.element_size() + lse_h.numel() * 4),
               "us_per_step": e2e_max * 1e6,
               "includes": "host plan + tile upload + q/kv_indices H2D + run + o/lse D2H"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = prefill_cpu_baseline(w, dev, stride=8)

    if rank == 0:
        lens = w.kv_lens()
        cfg = {"workload": w.name, "batch": w.batch, "num_qo_heads": w.num_qo_heads,
               "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim,
               "page_size": w.page_size, "kv_dtype": w.dtype, "accumulate": "f32",
               "kv_len": int(lens[0]) if len(set(lens.tolist())) == 1 else int(lens.sum()),
               "qo_len": int(w.qo_lens[0]) if len(set(w.qo_lens.tolist())) == 1
               else int(w.qo_lens.sum()),
               "causal": True, "flops_per_step": flops, "pool_pages": w.num_pages,
               "l2": "flushed before every timed step: 256 MB write, then a 256 MB read of "
                     "another buffer (both untimed)",
               "parallelism": f"replicas x{world}"}
        print(json.dumps({
            "metric": PREFILL_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "us_per_step": ms * 1e3, "pct_of_peak": 100.0 * achieved / peak,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic (seeded splitmix64 + Box-Muller, N(0,1))",
            "config": cfg,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak,
                         "peak_kind": peak_kind + " (bf16 cuBLAS burst; fp16 has the same "
                                                  "nominal dense rate)",
                         "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                         "kernel": "paged_prefill_kernel"},
            "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks, "gpu_launches": args.steps,
            "plan_us": plan_us, "setup_us": setup_us,
            "step_ms_p10_p50_p90": [float(np.percentile(step_ms, p)) for p in (10, 50, 90)],
        }))


def make_decode(w, args, dev_t, C, rope_theta=0.0):
    """Plan (and workspace) for a decode workload, in the bench's launch configuration."""
    from serving_attention_paged_b200.wrapper import PagedDecode
    return PagedDecode(w.kv_indptr, w.last_page_len, num_qo_heads=w.num_qo_heads,
                       num_kv_heads=w.num_kv_heads, page_size=w.page_size, dtype=w.dtype,
                       sm_scale=w.sm_scale, num_pages=w.num_pages, prefix_len=w.prefix_len,
                       device=dev_t, min_chunk_tokens=args.min_chunk_tokens,
                       ctas_per_sm=args.ctas_per_sm or None,
                       flags={"auto": 0, "cuda_cores": C.PA_FLAG_CUDA_CORES,
                              "tensor_cores": C.PA_FLAG_TENSOR_CORES}[args.kernel],
                       piece_cost_tokens=args.piece_cost_tokens, kv_dtype=w.kv_dtype,
                       k_scale=w.k_scale, v_scale=w.v_scale, rope_theta=rope_theta)


def step_stats(step_ms):
    return {"us_p10_p50_p90": [round(float(np.percentile(step_ms, p)) * 1e3, 2)
                               for p in (10, 50, 90)],
            "us_mean": round(sum(step_ms) / len(step_ms) * 1e3, 2)}


def decode_kernel_name(C, pd):
    return "paged_decode_tc_kernel" if C.pa_plan_uses_tensor_cores(pd.plan) else \
        "paged_decode_kernel"


def extra_decode(key, args, dev_t, stream, flush_l2, peak, C, rope_theta=0.0):
    """One more decode workload, timed like the headline (1 GPU, own clocks):
    µs per step, effective GB/s and % of the HBM peak."""
    import torch
    w = workload(key)
    dev = w.materialize(dev_t)
    pd = make_decode(w, args, dev_t, C, rope_theta)
    o, lse = pd.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"],
                    prefix_indices=dev.get("prefix_indices"))

    def step():
        pd.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"], o, lse,
               prefix_indices=dev.get("prefix_indices"), stream=stream)

    ms, step_ms, clocks = timed_steps(step, flush_l2, args, stream, dev_t, 1,
                                      soak_seconds=EXTRA_SOAK_S)
    nbytes = w.kv_bytes()
    gbs = nbytes / (ms * 1e-3) / 1e9
    entry = {"workload": w.name, **step_stats(step_ms), "gb_s": round(gbs, 1),
             "pct_of_peak": round(100.0 * gbs / peak, 2), "kv_bytes_per_step": nbytes,
             "kernel": decode_kernel_name(C, pd), "sm_mhz": clocks["sm_mhz"],
             "clock_reasons": clocks["reasons"]}
    if w.kv_dtype:
        entry["kv_cache"] = {"format": w.kv_dtype, "k_scale": w.k_scale, "v_scale": w.v_scale,
                             "bytes_per_element": 1}
    if rope_theta:
        entry["rope_theta"] = rope_theta
    if w.prefix_len:
        # the prefix level with a near-empty second level: the same cascade with
        # every suffix cut to its first token (the decode level then reads one
        # token per request and merges the prefix chunks of each row)
        one_indptr = np.arange(w.batch + 1, dtype=np.int32)
        one_last = np.ones(w.batch, dtype=np.int32)
        first_pages = dev["kv_indices"][torch.from_numpy(w.kv_indptr[:-1].astype(np.int64))
                                        .to(dev_t)].contiguous()
        from serving_attention_paged_b200.wrapper import PagedDecode
        pp = PagedDecode(one_indptr, one_last, num_qo_heads=w.num_qo_heads,
                         num_kv_heads=w.num_kv_heads, page_size=w.page_size, dtype=w.dtype,
                         sm_scale=w.sm_scale, num_pages=w.num_pages, prefix_len=w.prefix_len,
                         device=dev_t)

        def prefix_step():
            pp.run(dev["q"], dev["k_pool"], dev["v_pool"], first_pages, o, lse,
                   prefix_indices=dev["prefix_indices"], stream=stream)

        pms, pstep_ms, _ = timed_steps(prefix_step, flush_l2, args, stream, dev_t, 1,
                                       soak_seconds=0.0)
        flops = 4 * w.batch * w.num_qo_heads * w.prefix_len * w.head_dim
        tpeak, tkind = measured_tensor_peak()
        tf = flops / (pms * 1e-3) / 1e12
        entry["prefix_level"] = {
            **step_stats(pstep_ms), "flops_per_step": flops, "tflop_s": round(tf, 1),
            "pct_of_tensor_peak": round(100.0 * tf / tpeak, 2), "tensor_peak_kind": tkind,
            "includes": "cascade_prefix_kernel + a decode launch over one suffix token per "
                        "request that merges the prefix chunks of every row"}
    del dev, o, lse
    torch.cuda.empty_cache()
    return w, entry, ms


def launch_floor(args, dev_t, stream, flush_l2):
    """Event-timed cost of one near-empty kernel in the bench's timing pattern
    (L2 flush, start event, one kernel, end event): the fixed per-step floor."""
    import torch
    x = torch.zeros(1, device=dev_t)

    def step():
        x.add_(1.0)

    ms, step_ms, _ = timed_steps(step, flush_l2, args, stream, dev_t, 1, soak_seconds=0.0)
    return step_stats(step_ms)


def read_floor(args, dev_t, stream, flush_l2, nbytes):
    """Event-timed cost of reading `nbytes` from HBM with one library reduction
    (torch.sum over an fp16 buffer of that size) in the bench's timing pattern:
    what streaming a single-request step's bytes costs at all, as a reference
    for that step's time."""
    import torch
    buf = torch.ones(nbytes // 2, dtype=torch.float16, device=dev_t)
    out = torch.empty((), dtype=torch.float32, device=dev_t)

    def step():
        torch.sum(buf, dim=0, dtype=torch.float32, out=out)

    ms, step_ms, _ = timed_steps(step, flush_l2, args, stream, dev_t, 1, soak_seconds=0.0)
    del buf
    return step_stats(step_ms)


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev_t = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev_t,
                                timeout=datetime.timedelta(seconds=120))

    from serving_attention_paged_b200 import build
    if rank == 0 or world == 1:
        build.build()
    if world > 1:
        dist.barrier()
    from serving_attention_paged_b200 import pagedattn as C

    w = workload(args.workload)
    dev = w.materialize(dev_t)
    stream = torch.cuda.current_stream(dev_t)
    if w.qo_lens is not None:
        run_prefill(args, w, dev, stream, dev_t, world, rank)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return
    t0 = time.perf_counter()
    pd = make_decode(w, args, dev_t, C)
    tensor_cores = C.pa_plan_uses_tensor_cores(pd.plan)
    setup_us = (time.perf_counter() - t0) * 1e6
    reps = 20
    t0 = time.perf_counter()
    for _ in range(reps):
        (C.pa_cascade_plan_create(pd.problem, w.prefix_len, w.kv_indptr, w.last_page_len)
         if w.prefix_len else C.pa_plan_create(pd.problem, w.kv_indptr, w.last_page_len))
    plan_us = (time.perf_counter() - t0) * 1e6 / reps
    o, lse = pd.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"],
                    prefix_indices=dev.get("prefix_indices"))
    launches_per_step = 2 if (w.prefix_len and w.batch) else 1

    def step():
        pd.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["kv_indices"], o, lse,
               prefix_indices=dev.get("prefix_indices"), stream=stream)

    flush_l2 = make_l2_flush(dev_t)
    ms, step_ms, clocks = timed_steps(step, flush_l2, args, stream, dev_t, world,
                                      soak_seconds=args.soak_seconds)

    nbytes = w.kv_bytes()
    value = aggregate_gbs(world, nbytes, ms * 1e-3)
    peak, peak_kind = measured_peak()
    achieved = nbytes / (ms * 1e-3) / 1e9  # one GPU's launch: the dominant (only) kernel
    decode_kernel = "paged_decode_tc_kernel" if tensor_cores else "paged_decode_kernel"
    kernel_sources = list(KERNEL_SOURCES["decode_tc" if tensor_cores else "decode"])
    if w.prefix_len:
        kernel_sources += KERNEL_SOURCES["cascade"]
    traffic = profiled_traffic(kernel_sources, w.name)

    # end to end through the public API from host buffers
    e2e = None
    if not args.no_e2e:
        q_h = dev["q"].cpu().pin_memory()
        idx_h = dev["kv_indices"].cpu().pin_memory()
        o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        lse_h = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        q_d = torch.empty_like(dev["q"])
        idx_d = torch.empty_like(dev["kv_indices"])
        e2e_s = []
        for i in range(max(args.warmup, 3) + args.steps):
            flush_l2()
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            plan = C.pa_cascade_plan_create(pd.problem, w.prefix_len, w.kv_indptr,
                                            w.last_page_len) if w.prefix_len else \
                C.pa_plan_create(pd.problem, w.kv_indptr, w.last_page_len)
            C.pa_plan_upload(plan, pd.workspace, pd.workspace.numel(), stream)
            q_d.copy_(q_h, non_blocking=True)
            idx_d.copy_(idx_h, non_blocking=True)
            if w.prefix_len:
                C.pa_cascade_run(plan, q_d, dev["k_pool"], dev["v_pool"], dev["prefix_indices"],
                                 idx_d, o, lse, pd.workspace, pd.workspace.numel(), stream)
            else:
                C.pa_run(plan, q_d, dev["k_pool"], dev["v_pool"], idx_d, o, lse, pd.workspace,
                         pd.workspace.numel(), stream)
            o_h.copy_(o, non_blocking=True)
            lse_h.copy_(lse, non_blocking=True)
            torch.cuda.synchronize()
            if i >= max(args.warmup, 3):
                e2e_s.append(time.perf_counter() - t0)
        e2e_max = max_over_ranks(sum(e2e_s) / len(e2e_s), dev_t)
        items = len(pd.work_items())
        n_cta = len(C.pa_plan_cta_indptr(pd.plan)) - 1
        h2d = (q_h.numel() * q_h.element_size() + idx_h.numel() * 4 + items * 24 +
               (n_cta + 1) * 4 + (w.batch * w.num_kv_heads + 1) * 4)
        e2e = {"value": aggregate_gbs(world, nbytes, e2e_max), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(o_h.numel() * o_h.element_size() + lse_h.numel() * 4),
               "us_per_step": e2e_max * 1e6,
               "includes": "host plan + work-list upload + q/kv_indices H2D + run + o/lse D2H"}
        del q_h, idx_h, o_h, lse_h, q_d, idx_d

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, dev, CPU_BASELINE_SECONDS)

    # Every other configuration, timed the same way on this GPU (1 GPU only:
    # they characterise the kernels; the headline above is the job's number).
    extras = {}
    if world == 1 and not args.headline_only and w.name == "vector_sparse_decode":
        del dev, o, lse
        torch.cuda.empty_cache()
        tw, twin, _ = extra_decode("4c", args, dev_t, stream, flush_l2, peak, C)
        extras["vector_sparse_vs_contiguous"] = {
            "ratio": round(value / twin["gb_s"], 4), "target": 0.85,
            "page_size_1_gb_s": round(value, 1), "contiguous": twin}
        per = {}
        for key in (1, 2, 3, 5):
            kw, entry, _ = extra_decode(str(key), args, dev_t, stream, flush_l2, peak, C)
            per[str(key)] = entry
        # 8-bit (E4M3) caches of workloads 2 and 3: GB/s on the halved bytes
        for key in ("2f8", "3f8"):
            _, entry, _ = extra_decode(key, args, dev_t, stream, flush_l2, peak, C)
            per[key] = entry
        # rotary positions on the fly, workload 2: the cost against plain decode
        _, rope, _ = extra_decode("2", args, dev_t, stream, flush_l2, peak, C, rope_theta=1e4)
        rope["time_vs_plain"] = round(rope["us_mean"] / per["2"]["us_mean"], 3)
        per["2rope"] = rope
        per["1"]["launch_floor"] = launch_floor(args, dev_t, stream, flush_l2)
        per["1"]["launch_floor"]["what"] = (
            "the same timing pattern (flush, start event, one 1-element torch kernel, end "
            "event): the fixed cost every event-timed step carries")
        w1_bytes = workload("1").kv_bytes()
        per["1"]["read_floor"] = read_floor(args, dev_t, stream, flush_l2, w1_bytes)
        per["1"]["read_floor"]["what"] = (
            f"the same timing pattern around torch.sum over {w1_bytes} bytes of fp16 (one "
            "library reduction reading the step's byte count from HBM)")
        pw = workload("6")
        pdev = pw.materialize(dev_t)
        per["6"] = prefill_timing(args, pw, pdev, stream, dev_t, 1, flush_l2)[0]
        del pdev
        torch.cuda.empty_cache()
        extras["per_config"] = per

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "us_per_step": ms * 1e3, "pct_of_peak": 100.0 * achieved / peak,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.kv_dtype or w.dtype,
            "data": "synthetic (seeded splitmix64 + Box-Muller, N(0,1))",
            "config": dict(workload_config(w), parallelism=f"replicas x{world}"),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": traffic,
                         "kernel": decode_kernel if not w.prefix_len
                         else f"cascade step (prefix kernel + {decode_kernel})"},
            "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
            "gpu_launches": args.steps * launches_per_step,
            "plan_us": plan_us, "setup_us": setup_us,
            "step_ms_p10_p50_p90": [float(np.percentile(step_ms, p)) for p in (10, 50, 90)],
            **extras,
        }
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
