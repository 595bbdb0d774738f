"""Benchmark of attention over a KV cache on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: GQA split-K decode -- 16 sequences x 1 query row, 32 query heads over
8 KV heads, head_dim 128, bf16 KV cache [16 x 8192 cells, 8, 128] with
per-sequence lengths uniform in [1024, 8192] (seed 1002), bf16 output, slice
count from the planner.  One step = one attn_decode call (the balanced
stream kernel + split_k_reduce) over one batch.  The metric is attention GB/s: the algorithmic
bytes of a step (K and V rows of every visible cell, Q and the output) over
the step time, with the HBM roofline of the dominant kernel beside it.

Timing: W untimed warm-up steps, then K steps between a barrier and a device
synchronize, timed with CUDA events on the launching stream, max over ranks.
Each step reads a different one of three resident input sets (~0.9 GB of K/V
in all), so a step never finds the previous step's cache in L2 (126 MB).

The line's "parts" object times the other two operations on their own
workloads, per call with the L2 flushed before each call: maskless
selected-key attention (2048 rows, GQA 12, D 256, fp16 cache of 32768 cells;
effective GB/s of the gathered K/V rows) and causal prefill (2048 rows over
14048 cells, Hq 64 / Hkv 8, D 128, bf16; TFLOP/s over the visible pairs on
the tensor cores), draft-tree decode rows (tree mask + attn_decode), the
decode batch over an e4m3 cache with per (cell, KV head) scales (GB/s of the
visible codes and scales, Q and out), and the unified-cache semantics sweep through attn_decode and attn_prefill (GB/s of the
visible K/V rows, mask rows and cell metadata), each with the roofline of its
main kernel.
--profile-op {decode,selected,prefill,semantics} only runs W + K calls of one operation
(the command the ncu summaries under profiles/ are taken on).

--impl reference times the FP64 CPU oracle on the host cores on a bounded
sample of the same workload (the pages ship no code; the oracle is the
baseline arm).  Under torchrun every rank runs its own batch (weak scaling;
the path has no collective); only a scalar max of the step time crosses ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import attention_split_attn_b200 as A                      # noqa: E402
from attention_split_attn_b200 import workloads as W       # noqa: E402

METRIC = "attention GB/s (decode, % HBM peak); prefill TFLOP/s (% bf16 tensor peak)"
WORKLOAD = "gqa_decode: 16 seq x 1 row, Hq 32 / Hkv 8, D 128, bf16 KV, len U[1024,8192], bf16 out"
N_SETS = 3


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws == 1:
        return 0, 1, 0
    import torch.distributed as dist
    import datetime
    rank, local = int(os.environ["RANK"]), int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", local))
    return rank, ws, local


def _max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


class Clocks:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def algorithmic_bytes(p) -> int:
    """K and V rows of every visible cell for its KV head, plus Q and out."""
    lens = (p.row_end - p.row_begin).to(torch.int64)
    kv = int(lens.sum()) * p.n_head_kv * p.head_dim * p.k.element_size() * 2
    q = p.q.numel() * p.q.element_size()
    o = p.n_rows * p.n_head_q * p.head_dim * torch.empty((), dtype=p.out_dtype).element_size()
    return kv + q + o


def run_reference(args, rank, world):
    """The FP64 oracle on the host cores, on a bounded sample of the workload."""
    if rank != 0:
        return
    import oracle
    p = W.gqa_decode(poison_unused=False)
    rows = [0, 1]                       # a bounded sample: 2 of the 16 rows
    sub = p.row_subset(rows)
    bytes_per_step = algorithmic_bytes(sub)
    cores = os.cpu_count() or 1
    prep = oracle.Prepared(sub)
    for _ in range(max(0, args.warmup)):
        prep.run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        prep.run()
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    gbs = bytes_per_step / dt / 1e9
    line = {"metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": WORKLOAD, "sample": "rows 0-1 of 16", "parallelism": "host threads"},
            "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": min(cores, len(rows)),
                             "kind": "oracle", "sample": "rows 0-1 of the 16-row batch (one thread per row)"},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def cpu_baseline():
    """Oracle throughput on the host cores over the whole 16-row batch, repeated
    for about 10 s."""
    import oracle
    p = W.gqa_decode(poison_unused=False)
    nbytes = algorithmic_bytes(p)
    cores = os.cpu_count() or 1
    prep = oracle.Prepared(p)
    prep.run(n_threads=cores)
    t0, n = time.perf_counter(), 0
    while True:
        prep.run(n_threads=cores)
        n += 1
        if time.perf_counter() - t0 > 10.0:
            break
    dt = (time.perf_counter() - t0) / n
    # one thread, rows 0-1 (the 1-thread figure)
    rate1, _, n1 = _oracle_rate(p, [0, 1], algorithmic_bytes, budget_s=2.0, threads=1)
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": min(cores, p.n_rows), "kind": "oracle",
            "sample": f"the full 16-row batch, {n} repetitions (~10 s), one thread per row",
            "value_1thread": rate1 / 1e9, "sample_1thread": f"rows 0-1 on one thread, {n1} repetitions (~2 s)"}


def _oracle_rate(p, rows, amount_fn, budget_s=2.0, threads=0):
    """The FP64 oracle as it stands on rows `rows` of problem p, repeated for
    about budget_s on the host cores (one thread per row, or `threads`);
    returns (amount_fn(rows) per second, threads used, repetitions)."""
    import oracle
    sub = p.row_subset(rows)
    prep = oracle.Prepared(sub)
    n_thr = threads or min(os.cpu_count() or 1, len(rows))
    prep.run(n_threads=n_thr)
    t0, n = time.perf_counter(), 0
    while True:
        prep.run(n_threads=n_thr)
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = (time.perf_counter() - t0) / n
    return amount_fn(sub) / dt, n_thr, n


def _part_baseline(p, rows, amount_fn, unit, scale, what):
    rate, thr, n = _oracle_rate(p, rows, amount_fn)
    return {"value": rate / scale, "unit": unit, "cores": thr, "kind": "oracle",
            "sample": f"{what}, {n} repetitions (~2 s)"}


def run_ours(args, rank, world, local):
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    A.load_library()
    hbm_peak, _, peak_kind = _peaks()

    # three resident input sets of the same shape (different seeds per set and rank)
    sets = []
    for i in range(N_SETS):
        p = W.gqa_decode(seed=1002 + 7919 * rank + 104729 * i, poison_unused=False)
        (q, k, v, out), kw = A.problem_kwargs(p, device=dev)
        a = A.make_args(q, k, v, out, **kw)
        ws = torch.empty(max(A.workspace_size(a, A.OP_DECODE), 256), dtype=torch.uint8, device=dev)
        sets.append(dict(p=p, args=a, ws=ws, keep=(q, k, v, out, kw), bytes=algorithmic_bytes(p)))
    S = A.workspace_size(sets[0]["args"], A.OP_DECODE)   # nonzero -> split
    launches_per_step = 2 if S > 0 else 1

    # a quick parity spot check outside the timed region (2 rows vs the oracle)
    if rank == 0:
        import oracle
        A.attn_decode_args(sets[0]["args"], ws=sets[0]["ws"])
        torch.cuda.synchronize()
        out = sets[0]["keep"][3][:2].double().cpu().numpy()
        ref = oracle.attn(sets[0]["p"].row_subset([0, 1]))
        nmse = float(((out - ref) ** 2).sum() / (ref ** 2).sum())
        assert nmse < 1e-5, f"parity spot check failed: NMSE {nmse}"

    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        st = sets[i % N_SETS]
        A.attn_decode_args(st["args"], ws=st["ws"])
    torch.cuda.synchronize()

    # the timed region: K whole steps, only a start and an end event
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    total_bytes = 0
    with Clocks(local) as clk:
        _barrier(world)
        torch.cuda.synchronize()
        t_start.record(stream)
        for i in range(args.steps):
            st = sets[i % N_SETS]
            A.attn_decode_args(st["args"], ws=st["ws"], stream=stream)
            total_bytes += st["bytes"]
        t_end.record(stream)
        torch.cuda.synchronize()
        _barrier(world)
    elapsed_ms = t_start.elapsed_time(t_end)
    elapsed_ms = _max_over_ranks(elapsed_ms, world)
    step_bytes = total_bytes / args.steps
    value = step_bytes * world * args.steps / (elapsed_ms * 1e-3) / 1e9

    # the dominant kernel, timed live on the launching stream: the same K steps
    # again through the timing hook (an event right after the main kernel; the
    # hook turns off the overlap of the combine with it, so it is a separate pass)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for e in (x for row in ev for x in row):
        e.record(stream)          # torch creates the handle on first record; the library re-records it
    torch.cuda.synchronize()
    for i in range(args.steps):
        st = sets[i % N_SETS]
        A.attn_decode_timed_args(st["args"], st["ws"], ev[i], stream=stream)
    torch.cuda.synchronize()
    main_ms = [e[0].elapsed_time(e[1]) for e in ev]
    kmean_ms = sum(main_ms) / len(main_ms)
    achieved = step_bytes / (kmean_ms * 1e-3) / 1e9
    traffic = _recorded_traffic("gqa_decode")

    e2e = run_e2e(args, sets, stream)
    with_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    parts = None if args.no_parts else run_parts(args, rank, dev, stream, with_cpu)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "rows_per_step": 16 * world, "slices": "planner",
                   "l2": "3 rotating input sets, each step's K/V (302 MB) larger than L2",
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"},
        "rows_per_s": 16 * world * args.steps / (elapsed_ms * 1e-3),
        "frac_of_hbm_peak": value / world / hbm_peak,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": traffic,
                     "kernel": "decode_stream_kernel + combine_kernel (balanced split-K; the stream kernel computes the row tile prefix)",
                     "kernel_ms": kmean_ms, "peak_kind": f"{peak_kind} hbm_gbs (burst copy)"},
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if parts is not None:
        line["parts"] = parts
        line["gpu_launches"] += sum(p_["gpu_launches"] for p_ in parts.values())
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    # one compact entry per workload, last on the line
    summ = {"gqa_decode": f"{value:.0f} GB/s whole step, kernel {achieved:.0f} GB/s = {achieved / hbm_peak:.3f} of HBM"}
    for name, pt in (parts or {}).items():
        r = pt.get("roofline")
        s_ = f"{pt['value']:.4g} {pt['unit'].split(' (')[0]}"
        if r:
            s_ += f", kernel {r['achieved']:.4g} {r['unit']} = {r['frac']:.3f} of {r['bound']}"
        if "cpu_baseline" in pt:
            s_ += f"; oracle {pt['cpu_baseline']['value']:.3g} {pt['cpu_baseline']['unit']} on {pt['cpu_baseline']['cores']} cores"
        summ[name] = s_
    line["summary"] = summ
    if rank == 0:
        print(json.dumps(line), flush=True)


def _recorded_traffic(part: str):
    """DRAM bytes per launch of the dominant kernel of bench part `part` from
    the committed ncu summary (profiles/traffic.json), if it was taken on the
    current sources of that kernel (else None)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f).get(part)
    if not d:
        return None
    m = hashlib.sha256()
    for name in d["sources"]:
        with open(os.path.join(ROOT, "attention_split_attn_b200", "csrc", name), "rb") as f:
            m.update(f.read())
    return d["dram_bytes_per_launch"] if m.hexdigest()[:16] == d["sources_sha256_16"] else None


class _L2Flush:
    """Writes a 256 MiB buffer (twice the L2) between timed calls."""

    def __init__(self, dev):
        self.buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def __call__(self):
        self.buf.fill_(1)


def _time_calls(call_timed, n, flush, stream):
    """n calls, each bracketed by its own events on the launching stream with
    an L2 flush before it; returns (mean whole-call ms, mean main-kernel ms)."""
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
    for e in (x for row in ev for x in row):
        e.record(stream)
    torch.cuda.synchronize()
    for i in range(n):
        flush()
        call_timed(ev[i])
    torch.cuda.synchronize()
    whole = [e[0].elapsed_time(e[2]) for e in ev]
    main = [e[0].elapsed_time(e[1]) for e in ev]
    return sum(whole) / n, sum(main) / n


def selected_bytes(p) -> int:
    """K and V rows of every distinct valid selected cell for each KV head,
    plus Q, the selection lists and the output."""
    sel = p.sel.numpy()
    n_valid = 0
    for row in sel:
        v = row[(row >= 0) & (row < p.n_cells)]
        n_valid += len(np.unique(v))
    kv = n_valid * p.n_head_kv * p.head_dim * p.k.element_size() * 2
    o = p.n_rows * p.n_head_q * p.head_dim * torch.empty((), dtype=p.out_dtype).element_size()
    return kv + p.q.numel() * p.q.element_size() + sel.size * 4 + o


def _selected_pairs(p) -> int:
    """Distinct valid selected (row, cell) pairs."""
    sel = p.sel.numpy()
    return sum(len(np.unique(row[(row >= 0) & (row < p.n_cells)])) for row in sel)


def prefill_flops(p) -> int:
    """4 D flops (QK^T and PV) per visible (row, cell, q head); visibility is
    carried by the mask in the causal prefill workload."""
    vis = int(torch.isfinite(p.mask).sum()) if p.mask is not None else p.n_rows * p.n_cells
    return 4 * p.head_dim * vis * p.n_head_q


def run_parts(args, rank, dev, stream, with_cpu=False):
    """The other workloads (tiny decode, selected-key, causal prefill,
    draft-tree rows, e4m3 decode, the semantics sweep), each timed per call
    (L2 flushed before every call), with the roofline of its main kernel and,
    with_cpu, the FP64 oracle timed beside it on a bounded sample."""
    hbm_peak, tc_peak, peak_kind = _peaks()
    flush = _L2Flush(dev)
    n = max(3, min(args.steps, 20))
    parts = {}

    # tiny decode (1 row, 4 q heads over 1 KV head, D 64, 128 FP32 keys, 4
    # slices): a latency case -- the mean time of one call over back-to-back
    # calls (inputs resident, no flush: they are 64 KB)
    p = W.tiny_decode()
    (q, k, v, out), kw = A.problem_kwargs(p, device=dev)
    ta = A.make_args(q, k, v, out, **kw)
    ws = torch.empty(max(A.workspace_size(ta, A.OP_DECODE), 256), dtype=torch.uint8, device=dev)
    for _ in range(20):
        A.attn_decode_args(ta, ws=ws, stream=stream)
    reps = 200
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        A.attn_decode_args(ta, ws=ws, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / reps
    tiny_bytes = 2 * p.k.numel() * 4 + p.q.numel() * 4 + p.n_rows * p.n_head_q * p.head_dim * 4
    parts["tiny_decode"] = {
        "workload": "tiny_decode: 1 row, Hq 4 / Hkv 1, D 64, 128 FP32 keys, 4 forced slices, f32 out",
        "value": us, "unit": "us per call (latency; back-to-back calls)", "higher_is_better": False,
        "rows_per_s": 1e6 / us, "GBs": tiny_bytes / (us * 1e-6) / 1e9, "calls": reps,
        "gpu_launches": 2 * reps,   # (rows, heads, slices) grid kernel + split_k_reduce
    }
    if with_cpu:
        rate, thr, nrep = _oracle_rate(p, [0], lambda s_: 1, threads=1)
        parts["tiny_decode"]["cpu_baseline"] = {"value": 1e6 / rate, "unit": "us per call", "cores": 1,
                                                "kind": "oracle", "sample": f"the whole call, {nrep} repetitions"}
    del q, k, v, out, ta, ws, kw

    # maskless selected-key: 2048 rows, GQA 12, D 256, fp16 cache of 32768 cells
    p = W.selected_prefill()
    (q, k, v, out), kw = A.problem_kwargs(p, device=dev)
    sel = kw.pop("sel")
    sa = A.make_selected_args(q, k, v, out, sel, **kw)
    ws = torch.empty(max(A.selected_workspace_size(sa), 256), dtype=torch.uint8, device=dev)
    for _ in range(max(args.warmup, 3)):
        A.attn_selected_args(sa, ws=ws, stream=stream)
    whole, main = _time_calls(lambda e: A.attn_selected_timed_args(sa, ws, e, stream=stream), n, flush, stream)
    nbytes = selected_bytes(p)
    parts["selected"] = {
        "workload": "selected_prefill: 2048 rows, Hq 48 / Hkv 4, D 256, fp16 KV of 32768 cells, "
                    "2048-entry lists (5% dup, 3% invalid), f32 out",
        "value": nbytes / (whole * 1e-3) / 1e9, "unit": "GB/s (effective: gathered K/V bytes)",
        "ms_per_call": whole, "rows_per_s": p.n_rows / (whole * 1e-3), "calls": n,
        # compaction + gather (2048 rows x 4 KV heads fill the GPU: one part per row, no combine)
        "gpu_launches": 2 * n,
        "roofline": {"bound": "hbm", "achieved": nbytes / (main * 1e-3) / 1e9, "peak": hbm_peak,
                     "unit": "GB/s", "frac": nbytes / (main * 1e-3) / 1e9 / hbm_peak,
                     "traffic": _recorded_traffic("selected"),
                     "kernel": "select_bitmap_kernel + selected_kernel",
                     "kernel_ms": main, "algorithmic_bytes": nbytes,
                     "peak_kind": f"{peak_kind} hbm_gbs (burst copy); gathered rows are mostly L2 hits"},
    }
    if with_cpu:
        parts["selected"]["cpu_baseline"] = _part_baseline(p, list(range(0, 2048, 128)), selected_bytes, "GB/s",
                                                           1e9, "16 of the 2048 rows (every 128th)")
    del sa, ws

    # the masked per-cell route on the same workload (strix-llama.cpp PR #115,
    # "Measurements"): a dense F32 mask [2048 x 32768] from the lists, then the
    # tensor-core prefill kernel; same result, same effective-bytes metric
    ma = A.make_selected_args(q, k, v, out, sel, **kw)
    mws = torch.empty(max(A.selected_masked_workspace_size(ma), 256), dtype=torch.uint8, device=dev)
    for _ in range(max(args.warmup, 3)):
        A.attn_selected_masked_args(ma, ws=mws, stream=stream)
    nm = max(3, min(args.steps, 5))
    whole_m, main_m = _time_calls(lambda e: A.attn_selected_masked_timed_args(ma, mws, e, stream=stream), nm,
                                  flush, stream)
    sflops = 4 * p.head_dim * p.n_head_q * _selected_pairs(p)
    parts["selected_masked"] = {
        "workload": "selected_prefill through the masked per-cell route: F32 mask 2048 x 32768 from the lists, "
                    "then the dense tensor-core pass (tile classifier skips tiles no row selected)",
        "value": nbytes / (whole_m * 1e-3) / 1e9, "unit": "GB/s (effective: gathered K/V bytes, as selected)",
        "ms_per_call": whole_m, "vs_selected_kernel": whole_m / whole, "calls": nm,
        "gpu_launches": 3 * nm,   # mask builder + tile classifier + tensor-core kernel
        "roofline": {"bound": "tensor", "achieved": sflops / (main_m * 1e-3) / 1e12, "peak": tc_peak,
                     "unit": "TFLOP/s", "frac": sflops / (main_m * 1e-3) / 1e12 / tc_peak, "traffic": _recorded_traffic("selected_masked"),
                     "kernel": "sel_mask_kernel + prefill_classify_kernel + prefill_kernel<f16, 256>",
                     "kernel_ms": main_m, "algorithmic_flops": sflops,
                     "peak_kind": f"{peak_kind} bf16_tflops (burst cuBLAS); flops of the selected pairs only"},
    }
    del q, k, v, out, sel, ma, mws, kw

    # causal prefill: 2048 rows over 14048 cells, Hq 64 / Hkv 8, D 128, bf16
    p = W.causal_prefill()
    (q, k, v, out), kw = A.problem_kwargs(p, device=dev)
    pa = A.make_args(q, k, v, out, **kw)
    ws = torch.empty(max(A.workspace_size(pa, A.OP_PREFILL), 256), dtype=torch.uint8, device=dev)
    for _ in range(max(args.warmup, 3)):
        A.attn_prefill_args(pa, ws=ws, stream=stream)
    whole, main = _time_calls(lambda e: A.attn_prefill_timed_args(pa, ws, e, stream=stream), n, flush, stream)
    flops = prefill_flops(p)
    parts["prefill"] = {
        "workload": "causal_prefill: 2048 rows over 14048 cells (depth 12000), Hq 64 / Hkv 8, D 128, "
                    "bf16, softcap 50, ALiBi, sinks, f32 causal mask",
        "value": flops / (whole * 1e-3) / 1e12, "unit": "TFLOP/s",
        "ms_per_call": whole, "rows_per_s": p.n_rows / (whole * 1e-3), "calls": n,
        "gpu_launches": 2 * n,
        "roofline": {"bound": "tensor", "achieved": flops / (main * 1e-3) / 1e12, "peak": tc_peak,
                     "unit": "TFLOP/s", "frac": flops / (main * 1e-3) / 1e12 / tc_peak,
                     "traffic": _recorded_traffic("prefill"),
                     "kernel": "prefill_classify_kernel + prefill_kernel (tcgen05)",
                     "kernel_ms": main, "algorithmic_flops": flops,
                     "peak_kind": f"{peak_kind} bf16_tflops (burst cuBLAS)"},
    }
    if with_cpu:
        parts["prefill"]["cpu_baseline"] = _part_baseline(p, [128 * i + 64 for i in range(16)], prefill_flops,
                                                          "TFLOP/s", 1e12, "16 of the 2048 rows (one per row tile)")
    del q, k, v, out, pa, ws, kw

    # the causal prefill workload over an e4m3 cache (K and V quantized per
    # (cell, KV head), amax / 448): attn_prefill widens the codes into its
    # workspace and runs the same tensor-core path; TensorFold PR #911 puts
    # its e4m3 prefill within 5% of bf16.
    pq = W.causal_prefill()
    kq, ksq = W.quantize_kv(pq.k.to(torch.float32), "e4m3")
    vq, vsq = W.quantize_kv(pq.v.to(torch.float32), "e4m3")
    pq = dataclasses.replace(pq, k=kq, v=vq, k_scale=ksq, v_scale=vsq)
    (q, k, v, out), kw = A.problem_kwargs(pq, device=dev)
    pa = A.make_args(q, k, v, out, **kw)
    ws = torch.empty(max(A.workspace_size(pa, A.OP_PREFILL), 256), dtype=torch.uint8, device=dev)
    for _ in range(max(args.warmup, 3)):
        A.attn_prefill_args(pa, ws=ws, stream=stream)
    whole_q, main_q = _time_calls(lambda e: A.attn_prefill_timed_args(pa, ws, e, stream=stream), n, flush, stream)
    parts["fp8_prefill"] = {
        "workload": "causal_prefill over an e4m3 cache (per (cell, KV head) F32 scales): widening kernel + the "
                    "bf16 tensor-core prefill",
        "value": flops / (whole_q * 1e-3) / 1e12, "unit": "TFLOP/s",
        "ms_per_call": whole_q, "vs_bf16_prefill": whole_q / parts["prefill"]["ms_per_call"], "calls": n,
        "gpu_launches": 3 * n,   # widening + classifier + tensor-core kernel
        "roofline": {"bound": "tensor", "achieved": flops / (main_q * 1e-3) / 1e12, "peak": tc_peak,
                     "unit": "TFLOP/s", "frac": flops / (main_q * 1e-3) / 1e12 / tc_peak, "traffic": None,
                     "kernel": "dequant_kernel + prefill_classify_kernel + prefill_kernel (tcgen05)",
                     "kernel_ms": main_q, "algorithmic_flops": flops,
                     "peak_kind": f"{peak_kind} bf16_tflops (burst cuBLAS)"},
    }
    del q, k, v, out, pa, ws, kw, pq, kq, vq

    # draft-tree decode rows: 16 nodes of a binary draft tree over 130856 keys
    # (the depth of TensorFold PR #2595's long-context receipt), GQA heads;
    # a call = the tree mask kernel + attn_prefill, whose tiles then hold the
    # 16 rows x the 4 q heads of a KV group (packed rows), so each K/V tile
    # is read once for all of them; the same rows through attn_decode (each
    # row streams the prefix) are timed beside it.  Algorithmic bytes: the K/V
    # rows of every cell some row sees, once (the rows share the prefix), the
    # mask, Q and the output; rows_per_s and the per-row view are beside it.
    p = W.tree_decode(width=16, visible=130856)
    (q, k, v, out), kw = A.problem_kwargs(p, device=dev)
    kw.pop("mask")
    parent = p.tree_parent.to(dev)
    tmask = torch.empty((p.n_rows, p.n_cells), dtype=torch.float32, device=dev)
    ta = A.make_args(q, k, v, out, mask=tmask, **kw)
    ws = torch.empty(max(A.workspace_size(ta, A.OP_DECODE), 256), dtype=torch.uint8, device=dev)
    wsp = torch.empty(max(A.workspace_size(ta, A.OP_PREFILL), 256), dtype=torch.uint8, device=dev)
    vis = int(torch.isfinite(p.mask).sum())
    cells = int(torch.isfinite(p.mask).any(dim=0).sum())
    kv_cell = p.n_head_kv * p.head_dim * p.k.element_size() * 2
    rest = p.n_rows * p.n_cells * 4 + p.q.numel() * p.q.element_size() + p.n_rows * p.n_head_q * p.head_dim * 2
    tbytes = cells * kv_cell + rest

    def tree_call_decode(e):
        e[0].record(stream)
        A.tree_mask(parent, p.tree_prefix, p.n_cells, mask=tmask, stream=stream)
        A.attn_decode_args(ta, ws=ws, stream=stream)
        e[1].record(stream)
        e[2].record(stream)

    def tree_call(e):
        e[0].record(stream)
        A.tree_mask(parent, p.tree_prefix, p.n_cells, mask=tmask, stream=stream)
        A.attn_prefill_args(ta, ws=wsp, stream=stream)
        e[1].record(stream)
        e[2].record(stream)

    for _ in range(max(args.warmup, 3)):
        tree_call_decode([torch.cuda.Event(enable_timing=True) for _ in range(3)])
        tree_call([torch.cuda.Event(enable_timing=True) for _ in range(3)])
    whole_dec, _ = _time_calls(tree_call_decode, n, flush, stream)
    whole, main = _time_calls(tree_call, n, flush, stream)
    parts["tree_decode"] = {
        "workload": "tree_decode: 16 draft-tree rows (binary heap order) over 130856 keys, Hq 32 / Hkv 8, D 128, "
                    "bf16 KV and out; tree mask + attn_prefill (packed rows)",
        "value": tbytes / (whole * 1e-3) / 1e9, "unit": "GB/s (K/V of every visible cell once + mask)",
        "per_row_GBs": (vis * kv_cell + rest) / (whole * 1e-3) / 1e9,
        "ms_per_call": whole, "ms_attn_decode": whole_dec, "rows_per_s": p.n_rows / (whole * 1e-3), "calls": n,
        "gpu_launches": 3 * n,   # tree mask + classifier + tensor-core kernel
        "roofline": {"bound": "hbm", "achieved": tbytes / (main * 1e-3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                     "frac": tbytes / (main * 1e-3) / 1e9 / hbm_peak, "traffic": _recorded_traffic("tree_decode"), "kernel_ms": main,
                     "algorithmic_bytes": tbytes,
                     "peak_kind": f"{peak_kind} hbm_gbs (burst copy); K/V of the tree's KV groups read once"},
    }
    if with_cpu:
        parts["tree_decode"]["cpu_baseline"] = _part_baseline(
            p, list(range(p.n_rows)), lambda s_: tbytes, "GB/s", 1e9, "all 16 rows")
    del q, k, v, out, ta, ws, kw, tmask

    # one long row (130856 cached keys, the depth of TensorFold PR #2595's
    # long-context receipt), Hq 32 / Hkv 8, D 128, bf16: attn_decode (balanced
    # kernel + split_k_reduce), attn_decode_cluster (16-CTA clusters, DSMEM
    # fold, no workspace) and attn_decode_append (the step's append fused in)
    p = W.random_problem(1010, R=1, Hq=32, Hkv=8, D=128, N=130857, kv_dtype=torch.bfloat16,
                         out_dtype=torch.bfloat16, lengths=[130857])
    (q, k, v, out), kw = A.problem_kwargs(p, device=dev)
    la = A.make_args(q, k, v, out, **kw)
    ws = torch.empty(max(A.workspace_size(la, A.OP_DECODE), 256), dtype=torch.uint8, device=dev)
    kn = torch.randn((1, 8, 128), device=dev).to(torch.bfloat16)
    vn = torch.randn((1, 8, 128), device=dev).to(torch.bfloat16)
    lbytes = algorithmic_bytes(p)
    calls = {
        "decode": lambda: A.attn_decode_args(la, ws=ws, stream=stream),
        "cluster": lambda: A.attn_decode_cluster_args(la, stream=stream),
        "append": lambda: A.attn_decode_append_args(la, kn, vn, ws=ws, stream=stream),
    }
    lat = {}
    for name, fn in calls.items():
        for _ in range(max(args.warmup, 3)):
            fn()

        def timed(e, fn=fn):
            e[0].record(stream)
            fn()
            e[1].record(stream)
            e[2].record(stream)
        lat[name], _ = _time_calls(timed, n, flush, stream)
    parts["long_row_decode"] = {
        "workload": "long_row_decode: 1 row over 130857 cached keys, Hq 32 / Hkv 8, D 128, bf16 KV and out",
        "value": lbytes / (lat["cluster"] * 1e-3) / 1e9, "unit": "GB/s (attn_decode_cluster; K/V, Q, out)",
        "ms_per_call": lat["cluster"], "ms_attn_decode": lat["decode"], "ms_attn_decode_append": lat["append"],
        "GBs_attn_decode": lbytes / (lat["decode"] * 1e-3) / 1e9, "calls": n,
        "gpu_launches": n * (1 + 2 + 2),   # cluster; decode (stream + combine); append (stream + combine)
        "roofline": {"bound": "hbm", "achieved": lbytes / (lat["cluster"] * 1e-3) / 1e9, "peak": hbm_peak,
                     "unit": "GB/s", "frac": lbytes / (lat["cluster"] * 1e-3) / 1e9 / hbm_peak, "traffic": _recorded_traffic("long_row_decode"),
                     "kernel": "decode_cluster_kernel (one launch)", "kernel_ms": lat["cluster"],
                     "algorithmic_bytes": lbytes, "peak_kind": f"{peak_kind} hbm_gbs (burst copy)"},
    }
    del q, k, v, out, la, ws, kw

    # quantized GQA decode: the decode batch's shape (16 rows, lengths U[1024,
    # 8192], Hq 32 / Hkv 8, D 128) over an e4m3 cache with one F32 scale per
    # (cell, KV head) for K and for V (TensorFold PR #911).  Bytes: the K and V
    # codes and scales of every visible (cell, KV head), Q and out.
    p = W.quantized_decode(fmt="e4m3")
    (q, k, v, out), kw = A.problem_kwargs(p, device=dev)
    qa = A.make_args(q, k, v, out, **kw)
    qws_n = A.workspace_size(qa, A.OP_DECODE)
    ws = torch.empty(max(qws_n, 256), dtype=torch.uint8, device=dev)
    lens = int((p.row_end - p.row_begin).to(torch.int64).sum())
    qbytes = (lens * p.n_head_kv * (2 * p.head_dim + 2 * 4) + p.q.numel() * p.q.element_size()
              + p.n_rows * p.n_head_q * p.head_dim * 2)
    for _ in range(max(args.warmup, 3)):
        A.attn_decode_args(qa, ws=ws, stream=stream)
    whole, main = _time_calls(lambda e: A.attn_decode_timed_args(qa, ws, e, stream=stream), n, flush, stream)
    parts["fp8_decode"] = {
        "workload": "quantized_decode: 16 seq x 1 row, Hq 32 / Hkv 8, D 128, e4m3 KV with per (cell, KV head) "
                    "F32 scales, len U[1024,8192], bf16 out",
        "value": qbytes / (whole * 1e-3) / 1e9, "unit": "GB/s (visible K/V codes + scales, Q, out)",
        "ms_per_call": whole, "calls": n,
        "gpu_launches": (2 if qws_n > 0 else 1) * n,   # decode kernel (+ split_k_reduce)
        "roofline": {"bound": "hbm", "achieved": qbytes / (main * 1e-3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                     "frac": qbytes / (main * 1e-3) / 1e9 / hbm_peak, "traffic": _recorded_traffic("fp8_decode"), "kernel_ms": main,
                     "algorithmic_bytes": qbytes,
                     "kernel": "decode_stream_kernel<e4m3> (codes widened to f16 for the tensor cores) + combine_kernel",
                     "peak_kind": f"{peak_kind} hbm_gbs (burst copy)"},
    }
    if with_cpu:
        parts["fp8_decode"]["cpu_baseline"] = _part_baseline(
            p, list(range(p.n_rows)), lambda s_: qbytes, "GB/s", 1e9, "all 16 rows")
    del q, k, v, out, qa, ws, kw

    # semantics sweep: unified fp16 cache of 8 interleaved sequences, 256 rows,
    # per-cell sequence ids and positions, F32 mask, NaN cells, sinks; through
    # attn_decode (planner slices) and attn_prefill.  Bytes: the K and V rows of
    # every visible (cell, KV head), the F32 mask rows and the cell metadata
    # each row scans, Q and the output.
    p = W.semantics_sweep()
    (q, k, v, out), kw = A.problem_kwargs(p, device=dev)
    vis = _visible_cells(p)
    nbytes = (vis * p.n_head_kv * p.head_dim * p.k.element_size() * 2
              + p.n_rows * p.n_cells * (4 + 8) + p.q.numel() * p.q.element_size()
              + p.n_rows * p.n_head_q * p.head_dim * 4)
    for name, op, call in (("semantics_decode", A.OP_DECODE, A.attn_decode_timed_args),
                           ("semantics_prefill", A.OP_PREFILL, A.attn_prefill_timed_args)):
        a = A.make_args(q, k, v, out, **kw)
        ws = torch.empty(max(A.workspace_size(a, op), 256), dtype=torch.uint8, device=dev)
        for _ in range(max(args.warmup, 3)):
            (A.attn_decode_args if op == A.OP_DECODE else A.attn_prefill_args)(a, ws=ws, stream=stream)
        whole, main = _time_calls(lambda e: call(a, ws, e, stream=stream), n, flush, stream)
        parts[name] = {
            "workload": "semantics_sweep: unified fp16 cache of 8 interleaved sequences, 256 rows with lengths "
                        "log-uniform in [1, 65536], Hq 16 / Hkv 4, D 128, F32 mask with -inf/+inf, NaN cells, sinks",
            "value": nbytes / (whole * 1e-3) / 1e9, "unit": "GB/s (visible K/V + mask + cell metadata)",
            "ms_per_call": whole, "rows_per_s": p.n_rows / (whole * 1e-3), "calls": n,
            # visible lists + gather + split_k_reduce (long rows are split into parts)
            "gpu_launches": 3 * n,
            "roofline": {"bound": "hbm", "achieved": nbytes / (main * 1e-3) / 1e9, "peak": hbm_peak,
                         "unit": "GB/s", "frac": nbytes / (main * 1e-3) / 1e9 / hbm_peak, "traffic": _recorded_traffic("semantics"),
                         "kernel_ms": main, "algorithmic_bytes": nbytes,
                         "peak_kind": f"{peak_kind} hbm_gbs (burst copy); semantics case, no target"},
        }
    if with_cpu:
        base = _part_baseline(p, list(range(p.n_rows)), lambda s_: nbytes, "GB/s", 1e9, "all 256 rows")
        parts["semantics_decode"]["cpu_baseline"] = base
        parts["semantics_prefill"]["cpu_baseline"] = base
    return parts


def _visible_cells(p) -> int:
    """Number of visible (row, cell) pairs: same sequence, causal, mask not -inf."""
    cs, cp = p.cell_seq.numpy(), p.cell_pos.numpy()
    rs, rp = p.row_seq.numpy(), p.row_pos.numpy()
    m = p.mask.numpy()
    total = 0
    for r in range(p.n_rows):
        total += int(((cs == rs[r]) & (cp <= rp[r]) & (m[r] != -np.inf)).sum())
    return total


def run_profile_op(args, local):
    """--profile-op: W + K plain calls of one operation on its benchmark
    workload and nothing else (the command the ncu summaries are taken on)."""
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    A.load_library()
    op = args.profile_op
    if op == "decode":
        p = W.gqa_decode(poison_unused=False)
        (q, k, v, out), kw = A.problem_kwargs(p, device=dev)
        a = A.make_args(q, k, v, out, **kw)
        ws = torch.empty(max(A.workspace_size(a, A.OP_DECODE), 256), dtype=torch.uint8, device=dev)
        call = lambda: A.attn_decode_args(a, ws=ws)
    elif op == "semantics":
        p = W.semantics_sweep()
        (q, k, v, out), kw = A.problem_kwargs(p, device=dev)
        a = A.make_args(q, k, v, out, **kw)
        ws = torch.empty(max(A.workspace_size(a, A.OP_DECODE), 256), dtype=torch.uint8, device=dev)
        call = lambda: A.attn_decode_args(a, ws=ws)
    elif op in ("selected", "selected_masked"):
        p = W.selected_prefill()
        (q, k, v, out), kw = A.problem_kwargs(p, device=dev)
        sel = kw.pop("sel")
        a = A.make_selected_args(q, k, v, out, sel, **kw)
        if op == "selected":
            ws = torch.empty(max(A.selected_workspace_size(a), 256), dtype=torch.uint8, device=dev)
            call = lambda: A.attn_selected_args(a, ws=ws)
        else:
            ws = torch.empty(max(A.selected_masked_workspace_size(a), 256), dtype=torch.uint8, device=dev)
            call = lambda: A.attn_selected_masked_args(a, ws=ws)
    elif op == "fp8":
        p = W.quantized_decode(fmt="e4m3")
        (q, k, v, out), kw = A.problem_kwargs(p, device=dev)
        a = A.make_args(q, k, v, out, **kw)
        ws = torch.empty(max(A.workspace_size(a, A.OP_DECODE), 256), dtype=torch.uint8, device=dev)
        call = lambda: A.attn_decode_args(a, ws=ws)
    elif op == "tree":
        # the bench's tree rows: the host-built tree mask, attn_prefill (packed rows)
        p = W.tree_decode(width=16, visible=130856)
        (q, k, v, out), kw = A.problem_kwargs(p, device=dev)
        a = A.make_args(q, k, v, out, **kw)
        ws = torch.empty(max(A.workspace_size(a, A.OP_PREFILL), 256), dtype=torch.uint8, device=dev)
        call = lambda: A.attn_prefill_args(a, ws=ws)
    elif op == "long_row":
        p = W.random_problem(1010, R=1, Hq=32, Hkv=8, D=128, N=130857, kv_dtype=torch.bfloat16,
                             out_dtype=torch.bfloat16, lengths=[130857])
        (q, k, v, out), kw = A.problem_kwargs(p, device=dev)
        a = A.make_args(q, k, v, out, **kw)
        call = lambda: A.attn_decode_cluster_args(a)
    else:
        p = W.causal_prefill()
        (q, k, v, out), kw = A.problem_kwargs(p, device=dev)
        a = A.make_args(q, k, v, out, **kw)
        ws = torch.empty(max(A.workspace_size(a, A.OP_PREFILL), 256), dtype=torch.uint8, device=dev)
        call = lambda: A.attn_prefill_args(a, ws=ws)
    for _ in range(args.warmup + args.steps):
        call()
    torch.cuda.synchronize()
    A.check_device_status()
    print(json.dumps({"profile_op": op, "calls": args.warmup + args.steps}), flush=True)


def run_e2e(args, sets, stream):
    """The same step through the C ABI from pinned HOST buffers: every step
    copies its inputs (Q, the K/V rows each sequence uses, row ranges) to the
    device, runs attn_decode, and reads the output back."""
    st0 = sets[0]
    p = st0["p"]
    q, k, v, out, kw = st0["keep"]
    b = p.row_begin.tolist()
    e = p.row_end.tolist()
    host = {"q": p.q.pin_memory(), "rb": p.row_begin.pin_memory(), "re": p.row_end.pin_memory(),
            "out": torch.empty(out.shape, dtype=out.dtype).pin_memory()}
    host_k = [p.k[b[i]:e[i]].contiguous().pin_memory() for i in range(len(b))]
    host_v = [p.v[b[i]:e[i]].contiguous().pin_memory() for i in range(len(b))]
    h2d = (host["q"].numel() * host["q"].element_size() + 2 * host["rb"].numel() * 4
           + sum(t.numel() * t.element_size() for t in host_k + host_v))
    d2h = host["out"].numel() * host["out"].element_size()

    def step():
        q.copy_(host["q"], non_blocking=True)
        kw["row_begin"].copy_(host["rb"], non_blocking=True)
        kw["row_end"].copy_(host["re"], non_blocking=True)
        for i in range(len(b)):
            k[b[i]:e[i]].copy_(host_k[i], non_blocking=True)
            v[b[i]:e[i]].copy_(host_v[i], non_blocking=True)
        A.attn_decode_args(st0["args"], ws=st0["ws"])
        host["out"].copy_(out, non_blocking=True)

    for _ in range(2):
        step()
    torch.cuda.synchronize()
    n = max(3, min(args.steps, 10))
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(n):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / n
    return {"value": st0["bytes"] / (ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": ms}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-parts", action="store_true", help="time the decode workload only")
    ap.add_argument("--profile-op", choices=["decode", "selected", "prefill", "semantics", "selected_masked", "fp8",
                                             "tree", "long_row"], default=None,
                    help="only run W + K calls of one operation (for ncu captures); prints no bench line")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup
    rank, world, local = _dist()
    try:
        if args.profile_op:
            run_profile_op(args, local)
        elif args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
