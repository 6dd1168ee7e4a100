"""Benchmark: paged GQA decode (Llama-3.1-70B shapes) through libsplitkv on B200.

One step = the decode workload run twice, as the configuration states: K/V with identical
strides, then V as a strided column slice of a 2x-wide buffer (independent strides).  Each run is
the attention kernel (split-KV partials) followed by the plan's merge pass.  Batch 64, q_len 1,
64 query / 8 KV heads, head_dim 128, page_size 16, KV lengths U[1024, 8192], permuted pages,
bf16 N(0,1) data (seeded, synthetic).  The KV cache is resident device state (uploaded once);
the KV working set (2 x 1.2 GB) is far larger than the 126 MB L2, so every step reads it from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
    torchrun --nproc-per-node N bench.py --gpus N ...     (one rank per GPU, weak scaling)

Prints ONE JSON line (rank 0).  ``value`` = achieved KV GB/s over all ranks (algorithmic KV bytes:
exactly L_r tokens x Hk x D x 2 tensors x 2 bytes per request, per run) / max-over-ranks device time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention: achieved KV GB/s (% of HBM peak), µs per decode step"
NOMINAL_HBM_GBS = 8000.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
KERNEL_SOURCES = ["split_kv_merge_b200/csrc/gqa_tc_wide.cu", "split_kv_merge_b200/csrc/gqa_tc_wide_body.cuh",
                  "split_kv_merge_b200/csrc/tc_ptx.cuh"]


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK), "fallback"


def _kernel_hash(paths):
    h = hashlib.sha256()
    for rel in paths:
        p = os.path.join(ROOT, rel)
        if os.path.exists(p):
            with open(p, "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:16]


def _traffic_record(kernel_name, src_hash):
    """DRAM bytes per launch from the committed ncu summary, only if it was taken on this exact
    kernel source (else null)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        recs = json.load(f)
    r = recs.get(kernel_name)
    if not r or r.get("source_hash") != src_hash:
        return None
    return r


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self.thread is not None:
                self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() in ("active", "1", "yes"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def _physical_gpu(local: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [x.strip() for x in vis.split(",") if x.strip()]
    if local < len(ids) and ids[local].isdigit():
        return int(ids[local])
    return local


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def aggregate_over_ranks(local_ms: float, local_bytes: int, device=None):
    """Whole-job numbers: the slowest rank's device time and the bytes all ranks processed
    (all-reduce MAX / SUM over the default process group; identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(local_ms), int(local_bytes)
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    b = torch.tensor([int(local_bytes)], dtype=torch.int64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(b, op=dist.ReduceOp.SUM)
    return float(t.item()), int(b.item())


def _kv_bytes(case):
    L = case.kv_lengths()
    return int(L.sum()) * case.num_kv_heads * case.head_dim * 2 * 2


def _cpu_baseline(cases, budget_s=12.0):
    """The oracle as it stands, on the host cores, over a bounded sample of the same workload:
    requests of both stride variants in order until ~budget_s seconds have passed."""
    import oracle.attention as OA
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        threads = 1
    done_bytes, n_req, t0 = 0, 0, time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        for c in cases:
            for r in range(c.batch):
                OA.paged_attention(c.q, c.k, c.v, c.qo_indptr, c.kv_indptr, c.kv_indices, c.kv_last_page_len,
                                   c.page_size, c.sm_scale, requests=[r])
                L = int(c.kv_lengths()[r])
                done_bytes += L * c.num_kv_heads * c.head_dim * 4
                n_req += 1
                if time.perf_counter() - t0 >= budget_s:
                    break
            if time.perf_counter() - t0 >= budget_s:
                break
    dt = time.perf_counter() - t0
    return {"value": done_bytes / dt / 1e9, "unit": "GB/s", "cores": int(threads), "kind": "oracle",
            "sample": f"{n_req} requests of the same decode workload (float64 numpy oracle, "
                      f"{dt:.1f} s, {os.cpu_count()} host cores visible)"}


def _make_cases(rank: int, batch: int = 64):
    from workloads import llama70b_decode_case
    seed = 2 + 1000 * rank   # each rank holds its own batch of requests (weak scaling)
    return [llama70b_decode_case(independent_v=False, seed=seed, batch=batch),
            llama70b_decode_case(independent_v=True, seed=seed, batch=batch)]


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    cases = _make_cases(0)
    per_step = []
    budget = max(0.2, min(args.ref_budget, 150.0 / (args.steps + args.warmup)))   # whole run ~ minutes
    for _ in range(args.warmup):
        _cpu_baseline(cases, budget_s=budget)
    for _ in range(args.steps):
        per_step.append(_cpu_baseline(cases, budget_s=budget))
    value = statistics.median(x["value"] for x in per_step)
    kv = sum(_kv_bytes(c) for c in cases)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": kv / (value * 1e9) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": _config(cases, None),
            "cpu_baseline": {**per_step[-1], "value": value},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def _config(cases, plans):
    c = cases[0]
    L = c.kv_lengths()
    cfg = {"workload": "Llama-3.1-70B-shaped paged decode, run twice per step (equal K/V strides; V a column "
                       "slice of a 2x-wide buffer)",
           "batch": c.batch, "q_len": 1, "num_qo_heads": c.num_qo_heads, "num_kv_heads": c.num_kv_heads,
           "head_dim": c.head_dim, "page_size": c.page_size, "kv_len_range": [1024, 8192],
           "kv_tokens_per_run": int(L.sum()), "kv_bytes_per_step": sum(_kv_bytes(x) for x in cases),
           "l2": "no flush: 2.4 GB KV working set per step > 126 MB L2", "parallelism": "replicas (independent "
                                                                                    "request batches per GPU)"}
    if plans is not None:
        cfg["split_policy"] = "balanced"
        cfg["plans"] = [p.info.as_dict() for p in plans]
    return cfg


def run_ours(args):
    import torch
    import split_kv_merge_b200 as skv
    from workloads.device import paged_to_device

    ws, rank, local = _dist()
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cases = _make_cases(rank, args.batch)
    kv_bytes_step = sum(_kv_bytes(c) for c in cases)
    runs = []
    for c in cases:
        d = paged_to_device(c, dev)
        plan = skv.plan_paged(c.qo_indptr, c.kv_indptr, c.kv_last_page_len, c.page_size, c.num_qo_heads,
                              c.num_kv_heads, c.head_dim, "balanced", 0).to(dev)
        n_part = plan.info.num_partial_rows
        o = torch.empty(c.q.shape[0], c.num_qo_heads, c.head_dim, dtype=torch.float32, device=dev)
        lse = torch.empty(c.q.shape[0], c.num_qo_heads, dtype=torch.float32, device=dev)
        o_part = torch.empty(max(1, n_part), c.num_qo_heads, c.head_dim, dtype=torch.float32, device=dev)
        lse_part = torch.empty(max(1, n_part), c.num_qo_heads, dtype=torch.float32, device=dev)
        runs.append(dict(c=c, d=d, plan=plan, o=o, lse=lse, o_part=o_part, lse_part=lse_part))
    stream = torch.cuda.current_stream(dev)

    def launch(run, ev=None):
        # one skv_paged_attn_fwd call (attention, then the merge pass with programmatic dependent
        # launch); with `ev`, the two phases as separate calls with `ev` recorded between them (an
        # event between the kernels also ends the merge's early launch, so this form is used only
        # to time the attention kernel alone)
        c, d = run["c"], run["d"]
        if ev is None:
            skv.paged_attn_fwd(d["q"], d["k"], d["v"], d["kv_indptr"], d["kv_indices"], d["kv_last_page_len"],
                               run["plan"], run["o"], run["lse"], run["o_part"], run["lse_part"], None, c.sm_scale,
                               c.num_pages, stream)
            return
        skv.paged_attn_fwd(d["q"], d["k"], d["v"], d["kv_indptr"], d["kv_indices"], d["kv_last_page_len"],
                           run["plan"], run["o"], run["lse"], run["o_part"], run["lse_part"], None, c.sm_scale,
                           c.num_pages, stream, phase="partial")
        ev.record(stream)
        skv.merge_plan(run["o_part"], run["lse_part"], run["plan"], c.num_qo_heads, c.head_dim, run["o"],
                       run["lse"], stream)

    for _ in range(args.warmup):
        for run in runs:
            launch(run)
    torch.cuda.synchronize(dev)

    def barrier():
        if ws > 1:
            import torch.distributed as dist
            dist.barrier()

    # ---------------------------------------------------------------- device-timed region
    # K steps of the public call (events only between runs), then -- for the roofline of the
    # attention kernel -- the same K steps again as two phases with an event between them
    n_ev = args.steps * len(runs)
    ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    ev_c = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    ra = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    rb = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    rc = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(_physical_gpu(local)) as clk:
        time.sleep(0.15)
        start.record(stream)
        i = 0
        for _ in range(args.steps):
            for run in runs:
                ev_a[i].record(stream)
                launch(run)
                ev_c[i].record(stream)
                i += 1
        end.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        i = 0
        for _ in range(args.steps):
            for run in runs:
                ra[i].record(stream)
                launch(run, rb[i])
                rc[i].record(stream)
                i += 1
        torch.cuda.synchronize(dev)
        time.sleep(0.1)
    barrier()
    total_ms = start.elapsed_time(end)
    run_ms = [ev_a[j].elapsed_time(ev_c[j]) for j in range(n_ev)]
    attn_ms = [ra[j].elapsed_time(rb[j]) for j in range(n_ev)]
    merge_ms = [rb[j].elapsed_time(rc[j]) for j in range(n_ev)]
    total_ms, total_bytes = aggregate_over_ranks(total_ms, kv_bytes_step * args.steps, dev)
    value = total_bytes / (total_ms * 1e-3) / 1e9
    ms_per_step = total_ms / args.steps

    # ---------------------------------------------------------------- end-to-end through the public API
    e2e = _e2e(args, runs, dev, stream, skv, torch)

    if rank != 0:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return 0
    peaks, peak_src = _peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK["hbm_gbs"]))
    attn_avg_ms = statistics.mean(attn_ms)
    per_launch_bytes = kv_bytes_step / len(runs)
    achieved = per_launch_bytes / (attn_avg_ms * 1e-3) / 1e9
    kernel = {1: "gqa_simt_kernel", 2: "gqa_tc_decode_kernel", 3: "gqa_tc_wide_kernel"}.get(
        runs[0]["plan"].info.kernel, "unknown")
    src_hash = _kernel_hash(KERNEL_SOURCES)
    tr = _traffic_record(kernel, src_hash)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": _config(cases, [r["plan"] for r in runs]),
        "us_per_step": round(ms_per_step * 1e3, 2),
        "us_per_run": {"equal_strides": round(statistics.median(run_ms[0::2]) * 1e3, 2),
                       "independent_v_strides": round(statistics.median(run_ms[1::2]) * 1e3, 2)},
        "pct_hbm": {"of_nominal_8TBps": round(100 * value / ws / NOMINAL_HBM_GBS, 2),
                    f"of_{peak_src}_{hbm:.0f}GBps": round(100 * value / ws / hbm, 2)},
        "roofline": {"bound": "hbm", "kernel": kernel, "achieved": round(achieved, 2), "peak": hbm, "unit": "GB/s",
                     "frac": round(achieved / hbm, 4), "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"
                     if peak_src == "measured" else "fallback 6650 GB/s",
                     "traffic": None if tr is None else tr["bytes_per_launch"],
                     "algorithmic_bytes_per_launch": int(per_launch_bytes),
                     "avg_launch_us": round(attn_avg_ms * 1e3, 2),
                     "merge_avg_us": round(statistics.mean(merge_ms) * 1e3, 2),
                     "how": "attention kernel timed with CUDA events around each of its launches in a second "
                            "pass of the same steps right after the timed region (an event between the "
                            "attention and merge kernels ends the merge's programmatic early launch, so the "
                            "timed region itself records events only between runs)"},
        "e2e": e2e,
        "gpu_launches": args.steps * sum(1 + (1 if r["plan"].info.num_merge_rows > 0 else 0) for r in runs),
        "clocks": clk.summary(),
        "kernel_source_hash": src_hash,
    }
    if ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = _cpu_baseline(cases)
    if ws == 1 and not args.no_configs:
        del runs
        torch.cuda.empty_cache()
        line["configs"] = all_configs(args, dev, stream, skv, torch)
    print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def _e2e(args, runs, dev, stream, skv, torch):
    """Same metric through the public API with every step's inputs and outputs in host memory
    (``PagedDecodePipeline``): each step plans both runs on the host, copies their q, page tables
    and plans from pinned host memory, runs both phases and copies O and LSE back into pinned host
    memory; the host work and the copies of step k + 1 overlap the kernels of step k (two buffer
    sets, input / compute / output streams).  Wall clock from the first submit to the last
    result read."""
    pipes = []
    for run in runs:
        c = run["c"]
        q_h = torch.from_numpy(np.ascontiguousarray(c.q).view(np.int16)).view(torch.bfloat16).pin_memory()
        pipe = skv.PagedDecodePipeline(run["d"]["k"], run["d"]["v"], c.num_qo_heads, max_rows=c.q.shape[0],
                                       max_batch=c.batch, max_page_ids=len(c.kv_indices), sm_scale=c.sm_scale,
                                       num_pages=c.num_pages)
        pipes.append((pipe, q_h, c))
    steps = max(3, min(args.steps, args.e2e_steps))

    def submit():
        return [p.submit(q_h, c.qo_indptr, c.kv_indptr, c.kv_indices, c.kv_last_page_len) for p, q_h, c in pipes]

    def read(tickets):
        for (p, _, _), t in zip(pipes, tickets):
            p.result(t)

    for _ in range(3):  # warm-up: buffers at their final sizes
        read(submit())
    h2d0 = sum(p.h2d_bytes for p, _, _ in pipes)
    d2h0 = sum(p.d2h_bytes for p, _, _ in pipes)
    t0 = time.perf_counter()
    prev = None
    for _ in range(steps):
        cur = submit()
        if prev is not None:
            read(prev)
        prev = cur
    read(prev)
    dt = time.perf_counter() - t0
    h2d = sum(p.h2d_bytes for p, _, _ in pipes) - h2d0
    d2h = sum(p.d2h_bytes for p, _, _ in pipes) - d2h0
    kv = sum(_kv_bytes(r["c"]) for r in runs)
    return {"value": round(kv * steps / dt / 1e9, 2), "unit": "GB/s", "steps": steps,
            "h2d_bytes_per_step": h2d // steps, "d2h_bytes_per_step": d2h // steps,
            "ms_per_step": round(dt / steps * 1e3, 4),
            "how": "PagedDecodePipeline: host planning + pinned H2D of q, page table and plan + both phases + "
                   "D2H of O and LSE every step; next step's host work and copies overlap this step's kernels, "
                   "and the two runs of a step (one pipeline each, own streams) may overlap on the GPU where "
                   "one kernel's tail leaves SMs free, which the device-timed region (one stream) does not do"}


# ----------------------------------------------------------------------------- other configurations
CONFIG_NAMES = (["tiny", "llama70b_e4m3", "shared_kv"] + [f"mla_h{h}_q{q}_{d}" for h in (16, 128) for q in (1, 4)
                                                          for d in ("bf16", "e4m3")]
                + ["mla_h16_q4_bf16_causal", "pod", "pod_two_launches", "route", "fetch_splice"])
L2_FLUSH_BYTES = 512 << 20   # > 126 MB L2: written before every timed call


def _threads_used():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        return 1


def _time_calls(step, steps, warmup, torch, stream, flush):
    """Mean device time (ms) of one call: `warmup` untimed calls, then `steps` calls each
    bracketed by CUDA events on the launching stream, with L2 flushed (a 512 MB write) before
    every timed call."""
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in ev)


def _sampled(units, budget_s):
    """Run oracle sample units (callables returning the (bytes, FLOPs) they covered) until
    budget_s has passed; returns ((bytes, FLOPs) done, seconds, units run).  At least one runs."""
    done, n, t0 = np.zeros(2), 0, time.perf_counter()
    for u in units:
        done += np.asarray(u(), dtype=np.float64)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    return done, time.perf_counter() - t0, n


def _setup_config(name, dev, skv, torch, stream):
    """Device inputs, the timed call and its algorithmic bytes / FLOPs for one configuration, plus
    the oracle sample units (each returns the algorithmic bytes and FLOPs it covered) and the
    kernel it runs."""
    import oracle.attention as OA
    from workloads import fetch_splice_case, mla_decode_case, route_case, shared_kv_prefill_case, tiny_gqa_case
    from workloads.device import mla_to_device, paged_to_device, route_to_device, splice_to_device
    from workloads import llama70b_decode_case
    e = {}
    if name in ("tiny", "shared_kv", "llama70b_e4m3"):
        c = {"tiny": tiny_gqa_case, "shared_kv": shared_kv_prefill_case,
             "llama70b_e4m3": lambda: llama70b_decode_case(kv_dtype="e4m3")}[name]()
        d = paged_to_device(c, dev)
        pol, par = {"tiny": ("fixed", 2), "shared_kv": ("none", 0), "llama70b_e4m3": ("balanced", 0)}[name]
        plan = skv.plan_paged(c.qo_indptr, c.kv_indptr, c.kv_last_page_len, c.page_size, c.num_qo_heads,
                              c.num_kv_heads, c.head_dim, pol, par).to(dev)
        n = max(1, plan.info.num_partial_rows)
        o = torch.empty(c.q.shape[0], c.num_qo_heads, c.head_dim, device=dev)
        lse = torch.empty(c.q.shape[0], c.num_qo_heads, device=dev)
        op = torch.empty(n, c.num_qo_heads, c.head_dim, device=dev)
        lp = torch.empty(n, c.num_qo_heads, device=dev)
        e["step"] = lambda: skv.paged_attn_fwd(d["q"], d["k"], d["v"], d["kv_indptr"], d["kv_indices"],
                                               d["kv_last_page_len"], plan, o, lse, op, lp, None, c.sm_scale,
                                               c.num_pages, stream, kv_scale=c.kv_scale)
        L = c.kv_lengths()
        q_rows = np.diff(c.qo_indptr)
        per_tok = c.num_kv_heads * c.head_dim * 2 * (1 if c.kv_dtype == "e4m3" else 2)
        e["bytes"] = int(L[0] if name == "shared_kv" else L.sum()) * per_tok   # the shared KV is read once
        e["flops"] = float(np.sum(q_rows * L)) * c.num_qo_heads * 4 * c.head_dim
        e["launches"] = 1 + (1 if plan.info.num_merge_rows else 0)
        e["kernel"] = plan.info.kernel
        e["dtype"] = c.kv_dtype
        unit_work = lambda r: (float(L[r]) * per_tok, float(q_rows[r] * L[r]) * c.num_qo_heads * 4 * c.head_dim)
        e["oracle_units"] = (lambda r=r: (OA.paged_attention(c.q, c.k, c.v, c.qo_indptr, c.kv_indptr, c.kv_indices,
                                                            c.kv_last_page_len, c.page_size, c.sm_scale,
                                                            requests=[r], kv_dtype=c.kv_dtype,
                                                            kv_scale=c.kv_scale), unit_work(r))[1]
                             for r in range(c.batch))
        e["oracle_what"] = "requests (query batches)" if name == "shared_kv" else "requests"
    elif name.startswith("mla_"):
        parts = name.split("_")
        H, q, dt = int(parts[1][1:]), int(parts[2][1:]), parts[3]
        causal = len(parts) > 4 and parts[4] == "causal"
        c = mla_decode_case(H, q, dt)
        d = mla_to_device(c, dev)
        o = torch.empty(c.batch, q, H, 512, device=dev)
        lse = torch.empty(c.batch, q, H, device=dev)
        if causal:
            cm = skv.CausalMlaDecode(q, H, c.kv_indptr, c.kv_indices, c.kv_last_page_len, c.page_size, c.num_pages,
                                     dev, dt)
            e["step"] = lambda: cm(d["q_nope"], d["q_pe"], d["ckv"], d["kpe"], o, lse, sm_scale=c.sm_scale,
                                   kv_scale=c.kv_scale, stream=stream)
            e["launches"] = cm.launches()
            e["kernel"] = [cm.prefix_plan.info.kernel, cm.diag_plan.info.kernel]
        else:
            plan = skv.plan_mla(q, c.kv_indptr, c.kv_last_page_len, c.page_size, H, "balanced", 0,
                                kv_dtype=dt).to(dev)
            n = max(1, plan.info.num_partial_rows)
            op = torch.empty(n, H, 512, device=dev)
            lp = torch.empty(n, H, device=dev)
            e["step"] = lambda: skv.mla_decode_fwd(d["q_nope"], d["q_pe"], d["ckv"], d["kpe"], d["kv_indptr"],
                                                   d["kv_indices"], d["kv_last_page_len"], plan, o, lse, op, lp,
                                                   None, c.sm_scale, c.kv_scale, c.num_pages, stream)
            e["launches"] = 1 + (1 if plan.info.num_merge_rows else 0)
            e["kernel"] = plan.info.kernel
        L = c.kv_lengths()
        per_tok = 1152 if dt == "bf16" else 576
        e["bytes"] = int(L.sum()) * per_tok
        # causal: position i of q_len sees L - q_len + 1 + i keys
        vis = (lambda l: q * l - q * (q - 1) / 2) if causal else (lambda l: q * l)
        e["flops"] = float(sum(vis(float(x)) for x in L)) * H * 2 * (576 + 512)
        e["dtype"] = dt
        unit_work = lambda r: (float(L[r]) * per_tok, vis(float(L[r])) * H * 2 * (576 + 512))
        e["oracle_units"] = (lambda r=r: (OA.mla_decode(c.q_nope, c.q_pe, c.ckv, c.kpe, c.kv_indptr, c.kv_indices,
                                                       c.kv_last_page_len, c.page_size, c.sm_scale, c.kv_dtype,
                                                       c.kv_scale, requests=[r], causal=causal), unit_work(r))[1]
                             for r in range(c.batch))
        e["oracle_what"] = "requests"
    elif name in ("pod", "pod_two_launches"):
        # a Llama-shaped POD batch: 48 decode requests + 2 prefill requests (1024 query tokens over
        # 2048 KV tokens each), one attention launch or one launch per kind
        from workloads import pod_case
        c = pod_case()
        d = paged_to_device(c, dev)
        pod = skv.PodAttention(c.qo_indptr, c.kv_indptr, c.kv_last_page_len, c.page_size, c.num_qo_heads,
                               c.num_kv_heads, c.head_dim, dev, fused=name == "pod")
        o = torch.empty(c.q.shape[0], c.num_qo_heads, c.head_dim, device=dev)
        lse = torch.empty(c.q.shape[0], c.num_qo_heads, device=dev)
        e["step"] = lambda: pod(d["q"], d["k"], d["v"], d["kv_indptr"], d["kv_indices"], d["kv_last_page_len"], o,
                                lse, sm_scale=c.sm_scale, num_pages=c.num_pages, stream=stream)
        L = c.kv_lengths()
        q_rows = np.diff(c.qo_indptr)
        per_tok = c.num_kv_heads * c.head_dim * 4
        e["bytes"] = int(L.sum()) * per_tok
        e["flops"] = float(np.sum(q_rows * L)) * c.num_qo_heads * 4 * c.head_dim
        e["launches"] = pod.launches()
        e["kernel"] = {"decode_sms": pod.decode_sms, "plans": [p.info.kernel for p in pod.plans]}
        e["dtype"] = "bf16"
        unit_work = lambda r: (float(L[r]) * per_tok, float(q_rows[r] * L[r]) * c.num_qo_heads * 4 * c.head_dim)
        e["oracle_units"] = (lambda r=r: (OA.paged_attention(c.q, c.k, c.v, c.qo_indptr, c.kv_indptr, c.kv_indices,
                                                            c.kv_last_page_len, c.page_size, c.sm_scale,
                                                            requests=[r]), unit_work(r))[1]
                             for r in list(range(c.batch - 2, c.batch)) + list(range(c.batch - 2)))
        e["oracle_what"] = "requests (prefill first)"
    elif name == "route":
        c = route_case()
        d = route_to_device(c, dev)
        rm = skv.RouteMerge(c.sel, c.num_heads, dev)
        out_o = torch.empty(c.sel.shape[0], c.num_heads, 512, device=dev)
        out_l = torch.empty(c.sel.shape[0], c.num_heads, device=dev)
        e["step"] = lambda: rm(d["q_nope"], d["q_pe"], d["ckv"], d["kpe"], d["sel_cqk"], sm_scale=c.sm_scale,
                               stream=stream, o=out_o, lse=out_l)
        e["bytes"] = int(c.sel.size) * 1152              # gathered rows
        e["flops"] = float(c.sel.size) * c.num_heads * 2 * (576 + 512)
        e["launches"] = c.num_chunks + 1
        e["kernel"] = rm.plan.info.kernel
        e["dtype"] = "bf16"
        u = c.union_mla()
        per_q = (c.num_chunks * c.sel.shape[2] * 1152.0, c.num_chunks * c.sel.shape[2] * c.num_heads * 2.0 * 1088)
        e["oracle_units"] = (lambda qq=qq: (OA.mla_decode(u.q_nope, u.q_pe, u.ckv, u.kpe, u.kv_indptr, u.kv_indices,
                                                         u.kv_last_page_len, 1, u.sm_scale, requests=[qq]),
                                            per_q)[1]
                             for qq in range(c.sel.shape[0]))
        e["oracle_what"] = "queries (attention over the union of their selections)"
    elif name == "fetch_splice":
        # fetch's local compute: every chunk of the route corpus moved into a requester's paged
        # cache and re-rotated (all chunks in one call); bytes = each row read once and written once
        import oracle.splice as OS
        c = fetch_splice_case()
        d = splice_to_device(c, dev)
        sp = skv.splice_params(d["src_ckv"], d["src_kpe"], d["src_pages"], d["dst_ckv"], d["dst_kpe"],
                               d["dst_pages"], rope_theta=c.rope_theta)
        chunks = skv.splice_chunks([(int(c.src_start[ch]), int(c.dst_start[ch]), c.chunk_tokens, int(c.delta[ch]))
                                    for ch in range(c.num_chunks)])
        e["step"] = lambda: skv.splice_launch(sp, chunks, stream)
        e["bytes"] = 2 * c.num_chunks * c.chunk_tokens * 1152
        e["flops"] = 0.0
        e["launches"] = 1
        e["kernel"] = "splice"
        e["dtype"] = "bf16"
        freq = OS.rope_inv_freq(c.rope_theta)
        blk = 256
        e["oracle_units"] = (lambda ch=ch, t0=t0: (OS.splice_rows(
            c.src[..., :512], c.src[..., 512:], c.src_pages, int(c.src_start[ch]) + t0, c.dst_pages, c.dst_page_size,
            int(c.dst_start[ch]) + t0, blk, int(c.delta[ch]), freq), (2.0 * blk * 1152, 0.0))[1]
            for t0 in range(0, c.chunk_tokens, blk) for ch in range(c.num_chunks))
        e["oracle_what"] = f"blocks of {blk} tokens"
    else:
        raise SystemExit(f"unknown workload {name}")
    return e


def _config_entry(name, args, dev, stream, skv, torch, flush, peaks, peak_src, cpu_budget):
    """One configuration: device time per call (attention + merge, inputs resident, L2 flushed
    before each timed call), roofline fraction against the measured peaks, and the oracle timed on
    the host cores over a bounded sample of the same inputs."""
    e = _setup_config(name, dev, skv, torch, stream)
    hbm = float(peaks.get("hbm_gbs", FALLBACK["hbm_gbs"]))
    tf_bf16 = float(peaks.get("bf16_tflops", FALLBACK["bf16_tflops"]))
    fp8 = e["dtype"] == "e4m3"
    tf = tf_bf16 * (2.0 if fp8 else 1.0)
    tf_src = (f"{peak_src} bf16 x 2 (nominal fp8 : bf16 dense ratio; e4m3 MMAs)" if fp8
              else f"{peak_src} bf16 burst")
    steps = max(3, min(args.steps, args.config_steps))
    ms = _time_calls(e["step"], steps, max(3, min(args.warmup, 5)), torch, stream, flush)
    t_mem, t_tc = e["bytes"] / (hbm * 1e9), e["flops"] / (tf * 1e12)
    bound = "hbm" if t_mem >= t_tc else "tensor"
    gbs = e["bytes"] / (ms * 1e-3) / 1e9
    tfs = e["flops"] / (ms * 1e-3) / 1e12
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(gbs / hbm, 4), "peak_source": f"{peak_src} hbm_gbs"}
    else:
        roof = {"bound": "tensor", "achieved": round(tfs, 1), "peak": round(tf, 1), "unit": "TFLOP/s",
                "frac": round(tfs / tf, 4), "peak_source": tf_src}
    out = {"us": round(ms * 1e3, 2), "GBps": round(gbs, 1), "TFLOPs": round(tfs, 2), "kv_bytes": e["bytes"],
           "flops": e["flops"], "roofline": roof, "kernel": e["kernel"], "launches_per_call": e["launches"],
           "dtype": e["dtype"], "timed_calls": steps, "l2": "flushed (512 MB write) before every timed call"}
    if cpu_budget > 0:
        done, dt, n = _sampled(e["oracle_units"], cpu_budget)
        work, scale = (done[0], 1e9) if roof["unit"] == "GB/s" else (done[1], 1e12)
        out["cpu_baseline"] = {"value": work / dt / scale, "unit": roof["unit"], "cores": int(_threads_used()),
                               "kind": "oracle",
                               "sample": f"{n} {e['oracle_what']} of the same inputs, float64 numpy oracle, "
                                         f"{dt:.1f} s on {os.cpu_count()} visible host cores; rate extrapolates "
                                         f"linearly to the whole configuration"}
    return out


def _flush_buffer(torch, dev):
    return torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)


def run_workload(args):
    """One JSON line per named configuration (the entries of the default line's ``configs``)."""
    import torch
    import split_kv_merge_b200 as skv
    peaks, src = _peaks()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    flush = _flush_buffer(torch, dev)
    names = args.workload.split(",")
    if names == ["all"]:
        names = list(CONFIG_NAMES)
    for name in names:
        line = {"workload": name, **_config_entry(name, args, dev, stream, skv, torch, flush, peaks, src,
                                                  0.0 if args.no_cpu_baseline else args.config_cpu_budget)}
        print(json.dumps(line), flush=True)
    return 0


def all_configs(args, dev, stream, skv, torch):
    """The ``configs`` object of the default line: every configuration other than the headline."""
    peaks, src = _peaks()
    flush = _flush_buffer(torch, dev)
    out = {}
    for name in CONFIG_NAMES:
        out[name] = _config_entry(name, args, dev, stream, skv, torch, flush, peaks, src,
                                  0.0 if args.no_cpu_baseline else args.config_cpu_budget)
        torch.cuda.empty_cache()
    del flush
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--ref-budget", type=float, default=8.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=64, help="requests per GPU (64 = the benchmark workload; "
                                                          "smaller only for profiler captures)")
    ap.add_argument("--workload", default="llama70b",
                    help="llama70b (the benchmark line) | tiny | llama70b_e4m3 | shared_kv | "
                         "mla_h{16,128}_q{1,4}_{bf16,e4m3} | "
                         "mla_h16_q4_bf16_causal | pod | pod_two_launches | route | fetch_splice | all (one line "
                         "per configuration)")
    ap.add_argument("--no-configs", action="store_true", help="default line without the per-configuration block")
    ap.add_argument("--config-steps", type=int, default=20, help="timed calls per configuration (at most --steps)")
    ap.add_argument("--config-cpu-budget", type=float, default=2.0,
                    help="seconds of oracle work per configuration for its cpu_baseline")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.workload != "llama70b":
        return run_workload(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
