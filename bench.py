#!/usr/bin/env python
"""Benchmark of the B200 paged latent-attention path (one ``mla_run`` per step).

Default workload: batch-64 decode (q_len 1, H = 128, kv lens ~ U{512..8192},
page_size 64), whose headline metric is KV GB/s (KV bytes = kv_len x 576 x 2 per
row, read once for all heads).  A step is one full pass of the hot path (attention
kernel + split-KV merge kernel) over one batch whose inputs are already in HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the fp64 CPU oracle on a bounded sample

Under torchrun (N > 1) every rank runs an independent replica of the workload on its
own GPU (the path has no cross-GPU exchange); ``value`` sums the ranks' bytes over the
slowest rank's device time.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA attn: decode KV GB/s (frac of HBM peak); prefill TFLOP/s (frac of bf16 peak)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLOP_PER_VISIT = 2 * 576 + 2 * 512  # QK^T over 576 columns + P.V over 512 columns
KV_BYTES_PER_KEY = 576 * 2
L2_BYTES = 126 * 1024 * 1024


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="decode_b64")
    ap.add_argument("--no-others", action="store_true", help="skip the other workloads' summary")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle CPU-baseline budget (0: skip)")
    ap.add_argument("--soak", type=float, default=1.5, help="untimed seconds of steps while clocks are sampled")
    ap.add_argument("--copies", type=int, default=0, help="HBM copies of the inputs to rotate (0: auto)")
    ap.add_argument("--no-next", action="store_true",
                    help="skip the measurements of graph replay, append, cascade and plan reuse")
    return ap.parse_args()


# ------------------------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def work_of(d):
    """Algorithmic work of a workload: KV bytes (each row's keys once), score/value
    flops over visible (query, head, key) triples, and the other bytes moved."""
    kv_bytes = sum(int(k) * KV_BYTES_PER_KEY for k in d.kv_lens)
    visits = 0
    for q, k in zip(d.q_lens, d.kv_lens):
        if d.causal:
            visits += sum(min(k, max(0, k - q + i + 1)) for i in range(q))
        else:
            visits += q * k
    T, H = d.total_tokens, d.num_heads
    flops = visits * H * FLOP_PER_VISIT
    other = T * H * (576 * 2 + 512 * 2 + (4 if d.return_lse else 0))
    return {"kv_bytes": kv_bytes, "flops": flops, "visits": visits * H, "other_bytes": other}


class ClockSampler:
    """nvidia-smi samples (every 100 ms) of SM clock and throttle reasons."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clk_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    rows.append(parts)
                except Exception:
                    pass
        os.unlink(self.path)
        if not rows:
            return None
        def num(x):
            try:
                return float(x)
            except ValueError:
                return float("nan")
        busy = [r for r in rows if num(r[4]) >= 50] or rows
        sm = [num(r[1]) for r in busy if not math.isnan(num(r[1]))]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in busy:
            for nm, v in zip(names, r[6:10]):
                if v.strip().lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": num(rows[0][2]),
                "reasons": sorted(reasons),
                "samples": len(rows), "samples_busy": len(busy),
                "power_w_max": max(num(r[3]) for r in rows)}


def kernel_traffic(workload: str):
    """DRAM bytes per launch of the attention kernel from the committed ncu summary, if
    the kernel source still hashes to what was profiled; else None."""
    path = os.path.join(ROOT, "profiles", f"mla_attn_kernel__{workload}.txt")
    src = os.path.join(ROOT, "paged_head_latent_mla_b200", "csrc", "mla_attn.cu")
    try:
        kv = {}
        with open(path) as f:
            for line in f:
                if ":" in line:
                    k, v = line.split(":", 1)
                    kv[k.strip()] = v.strip()
        with open(src, "rb") as f:
            h = hashlib.sha256(f.read()).hexdigest()[:16]
        if kv.get("kernel_source_sha256_16") != h:
            return None
        return float(kv["dram_bytes_per_launch"])
    except Exception:
        return None


# ------------------------------------------------------------------------------- oracle legs
def oracle_sample(d, budget_s: float, max_rows=None):
    """Run the fp64 oracle row by row (rows in order) until `budget_s` of wall time;
    return (seconds, kv bytes covered, rows done, threads)."""
    from oracle import mla_oracle as O

    qo = d.qo_indptr.numpy()
    B = len(qo) - 1
    t0 = time.perf_counter()
    done, kvb = 0, 0
    for b in range(B if max_rows is None else min(B, max_rows)):
        toks = range(int(qo[b]), int(qo[b + 1]))
        O.mla_attention(d.q_nope, d.q_pe, d.cache, d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len,
                        d.page_size, d.sm_scale, causal=d.causal, tokens=toks)
        done += 1
        kvb += int(d.kv_lens[b]) * KV_BYTES_PER_KEY
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info

        threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=os.cpu_count())
    except Exception:
        threads = os.cpu_count()
    return dt, kvb, done, threads


L2_NOTE = ("GPU arm: inputs rotated over HBM copies (at least 3x L2 in total where memory allows), never "
           "L2-resident between steps")


def config_of(name, d):
    """The workload description both arms print (identical dicts for the same workload)."""
    w = work_of(d)
    return {"workload": name, "description": d.description, "kv_bytes_per_step": w["kv_bytes"],
            "flops_per_step": w["flops"], "l2": L2_NOTE}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from workloads import make_config

    d = make_config(args.workload)
    per_step = max(0.5, min(4.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(d, per_step)
    times, kvbs, rows = [], [], 0
    threads = os.cpu_count()
    for _ in range(args.steps):
        dt, kvb, n, threads = oracle_sample(d, per_step)
        times.append(dt)
        kvbs.append(kvb)
        rows = n
    total_t, total_b = sum(times), sum(kvbs)
    value = total_b / total_t / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(args.workload, d),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"each step: the first {rows} rows of {args.workload} (all their queries), "
                                   f"fp64 NumPy oracle, ~{per_step:.1f} s budget"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------- native leg
def make_runner(d, device, n_copies, timing=True, plan_kw=None):
    """Plan once; keep `n_copies` copies of the inputs in HBM and rotate through them so
    consecutive steps never find their inputs in L2.  With `timing` the plan records CUDA
    events around each of its launches (kernel durations for the roofline); those events
    sit between the attention and merge launches."""
    import ctypes

    import torch

    import paged_head_latent_mla_b200 as M

    plan = M.mla_plan(d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len, num_heads=d.num_heads,
                      page_size=d.page_size, num_pages=d.num_pages, sm_scale=d.sm_scale, causal=d.causal,
                      debug_flags=M.MLA_DEBUG_KERNEL_TIMING if timing else 0, **(plan_kw or {}))
    copies = []
    for _ in range(n_copies):
        copies.append((d.q_nope.to(device), d.q_pe.to(device), d.cache.to(device)))
    T, H = d.total_tokens, d.num_heads
    out = torch.empty((T, H, 512), dtype=torch.bfloat16, device=device)
    lse = torch.empty((T, H), dtype=torch.float32, device=device) if d.return_lse else None
    lib = M.load_library()
    stream = ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    args = [(plan.handle, ctypes.c_void_p(qn.data_ptr()), ctypes.c_void_p(qp.data_ptr()),
             ctypes.c_void_p(c.data_ptr()), ctypes.c_void_p(out.data_ptr()),
             ctypes.c_void_p(lse.data_ptr() if lse is not None else 0), stream) for (qn, qp, c) in copies]
    state = {"i": 0}

    def step():
        a = args[state["i"] % len(args)]
        state["i"] += 1
        st = lib.mla_run(*a)
        if st != 0:
            raise M.MlaError(st, "mla_run")

    return plan, step, out, lse, copies


def input_bytes(d):
    return d.cache.numel() * 2 + d.q_nope.numel() * 2 + d.q_pe.numel() * 2


def time_workload(d, device, steps, warmup, dist=None, soak_s=0.0, sampler=None, copies=0, plan_kw=None):
    """Time K steps of the workload on resident inputs.

    The timed region runs the steps through a plan that records CUDA events around each
    of its launches (before the attention kernel, between it and the merge kernel, after
    the merge), so the step time and the per-kernel durations come from the same K steps
    under the same clocks: a kernel can never read longer than the step that contains it.
    The region is bracketed by a barrier and a device synchronise and timed with CUDA
    events on the launch stream.  Afterwards the same K steps run once more through a
    plain plan (no events between the launches, the merge set up while the attention
    drains): the product path's own step time, reported beside the headline."""
    import torch

    import paged_head_latent_mla_b200 as M

    n_copies = copies or max(1, min(4, math.ceil(3 * L2_BYTES / max(1, input_bytes(d)))))
    free, _ = torch.cuda.mem_get_info(device)
    while n_copies > 1 and n_copies * input_bytes(d) > 0.6 * free:
        n_copies -= 1
    tplan, tstep, out, lse, copies_ = make_runner(d, device, n_copies, timing=True, plan_kw=plan_kw)
    plan = M.mla_plan(d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len, num_heads=d.num_heads,
                      page_size=d.page_size, num_pages=d.num_pages, sm_scale=d.sm_scale, causal=d.causal,
                      **(plan_kw or {}))
    lib = M.load_library()
    import ctypes
    stream = ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    pargs = [(plan.handle, ctypes.c_void_p(qn.data_ptr()), ctypes.c_void_p(qp.data_ptr()),
              ctypes.c_void_p(c.data_ptr()), ctypes.c_void_p(out.data_ptr()),
              ctypes.c_void_p(lse.data_ptr() if lse is not None else 0), stream) for (qn, qp, c) in copies_]
    pstate = {"i": 0}

    def pstep():
        a_ = pargs[pstate["i"] % len(pargs)]
        pstate["i"] += 1
        st_ = lib.mla_run(*a_)
        if st_ != 0:
            raise M.MlaError(st_, "mla_run")

    info = M.mla_plan_get_info(tplan)
    for _ in range(warmup):
        tstep()
        pstep()
    torch.cuda.synchronize(device)
    for pl in (plan, tplan):
        st = M.mla_plan_check(pl)
        if st != 0:
            raise M.MlaError(st, "warm-up")
    if sampler is not None:
        sampler.start()
    if soak_s > 0:  # untimed: brings the clocks to their level under this load, sampled
        t_end = time.perf_counter() + soak_s
        while time.perf_counter() < t_end:
            for _ in range(20):
                tstep()
            torch.cuda.synchronize(device)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e2 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        tstep()
    e1.record()
    torch.cuda.synchronize(device)
    if dist is not None:
        dist.barrier()
    # The product path without events between its launches, the same steps, enqueued
    # at once so that it runs under the same (power-capped) clocks; a pause here would
    # let the clocks recover and flatter it.
    for _ in range(steps):
        pstep()
    e2.record()
    torch.cuda.synchronize(device)
    clocks = sampler.stop() if sampler is not None else None
    ms = e0.elapsed_time(e1)
    ms_plain = e1.elapsed_time(e2)
    attn_ms, merge_ms = M.mla_plan_kernel_times(tplan, capacity=min(steps, 256))
    for pl in (plan, tplan):
        st = M.mla_plan_check(pl)
        if st != 0:
            raise M.MlaError(st, "timed steps")
    res = {"ms_total": ms, "ms_per_step": ms / steps, "ms_per_step_plain": ms_plain / steps,
           "attn_ms": float(attn_ms.mean()),
           "attn_ms_median": float(statistics.median(attn_ms.tolist())), "attn_ms_min": float(attn_ms.min()),
           "merge_ms": float(merge_ms.mean()), "info": info, "n_copies": n_copies, "clocks": clocks,
           "launches": steps * (1 + (1 if info["num_merge"] > 0 else 0))}
    plan.destroy()
    tplan.destroy()
    del copies_, out, lse
    torch.cuda.empty_cache()
    return res


def time_e2e(d, device, steps, warmup):
    """The public API end to end with host buffers.  Every step plans from host tables
    (mla_plan: uploads the work lists and page table), copies the step's queries from
    pinned host memory, runs, and copies out/lse back to pinned host memory.  Steps are
    pipelined two deep the way a serving loop overlaps them: step i's queries go up on a
    copy stream while step i-1 computes, and step i-1's result comes down on another
    while step i computes (separate device buffers per step parity).  Each plan's status
    is read when it is retired, two steps later.  The timed region covers `steps`
    complete steps, from before the first plan to the last result on the host, on the
    device clock."""
    import torch

    import paged_head_latent_mla_b200 as M

    T, H = d.total_tokens, d.num_heads
    cache = d.cache.to(device)  # the KV cache is resident state, written by earlier steps
    qn_h = d.q_nope.pin_memory()
    qp_h = d.q_pe.pin_memory()
    bufs = []
    for _ in range(2):
        bufs.append({
            "qn": torch.empty_like(qn_h, device=device),
            "qp": torch.empty_like(qp_h, device=device),
            "out": torch.empty((T, H, 512), dtype=torch.bfloat16, device=device),
            "lse": torch.empty((T, H), dtype=torch.float32, device=device) if d.return_lse else None,
            "out_h": torch.empty((T, H, 512), dtype=torch.bfloat16).pin_memory(),
            "lse_h": torch.empty((T, H), dtype=torch.float32).pin_memory() if d.return_lse else None,
            "uploaded": torch.cuda.Event(), "computed": torch.cuda.Event(), "downloaded": torch.cuda.Event(),
        })
    s_up, s_run, s_down = torch.cuda.Stream(device), torch.cuda.Stream(device), torch.cuda.Stream(device)
    h2d = [0]
    live = []  # (plan) of steps not yet retired

    def retire(plan):
        st = M.mla_plan_check(plan)  # waits for that step's launches, reads its status word
        if st != 0:
            raise M.MlaError(st, "e2e")
        plan.destroy()

    def one(i):
        b = bufs[i % 2]
        # the plan's upload goes on the upload stream ahead of the queries (on the compute
        # stream it would wait for step i-1's run, then queue behind step i+1's query copy
        # in the copy engine); `uploaded` orders the run after both
        plan = M.mla_plan(d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len, num_heads=H,
                          page_size=d.page_size, num_pages=d.num_pages, sm_scale=d.sm_scale, causal=d.causal,
                          stream=s_up.cuda_stream)
        info = M.mla_plan_get_info(plan)
        with torch.cuda.stream(s_up):
            s_up.wait_event(b["computed"])  # step i-2 has finished reading these buffers
            b["qn"].copy_(qn_h, non_blocking=True)
            b["qp"].copy_(qp_h, non_blocking=True)
            b["uploaded"].record(s_up)
        with torch.cuda.stream(s_run):
            s_run.wait_event(b["uploaded"])
            s_run.wait_event(b["downloaded"])  # step i-2's result has left `out`
            M.mla_run(plan, b["qn"], b["qp"], cache, out=b["out"], lse=b["lse"], stream=s_run.cuda_stream)
            b["computed"].record(s_run)
        with torch.cuda.stream(s_down):
            s_down.wait_event(b["computed"])
            b["out_h"].copy_(b["out"], non_blocking=True)
            if b["lse"] is not None:
                b["lse_h"].copy_(b["lse"], non_blocking=True)
            b["downloaded"].record(s_down)
        live.append(plan)
        if len(live) > 2:
            retire(live.pop(0))
        # work list, merge list and references, append rows, page table
        plan_bytes = (32 * info["num_work"] + 16 * info["num_merge"] + 4 * info["num_merge_refs"] + 4 * T +
                      4 * int(d.kv_indptr[-1]))
        h2d[0] = plan_bytes + qn_h.numel() * 2 + qp_h.numel() * 2

    for i in range(warmup):
        one(i)
    while live:
        retire(live.pop(0))
    torch.cuda.synchronize(device)
    # device clock: from an event the upload stream passes before the first step's plan
    # upload to one the download stream passes after the last result reached the host
    # (host planning time shows up as device idle time inside the span)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    for i in range(steps):
        one(i)
    for b in bufs:
        s_down.wait_event(b["downloaded"])
    e1.record(s_down)
    e1.synchronize()
    while live:
        retire(live.pop(0))
    ms = e0.elapsed_time(e1) / steps
    d2h = T * H * 512 * 2 + (T * H * 4 if d.return_lse else 0) + 4
    del cache, bufs
    torch.cuda.empty_cache()
    return ms, h2d[0], d2h


def time_e2e_cpp(d, steps, warmup, device_index=0):
    """The same end-to-end loop as time_e2e, written as a C++ client of the C ABI
    (tests/c/e2e_driver.cpp): per step mla_plan from host tables, H2D of the queries from
    pinned memory, mla_run, D2H of the result to pinned memory, pipelined two deep on
    three streams, each plan retired two steps later.  Returns (ms/step, h2d bytes, d2h
    bytes), or a dict with an error when no compiler is at hand or the run fails."""
    import shutil

    import numpy as np
    import torch

    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        return {"error": "no C++ compiler"}
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    pkg = os.path.join(ROOT, "paged_head_latent_mla_b200")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "e2e_driver")
        r = subprocess.run([cxx, "-O2", "-std=c++17", "-I", os.path.join(ROOT, "include"), "-I",
                            os.path.join(cuda, "include"), os.path.join(ROOT, "tests", "c", "e2e_driver.cpp"),
                            "-L", pkg, "-l:libmla_b200.so", "-L", os.path.join(cuda, "lib64"), "-lcudart",
                            "-Wl,-rpath," + pkg + ":" + os.path.join(cuda, "lib64"), "-o", exe],
                           capture_output=True, text=True)
        if r.returncode != 0:
            return {"error": r.stderr[-300:]}
        hdr = np.array([d.num_heads, d.page_size, d.num_pages, d.batch, 1 if d.causal else 0], np.int32)
        with open(os.path.join(tmp, "tables"), "wb") as f:
            for a in (hdr, d.qo_indptr.numpy(), d.kv_indptr.numpy(), d.kv_indices.numpy(),
                      d.last_page_len.numpy()):
                f.write(np.ascontiguousarray(a, dtype=np.int32).tobytes())
        for name, t in (("q_nope.bin", d.q_nope), ("q_pe.bin", d.q_pe), ("cache.bin", d.cache)):
            with open(os.path.join(tmp, name), "wb") as f:
                f.write(t.contiguous().view(torch.int16).numpy().tobytes())
        with open(os.path.join(tmp, "lse"), "wb") as f:
            f.write(np.array([1 if d.return_lse else 0], np.int32).tobytes())
        r = subprocess.run([exe, tmp, str(steps), str(warmup), repr(float(d.sm_scale)), str(device_index)],
                           capture_output=True, text=True, timeout=300)
        if r.returncode != 0:
            return {"error": f"rc {r.returncode}: {r.stderr[-300:]}"}
        out = dict(line.split() for line in r.stdout.strip().splitlines())
        if int(out["status"]) != 0:
            return {"error": f"device status {out['status']}"}
        return float(out["ms_per_step"]), int(out["h2d_bytes_per_step"]), int(out["d2h_bytes_per_step"])


def summarise(d, res, peaks):
    w = work_of(d)
    s = res["ms_per_step"] * 1e-3
    a = res["attn_ms"] * 1e-3
    return {
        "us_per_step": res["ms_per_step"] * 1e3,
        "us_per_step_plain": res["ms_per_step_plain"] * 1e3,
        "attn_kernel_us": res["attn_ms"] * 1e3,
        "attn_kernel_us_median": res["attn_ms_median"] * 1e3,
        "attn_kernel_us_min": res["attn_ms_min"] * 1e3,
        "merge_kernel_us": res["merge_ms"] * 1e3,
        "kv_gbs": w["kv_bytes"] / s / 1e9,
        "tflops": w["flops"] / s / 1e12,
        "attn_kernel_kv_gbs": w["kv_bytes"] / a / 1e9,
        "attn_kernel_tflops": w["flops"] / a / 1e12,
        "frac_hbm": w["kv_bytes"] / s / 1e9 / peaks["hbm_gbs"],
        "frac_tensor": w["flops"] / s / 1e12 / peaks["bf16_tflops"],
        "work_items": res["info"]["num_work"],
        "split_tiles": res["info"]["num_merge"],
        "kv_bytes": w["kv_bytes"],
        "flops": w["flops"],
        "clocks": res.get("clocks"),
    }


def _events_ms(fn, device, n, flush=None):
    """Mean device time of `fn` over n calls, each bracketed by its own CUDA events on the
    current stream; `flush` (outside the events) runs before every call."""
    import torch

    ms = 0.0
    for _ in range(n):
        if flush is not None:
            flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize(device)
        ms += a.elapsed_time(b)
    return ms / n


def measure_next_rows(device, peaks):
    """The entry points around the attention, each on its own workload:
    * graph replay: the tiny decode step replayed from a captured CUDA graph (a graph
      plan) against the same step launched eagerly, device time per step (L2-warm: the
      step reads 215 KB, so this is launch latency);
    * append: mla_append_kv of the mixed chunked-prefill step's 4156 tokens (1152 B read
      and written per token), L2 flushed before each launch, against HBM bandwidth; and
      mla_run_append against mla_run per step (decode_b64, mixed_prefill), the cost the
      append adds when the attention is its programmatic dependent;
    * cascade: the speculative shared-prefix rows at 16 heads with and without the cascade;
    * plan reuse: host time of mla_plan_update on an unchanged decode step (skipped
      re-plan) against a changed one and a fresh mla_plan."""
    import torch

    import paged_head_latent_mla_b200 as M
    from workloads import make_config, make_custom

    res = {}
    stream = torch.cuda.current_stream(device)

    # --- graph replay vs eager, tiny decode
    d = make_config("tiny_decode")
    qn, qp, cache = d.q_nope.to(device), d.q_pe.to(device), d.cache.to(device)
    T, H = d.total_tokens, d.num_heads
    out = torch.empty((T, H, 512), dtype=torch.bfloat16, device=device)
    lse = torch.empty((T, H), dtype=torch.float32, device=device)
    eager = M.mla_plan(d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len, num_heads=H,
                       page_size=d.page_size, num_pages=d.num_pages, sm_scale=d.sm_scale, causal=d.causal)
    gplan = M.mla_plan(d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len, num_heads=H,
                       page_size=d.page_size, num_pages=d.num_pages, sm_scale=d.sm_scale, causal=d.causal,
                       graph_max_batch=d.batch, graph_max_tokens=T, graph_max_page_ids=int(d.kv_indptr[-1]))
    n = 200
    for _ in range(5):
        M.mla_run(eager, qn, qp, cache, out=out, lse=lse)
        M.mla_run(gplan, qn, qp, cache, out=out, lse=lse)
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(n):
        M.mla_run(eager, qn, qp, cache, out=out, lse=lse)
    b.record()
    torch.cuda.synchronize(device)
    eager_us = a.elapsed_time(b) / n * 1e3
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(device)
    s.wait_stream(stream)
    with torch.cuda.graph(g, stream=s):
        for _ in range(10):
            M.mla_run(gplan, qn, qp, cache, out=out, lse=lse)
    torch.cuda.synchronize(device)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize(device)
    a.record()
    for _ in range(n // 10):
        g.replay()
    b.record()
    torch.cuda.synchronize(device)
    graph_us = a.elapsed_time(b) / n * 1e3
    for pl in (eager, gplan):
        if M.mla_plan_check(pl) != 0:
            raise M.MlaError(M.mla_plan_check(pl), "graph replay")
    res["graph_replay_tiny_decode"] = {
        "eager_us_per_step": eager_us, "graph_us_per_step": graph_us,
        "work_capacity": M.mla_plan_get_info(gplan)["work_capacity"],
        "note": "10 steps per captured graph; both on the same inputs, L2-warm (215 KB per step)"}
    del g
    eager.destroy()
    gplan.destroy()

    # --- append bandwidth, mixed chunked-prefill tokens
    d = make_config("mixed_prefill")
    T = d.total_tokens
    cache = d.cache.to(device)
    kv_new = (torch.randn((T, 576), generator=torch.Generator().manual_seed(5)) * 0.5).to(torch.bfloat16).to(device)
    plan = M.mla_plan(d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len, num_heads=d.num_heads,
                      page_size=d.page_size, num_pages=d.num_pages, sm_scale=d.sm_scale, causal=d.causal)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
    for _ in range(3):
        M.mla_append_kv(plan, kv_new, cache)
    ms = _events_ms(lambda: M.mla_append_kv(plan, kv_new, cache), device, 20, flush=lambda: flush.fill_(1.0))
    moved = 2 * 1152 * T
    res["append_mixed_prefill"] = {"tokens": T, "us": ms * 1e3, "bytes": moved, "gbs": moved / (ms * 1e-3) / 1e9,
                                   "frac_hbm": moved / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                   "note": "L2 flushed before each launch; 1152 B read + 1152 B written per token"}
    plan.destroy()
    del cache, flush, kv_new
    torch.cuda.empty_cache()

    # --- the append fused ahead of the attention (mla_run_append, the attention launched as
    # its programmatic dependent) against the attention alone, per step
    fused = {}
    for name in ("decode_b64", "mixed_prefill"):
        d = make_config(name)
        T = d.total_tokens
        qn, qp, cache = d.q_nope.to(device), d.q_pe.to(device), d.cache.to(device)
        kv_new = (torch.randn((T, 576), generator=torch.Generator().manual_seed(6)) * 0.5).to(torch.bfloat16)
        kv_new = kv_new.to(device)
        out = torch.empty((T, d.num_heads, 512), dtype=torch.bfloat16, device=device)
        plan = M.mla_plan(d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len, num_heads=d.num_heads,
                          page_size=d.page_size, num_pages=d.num_pages, sm_scale=d.sm_scale, causal=d.causal)
        # the two variants alternate in short batches, so both see the same clocks (steps of
        # milliseconds at the power cap drift the SM clock over a long sequence)
        variants = (("run", {}), ("run_append", {"kv_new": kv_new}))
        for _ in range(3):
            for _, kw in variants:
                M.mla_run(plan, qn, qp, cache, out=out, **kw)
        torch.cuda.synchronize(device)
        times = {label: 0.0 for label, _ in variants}
        batches, per_batch = 4, 5  # short batches keep launches queued back to back
        for _ in range(batches):
            for label, kw in variants:
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                for _ in range(per_batch):
                    M.mla_run(plan, qn, qp, cache, out=out, **kw)
                b.record()
                b.synchronize()
                times[label] += a.elapsed_time(b) / (batches * per_batch) * 1e3
        if M.mla_plan_check(plan) != 0:
            raise M.MlaError(M.mla_plan_check(plan), "run_append")
        plan.destroy()
        fused[name] = {"tokens": T, "run_us": times["run"], "run_append_us": times["run_append"],
                       "append_cost_us": times["run_append"] - times["run"]}
        del qn, qp, cache, kv_new, out
        torch.cuda.empty_cache()
    res["run_append_vs_run"] = fused

    # --- cascade on/off: the speculative shared-prefix rows with 16 query heads (with 128
    # heads a token fills a query tile by itself and the planner applies no cascade)
    t = make_config("spec_shared_prefix", tables_only=True)
    d = make_custom(t.q_lens, t.kv_lens, 16, 64, shared_group=8, shared_pages=16, seed=0,
                    name="spec_shared_prefix_h16")
    base = summarise(d, time_workload(d, device, 20, 3), peaks)
    casc_res = time_workload(d, device, 20, 3, plan_kw={"cascade": True})
    casc = summarise(d, casc_res, peaks)
    res["cascade_spec_shared_prefix_h16"] = {
        "off_tflops": base["tflops"], "on_tflops": casc["tflops"],
        "off_us": base["us_per_step"], "on_us": casc["us_per_step"],
        "off_kv_gbs": base["kv_gbs"], "on_kv_gbs": casc["kv_gbs"],
        "cascade_items": casc_res["info"]["num_cascade"], "work_items": casc_res["info"]["num_work"],
        "note": "rows, lengths and prefix groups of spec_shared_prefix with H=16: a prefix tile packs two rows' "
                "4 x 16 query rows; TFLOP/s and GB/s count the same algorithmic work either way"}
    del d
    torch.cuda.empty_cache()

    # --- plan reuse, host time
    d = make_config("decode_b64", tables_only=True)
    d2 = make_config("decode_b64", seed=1, tables_only=True)
    plan = M.mla_plan(d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len, num_heads=d.num_heads,
                      page_size=d.page_size, num_pages=max(d.num_pages, d2.num_pages), sm_scale=d.sm_scale,
                      causal=d.causal)
    tabs = [(x.qo_indptr.numpy(), x.kv_indptr.numpy(), x.kv_indices.numpy(), x.last_page_len.numpy()) for x in (d, d2)]

    def host_us(fn, n=100):
        t0 = time.perf_counter()
        for i in range(n):
            fn(i)
        return (time.perf_counter() - t0) / n * 1e6

    sid = torch.cuda.current_stream(device).cuda_stream  # given once, as a serving loop would
    reuse_us = host_us(lambda i: M.mla_plan_update(plan, *tabs[0], stream=sid))
    replan_us = host_us(lambda i: M.mla_plan_update(plan, *tabs[i % 2], stream=sid))

    # fresh plans, each destroyed two steps later (as a pipelined serving loop retires
    # them); only the mla_plan calls are timed
    live, spent = [], 0.0
    for i in range(103):
        t0 = time.perf_counter()
        pl = M.mla_plan(*tabs[i % 2], num_heads=d.num_heads, page_size=d.page_size,
                        num_pages=max(d.num_pages, d2.num_pages), sm_scale=d.sm_scale, causal=d.causal,
                        stream=sid)
        if i >= 3:
            spent += time.perf_counter() - t0
        live.append(pl)
        if len(live) > 2:
            live.pop(0).destroy()
    for pl in live:
        pl.destroy()
    fresh_us = spent / 100 * 1e6
    torch.cuda.synchronize(device)
    plan.destroy()
    res["plan_reuse_decode_b64"] = {"unchanged_update_us": reuse_us, "changed_update_us": replan_us,
                                    "fresh_plan_us": fresh_us,
                                    "cpp": plan_timer_cpp(d, d2),
                                    "note": "host wall time per call, from numpy tables (binding included); "
                                            "'cpp': the same calls from a C++ client of the C ABI"}
    return res


def plan_timer_cpp(d, d2, iters=200):
    """Host time of mla_plan / mla_plan_update on the steps' tables, measured by the C++
    client tests/c/plan_timer.cpp through the C ABI (real plans on the current device:
    uploads enqueued, no synchronisation).  None if no C++ compiler is at hand."""
    import shutil

    import numpy as np

    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        return None
    pkg = os.path.join(ROOT, "paged_head_latent_mla_b200")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "plan_timer")
        r = subprocess.run([cxx, "-O2", "-std=c++17", "-I", os.path.join(ROOT, "include"),
                            os.path.join(ROOT, "tests", "c", "plan_timer.cpp"), "-L", pkg, "-l:libmla_b200.so",
                            "-Wl,-rpath," + pkg, "-o", exe], capture_output=True, text=True)
        if r.returncode != 0:
            return {"error": r.stderr[-300:]}
        tables = os.path.join(tmp, "steps.tables")
        with open(tables, "wb") as f:
            for x in (d, d2):
                hdr = np.array([x.num_heads, x.page_size, max(d.num_pages, d2.num_pages), x.batch,
                                1 if x.causal else 0], np.int32)
                for a in (hdr, x.qo_indptr.numpy(), x.kv_indptr.numpy(), x.kv_indices.numpy(),
                          x.last_page_len.numpy()):
                    f.write(np.ascontiguousarray(a, dtype=np.int32).tobytes())
        env = dict(os.environ)
        r = subprocess.run([exe, tables, str(iters), "0"], capture_output=True, text=True, timeout=300, env=env)
        if r.returncode != 0:
            return {"error": f"rc {r.returncode}: {r.stderr[-300:]}"}
        out = {}
        for line in r.stdout.strip().splitlines():
            k, v = line.split()
            out[k + "_us"] = float(v)
        return out


def reduce_max_over_ranks(x: float, dist, device) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    if dist is None:
        return x
    import torch

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job GB/s: every rank's bytes over the slowest rank's time."""
    return world * bytes_per_rank / (ms_max * 1e-3) / 1e9


def run_native(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as tdist

        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local))
        dist = tdist
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)

    from paged_head_latent_mla_b200 import _build

    _build.build()
    from workloads import CONFIG_NAMES, make_config

    peaks, peak_kind = load_peaks()
    d = make_config(args.workload)
    w = work_of(d)
    sampler = ClockSampler(local)
    res = time_workload(d, device, args.steps, max(3, args.warmup), dist=dist, soak_s=args.soak, sampler=sampler,
                        copies=args.copies)
    ms = reduce_max_over_ranks(res["ms_per_step"], dist, device)
    value = job_throughput(w["kv_bytes"], world, ms)
    summ = summarise(d, res, peaks)

    e2e = None
    if not args.no_e2e:
        e2e_steps = max(5, min(args.steps, 30))
        py_ms, py_h2d, py_d2h = time_e2e(d, device, e2e_steps, 3)
        py_ms = reduce_max_over_ranks(py_ms, dist, device)
        loop = ("per step: mla_plan from host tables (its upload on the copy stream) + H2D of queries from pinned "
                "memory + mla_run + D2H of out/lse to pinned memory; steps pipelined two deep on separate copy "
                "and compute streams; each "
                "plan's status word read two steps later; CUDA events from before the first plan to the last "
                "result on the host")
        e2e_python = {"value": job_throughput(w["kv_bytes"], world, py_ms), "unit": "GB/s",
                      "h2d_bytes_per_step": int(py_h2d), "d2h_bytes_per_step": int(py_d2h), "ms_per_step": py_ms,
                      "client": "Python binding (paged_head_latent_mla_b200)"}
        cpp = time_e2e_cpp(d, e2e_steps, 3, device_index=device.index)
        # every rank takes the same collective steps: a failed C++ run reports inf
        cpp_ms = reduce_max_over_ranks(cpp[0] if isinstance(cpp, tuple) else float("inf"), dist, device)
        if isinstance(cpp, tuple) and cpp_ms != float("inf"):
            e2e = {"value": job_throughput(w["kv_bytes"], world, cpp_ms), "unit": "GB/s",
                   "h2d_bytes_per_step": cpp[1], "d2h_bytes_per_step": cpp[2], "ms_per_step": cpp_ms,
                   "client": "C++ through the C ABI (tests/c/e2e_driver.cpp)", "includes": loop,
                   "python": e2e_python}
        else:
            e2e = dict(e2e_python, includes=loop,
                       cpp_error=cpp.get("error") if isinstance(cpp, dict) else "failed on another rank")

    others = {}
    cpu = None
    if rank == 0 and world == 1:
        if not args.no_others:
            for name in CONFIG_NAMES:
                if name == args.workload:
                    continue
                od = make_config(name)
                ores = time_workload(od, device, max(10, min(args.steps, 50)), 3, soak_s=0.5,
                                     sampler=ClockSampler(local))
                others[name] = {k: (round(v, 4) if isinstance(v, float) else v)
                                for k, v in summarise(od, ores, peaks).items()}
                del od
        if args.cpu_seconds > 0:
            dt, kvb, rows, threads = oracle_sample(d, args.cpu_seconds)
            cpu = {"value": kvb / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
                   "sample": f"first {rows} of {d.batch} rows of {args.workload} (all heads), fp64 NumPy "
                             f"oracle, {dt:.1f} s wall"}

    next_rows = None
    if rank == 0 and world == 1 and not args.no_next:
        next_rows = measure_next_rows(device, peaks)

    attn_s = res["attn_ms"] * 1e-3
    traffic = kernel_traffic(args.workload)
    roofline = {
        "bound": "hbm",
        "kernel": "mla_attn_kernel",
        "achieved": w["kv_bytes"] / attn_s / 1e9,
        "peak": peaks["hbm_gbs"],
        "unit": "GB/s",
        "frac": w["kv_bytes"] / attn_s / 1e9 / peaks["hbm_gbs"],
        "traffic": traffic,
        "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback",
        "algorithmic_bytes_per_launch": w["kv_bytes"],
        "kernel_us": res["attn_ms"] * 1e3,
        "kernel_us_median": res["attn_ms_median"] * 1e3,
        "kernel_us_min": res["attn_ms_min"] * 1e3,
        "tensor_achieved_tflops": w["flops"] / attn_s / 1e12,
        "tensor_frac": w["flops"] / attn_s / 1e12 / peaks["bf16_tflops"],
        "note": "decode at H=128 does 242 flop per KV byte, just under the ridge; both fractions are reported",
    }
    rooflines_other = {}
    for name in ("mixed_prefill", "spec_shared_prefix"):
        o = others.get(name)
        if not o:
            continue
        achieved = o["flops"] / (o["attn_kernel_us"] * 1e-6) / 1e12
        rooflines_other[name] = {
            "bound": "tensor", "kernel": "mla_attn_kernel", "achieved": achieved,
            "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
            "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
            "peak_sustained": peaks["bf16_tflops_sustained"],
            "traffic": kernel_traffic(name),
            "peak_source": f"{peak_kind} (MEASURED_PEAKS.json bf16_tflops burst; bf16_tflops_sustained beside)"
                           if peak_kind == "measured" else "fallback",
            "algorithmic_flops_per_launch": o["flops"], "kernel_us": o["attn_kernel_us"],
            "step_us": o["us_per_step"],
            "note": "2176 flop per visible (query row x head x key); kernel and step from the same timed steps",
        }
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(3, args.warmup),
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": config_of(args.workload, d),
        "parallelism": f"replicas x{world}",
        "l2_detail": f"inputs rotated over {res['n_copies']} HBM copies ({input_bytes(d) / 1e6:.0f} MB each)",
        "roofline": roofline,
        "rooflines_other": rooflines_other,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": res["launches"],
        "clocks": res["clocks"],
        "tflops": summ["tflops"],
        "frac_tensor": summ["frac_tensor"],
        "us_per_step_plain": summ["us_per_step_plain"],
        "others": others,
        "next_rows": next_rows,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
