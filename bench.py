#!/usr/bin/env python
"""Decode-attention benchmark (one JSON line on rank 0).

A step is one whole decode pass over one batch: plan (host split of the KV
tiles over thread blocks) + the split-KV kernel (TMA tile loads, scores,
online softmax, partial states) + the split-segment merge kernel (exact
log-sum-exp merge, launched as a programmatic dependent of the first).
Default workload: batched paged decode, batch 64, 32 query / 8 kv heads,
head_dim 128, per-request kv_len uniform in [512, 16384] (seed 4), 16-token
pages in a random permutation of the pool, bf16 K/V ~ N(0,1).  Its K/V
(about 2.2 GB) are larger than L2, so no flush is needed between steps.

value       = KV bytes read by all ranks / device time (CUDA events, max over
              ranks), in GB/s; tokens/s = requests decoded per second.
e2e         = the same metric through the C ABI with host buffers: every step
              copies q, K, V, kv_indptr and page_table host->device from pinned
              memory and reads out and lse back.
roofline    = algorithmic bytes per pass / the pass's average duration in the
              timed region (events on the launching stream), against the
              measured HBM copy bandwidth; isolated_launch_us is the mean
              (isolated_launch_us_median the median) of single launches each
              bracketed by its own events.
cpu_baseline= the fp64 oracle on the host cores on a bounded sample.

--impl reference times the oracle (this tier's reference arm) on the same
workload and metric.  Multi-GPU: one process per GPU (torchrun); every rank
decodes its own copy of the batch (weak scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import ctypes
import glob
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode attention achieved HBM GB/s (% of B200 peak) and tokens/sec at 1 GPU"
HEADLINE = "paged_b64_gqa4_L512-16384"
SWEEP = ["gqa4_d64_L512", "gemma3_1b_global_L8192", "gemma3_1b_local_w512_L8192",
         "llama2_7b_mha_L1024", "llama2_7b_mha_L4096", "llama2_7b_mha_L16384",
         "llama2_7b_mha_L32768", "fp8_gqa8_L131072",
         # several query tokens per request
         "paged_b64_gqa4_q2_L512-16384", "paged_b64_gqa4_q4_L512-16384",
         "paged_b64_gqa4_q8_L512-16384", "llama2_7b_mha_q8_L32768",
         # query groups wider than 8 (row teams)
         "llama3_405b_tp8_gqa16_paged_b64_L512-16384",
         # INT4 KV cache
         "int4_gqa8_L131072", "int4_paged_b64_gqa4_L512-16384",
         # logit soft-capping
         "gemma2_2b_softcap50_L8192"]
FALLBACK_HBM_GBS = 6650.0
# unified max at phi = 4: the scaled scores of these inputs are N(0, 1), whose
# maximum over 10^4..10^5 keys is about 4.4
UNIFIED_PHI = 4.0


def sweep_jobs(headline=HEADLINE):
    """Every (workload, mode) the sweep times; mode is the planner's choice
    ("auto"), a forced dataflow ("simt", "mma") or the unified max at
    UNIFIED_PHI ("unified_max").  The parity tests run the same list."""
    jobs = [(name, "auto") for name in SWEEP]
    jobs += [(headline, "simt"), (headline, "mma"),
             ("fp8_gqa8_L131072", "simt"), ("fp8_gqa8_L131072", "mma"),
             ("llama2_7b_mha_L32768", "simt"), ("llama2_7b_mha_L32768", "mma"),
             # 16 and 32 rows: the warp-level products beside the tcgen05 ones
             ("paged_b64_gqa4_q4_L512-16384", "mma"), ("paged_b64_gqa4_q8_L512-16384", "mma"),
             ("llama3_405b_tp8_gqa16_paged_b64_L512-16384", "mma"),
             (headline, "unified_max"), ("fp8_gqa8_L131072", "unified_max")]
    return jobs


def sweep_key(name, mode):
    return name if mode == "auto" else f"{name}[{mode}]"


def make_runner(x, mode, device="cuda"):
    """The launch configuration the sweep times for (workload, mode)."""
    if mode == "unified_max":
        return Runner(x, device=device, softmax_phi=UNIFIED_PHI)
    return Runner(x, path=mode, device=device)


def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_hash():
    """Hash of the kernel sources (the measured dataflow table, planner data
    that leaves the kernels as they are, is not part of it)."""
    h = hashlib.sha256()
    for p in sorted(glob.glob(os.path.join(ROOT, "gqa_decode_attention_split_b200", "csrc", "*"))):
        if p.endswith("fa_tuning_b200.inc"):
            continue
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on
    the current kernel sources."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        e = t.get(workload)
        if e and e.get("source_hash") == source_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_index(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return local_rank


# ------------------------------------------------------------ device side
class Runner:
    """Holds the device copies of one workload and the raw C-ABI arguments so
    a step is two C calls (plan, run) with no Python allocation."""

    def __init__(self, x, path="auto", device="cuda", softmax_phi=None):
        import torch
        from gqa_decode_attention_split_b200 import binding
        self.torch = torch
        self.binding = binding
        self.lib = binding.load_library()
        self.x = x
        bits = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device)
        quant = x.kv_dtype != "bf16"  # fp8 / int4 codes (bytes) with per-head scales
        self.q = bits(x.q)
        if quant:
            self.k = torch.from_numpy(np.ascontiguousarray(x.k)).to(device)
            self.v = torch.from_numpy(np.ascontiguousarray(x.v)).to(device)
            self.ks = torch.from_numpy(x.k_scale).to(device)
            self.vs = torch.from_numpy(x.v_scale).to(device)
        else:
            self.k, self.v = bits(x.k), bits(x.v)
            self.ks = self.vs = None
        self.ind = torch.from_numpy(x.kv_indptr).to(device)
        self.pt = torch.from_numpy(x.page_table).to(device) if x.paged else None
        self.ind_host = np.ascontiguousarray(x.kv_indptr, dtype=np.int32)
        self.desc = binding.DecodeDesc(
            batch=x.batch, qo_heads=x.qo_heads, kv_heads=x.kv_heads, head_dim=x.head_dim,
            kv_dtype={"bf16": 0, "fp8_e4m3": 1, "int4": 2}[x.kv_dtype], paged=int(x.paged),
            page_size=int(x.page_size),
            window=int(x.window), sm_scale=float(x.sm_scale),
            path={"auto": 0, "simt": 1, "mma": 2, "tc": 3}[path], num_ctas=0, q_len=int(x.q_len),
            logit_cap=float(x.logit_cap), unified_max=0 if softmax_phi is None else 1,
            softmax_phi=0.0 if softmax_phi is None else float(softmax_phi))
        p = binding.plan(x.batch, x.qo_heads, x.kv_heads, x.head_dim, x.kv_indptr,
                         kv_dtype=x.kv_dtype, paged=x.paged, page_size=x.page_size,
                         window=x.window, sm_scale=x.sm_scale, path=path, q_len=x.q_len,
                         logit_cap=x.logit_cap, softmax_phi=softmax_phi)
        self.info = p.info()
        self.ws = p.new_workspace(device)
        rows = (x.batch, x.qo_heads) if x.q_len == 1 else (x.batch, x.q_len, x.qo_heads)
        self.out = torch.empty(rows + (x.head_dim,), dtype=torch.bfloat16, device=device)
        self.lse = torch.empty(rows, dtype=torch.float32, device=device)
        ptr = lambda t: None if t is None else t.data_ptr()
        self.stream = torch.cuda.current_stream()
        self.args = (ptr(self.q), ptr(self.k), ptr(self.v), int(self.k.shape[0]), ptr(self.pt),
                     int(self.pt.stride(0)) if self.pt is not None else 0, ptr(self.ind),
                     ptr(self.ks), ptr(self.vs), ptr(self.out), ptr(self.lse), ptr(self.ws),
                     int(self.ws.numel()), self.stream.cuda_stream or None)
        self._handle = ctypes.c_void_p()
        self._wsb = ctypes.c_size_t()

    def run_only(self, plan_handle):
        """One pass with a plan made beforehand (no host planning)."""
        st = self.lib.fa_decode_run(plan_handle, *self.args)
        if st != 0:
            raise RuntimeError(f"fa_decode_run failed: {st}")

    def make_plan(self):
        h = ctypes.c_void_p()
        wsb = ctypes.c_size_t()
        st = self.lib.fa_decode_plan(ctypes.byref(self.desc), self.ind_host.ctypes.data, 0,
                                     ctypes.byref(h), ctypes.byref(wsb))
        if st != 0:
            raise RuntimeError(f"fa_decode_plan failed: {st}")
        return h

    def step(self):
        """plan + run (the whole hot path for one batch)."""
        lib = self.lib
        st = lib.fa_decode_plan(ctypes.byref(self.desc), self.ind_host.ctypes.data, 0,
                                ctypes.byref(self._handle), ctypes.byref(self._wsb))
        if st != 0:
            raise RuntimeError(f"fa_decode_plan failed: {st}")
        st = lib.fa_decode_run(self._handle, *self.args)
        lib.fa_plan_destroy(self._handle)
        if st != 0:
            raise RuntimeError(f"fa_decode_run failed: {st}")

    def check_status(self):
        flags = self.binding.decode_status(self.ws)
        if flags:
            raise RuntimeError(f"device check flags {flags}")


def time_steps(fn, steps, stream):
    import torch
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def per_launch_ms(fn, reps, stream, flush=None):
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for a, b in evs:
        if flush is not None:
            flush()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def device_launch_ms(runner, reps, flush=None):
    """Device time of single passes: the plan is made once, outside the
    timed region, and each pass is queued behind GPU work (the L2 flush, or
    a short device-side delay when there is nothing to flush), so the start
    event fires only once the host has already enqueued the pass: host
    planning and launch overhead stay outside the bracket."""
    import torch
    h = runner.make_plan()
    try:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        for a, b in evs:
            if flush is not None:
                flush()
            else:
                torch.cuda._sleep(40000)  # about 20 us at the B200's clocks
            a.record(runner.stream)
            runner.run_only(h)
            b.record(runner.stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in evs]
    finally:
        runner.lib.fa_plan_destroy(h)


def l2_flusher(device="cuda"):
    import torch
    buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
    return lambda: buf.fill_(1)


def e2e_measure(x, runner, steps):
    """Same metric through the C ABI with host buffers (pinned), copies in the
    timed region."""
    import torch
    hq = torch.from_numpy(np.ascontiguousarray(x.q).view(np.int16)).pin_memory()
    quant = x.kv_dtype != "bf16"
    conv = (lambda a: torch.from_numpy(np.ascontiguousarray(a))) if quant else \
        (lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)))
    hk, hv = conv(x.k).pin_memory(), conv(x.v).pin_memory()
    hind = torch.from_numpy(x.kv_indptr).pin_memory()
    hpt = torch.from_numpy(x.page_table).pin_memory() if x.paged else None
    hks = torch.from_numpy(x.k_scale).pin_memory() if quant else None
    hvs = torch.from_numpy(x.v_scale).pin_memory() if quant else None
    out_h = torch.empty(runner.out.shape, dtype=runner.out.dtype).pin_memory()
    lse_h = torch.empty(runner.lse.shape, dtype=runner.lse.dtype).pin_memory()
    pairs = [(runner.q, hq), (runner.k, hk), (runner.v, hv), (runner.ind, hind)]
    if hpt is not None:
        pairs.append((runner.pt, hpt))
    if quant:
        pairs += [(runner.ks, hks), (runner.vs, hvs)]
    h2d = sum(h.numel() * h.element_size() for _, h in pairs)
    d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * lse_h.element_size()

    def step():
        for d, h in pairs:
            d.copy_(h, non_blocking=True)
        runner.step()
        out_h.copy_(runner.out, non_blocking=True)
        lse_h.copy_(runner.lse, non_blocking=True)

    step()
    torch.cuda.synchronize()
    ms = time_steps(step, steps, runner.stream) / steps
    return ms, h2d, d2h


# ------------------------------------------------------------ multi-rank
def max_over_ranks(value, world, device):
    """The largest of one float per rank (every rank gets it); the identity on
    one rank.  Every rank must call it at the same point."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(kv_bytes, batch, ms_total, steps, world):
    """Whole-job figures for `steps` steps that took ms_total (the slowest
    rank's device time) with every rank decoding its own batch."""
    ms_step = ms_total / steps
    return {"ms_per_step": ms_step,
            "value": world * kv_bytes / (ms_step * 1e-3) / 1e9,
            "tokens_per_s": world * batch / (ms_step * 1e-3)}


# --------------------------------------------------------------- CPU side
def oracle_sample(x, budget_s, max_requests=None):
    """Time the fp64 oracle on whole requests of x (all their heads) for about
    budget_s seconds.  Returns (seconds, kv bytes, requests, threads)."""
    from oracle import oracle
    threads = int(os.environ.get("OMP_NUM_THREADS", len(os.sched_getaffinity(0))))
    order = list(range(x.batch))
    done_b, t_total, nbytes = 0, 0.0, 0
    vis = x.visible_lens()
    per_tok = x.kv_heads * x.head_dim * x.elem_bytes * 2
    for b in order:
        per = x.q_len * x.qo_heads  # rows of one request
        rows = np.arange(b * per, (b + 1) * per)
        t0 = time.perf_counter()
        oracle.decode_rows(x, rows, nthreads=threads)
        t_total += time.perf_counter() - t0
        nbytes += int(vis[b]) * per_tok
        done_b += 1
        if t_total >= budget_s or (max_requests and done_b >= max_requests):
            break
    return t_total, nbytes, done_b, threads


def cpu_baseline(x, budget_s=12.0):
    t, nbytes, nreq, threads = oracle_sample(x, budget_s)
    return {"value": round(nbytes / t / 1e9, 4), "unit": "GB/s", "cores": threads,
            "kind": "oracle", "tokens_per_s": round(nreq * x.q_len / t, 3),
            "sample": f"fp64 oracle over {nreq} whole request(s) of {x.name} "
                      f"({nbytes / 1e9:.3f} GB of K/V) in {t:.2f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    from gqa_decode_attention_split_b200 import synth
    x = synth.workload(args.workload)
    total_budget = 150.0
    per_step = max(0.5, total_budget / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(x, per_step)
    times, byts, reqs = [], [], []
    threads = 0
    for _ in range(args.steps):
        t, nbytes, nreq, threads = oracle_sample(x, per_step)
        times.append(t)
        byts.append(nbytes)
        reqs.append(nreq)
    t, nbytes, nreq = sum(times), sum(byts), sum(reqs)
    value = nbytes / t / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * t / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(x, world),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                             "kind": "oracle",
                             "sample": f"each step: fp64 oracle over whole requests of {x.name} "
                                       f"for about {per_step:.1f} s ({nreq} requests in total)"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "tokens_per_s": round(nreq / t, 3)}
    print(json.dumps(line), flush=True)


def workload_config(x, world):
    lens = x.kv_lens
    return {"workload": x.name, "batch": x.batch, "qo_heads": x.qo_heads,
            "kv_heads": x.kv_heads, "head_dim": x.head_dim, "kv_dtype": x.kv_dtype,
            "paged": bool(x.paged), "page_size": x.page_size, "window": x.window,
            "q_len": x.q_len, "logit_cap": x.logit_cap,
            "kv_len_min": int(lens.min()), "kv_len_max": int(lens.max()),
            "kv_tokens": int(lens.sum()), "kv_bytes_per_step_per_gpu": x.kv_bytes(),
            "l2": "inputs larger than L2 (no flush)" if x.kv_bytes() > 256e6
            else "L2 flushed (256 MB write) before every timed launch",
            "parallelism": f"replicas x{world} (independent batches, no collective)"}


# ------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--path", default="auto", choices=["auto", "simt", "mma", "tc"])
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--sweep-cpu-s", type=float, default=1.5,
                    help="seconds of oracle time per sweep workload (its cpu_baseline)")
    ap.add_argument("--profile", type=int, default=0,
                    help="profiler driver: run --warmup steps, then N steps, print nothing")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    from gqa_decode_attention_split_b200 import synth

    x = synth.workload(args.workload)
    runner = Runner(x, path=args.path)
    stream = runner.stream
    if args.profile:
        for _ in range(args.warmup + args.profile):
            runner.step()
        torch.cuda.synchronize()
        runner.check_status()
        return
    for _ in range(args.warmup):
        runner.step()
    torch.cuda.synchronize()
    runner.check_status()
    sampler = ClockSampler(gpu_index(local_rank))
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ms_total = time_steps(runner.step, args.steps, stream)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms_total = max_over_ranks(ms_total, world, "cuda")
    kv_bytes = x.kv_bytes()
    agg = aggregate(kv_bytes, x.batch * x.q_len, ms_total, args.steps, world)  # query tokens
    ms_step, value, tokens = agg["ms_per_step"], agg["value"], agg["tokens_per_s"]

    # dominant kernel: its average duration in the timed region (CUDA events on
    # the launching stream around the back-to-back passes; the decode kernel is
    # 98.7% of a pass in the launch list, the split-merge kernel the rest, so
    # the pass time is used as the decode kernel's, slightly conservatively).
    # Isolated launches, each bracketed by its own events, are reported too.
    peak, peak_kind = hbm_peak()
    achieved = kv_bytes / (ms_step * 1e-3) / 1e9
    launch_ms = per_launch_ms(runner.step, min(args.steps, 100), stream,
                              flush=None if kv_bytes > 256e6 else l2_flusher())
    mean_launch = max_over_ranks(statistics.mean(launch_ms), world, "cuda")
    median_launch = max_over_ranks(statistics.median(launch_ms), world, "cuda")
    traffic = ncu_traffic(x.name)
    runner.check_status()

    e2e = None
    if not args.no_e2e:
        ms_e2e, h2d, d2h = e2e_measure(x, runner, args.e2e_steps)
        ms_e2e = max_over_ranks(ms_e2e, world, "cuda")
        e2e = {"value": round(world * kv_bytes / (ms_e2e * 1e-3) / 1e9, 3), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(ms_e2e, 3), "steps": args.e2e_steps,
               "tokens_per_s": round(world * x.batch * x.q_len / (ms_e2e * 1e-3), 1)}

    sweep = None
    if rank == 0 and world == 1 and not args.no_sweep:
        sweep = {}
        flush = l2_flusher()
        cache = {x.name: x}
        cpu_cache = {}
        for name, mode in sweep_jobs(x.name):
            key = sweep_key(name, mode)
            try:
                y = cache.get(name) or synth.workload(name)
                cache = {x.name: x, name: y}
                r = make_runner(y, mode)
                for _ in range(5):
                    r.step()
                big = y.kv_bytes() > 256e6
                ms = per_launch_ms(r.step, 30, r.stream, flush=None if big else flush)
                med = statistics.median(ms)
                dev_ms = device_launch_ms(r, 30, flush=None if big else flush)
                dmed = statistics.median(dev_ms)
                loop_us = None
                if big:  # back to back, as in the timed region (inputs exceed L2)
                    loop_us = 1e3 * time_steps(r.step, 50, r.stream) / 50
                r.check_status()
                gbps = y.kv_bytes() / (med * 1e-3) / 1e9
                dgbps = y.kv_bytes() / (dmed * 1e-3) / 1e9
                entry = {"us": round(med * 1e3, 2), "gbps": round(gbps, 1),
                         "frac": round(gbps / peak, 4),
                         "device_us": round(dmed * 1e3, 2),
                         "device_frac": round(dgbps / peak, 4),
                         "back_to_back_us": None if loop_us is None else round(loop_us, 2),
                         "back_to_back_frac": None if loop_us is None else
                         round(y.kv_bytes() / (loop_us * 1e-6) / 1e9 / peak, 4),
                         "tokens_per_s": round(y.batch * y.q_len / (med * 1e-3), 1),
                         "path": {1: "simt", 2: "mma", 3: "tc"}.get(r.info["path"], str(r.info["path"])),
                         "ctas": r.info["num_ctas"], "kv_bytes": y.kv_bytes()}
                del r
                torch.cuda.empty_cache()
                # the oracle on a bounded sample of the same workload (the
                # definition is the same with or without the unified max)
                if not args.no_cpu_baseline:
                    if name not in cpu_cache:
                        cpu_cache[name] = cpu_baseline(y, budget_s=args.sweep_cpu_s)
                    entry["cpu_baseline"] = cpu_cache[name]
                sweep[key] = entry
            except Exception as e:  # keep the headline line even if a sweep entry fails
                sweep[key] = {"error": str(e)[:300]}
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(x)

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": x.kv_dtype,
                "data": "synthetic", "config": workload_config(x, world),
                "tokens_per_s": round(tokens, 1), "frac_of_peak": round(value / world / peak, 4),
                "path": {1: "simt", 2: "mma", 3: "tc"}[runner.info["path"]],
                "num_ctas": runner.info["num_ctas"],
                "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                             "unit": "GB/s", "frac": round(achieved / peak, 4),
                             "traffic": traffic, "peak_source": peak_kind,
                             "launch_us": round(ms_step * 1e3, 2),
                             "isolated_launch_us": round(mean_launch * 1e3, 2),
                             "isolated_launch_us_median": round(median_launch * 1e3, 2),
                             "algorithmic_bytes_per_launch": kv_bytes},
                # per step: the decode kernel, plus the split-merge kernel when
                # some segment is split over blocks
                "gpu_launches": args.steps * runner.info["launches"],
                "clocks": clocks, "e2e": e2e,
                "cpu_baseline": cpu, "sweep": sweep}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
