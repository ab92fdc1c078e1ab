#!/usr/bin/env python3
"""Benchmark of the GQA attention forward on B200.

Default workload: prefill GQA, B=64, Hq=32, Hk=8, Sq=Sk=2048, d=128, bf16 Q/K/V ~ N(0,1)
(seeded, synthetic), causal, scale 1/sqrt(128), pack_gqa / num_splits from the heuristic.
One step = one forward over the whole batch.  Rank 0 prints one JSON line.  Besides the
headline (the step timed over --steps launches), the line carries:
  "sustained"  the same step over a timed region of at least 1.2 s, against the sustained
               GEMM peak (power and clocks settle over such a region);
  "decode"     the metric's decode half: B=256, Sq=1, Sk=8192, Hq=32, Hk=8, d=128
               (K and V 8.6 GB), device-timed like the headline, in HBM GB/s against
               the measured copy bandwidth, with its own CPU-oracle baseline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

--impl reference times the fp64 CPU oracle (the only reference this project has) on the
box's host cores, on bounded samples of the same workload.  Other flags (--B, --Sq, ...)
select another shape for ad-hoc measurement; ``--sweep prefill|decode|kvcache|paged|fp8`` prints
one line per configuration of the batch-sensitivity sweep, the decode grid, the KV-cache
entry point (per-sequence lengths, bf16 output), the paged KV cache next to the dense one, or
the e4m3 entry point next to bf16 inputs of the same shapes.
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
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "GQA fwd TFLOPS & tokens/s (Hq32 Hk8 d128 S2K, B16-256); decode HBM GB/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
CSRC_DIR = os.path.join(ROOT, "gqa_exact_attention_b200", "csrc")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# nominal (datasheet) peaks of one B200, the second denominator every fraction is given
# against: dense bf16 tensor throughput and HBM3e bandwidth
SPEC_PEAKS = {"tensor": 2250.0, "hbm": 8000.0}


def with_spec(roof):
    """Add the nominal peak and the fraction of it beside the measured one."""
    roof["spec_peak"] = SPEC_PEAKS[roof["bound"]]
    roof["frac_of_spec"] = roof["achieved"] / roof["spec_peak"]
    return roof


# ----------------------------------------------------------------- work accounting

def causal_pairs(Sq, Sk):
    """Number of (query, key) pairs the causal mask allows (bottom-right aligned)."""
    tot = 0
    off = Sk - Sq
    # row i allows min(Sk, max(0, i + 1 + off)) keys
    lo = max(0, -off)  # first row with at least one key
    full_from = max(lo, Sk - off - 1)  # rows from here see all Sk keys
    full_from = min(max(full_from, lo), Sq)
    # rows lo .. full_from-1: i + 1 + off keys
    n = full_from - lo
    if n > 0:
        a = lo + 1 + off
        tot += n * a + n * (n - 1) // 2
    tot += (Sq - full_from) * Sk
    return tot


def flops(B, Sq, Sk, Hq, d, causal):
    """4 B Hq Sq Sk d for non-causal; the allowed pairs (Sq Sk / 2 when Sq = Sk, up to
    the diagonal term) for causal: 2 flops per multiply-add in QK^T and in PV."""
    pairs = causal_pairs(Sq, Sk) if causal else Sq * Sk
    if causal and Sq == Sk:
        pairs = Sq * Sk / 2  # the pages' convention: halved for causal
    return 4.0 * B * Hq * d * pairs


def hbm_bytes(B, Sq, Sk, Hq, Hk, d):
    """Algorithmic bytes: read Q, K, V once (bf16), write O (fp32) and LSE (fp32)."""
    return 2 * B * Sq * Hq * d + 2 * 2 * B * Sk * Hk * d + 4 * B * Sq * Hq * d + 4 * B * Hq * Sq


# ----------------------------------------------------------------- environment

def load_peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            pk = json.load(f)
        return pk, "measured"
    return FALLBACK_PEAKS, "fallback"


def kernel_hash():
    """sha256[:16] over the library's sources (kernels, host plan and schedule, headers):
    any change that can move the kernel's DRAM traffic invalidates the stored counters."""
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC_DIR)):
        if name.endswith((".cu", ".cuh", ".cpp", ".h")):
            with open(os.path.join(CSRC_DIR, name), "rb") as f:
                h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def traffic_for(workload_key, pack_gqa, num_splits):
    """DRAM bytes per launch from a committed ncu capture, if it was taken on the current
    kernel source with the same resolved pack / split choice; else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        t = json.load(f)
    if t.get("kernel_sha256_16") != kernel_hash():
        return None
    e = t.get("workloads", {}).get(workload_key)
    if e is None or e.get("pack_gqa") != pack_gqa or e.get("num_splits") != num_splits:
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, smax, reasons = [], None, set()
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                clk, mx, util = float(parts[1]), float(parts[2]), float(parts[4])
            except ValueError:
                continue
            smax = mx
            if util >= 50:
                sm.append(clk)
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples_under_load": len(sm)}


# ----------------------------------------------------------------- distributed plumbing

def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}; launch N>1 with torchrun")
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = dist
    else:
        torch.cuda.set_device(0)
    return rank, world, local, pg


def barrier(pg):
    if pg is not None:
        pg.barrier()


def max_over_ranks(pg, x):
    """Max of a per-rank float over all ranks (the slowest rank sets the job's time)."""
    if pg is None:
        return x
    import torch
    dev = "cuda" if pg.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_throughput(per_rank_work, world, total_ms, steps):
    """Whole-job rate: every rank processes per_rank_work per step (weak scaling), and
    the job's time per step is the slowest rank's."""
    return world * per_rank_work / (total_ms / steps / 1e3)


# ----------------------------------------------------------------- CPU oracle timing

def oracle_sample(cfg, budget_s):
    """Time the fp64 oracle on whole batch elements of the workload until about
    budget_s seconds of CPU work; returns (flops/s, threads, description)."""
    import inputs
    import oracle
    B, Sq, Sk, Hq, Hk, d, causal = (cfg[k] for k in ("B", "Sq", "Sk", "Hq", "Hk", "d", "causal"))
    scale = 1.0 / math.sqrt(d)

    def one(nb, seed_off):
        # nb batch elements, all heads (regenerated from the same seeded definition)
        qs, ks = (nb, Sq, Hq, d), (nb, Sk, Hk, d)
        f = inputs.bf16_bits_to_f64
        q = f(inputs.bits_range(cfg["seed"], inputs.TID_Q, seed_off * Sq * Hq * d, nb * Sq * Hq * d)).reshape(qs)
        k = f(inputs.bits_range(cfg["seed"], inputs.TID_K, seed_off * Sk * Hk * d, nb * Sk * Hk * d)).reshape(ks)
        v = f(inputs.bits_range(cfg["seed"], inputs.TID_V, seed_off * Sk * Hk * d, nb * Sk * Hk * d)).reshape(ks)
        t0 = time.perf_counter()
        _, _, threads = oracle.attn_fwd(q, k, v, scale, causal, return_threads=True)
        return time.perf_counter() - t0, threads

    # calibrate on one sequence restricted to a few heads' worth of time
    t1, threads = one(1, 0)
    nb = max(1, min(B - 1 if B > 1 else 1, int(budget_s / max(t1, 1e-3))))
    # keep the fp64 copies of the sample within about 1 GB per tensor
    per_seq = max(Sq * Hq * d, Sk * Hk * d)
    nb = max(1, min(nb, (1 << 27) // per_seq))
    if nb > 1:
        tn, threads = one(nb, 1)
        total_t, total_b = t1 + tn, 1 + nb
    else:
        total_t, total_b = t1, 1
    rate = flops(total_b, Sq, Sk, Hq, d, causal) / total_t
    desc = (f"{total_b} of {B} sequences (all {Hq} heads, Sq={Sq}, Sk={Sk}), fp64 oracle, "
            f"{total_t:.1f} s")
    return rate, threads, desc


# ----------------------------------------------------------------- GPU arm

# The decode half of the metric: one new query token per sequence against its keys,
# B=256, Sk=8192 (K and V 8.6 GB, far above the 126 MB L2), Hq=32, Hk=8, d=128,
# non-causal, pack_gqa / num_splits from the heuristic.
DECODE_CFG = {"name": "decode B=256 Hq=32 Hk=8 Sq=1 Sk=8192 d=128 non-causal", "B": 256,
              "Sq": 1, "Sk": 8192, "Hq": 32, "Hk": 8, "d": 128, "causal": 0, "seed": 1003,
              "l2": "inputs larger than L2 (K and V 8590 MB read per step)"}


def time_steps(step, steps, stream, per_launch=True):
    """Time `steps` calls of step() on `stream` with CUDA events: (total ms, mean ms of
    one call measured by its own event pair)."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps if per_launch else 0)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(steps):
        if per_launch:
            ev[i][0].record(stream)
        step()
        if per_launch:
            ev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    total = t_start.elapsed_time(t_end)
    mean = statistics.mean(a.elapsed_time(b) for a, b in ev) if per_launch else total / steps
    return total, mean


def run_decode(args, pg, world, rank, dev, peaks, peak_src):
    """The decode workload, device-timed like the main step: the 'decode' object of the
    JSON line (HBM GB/s against the measured copy bandwidth)."""
    import torch

    import gqa_exact_attention_b200 as G
    import inputs
    c = DECODE_CFG
    B, Sq, Sk, Hq, Hk, d = (c[k] for k in ("B", "Sq", "Sk", "Hq", "Hk", "d"))
    pack, splits = G.gqa_attn_choose(B, Sq, Sk, Hq, Hk, d, 0)
    seed = c["seed"] + rank
    q = inputs.device_tensor(seed, inputs.TID_Q, (B, Sq, Hq, d), device=dev)
    k = inputs.device_tensor(seed, inputs.TID_K, (B, Sk, Hk, d), device=dev)
    v = inputs.device_tensor(seed, inputs.TID_V, (B, Sk, Hk, d), device=dev)
    out = torch.empty((B, Sq, Hq, d), dtype=torch.float32, device=dev)
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        G.gqa_attn_fwd(q, k, v, out=out, lse=lse, causal=0, pack_gqa=pack, num_splits=splits,
                       stream=stream)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(pg)
    torch.cuda.synchronize()
    total_ms, launch_ms = time_steps(step, args.steps, stream)
    barrier(pg)
    total_ms = max_over_ranks(pg, total_ms)
    launch_ms = max_over_ranks(pg, launch_ms)
    by = hbm_bytes(B, Sq, Sk, Hq, Hk, d)
    achieved = by / (launch_ms / 1e3) / 1e9
    obj = {
        "workload": c["name"], "value": round(job_throughput(by, world, total_ms, args.steps) / 1e9, 1),
        "unit": "GB/s", "ms_per_step": round(total_ms / args.steps, 4), "steps": args.steps,
        "tokens_per_s": round(world * B / (total_ms / args.steps / 1e3), 1),
        "pack_gqa": pack, "num_splits": splits, "l2": c["l2"],
        "gpu_launches": (1 + (1 if splits > 1 else 0)) * args.steps,
        "roofline": with_spec({"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                               "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                               "peak_source": f"{peak_src}:hbm_gbs",
                               "traffic": traffic_for(c["name"], pack, splits),
                               "kernel": "gqa_fwd_kernel"}),
    }
    del q, k, v, out, lse
    torch.cuda.empty_cache()
    return obj


def run_gpu(args, cfg):
    import torch

    import gqa_exact_attention_b200 as G
    import inputs  # seeded input generator (no attention arithmetic)

    rank, world, local, pg = dist_setup(args.gpus)
    dev = torch.device("cuda", local if world > 1 else 0)
    G.load()
    B, Sq, Sk, Hq, Hk, d, causal = (cfg[k] for k in ("B", "Sq", "Sk", "Hq", "Hk", "d", "causal"))
    pack, splits = G.gqa_attn_choose(B, Sq, Sk, Hq, Hk, d, causal) if (args.pack < 0 and args.splits <= 0) \
        else (args.pack, args.splits)
    if args.pack >= 0:
        pack = args.pack
    if args.splits > 0:
        splits = args.splits
    seed = cfg["seed"] + rank
    q = inputs.device_tensor(seed, inputs.TID_Q, (B, Sq, Hq, d), device=dev)
    k = inputs.device_tensor(seed, inputs.TID_K, (B, Sk, Hk, d), device=dev)
    v = inputs.device_tensor(seed, inputs.TID_V, (B, Sk, Hk, d), device=dev)
    out = torch.empty((B, Sq, Hq, d), dtype=torch.float32, device=dev)
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    launches_per_step = 1 + (1 if splits > 1 else 0)

    def step():
        G.gqa_attn_fwd(q, k, v, out=out, lse=lse, causal=causal, pack_gqa=pack,
                       num_splits=splits, stream=stream)

    sampler = ClockSampler(local if world > 1 else 0) if rank == 0 or world > 1 else None
    if sampler:
        sampler.start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- device-timed region: K steps, events per launch on the launching stream
    barrier(pg)
    torch.cuda.synchronize()
    total_ms, launch_ms = time_steps(step, args.steps, stream)
    barrier(pg)
    total_ms = max_over_ranks(pg, total_ms)
    launch_ms = max_over_ranks(pg, launch_ms)
    ms_per_step = total_ms / args.steps

    # ---- the same step over a timed region of at least a second (power and clocks
    # settle), reported against the sustained GEMM peak
    sus_steps = 0
    if not args.no_sustained:
        sus_steps = max(args.steps, min(4000, int(math.ceil(1200.0 / max(ms_per_step, 1e-3)))))
        barrier(pg)
        torch.cuda.synchronize()
        sus_total, _ = time_steps(step, sus_steps, stream, per_launch=False)
        barrier(pg)
        sus_total = max_over_ranks(pg, sus_total)
    if G.gqa_attn_device_status(reset=True) != 0:
        raise SystemExit("an in-kernel bounded wait timed out during the benchmark")

    # ---- end to end through the public API: pinned host inputs in, results out.  As a
    # serving loop would, transfers overlap compute: step i+1's inputs go up on one copy
    # stream and step i-1's results come down on another while step i computes (two
    # device buffer sets).  Every step still moves all of its inputs and results.
    q_h = q.cpu().pin_memory()
    k_h = k.cpu().pin_memory()
    v_h = v.cpu().pin_memory()
    out_h = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    lse_h = [torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True) for _ in range(2)]
    h2d = (q_h.numel() + k_h.numel() + v_h.numel()) * 2
    d2h = out_h[0].numel() * 4 + lse_h[0].numel() * 4
    bufs = [(q, k, v, out, lse),
            (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(out),
             torch.empty_like(lse))]
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)

    def e2e_run(n):
        """n pipelined steps; returns (start event on s_in, end event on s_out)."""
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        in_done, comp_done, out_done = [], [], []
        start.record(s_in)
        for i in range(n):
            j = i & 1
            qb, kb, vb, ob, lb = bufs[j]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(comp_done[i - 2])  # buffer set j's inputs are consumed
                qb.copy_(q_h, non_blocking=True)
                kb.copy_(k_h, non_blocking=True)
                vb.copy_(v_h, non_blocking=True)
                e = torch.cuda.Event()
                e.record(s_in)
                in_done.append(e)
            stream.wait_event(in_done[i])
            if i >= 2:
                stream.wait_event(out_done[i - 2])  # buffer set j's results are read out
            G.gqa_attn_fwd(qb, kb, vb, out=ob, lse=lb, causal=causal, pack_gqa=pack,
                           num_splits=splits, stream=stream)
            e = torch.cuda.Event()
            e.record(stream)
            comp_done.append(e)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[i])
                out_h[j].copy_(ob, non_blocking=True)
                lse_h[j].copy_(lb, non_blocking=True)
                e = torch.cuda.Event()
                e.record(s_out)
                out_done.append(e)
        end.record(s_out)
        return start, end

    e2e_run(2)
    torch.cuda.synchronize()
    e_steps = max(2, min(args.steps, 20))
    barrier(pg)
    torch.cuda.synchronize()
    e0, e1 = e2e_run(e_steps)
    torch.cuda.synchronize()
    barrier(pg)
    e2e_ms = max_over_ranks(pg, e0.elapsed_time(e1)) / e_steps
    del bufs
    peaks, peak_src = load_peaks()
    decode = None
    if cfg.get("with_decode"):
        decode = run_decode(args, pg, world, rank, dev, peaks, peak_src)
    clocks = sampler.stop() if sampler else None

    fl = flops(B, Sq, Sk, Hq, d, causal)
    by = hbm_bytes(B, Sq, Sk, Hq, Hk, d)
    decode_like = Sq * (Hq // Hk) <= 128 and not causal
    timed_s = total_ms / 1e3
    if decode_like:
        achieved = by / (launch_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"]}
        value = job_throughput(by, world, total_ms, args.steps) / 1e9
        unit = "GB/s"
        e2e_value = world * by / (e2e_ms / 1e3) / 1e9
    else:
        pk_key = "bf16_tflops_sustained" if timed_s > 1.0 else "bf16_tflops"
        achieved = fl / (launch_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks[pk_key], "unit": "TFLOP/s",
                "frac": achieved / peaks[pk_key]}
        value = job_throughput(fl, world, total_ms, args.steps) / 1e12
        unit = "TFLOP/s"
        e2e_value = world * fl / (e2e_ms / 1e3) / 1e12
    roof["peak_source"] = f"{peak_src}:" + ("hbm_gbs" if decode_like else pk_key)
    roof["traffic"] = traffic_for(cfg["name"], pack, splits)
    roof["kernel"] = "gqa_fwd_kernel"
    with_spec(roof)

    tokens = B * (Sq if Sq > 1 else 1)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) rounded to bf16)",
        "config": {"workload": cfg["name"], "B": B, "Sq": Sq, "Sk": Sk, "Hq": Hq, "Hk": Hk,
                   "d": d, "causal": bool(causal), "pack_gqa": pack, "num_splits": splits,
                   "out_dtype": "fp32", "l2": cfg["l2"],
                   "parallelism": f"replicas x{world} (independent batches, no collective)"},
        "tokens_per_s": round(world * tokens / (ms_per_step / 1e3), 1),
        "tflops": round(world * fl / (ms_per_step / 1e3) / 1e12, 3),
        "hbm_gbs": round(world * by / (ms_per_step / 1e3) / 1e9, 1),
        "roofline": roof,
        "e2e": {"value": round(e2e_value, 3), "unit": unit, "ms_per_step": round(e2e_ms, 3),
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "overlap": "step i+1 inputs up and step i-1 results down while step i computes "
                           "(pinned host memory, two device buffer sets, two copy streams)"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if sus_steps and not decode_like:
        sus_ms = sus_total / sus_steps
        sus_val = job_throughput(fl, world, sus_total, sus_steps) / 1e12
        pk = peaks["bf16_tflops_sustained"]
        line["sustained"] = {
            "value": round(sus_val, 3), "unit": unit, "steps": sus_steps,
            "timed_s": round(sus_total / 1e3, 3), "ms_per_step": round(sus_ms, 4),
            "gpu_launches": launches_per_step * sus_steps,
            "roofline": with_spec({"bound": "tensor", "achieved": fl / (sus_ms / 1e3) / 1e12,
                                   "peak": pk, "unit": "TFLOP/s",
                                   "frac": fl / (sus_ms / 1e3) / 1e12 / pk,
                                   "peak_source": f"{peak_src}:bf16_tflops_sustained"})}
    if decode is not None:
        line["decode"] = decode
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, threads, desc = oracle_sample(cfg, args.cpu_budget)
        if decode_like:
            cv = by / (fl / rate) / 1e9
        else:
            cv = rate / 1e12
        line["cpu_baseline"] = {"value": cv, "unit": unit, "cores": threads, "kind": "oracle",
                                "sample": desc}
        if decode is not None:
            dc = DECODE_CFG
            drate, dthreads, ddesc = oracle_sample(dc, min(args.cpu_budget, 8.0))
            dfl = flops(dc["B"], dc["Sq"], dc["Sk"], dc["Hq"], dc["d"], 0)
            dby = hbm_bytes(dc["B"], dc["Sq"], dc["Sk"], dc["Hq"], dc["Hk"], dc["d"])
            decode["cpu_baseline"] = {"value": dby / (dfl / drate) / 1e9, "unit": "GB/s",
                                      "cores": dthreads, "kind": "oracle", "sample": ddesc}
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_reference(args, cfg):
    """The fp64 oracle as it stands, on host cores, bounded samples of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    # torchrun gives every rank OMP_NUM_THREADS=1; here rank 0 works alone, so the oracle
    # gets the host's cores, as in a single-process run (set before its OpenMP starts)
    if int(os.environ.get("WORLD_SIZE", "1")) > 1 and os.environ.get("OMP_NUM_THREADS") == "1":
        os.environ["OMP_NUM_THREADS"] = str(len(os.sched_getaffinity(0)))
    B, Sq, Sk, Hq, Hk, d, causal = (cfg[k] for k in ("B", "Sq", "Sk", "Hq", "Hk", "d", "causal"))
    budget = max(2.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(cfg, budget / 4)
    rates, threads, desc = [], 1, ""
    t0 = time.perf_counter()
    for _ in range(args.steps):
        r, threads, desc = oracle_sample(cfg, budget)
        rates.append(r)
    wall = time.perf_counter() - t0
    fl = flops(B, Sq, Sk, Hq, d, causal)
    by = hbm_bytes(B, Sq, Sk, Hq, Hk, d)
    rate = statistics.mean(rates)
    decode_like = Sq * (Hq // Hk) <= 128 and not causal
    value, unit = ((by / (fl / rate) / 1e9, "GB/s") if decode_like else (rate / 1e12, "TFLOP/s"))
    line = {
        "metric": METRIC, "impl": "reference", "value": value, "unit": unit,
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * wall / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) rounded to bf16)",
        "config": {"workload": cfg["name"], "B": B, "Sq": Sq, "Sk": Sk, "Hq": Hq, "Hk": Hk,
                   "d": d, "causal": bool(causal), "out_dtype": "fp64", "l2": cfg["l2"]},
        "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
                         "sample": desc + " per step"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_sweep(args):
    """Kernel-only timings over the batch-size sweep (B 16..256, causal and not, every
    pack/split variant plus the heuristic's choice) or the decode grid (Sk 2K/8K/32K,
    B 32/128/256, splits 1/2/4/8 plus the heuristic's).  One JSON line per case; not the
    benchmark contract's line."""
    import torch

    import gqa_exact_attention_b200 as G
    import inputs
    torch.cuda.set_device(0)
    G.load()
    stream = torch.cuda.current_stream()
    peaks, _ = load_peaks()
    if args.sweep == "kvcache":
        return run_sweep_kvcache(args, peaks)
    if args.sweep == "paged":
        return run_sweep_paged(args, peaks)
    if args.sweep == "fp8":
        return run_sweep_fp8(args, peaks)
    if args.sweep == "prefill":
        cases = [(B, 2048, 2048, c, pk, sp) for B in (16, 32, 64, 128, 256) for c in (1, 0)
                 for (pk, sp) in [(-1, 0), (0, 1), (1, 1), (0, 2), (1, 2), (0, 4), (1, 4)]]
    else:
        cases = [(B, 1, Sk, 0, pk, sp) for Sk in (2048, 8192, 32768) for B in (32, 128, 256)
                 for (pk, sp) in [(-1, 0), (1, 1), (1, 2), (1, 4), (1, 8)]]
    cur = None
    for (B, Sq, Sk, causal, pk, sp) in cases:
        Hq, Hk, d = 32, 8, args.d
        if cur != (B, Sq, Sk):
            q = k = v = out = lse = None
            torch.cuda.empty_cache()
            q = inputs.device_tensor(1001, inputs.TID_Q, (B, Sq, Hq, d))
            k = inputs.device_tensor(1001, inputs.TID_K, (B, Sk, Hk, d))
            v = inputs.device_tensor(1001, inputs.TID_V, (B, Sk, Hk, d))
            out = torch.empty((B, Sq, Hq, d), dtype=torch.float32, device="cuda")
            lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device="cuda")
            cur = (B, Sq, Sk)
        rp, rs = G.gqa_attn_choose(B, Sq, Sk, Hq, Hk, d, causal) if (pk < 0 and sp <= 0) else (pk, sp)

        def step():
            G.gqa_attn_fwd(q, k, v, out=out, lse=lse, causal=causal, pack_gqa=rp,
                           num_splits=rs, stream=stream)
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        fl = flops(B, Sq, Sk, Hq, d, causal)
        by = hbm_bytes(B, Sq, Sk, Hq, Hk, d)
        line = {"sweep": args.sweep, "B": B, "Sq": Sq, "Sk": Sk, "d": d, "causal": bool(causal),
                "pack_gqa": rp, "num_splits": rs, "heuristic": pk < 0 and sp <= 0,
                "ms": round(ms, 4), "tflops": round(fl / ms / 1e9, 1),
                "hbm_gbs": round(by / ms / 1e6, 1),
                "tokens_per_s": round(B * (Sq if Sq > 1 else 1) / ms * 1e3, 1)}
        if args.sweep == "prefill":
            line["frac_of_measured_bf16"] = round(fl / ms / 1e9 / peaks["bf16_tflops"], 3)
        else:
            line["frac_of_measured_hbm"] = round(by / ms / 1e6 / peaks["hbm_gbs"], 3)
        print(json.dumps(line), flush=True)


def run_sweep_kvcache(args, peaks):
    """Kernel-only timings of gqa_attn_fwd_kvcache: decode against a KV cache of capacity
    8192 whose sequences have seeded lengths uniform in [1, 8192] (B 32/128/256), fp32 and
    bf16 output with the automatic split count, and fp32 with splits 1/2/4/8; and the
    prefill shape (B=16, S=2048) with bf16 output.  Bytes and flops count each sequence's
    own keys."""
    import numpy as np
    import torch

    import gqa_exact_attention_b200 as G
    import inputs
    stream = torch.cuda.current_stream()
    Hq, Hk, d = 32, 8, 128
    cases = [(B, 1, 8192, 0, "uniform", dt, 0) for B in (32, 128, 256) for dt in ("fp32", "bf16")]
    cases += [(B, 1, 8192, 0, "uniform", "fp32", sp) for B in (32, 128, 256) for sp in (1, 2, 4, 8)]
    cases += [(16, 2048, 2048, c, "full", "bf16", 0) for c in (0, 1)]
    for (B, Sq, Sk, causal, mix, dt, sp) in cases:
        q = inputs.device_tensor(1001, inputs.TID_Q, (B, Sq, Hq, d))
        k = inputs.device_tensor(1001, inputs.TID_K, (B, Sk, Hk, d))
        v = inputs.device_tensor(1001, inputs.TID_V, (B, Sk, Hk, d))
        rng = np.random.default_rng(7000 + B)
        lens = rng.integers(1, Sk + 1, size=B) if mix == "uniform" else np.full(B, Sk)
        sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        odt = torch.bfloat16 if dt == "bf16" else torch.float32
        out = torch.empty((B, Sq, Hq, d), dtype=odt, device="cuda")
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device="cuda")

        def step(st=stream):
            G.gqa_attn_fwd_kvcache(q, k, v, sl, out=out, lse=lse, causal=causal, num_splits=sp,
                                   stream=st)
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        graph = None
        if args.graph:
            # the call's launches (work order, forward, combine) captured once and replayed
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                step(torch.cuda.current_stream())
            graph.replay()
            torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            if graph is not None:
                graph.replay()
            else:
                step()
        e1.record(stream)
        torch.cuda.synchronize()
        if G.gqa_attn_device_status(reset=True) != 0:
            raise SystemExit("an in-kernel bounded wait timed out")
        ms = e0.elapsed_time(e1) / args.steps
        del graph
        keys = int(lens.sum())
        osz = 2 if dt == "bf16" else 4
        by = 2 * B * Sq * Hq * d + 2 * 2 * keys * Hk * d + osz * B * Sq * Hq * d + 4 * B * Hq * Sq
        fl = sum(flops(1, Sq, int(L), Hq, d, causal) for L in lens)
        line = {"sweep": "kvcache", "graph": bool(args.graph), "B": B, "Sq": Sq, "Sk_capacity": Sk, "lengths": mix,
                "num_splits": sp if sp > 0 else "auto",
                "mean_length": round(float(lens.mean()), 1), "causal": bool(causal), "out": dt,
                "ms": round(ms, 4), "hbm_gbs": round(by / ms / 1e6, 1),
                "frac_of_measured_hbm": round(by / ms / 1e6 / peaks["hbm_gbs"], 3),
                "tflops": round(fl / ms / 1e9, 1),
                "frac_of_measured_bf16": round(fl / ms / 1e9 / peaks["bf16_tflops"], 3)}
        print(json.dumps(line), flush=True)
        del q, k, v, out, lse
        torch.cuda.empty_cache()


def run_sweep_paged(args, peaks):
    """Kernel-only timings of gqa_attn_fwd_paged next to gqa_attn_fwd_kvcache on the same
    keys: decode against a capacity of 8192 keys per sequence, seeded lengths uniform in
    [1, 8192] (B 32/128/256), automatic schedule, fp32 output; page sizes 16, 64 and 256,
    pages handed out in a shuffled order.  Bytes count each sequence's own keys."""
    import numpy as np
    import torch

    import gqa_exact_attention_b200 as G
    import inputs
    stream = torch.cuda.current_stream()
    Hq, Hk, d, cap, Sq = 32, 8, 128, 8192, 1

    def timed(step):
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        if G.gqa_attn_device_status(reset=True) != 0:
            raise SystemExit("an in-kernel bounded wait timed out")
        return e0.elapsed_time(e1) / args.steps

    for B in (32, 128, 256):
        rng = np.random.default_rng(7000 + B)
        lens = rng.integers(1, cap + 1, size=B)
        sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        q = inputs.device_tensor(1001, inputs.TID_Q, (B, Sq, Hq, d))
        out = torch.empty((B, Sq, Hq, d), dtype=torch.float32, device="cuda")
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device="cuda")
        keys = int(lens.sum())
        by = 2 * B * Sq * Hq * d + 2 * 2 * keys * Hk * d + 4 * B * Sq * Hq * d + 4 * B * Hq * Sq
        k = inputs.device_tensor(1001, inputs.TID_K, (B, cap, Hk, d))
        v = inputs.device_tensor(1001, inputs.TID_V, (B, cap, Hk, d))
        ms_dense = timed(lambda: G.gqa_attn_fwd_kvcache(q, k, v, sl, out=out, lse=lse, stream=stream))
        del k, v
        torch.cuda.empty_cache()
        for ps in (16, 64, 256):
            need = (lens + ps - 1) // ps
            num_pages = int(need.sum())
            perm = rng.permutation(num_pages)
            table = np.zeros((B, cap // ps), dtype=np.int32)
            o = 0
            for b in range(B):
                table[b, :need[b]] = perm[o:o + need[b]]
                o += need[b]
            tt = torch.from_numpy(table).cuda()
            kp = inputs.device_tensor(1002, inputs.TID_K, (num_pages, ps, Hk, d))
            vp = inputs.device_tensor(1002, inputs.TID_V, (num_pages, ps, Hk, d))
            ms = timed(lambda: G.gqa_attn_fwd_paged(q, kp, vp, tt, sl, out=out, lse=lse, stream=stream))
            print(json.dumps({"sweep": "paged", "B": B, "Sk_capacity": cap, "page_size": ps,
                              "mean_length": round(float(lens.mean()), 1), "ms": round(ms, 4),
                              "hbm_gbs": round(by / ms / 1e6, 1),
                              "frac_of_measured_hbm": round(by / ms / 1e6 / peaks["hbm_gbs"], 3),
                              "dense_kvcache_ms": round(ms_dense, 4),
                              "dense_kvcache_gbs": round(by / ms_dense / 1e6, 1),
                              "paged_over_dense": round(ms_dense / ms, 3)}), flush=True)
            del kp, vp
            torch.cuda.empty_cache()


def run_sweep_fp8(args, peaks):
    """Kernel-only timings of gqa_attn_fwd_fp8 (e4m3 Q, K, V with per-tensor scales, fp32
    output) next to gqa_attn_fwd on bf16 inputs of the same shape, both under the automatic
    schedule: the decode grid (Sk 2K/8K/32K, B 32/128/256) against the measured copy
    bandwidth, and the prefill shape (B=64, Sq=Sk=2048, causal and not) against the e4m3
    tensor rate taken as twice the measured bf16 rate (the nominal dense ratio).  Bytes
    count 1 byte per Q/K/V element for e4m3, 2 for bf16."""
    import torch

    import gqa_exact_attention_b200 as G
    import inputs
    stream = torch.cuda.current_stream()
    Hq, Hk, d = 32, 8, 128
    scales = (1 / 16, 1 / 16, 1 / 8)
    cases = [(B, 1, Sk, 0) for Sk in (2048, 8192, 32768) for B in (32, 128, 256)]
    cases += [(64, 2048, 2048, c) for c in (1, 0)]

    def timed(step):
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        if G.gqa_attn_device_status(reset=True) != 0:
            raise SystemExit("an in-kernel bounded wait timed out")
        return e0.elapsed_time(e1) / args.steps

    for (B, Sq, Sk, causal) in cases:
        out = torch.empty((B, Sq, Hq, d), dtype=torch.float32, device="cuda")
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device="cuda")
        q = inputs.device_tensor(1001, inputs.TID_Q, (B, Sq, Hq, d))
        k = inputs.device_tensor(1001, inputs.TID_K, (B, Sk, Hk, d))
        v = inputs.device_tensor(1001, inputs.TID_V, (B, Sk, Hk, d))
        ms_bf16 = timed(lambda: G.gqa_attn_fwd(q, k, v, out=out, lse=lse, causal=causal,
                                               stream=stream))
        del q, k, v
        torch.cuda.empty_cache()
        q = inputs.e4m3_device_tensor(1001, inputs.TID_Q, (B, Sq, Hq, d), scales[0])
        k = inputs.e4m3_device_tensor(1001, inputs.TID_K, (B, Sk, Hk, d), scales[1])
        v = inputs.e4m3_device_tensor(1001, inputs.TID_V, (B, Sk, Hk, d), scales[2])
        ms = timed(lambda: G.gqa_attn_fwd_fp8(q, k, v, *scales, out=out, lse=lse, causal=causal,
                                              stream=stream))
        del q, k, v
        torch.cuda.empty_cache()
        fl = flops(B, Sq, Sk, Hq, d, causal)
        io = 4 * B * Sq * Hq * d + 4 * B * Hq * Sq  # fp32 out + LSE
        by8 = B * Sq * Hq * d + 2 * B * Sk * Hk * d + io
        by16 = 2 * (B * Sq * Hq * d + 2 * B * Sk * Hk * d) + io
        line = {"sweep": "fp8", "B": B, "Sq": Sq, "Sk": Sk, "causal": bool(causal),
                "ms": round(ms, 4), "bf16_ms": round(ms_bf16, 4),
                "speedup_over_bf16": round(ms_bf16 / ms, 3),
                "tflops": round(fl / ms / 1e9, 1), "hbm_gbs": round(by8 / ms / 1e6, 1),
                "bf16_hbm_gbs": round(by16 / ms_bf16 / 1e6, 1)}
        if Sq > 1:
            line["frac_of_e4m3_peak"] = round(fl / ms / 1e9 / (2 * peaks["bf16_tflops"]), 3)
            line["frac_of_measured_bf16"] = round(fl / ms / 1e9 / peaks["bf16_tflops"], 3)
        else:
            line["frac_of_measured_hbm"] = round(by8 / ms / 1e6 / peaks["hbm_gbs"], 3)
        print(json.dumps(line), flush=True)
        del out, lse
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--B", type=int, default=64)
    ap.add_argument("--Sq", type=int, default=2048)
    ap.add_argument("--Sk", type=int, default=2048)
    ap.add_argument("--Hq", type=int, default=32)
    ap.add_argument("--Hk", type=int, default=8)
    ap.add_argument("--d", type=int, default=128)
    ap.add_argument("--causal", type=int, default=1)
    ap.add_argument("--pack", type=int, default=-1)
    ap.add_argument("--splits", type=int, default=0)
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sustained", action="store_true",
                    help="skip the >= 1 s timed region of the main step")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the decode workload of the default line")
    ap.add_argument("--graph", action="store_true",
                    help="--sweep kvcache: replay each call from a CUDA graph")
    ap.add_argument("--sweep", choices=["prefill", "decode", "kvcache", "paged", "fp8"], default=None,
                    help="print one line per configuration of the batch sweep or decode grid")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    default = (args.B, args.Sq, args.Sk, args.Hq, args.Hk, args.d, args.causal) == (64, 2048, 2048, 32, 8, 128, 1)
    name = ("prefill B=64 Hq=32 Hk=8 Sq=Sk=2048 d=128 causal" if default else
            f"B={args.B} Hq={args.Hq} Hk={args.Hk} Sq={args.Sq} Sk={args.Sk} d={args.d} "
            f"{'causal' if args.causal else 'non-causal'}")
    in_bytes = 2 * (args.B * args.Sq * args.Hq * args.d + 2 * args.B * args.Sk * args.Hk * args.d)
    cfg = {"name": name, "B": args.B, "Sq": args.Sq, "Sk": args.Sk, "Hq": args.Hq, "Hk": args.Hk,
           "d": args.d, "causal": args.causal, "seed": 1001,
           "with_decode": default and not args.no_decode,
           "l2": (f"inputs larger than L2 ({in_bytes / 1e6:.0f} MB read per step)"
                  if in_bytes > 126e6 else f"inputs {in_bytes / 1e6:.1f} MB, L2-resident")}
    if args.impl == "reference":
        run_reference(args, cfg)
    elif args.sweep:
        run_sweep(args)
    else:
        run_gpu(args, cfg)


if __name__ == "__main__":
    main()
