#!/usr/bin/env python
"""Benchmark of the exact fused attention path on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
the forward (fa_fwd) and the backward (its two launches: prep and main)
of exact attention on the long-context causal workload B=4, H=16, N=4096,
d=128, bf16, Q/K/V/dO iid N(0, 1).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Rank 0 prints one JSON line. Multi-GPU runs (torchrun, one process per GPU)
give every rank its own batch of the same workload (weak scaling); the path has
no data exchange between ranks, so the only collectives are the barriers and
the max-over-ranks of the timings.

``--impl reference`` times the fp64 CPU oracle instead, on a bounded sample of
the same workload per step (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd/bwd TFLOP/s and % of B200 BF16 tensor peak (N=1K–64K)"
UNIT = "TFLOP/s"
L2_BYTES = 126 * 1024 * 1024

WORKLOADS = {
    "long_causal_d128": dict(B=4, H=16, N=4096, d=128, causal=True, fmt="bf16", mask=False,
                             desc="long-context causal attention B=4 H=16 N=4096 d=128 bf16, fwd+bwd"),
    "tiny_exact": dict(B=1, H=1, N=128, d=64, causal=False, fmt="fp16", mask=False,
                       desc="tiny exact check B=1 H=1 N=128 d=64 fp16, fwd+bwd (one CTA; latency bound)"),
    "gpt2_small": dict(B=8, H=12, N=1024, d=64, causal=False, fmt="bf16", mask=False,
                       desc="GPT-2-small-shaped attention B=8 H=12 N=1024 d=64 bf16, fwd+bwd"),
    "gpt2_small_causal": dict(B=8, H=12, N=1024, d=64, causal=True, fmt="bf16", mask=False,
                              desc="GPT-2-small-shaped causal attention B=8 H=12 N=1024 d=64 bf16, fwd+bwd"),
    "linear_memory_64k": dict(B=1, H=16, N=65536, d=64, causal=True, fmt="bf16", mask=False,
                              desc="linear-memory stress causal attention B=1 H=16 N=65536 d=64 bf16, fwd+bwd"),
    "block_sparse_8k": dict(B=2, H=16, N=8192, d=64, causal=False, fmt="bf16", mask=True,
                            desc="block-sparse attention B=2 H=16 N=8192 d=64 bf16, 128x128 tile mask, fwd+bwd"),
}
DEFAULT_WORKLOAD = "long_causal_d128"


# ----------------------------------------------------------------------------- helpers

def workload_density(w) -> float:
    if not w["mask"]:
        return 1.0
    import fa_synth
    m = fa_synth.block_mask_recipe(w["N"] // 128)
    return float(m.sum()) / m.size


def step_flops(w, density=None):
    """Algorithmic FLOPs: forward 4·B·H·N²·d, backward 2.5× that, halved for causal,
    scaled by the non-zero tile fraction for block-sparse."""
    if density is None:
        density = workload_density(w)
    f = 4.0 * w["B"] * w["H"] * w["N"] ** 2 * w["d"] * (0.5 if w["causal"] else 1.0) * density
    return f, 2.5 * f


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"bf16": float(p["bf16_tflops"]), "bf16_sustained": float(p.get("bf16_tflops_sustained", 0) or 0),
                "hbm": float(p["hbm_gbs"]), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"bf16": 1590.0, "bf16_sustained": 1400.0, "hbm": 6650.0, "source": "fallback"}


def load_traffic(kernel_key):
    """DRAM bytes per launch from a committed ncu capture, if the kernel source is unchanged since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel_key]
    except (OSError, KeyError, ValueError):
        return None
    import hashlib
    h = hashlib.sha256()
    for name in rec.get("sources", []):
        with open(os.path.join(ROOT, name), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != rec.get("sha256"):
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock/throttle sampling while the timed region runs."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, path: str):
        self.path = path
        self.proc = None
        try:
            self.fh = open(path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self, t0: float, t1: float):
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [x.strip() for x in line.split(",")]
                    if len(parts) < 8:
                        continue
                    try:
                        ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                        frac = float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                        rows.append((ts + frac, float(parts[1]), float(parts[2]), parts[4:8]))
                    except ValueError:
                        continue
        except OSError:
            return None
        if not rows:
            return None
        inside = [r for r in rows if t0 - 0.15 <= r[0] <= t1 + 0.15]
        use = inside if len(inside) >= 1 else rows
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in use for i, v in enumerate(r[3]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": reasons, "samples": len(use), "samples_in_timed_region": len(inside)}


def oracle_sample_step(vals, w, rows, head):
    """One bounded sample of the workload on the CPU oracle: forward and backward of
    the loss restricted to `rows` query rows of one head."""
    import oracle
    q, k, v, do = (vals[n][head] for n in ("q", "k", "v", "do"))
    scale = 1.0 / math.sqrt(w["d"])
    mask = None
    if w["mask"]:
        import fa_synth
        mask = fa_synth.block_mask_recipe(w["N"] // 128)
    oracle.backward_rows(q, k, v, do, scale, rows, causal=w["causal"], block_mask=mask)


def oracle_inputs(w, heads, seed=0):
    import fa_synth
    bits = fa_synth.attention_input_bits(w["B"], w["H"], w["N"], w["d"], w["fmt"], seed)
    return {n: fa_synth.bits_to_values(b.reshape((-1,) + b.shape[2:])[heads], w["fmt"]) for n, b in bits.items()}


def cpu_description():
    """Model name and logical core count of the host running the oracle."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        usable = os.cpu_count() or 1
    return {"cpu_model": model, "nproc": usable}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"), default=1)
    except ImportError:
        return 1


def sample_rows_for(w, n_rows):
    import numpy as np
    step = w["N"] // n_rows
    return np.arange(n_rows) * step + step // 2


def cpu_rate(w, vals, n_rows, budget_s, min_steps=1, max_steps=None):
    """Run oracle samples until `budget_s` seconds pass; returns (TFLOP/s, steps, seconds)."""
    f_fwd, f_bwd = step_flops(w)
    per_row = (f_fwd + f_bwd) / (w["B"] * w["H"] * w["N"])
    rows = sample_rows_for(w, n_rows)
    nheads = next(iter(vals.values())).shape[0]
    t0 = time.perf_counter()
    steps = 0
    while True:
        oracle_sample_step(vals, w, rows, steps % nheads)
        steps += 1
        el = time.perf_counter() - t0
        if steps >= min_steps and (el >= budget_s or (max_steps and steps >= max_steps)):
            break
    return per_row * n_rows * steps / el / 1e12, steps, el


# ----------------------------------------------------------------------------- multi-rank plumbing

def max_over_ranks(values, device=None, world=1):
    """Element-wise max of a list of floats over all ranks of the default process
    group (device times are reported as the slowest rank's)."""
    vals = [float(x) for x in values]
    if world == 1:
        return vals
    import torch
    import torch.distributed as dist
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_tflops(flops_per_rank_step, steps, world, ms_max):
    """Throughput of the whole job: every rank processes its own batch of the same
    size (weak scaling), so total work over the slowest rank's time."""
    return world * flops_per_rank_step * steps / (ms_max * 1e-3) / 1e12


def rank_seed(rank):
    """Seed of a rank's synthetic batch: each rank draws an independent batch."""
    return rank


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, w, rank, world):
    if rank != 0:
        return 0
    vals = oracle_inputs(w, list(range(min(4, w["B"] * w["H"]))))
    f_fwd, f_bwd = step_flops(w)
    per_row = (f_fwd + f_bwd) / (w["B"] * w["H"] * w["N"])
    # Size the per-step sample so warm-up plus timed steps stay within the budget.
    rows = sample_rows_for(w, 64)
    t0 = time.perf_counter()
    oracle_sample_step(vals, w, rows, 0)
    t_probe = max(time.perf_counter() - t0, 1e-4)
    n_rows = 64
    target = args.reference_seconds / max(1, args.steps + args.warmup)
    while n_rows < min(w["N"], 2048) and t_probe * (2 * n_rows) / 64 <= target:
        n_rows *= 2
    rows = sample_rows_for(w, n_rows)
    nheads = next(iter(vals.values())).shape[0]
    for s in range(args.warmup):
        oracle_sample_step(vals, w, rows, s % nheads)
    t0 = time.perf_counter()
    for s in range(args.steps):
        oracle_sample_step(vals, w, rows, s % nheads)
    el = time.perf_counter() - t0
    value = per_row * n_rows * args.steps / el / 1e12
    sample = f"{n_rows} of {w['N']} query rows of one (batch, head) per step, forward + backward of the loss on those rows"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(w, args.workload),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle", "sample": sample,
                         **cpu_description()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def input_bytes(w):
    return 4 * w["B"] * w["H"] * w["N"] * w["d"] * 2


def needs_l2_flush(w):
    """Inputs under twice the L2 size could stay cached between steps: flush instead."""
    return input_bytes(w) < 2 * L2_BYTES


def config_block(w, name):
    l2 = (f"L2 flushed between steps ({2 * L2_BYTES >> 20} MiB write outside the timed events); "
          if needs_l2_flush(w) else "inputs larger than L2 (no flush): ")
    return {"workload": w["desc"], "name": name, "B": w["B"], "H": w["H"], "N": w["N"], "d": w["d"],
            "causal": w["causal"], "block_sparse": w["mask"], "dtype": w["fmt"],
            "l2": l2 + str(round(input_bytes(w) / 2 ** 20)) + " MiB of Q/K/V/dO per step",
            "parallelism": "one independent batch per GPU"}


# ----------------------------------------------------------------------------- GPU arm

class Problem:
    """Device buffers of one workload (seeded synthetic inputs) and its launches
    through the binding of the C ABI."""

    def __init__(self, w, dev, seed):
        import numpy as np
        import torch

        import fa_synth
        import io_aware_exact_19_b200 as fa

        self.fa = fa
        self.w = w
        B, H, N, d = w["B"], w["H"], w["N"], w["d"]
        tdt = torch.bfloat16 if w["fmt"] == "bf16" else torch.float16
        bits = fa_synth.attention_input_bits(B, H, N, d, w["fmt"], seed=seed)
        self.host = {n: torch.from_numpy(b.view(np.int16)).view(tdt) for n, b in bits.items()}
        self.q, self.k, self.v, self.do = (self.host[n].to(dev) for n in ("q", "k", "v", "do"))
        self.mask = None
        if w["mask"]:
            self.mask = torch.from_numpy(fa_synth.block_mask_recipe(N // 128)).to(dev)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        self.dq, self.dk, self.dv = (torch.empty_like(t) for t in (self.q, self.k, self.v))
        self.ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
        self.stream = torch.cuda.current_stream()

    def fwd(self):
        fa, w = self.fa, self.w
        if self.mask is None:
            fa.fa_fwd(self.q, self.k, self.v, self.o, self.lse, w["causal"])
        else:
            fa.fa_blocksparse_fwd(self.q, self.k, self.v, self.o, self.lse, self.mask, w["causal"])

    def bwd_phase(self, ph):
        self.fa.fa_debug_bwd_phase(ph, self.q, self.k, self.v, self.o, self.lse, self.do, self.dq, self.dk, self.dv,
                                   self.ws, causal=self.w["causal"], block_mask=self.mask)

    def bwd(self):
        fa, w = self.fa, self.w
        if self.mask is None:
            fa.fa_bwd(self.q, self.k, self.v, self.o, self.lse, self.do, self.dq, self.dk, self.dv, self.ws,
                      w["causal"])
        else:
            fa.fa_blocksparse_bwd(self.q, self.k, self.v, self.o, self.lse, self.do, self.dq, self.dk, self.dv,
                                  self.ws, self.mask, w["causal"])

    def step(self, ev=None):
        """Forward, then the backward's two launches (prep, main); `ev` = four CUDA
        events recorded on the launching stream around them."""
        if ev is not None:
            ev[0].record(self.stream)
        self.fwd()
        if ev is not None:
            ev[1].record(self.stream)
        self.bwd_phase(0)
        if ev is not None:
            ev[2].record(self.stream)
        self.bwd_phase(1)
        if ev is not None:
            ev[3].record(self.stream)


def timed_steps(prob, steps, warmup, dev, flush_l2, between=None):
    """Run `warmup` untimed steps, then `steps` steps each bracketed by CUDA events
    on the launching stream. With `flush_l2`, a buffer twice the L2 size is written
    between steps, outside the events. Returns per-step (total, fwd, prep, main) ms."""
    import torch
    for _ in range(max(warmup, 3)):
        prob.step()
    torch.cuda.synchronize()
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if flush_l2 else None
    if between is not None:
        between()
    for s in range(steps):
        if flush is not None:
            flush.fill_(s & 0xFF)
        prob.step(events[s])
    torch.cuda.synchronize()
    return [(e[0].elapsed_time(e[3]), e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3]))
            for e in events]


def prep_bytes(w):
    """Algorithmic bytes of the backward's prep launch: read O, dO (16-bit) and lse;
    write D and lse in log2 units (fp32)."""
    return w["B"] * w["H"] * w["N"] * (w["d"] * 2 * 2 + 4 * 3)


def summarize(w, times, peaks):
    """Per-launch averages and rates of one workload's timed steps."""
    f_fwd, f_bwd = step_flops(w)
    n = len(times)
    fwd = sum(t[1] for t in times) / n
    prep = sum(t[2] for t in times) / n
    main = sum(t[3] for t in times) / n
    tot = sum(t[0] for t in times) / n
    bwd = prep + main
    return {
        "ms_per_step": tot, "step_tflops": (f_fwd + f_bwd) / (tot * 1e-3) / 1e12,
        "fwd_ms": fwd, "fwd_tflops": f_fwd / (fwd * 1e-3) / 1e12,
        "fwd_frac_of_measured_peak": f_fwd / (fwd * 1e-3) / 1e12 / peaks["bf16"],
        "bwd_ms": bwd, "bwd_tflops": f_bwd / (bwd * 1e-3) / 1e12,
        "bwd_frac_of_measured_peak": f_bwd / (bwd * 1e-3) / 1e12 / peaks["bf16"],
        "bwd_main_ms": main, "bwd_main_tflops": f_bwd / (main * 1e-3) / 1e12,
        "bwd_prep_ms": prep, "bwd_prep_gbs": prep_bytes(w) / (prep * 1e-3) / 1e9,
        "bwd_prep_frac_of_measured_hbm": prep_bytes(w) / (prep * 1e-3) / 1e9 / peaks["hbm"],
        # Algorithmic HBM bytes of the whole step (Q, K, V, dO read once; O, dQ, dK,
        # dV and lse written once) over its time: the figure that matters for the
        # small cases, which are latency rather than tensor bound.
        "step_min_hbm_gbs": (w["B"] * w["H"] * w["N"] * (w["d"] * 2 * 8 + 4)) / (tot * 1e-3) / 1e9,
        "vendor_peak_tflops": 2250.0,
        "fwd_frac_of_vendor_peak": f_fwd / (fwd * 1e-3) / 1e12 / 2250.0,
        "bwd_frac_of_vendor_peak": f_bwd / (bwd * 1e-3) / 1e12 / 2250.0,
        "steps": n,
    }


DECODE = dict(B=1, H=16, Nq=1, Nk=65536, d=64, fmt="bf16", causal=True,
              desc="decoding: one query row against a 64K key cache, B=1 H=16 d=64 bf16, split-KV forward")


def time_decode(dev, peaks, steps=50):
    """Split-KV forward (fa_fwd_splitkv) on the decoding shape, against the same
    forward without splitting (fa_fwd_qk). HBM bound: the bytes are K and V
    (read once) plus Q, O and lse. K and V (256 MiB) are larger than the L2 and
    every step streams each key range from its start, so no flush is needed (a
    written flush buffer would leave dirty lines whose write-back lands inside
    this HBM-bound step)."""
    import numpy as np
    import torch

    import fa_synth
    import io_aware_exact_19_b200 as fa

    w = DECODE
    B, H, Nq, Nk, d = w["B"], w["H"], w["Nq"], w["Nk"], w["d"]
    bq = fa_synth.attention_input_bits(B, H, Nq, d, w["fmt"], seed=11)
    bk = fa_synth.attention_input_bits(B, H, Nk, d, w["fmt"], seed=12)
    to = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(dev)
    q, k, v = to(bq["q"]), to(bk["k"]), to(bk["v"])
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
    ns = fa.fa_fwd_splitkv_splits(B, H, Nq, Nk)
    ws = torch.empty(fa.fa_fwd_splitkv_workspace_size(B, H, Nq, d, ns), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def timed(fn):
        # Steps back to back between two events: a step is short (tens of
        # microseconds), so waiting for the host before each one would time the
        # launch calls rather than the device.
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    ms_split = timed(lambda: fa.fa_fwd_splitkv(q, k, v, o, lse, ns, ws, causal=w["causal"]))
    ms_plain = timed(lambda: fa.fa_fwd_qk(q, k, v, o, lse, causal=w["causal"]))
    status = fa.fa_device_status()
    nbytes = 2 * B * H * Nk * d * 2 + 2 * B * H * Nq * d * 2 + B * H * Nq * 4
    flops = 4.0 * B * H * Nq * Nk * d
    gbs = nbytes / (ms_split * 1e-3) / 1e9
    return {"workload": w["desc"], "n_splits": ns, "ms": ms_split, "hbm_gbs": gbs,
            "hbm_frac_of_measured_peak": gbs / peaks["hbm"], "tflops": flops / (ms_split * 1e-3) / 1e12,
            "unsplit_ms": ms_plain, "speedup_vs_unsplit": ms_plain / ms_split,
            "bytes_per_step": nbytes, "l2": "inputs larger than L2 (no flush): K and V 256 MiB per step",
            "device_status": int(status), "launches_per_step": 2, "steps": steps}


def time_dropout(dev, peaks, p_drop=0.1, steps=30):
    """The long-context causal workload with dropout on P (fa_fwd_dropout /
    fa_bwd_dropout, p = 0.1): forward and backward TFLOP/s under the same FLOP
    convention (dropout adds no credited FLOPs), beside the same calls at p = 0."""
    import torch

    import io_aware_exact_19_b200 as fa

    w = WORKLOADS["long_causal_d128"]
    prob = Problem(w, dev, 21)
    seed = 0x5EED
    f_fwd, f_bwd = step_flops(w)
    stream = torch.cuda.current_stream()
    out = {"workload": w["desc"] + ", dropout p=0.1 on P", "p_drop": p_drop, "steps": steps}
    for label, pd in (("dropout", p_drop), ("no_dropout", 0.0)):
        def fwd():
            fa.fa_fwd_dropout(prob.q, prob.k, prob.v, prob.o, prob.lse, pd, seed, causal=True)

        def bwd():
            fa.fa_bwd_dropout(prob.q, prob.k, prob.v, prob.o, prob.lse, prob.do, prob.dq, prob.dk, prob.dv, prob.ws,
                              pd, seed, causal=True)

        for _ in range(3):
            fwd()
            bwd()
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for e in ev:
            e[0].record(stream)
            fwd()
            e[1].record(stream)
            bwd()
            e[2].record(stream)
        torch.cuda.synchronize()
        fwd_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / steps
        bwd_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / steps
        out[label] = {"fwd_ms": fwd_ms, "fwd_tflops": f_fwd / (fwd_ms * 1e-3) / 1e12, "bwd_ms": bwd_ms,
                      "bwd_tflops": f_bwd / (bwd_ms * 1e-3) / 1e12,
                      "fwd_frac_of_measured_peak": f_fwd / (fwd_ms * 1e-3) / 1e12 / peaks["bf16"],
                      "bwd_frac_of_measured_peak": f_bwd / (bwd_ms * 1e-3) / 1e12 / peaks["bf16"]}
    out["device_status"] = int(fa.fa_device_status())
    return out


def time_fp8(dev, peaks, steps=50):
    """The long-context causal workload's forward with 8-bit (e4m3) Q, K, V
    (fa_fwd_fp8), TFLOP/s under the forward's FLOP convention. Its inputs (3 x 32
    MiB) are under twice the L2 size, so the L2 is flushed between steps."""
    import torch

    import fa_synth
    import io_aware_exact_19_b200 as fa

    w = WORKLOADS["long_causal_d128"]
    B, H, N, d = w["B"], w["H"], w["N"], w["d"]
    bits, sc = fa_synth.fp8_attention_input_bits(B, H, N, N, d, seed=31)
    q, k, v = (torch.from_numpy(bits[n]).to(dev) for n in ("q", "k", "v"))
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    f_fwd, _ = step_flops(w)
    run = lambda: fa.fa_fwd_fp8(q, k, v, sc["q"], sc["k"], sc["v"], o, lse, causal=True)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    tot = 0.0
    for i in range(steps):
        flush.fill_(i & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run()
        e1.record(stream)
        torch.cuda.synchronize()
        tot += e0.elapsed_time(e1)
    ms = tot / steps
    tf = f_fwd / (ms * 1e-3) / 1e12
    return {"workload": w["desc"].replace("bf16, fwd+bwd", "e4m3 Q/K/V, forward"), "fwd_ms": ms, "fwd_tflops": tf,
            "fwd_frac_of_measured_bf16_peak": tf / peaks["bf16"],
            "note": "S = Q K^T in e4m3 (kind::f8f6f4), P V in bf16", "l2": "L2 flushed between steps",
            "device_status": int(fa.fa_device_status()), "steps": steps}


def _time_pair(fwd, bwd, flush, steps, stream):
    """Mean device milliseconds of fwd and bwd (bwd may be None), L2 flushed before each step."""
    import torch

    for _ in range(3):
        fwd()
        if bwd is not None:
            bwd()
    torch.cuda.synchronize()
    tf = tb = 0.0
    for i in range(steps):
        flush.fill_(i & 0xFF)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(stream)
        fwd()
        ev[1].record(stream)
        if bwd is not None:
            bwd()
        ev[2].record(stream)
        torch.cuda.synchronize()
        tf += ev[0].elapsed_time(ev[1])
        tb += ev[1].elapsed_time(ev[2])
    return tf / steps, (tb / steps if bwd is not None else None)


def time_head_dims(dev, peaks, steps=30):
    """The long-context causal shape (B=4 H=16 N=4096, bf16) at head dimensions 32,
    96 and 256 (forward only: the backward supports d <= 128), and a chunked-prefill
    shape with N_q != N_k (1024 queries against 8192 keys, bottom-right causal,
    d = 128) through fa_fwd_qk / fa_bwd_qk. TFLOP/s count the allowed (query, key)
    pairs: 4 d per pair forward, 2.5 times that backward. L2 flushed between steps."""
    import torch

    import fa_synth
    import io_aware_exact_19_b200 as fa

    stream = torch.cuda.current_stream()
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    out = {}
    cases = [("d32", 4, 16, 4096, 4096, 32), ("d96", 4, 16, 4096, 4096, 96), ("d256", 4, 16, 4096, 4096, 256),
             ("nq1024_nk8192_d128", 4, 16, 1024, 8192, 128)]
    for label, B, H, Nq, Nk, d in cases:
        bq = fa_synth.attention_input_bits(B, H, Nq, d, "bf16", seed=41, names=("q", "do"))
        bk = fa_synth.attention_input_bits(B, H, Nk, d, "bf16", seed=42, names=("k", "v"))
        t = lambda b: torch.from_numpy(b.view("int16")).view(torch.bfloat16).to(dev)
        q, do, k, v = t(bq["q"]), t(bq["do"]), t(bk["k"]), t(bk["v"])
        o = torch.empty_like(q)
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
        fwd = lambda: fa.fa_fwd_qk(q, k, v, o, lse, causal=True)
        bwd = None
        if d <= 128:
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
            ws = torch.empty(fa.fa_bwd_workspace_size(B, H, Nq, d), dtype=torch.uint8, device=dev)
            bwd = lambda: fa.fa_bwd_qk(q, k, v, o, lse, do, dq, dk, dv, ws, causal=True)
        fms, bms = _time_pair(fwd, bwd, flush, steps, stream)
        pairs = Nq * (Nk - Nq) + Nq * (Nq + 1) / 2
        f_fwd = 4.0 * d * pairs * B * H
        rec = {"B": B, "H": H, "N_q": Nq, "N_k": Nk, "d": d, "causal": True, "fwd_ms": fms,
               "fwd_tflops": f_fwd / (fms * 1e-3) / 1e12,
               "fwd_frac_of_measured_peak": f_fwd / (fms * 1e-3) / 1e12 / peaks["bf16"]}
        if bms is not None:
            rec.update({"bwd_ms": bms, "bwd_tflops": 2.5 * f_fwd / (bms * 1e-3) / 1e12,
                        "bwd_frac_of_measured_peak": 2.5 * f_fwd / (bms * 1e-3) / 1e12 / peaks["bf16"]})
        out[label] = rec
        del q, k, v, do, o
        torch.cuda.empty_cache()
    out["device_status"] = int(fa.fa_device_status())
    out["l2"] = "L2 flushed between steps"
    return out


def run_gpu(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import io_aware_exact_19_b200 as fa

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    B, H, N, d = w["B"], w["H"], w["N"], w["d"]
    prob = Problem(w, dev, rank_seed(rank))

    for _ in range(max(args.warmup, 3)):
        prob.step()
    torch.cuda.synchronize()
    if fa.fa_device_status() != fa.FA_OK:
        raise RuntimeError("device status reported a time-out during warm-up")

    import tempfile
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(gpu_id, os.path.join(tempfile.gettempdir(), f"fa_bench_clocks_rank{rank}_{os.getpid()}.csv"))
    time.sleep(0.3)
    marks = {}

    def start():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        marks["t0"] = time.time()

    times = timed_steps(prob, args.steps, 0, dev, needs_l2_flush(w), between=start)
    t_wall1 = time.time()
    if world > 1:
        dist.barrier()
    time.sleep(0.2)
    sampler.stop()
    clocks = sampler.summary(marks["t0"], t_wall1)
    status = fa.fa_device_status()

    # Sum of the per-step spans (first to last launch of each step): the L2 flush
    # between steps, where there is one, stays outside.
    ms_total = sum(t[0] for t in times)
    main_sum = sum(t[3] for t in times)
    fwd_sum = sum(t[1] for t in times)
    ms_total, main_sum, fwd_sum = max_over_ranks([ms_total, main_sum, fwd_sum], dev, world)

    f_fwd, f_bwd = step_flops(w)
    value = whole_job_tflops(f_fwd + f_bwd, args.steps, world, ms_total)
    peaks = load_peaks()
    main_avg = main_sum / args.steps
    achieved = f_bwd / (main_avg * 1e-3) / 1e12
    breakdown = summarize(w, times, peaks)

    # ---- end to end through the C ABI: pinned host inputs in, results back to pinned host memory.
    # Two device buffer sets: step k's inputs are copied in (one stream) while step k-1
    # computes and step k-2's results are copied out (another stream), as a training or
    # serving loop would stream batches; every step still moves all of its inputs and
    # results between host and device inside the timed region.
    import copy
    pin = {n: t.pin_memory() for n, t in prob.host.items()}
    out_names = ("o", "lse", "dq", "dk", "dv")
    prob2 = copy.copy(prob)
    for n in ("q", "k", "v", "do") + out_names + ("ws",):
        setattr(prob2, n, torch.empty_like(getattr(prob, n)))
    bufs = (prob, prob2)
    out_host = [{n: torch.empty(getattr(prob, n).shape, dtype=getattr(prob, n).dtype, pin_memory=True)
                 for n in out_names} for _ in range(2)]
    e2e_steps = max(2, min(args.steps, 20))
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(steps, start):
        for k in range(steps):
            b = k % 2
            pb = bufs[b]
            with torch.cuda.stream(s_in):
                s_in.wait_event(computed[b] if k >= 2 else start)  # step k-2 has read these inputs
                for n in ("q", "k", "v", "do"):
                    getattr(pb, n).copy_(pin[n], non_blocking=True)
                in_ready[b].record(s_in)
            comp.wait_event(in_ready[b])
            if k >= 2:
                comp.wait_event(out_done[b])  # step k-2's results have been read back
            pb.fwd()
            pb.bwd()
            computed[b].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(computed[b])
                for n in out_names:
                    out_host[b][n].copy_(getattr(pb, n), non_blocking=True)
                out_done[b].record(s_out)
        comp.wait_event(out_done[0])
        comp.wait_event(out_done[1])

    w0 = torch.cuda.Event()
    w0.record(comp)
    e2e_run(2, w0)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    e2e_run(e2e_steps, e0)
    e1.record(comp)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks([e0.elapsed_time(e1)], dev, world)[0]
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = sum(t.numel() * t.element_size() for t in out_host[0].values())
    e2e_value = whole_job_tflops(f_fwd + f_bwd, e2e_steps, world, e2e_ms)
    del prob, prob2, bufs, out_host, pin

    # ---- the other workloads, each timed the same way (after the headline, outside its timed region)
    per_workload = {}
    if not args.no_per_workload:
        for name, ow in WORKLOADS.items():
            if name == args.workload:
                continue
            p2 = Problem(ow, dev, rank_seed(rank))
            steps = 10 if ow["N"] >= 32768 else 50
            t2 = timed_steps(p2, steps, 3, dev, needs_l2_flush(ow))
            st2 = fa.fa_device_status()
            tot = max_over_ranks([sum(t[0] for t in t2)], dev, world)[0]
            ff, fb = step_flops(ow)
            rec = {"workload": ow["desc"], "value": whole_job_tflops(ff + fb, steps, world, tot),
                   "unit": UNIT, "l2": config_block(ow, name)["l2"], "device_status": int(st2)}
            rec.update(summarize(ow, t2, peaks))
            per_workload[name] = rec
            del p2
            torch.cuda.empty_cache()
        per_workload["decode_splitkv_64k"] = time_decode(dev, peaks)
        torch.cuda.empty_cache()
        per_workload["long_causal_d128_dropout"] = time_dropout(dev, peaks)
        torch.cuda.empty_cache()
        per_workload["long_causal_d128_fp8_fwd"] = time_fp8(dev, peaks)
        torch.cuda.empty_cache()
        per_workload["head_dims_and_unequal_lengths"] = time_head_dims(dev, peaks)
        torch.cuda.empty_cache()

    if rank != 0:
        return 0

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        vals = oracle_inputs(w, list(range(min(4, B * H))))
        rate, n_steps, secs = cpu_rate(w, vals, 512 if N >= 4096 else min(N, 256), budget_s=12.0)
        cpu = {"value": rate, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{n_steps} samples x 512 of {N} query rows of one (batch, head), forward + backward "
                         f"of the loss on those rows, fp64, {secs:.1f} s", **cpu_description()}

    kernel_key = f"fa_bwd_main_kernel<{d},{'bf16' if w['fmt'] == 'bf16' else 'fp16'}>"
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w["fmt"], "data": "synthetic",
        "config": config_block(w, args.workload),
        "roofline": {"kernel": kernel_key, "bound": "tensor", "achieved": achieved, "peak": peaks["bf16"],
                     "unit": UNIT, "frac": achieved / peaks["bf16"],
                     "peak_source": f"{peaks['source']} bf16 dense burst" + (
                         "; fp16 MMAs run at the bf16 rate (nominal ratio 1)" if w["fmt"] == "fp16" else ""),
                     "traffic": load_traffic(kernel_key),
                     "flops_per_launch": f_bwd},
        "breakdown": breakdown,
        "per_workload": per_workload,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps,
                "note": "two device buffer sets: inputs of step k copied in while step k-1 computes and the "
                        "results of step k-2 are copied out (separate streams)"},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks,
        "device_status": int(status),
        "wall_s_timed_region": t_wall1 - marks["t0"],
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)
    return 0


def spawn_ranks(n, argv):
    """Run this script as n ranks, one process per GPU, under torch.distributed.run
    (rendezvous on 127.0.0.1); returns its exit status."""
    import socket
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        port = sock.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(n),
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="time only the selected workload (the default also times every other one)")
    ap.add_argument("--extra", choices=("decode_splitkv_64k", "long_causal_d128_dropout", "long_causal_d128_fp8_fwd",
                                        "head_dims_and_unequal_lengths"),
                    help="run only this one of the extra measurements (1 GPU) and print its record")
    ap.add_argument("--reference-seconds", type=float, default=120.0,
                    help="approximate CPU time budget of the reference arm (warm-up plus timed steps)")
    args = ap.parse_args(argv)
    w = WORKLOADS[args.workload]
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return spawn_ranks(args.gpus, sys.argv[1:] if argv is None else list(argv))
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; launch one process per GPU", file=sys.stderr)
        return 2
    if args.impl == "reference":
        return run_reference(args, w, rank, world)
    if args.extra:
        import torch
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        fn = {"decode_splitkv_64k": time_decode, "long_causal_d128_dropout": time_dropout,
              "long_causal_d128_fp8_fwd": time_fp8, "head_dims_and_unequal_lengths": time_head_dims}[args.extra]
        print(json.dumps({args.extra: fn(dev, load_peaks())}), flush=True)
        return 0
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_gpu(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
