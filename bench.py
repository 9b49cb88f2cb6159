#!/usr/bin/env python
"""Benchmark of the block-sparse attention hot path on B200.

One step = one pass of the whole path on the Wan2.1-14B-shaped self-attention
call (B=1, H=40, N=75600 = 21x45x80 tokens, d=128, bf16, topk=0.5): mean
pooling, block scores + top-k selection, and block-sparse attention over the
kept 128x64 tiles.  The timed step issues sparse_attn_select and then
block_sparse_attn_apply on one stream -- the same kernels, in the same order,
that the fused sparse_attn_topk call launches -- so that the attention kernel
can be timed on its own with CUDA events; the fused call is timed too.

Prints one JSON line (rank 0).  Metric: dense-equivalent TFLOPS
(4*B*H*N^2*d / step time), plus ms/call and the fraction of the measured bf16
tensor-core peak reached by the attention kernel on its kept tiles.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {b200,reference}]
                    [--workload W] [--call {topk,mask,cdf}] [--topk T] [--density P]
                    [--threshold C] [--causal] [--plan-reuse R] [--sweep]

--call mask times a caller-supplied random block mask at --density (compaction
then attention, or block_sparse_attn_fwd fused); --call cdf the cdfthreshd
selection at --threshold; --causal the causal variant; --plan-reuse R one
selection followed by R applies of its plan (the AB-Attention refresh pattern),
reporting the amortised time per call.  --sweep prints one line per row of the
workload table (every config and mode), without the CPU and end-to-end legs.

--steps K times exactly K steps; without it the bench picks enough steps for
~1 s of timed work (10 to 500) from one untimed step, so that the clock samples
fall inside the timed region.

Multi-GPU (torchrun, one rank per GPU): every rank runs its own independent
call (weak scaling, no collective on the data path); the step time is the
maximum over ranks.  --impl reference times the fp64 CPU oracle on a bounded
sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import csv
from datetime import datetime
import glob
import hashlib
import io
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_attention_14_b200 import workloads as W  # noqa: E402

METRIC = "ms/call and dense-equiv TFLOPS, Wan-14B-shaped topk=0.5, % of bf16 TC peak"
UNIT = "dense-equiv TFLOPS"
TF32_PER_BF16 = 1.1 / 2.25  # nominal dense TF32 / bf16 tensor-core ratio
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}
ATTN_SRCS = [os.path.join(ROOT, "block_sparse_attention_14_b200", "csrc", f)
             for f in ("bsa_attn.cu", "bsa_common.cuh")]
TRAFFIC_GLOB = os.path.join(ROOT, "profiles", "bsa_fwd*_kernel_*_ncu.md")


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=None,
                   help="timed steps (default: 10, or more so the timed region lasts ~1 s; at most 500)")
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["b200", "reference"], default="b200")
    p.add_argument("--workload", default="wan14b", choices=sorted(W.WORKLOADS))
    p.add_argument("--call", choices=["topk", "mask", "cdf"], default="topk")
    p.add_argument("--topk", type=float, default=0.5)
    p.add_argument("--density", type=float, default=0.5, help="caller-mask density (--call mask)")
    p.add_argument("--threshold", type=float, default=0.9, help="cdfthreshd threshold (--call cdf)")
    p.add_argument("--causal", action="store_true")
    p.add_argument("--plan-reuse", type=int, default=1,
                   help="applies of each selection's plan per step (amortised per call)")
    p.add_argument("--sweep", action="store_true", help="one line per row of the workload table")
    p.add_argument("--table", metavar="JSONL", default=None,
                   help="print the markdown table of a --sweep output file (no GPU work)")
    p.add_argument("--heads", type=int, default=0,
                   help="override H (small profiling case only; not a bench line)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-fused", action="store_true")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in PEAKS_FALLBACK}, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def attn_source_hash() -> str:
    """sha256[:16] of the attention kernel's sources (the kernel file and the
    device-helper header it inlines), concatenated."""
    h = hashlib.sha256()
    for path in ATTN_SRCS:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """Per-launch DRAM bytes of the attention kernel from a committed ncu summary
    (profiles/bsa_fwd*_kernel_*_ncu.md), valid only if it was taken on the current
    kernel source."""
    want = attn_source_hash()
    for path in sorted(glob.glob(TRAFFIC_GLOB)):
        with open(path) as f:
            for line in f:
                if line.startswith("traffic_bytes_per_launch:"):
                    parts = dict(x.split("=", 1) for x in line.split(":", 1)[1].split() if "=" in x)
                    if parts.get("workload") == workload and parts.get("source") == want:
                        return float(parts["bytes"])
    return None


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons every 50 ms.  Started before
    the warm-up (nvidia-smi takes a few hundred ms to emit its first row); stop()
    keeps the rows whose timestamps fall inside the timed region."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.path = None
        try:
            props = torch.cuda.get_device_properties(device)
            bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
        except Exception:
            bus = None
        self.bus = bus

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"]
            if self.bus:
                cmd.insert(1, f"--id={self.bus}")
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, t_begin: float, t_end: float):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for r in csv.reader(f):
                if len(r) >= 9:
                    try:
                        ts = datetime.strptime(r[0].strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    except ValueError:
                        continue
                    rows.append((ts, [x.strip() for x in r[1:]]))
        os.unlink(self.path)
        timed = [r for ts, r in rows if t_begin <= ts <= t_end]
        window = "timed region"
        if not timed:  # the timed region ended before nvidia-smi's first row
            timed, window = [r for _, r in rows], "whole run"
        rows = timed
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        loaded = [s for s in sm if s > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows),
                "window": window}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    """Maximum of a per-rank scalar (a step time) over all ranks."""
    if world == 1:
        return x
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(dense_flops_per_rank: float, step_s_max: float, world: int) -> float:
    """Weak scaling: every rank runs one call; throughput of all ranks over the slowest one."""
    return world * dense_flops_per_rank / step_s_max / 1e12


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# --------------------------------------------------------------- CPU oracle leg
def oracle_sample(q, k, v, wl: W.Workload, topk: float, budget_s: float):
    """Time the fp64 oracle on a bounded sample: the full selection of head (0, 0)
    and attention for as many of its query blocks as fit in `budget_s`.
    Returns the extrapolated full-call seconds and a description."""
    from oracle import bsa_oracle as O

    t0 = time.perf_counter()
    mask, _ = O.select(q[:1, :1], k[:1, :1], topk)
    t_sel = time.perf_counter() - t0
    qh, kh, vh = O.to_f64(q[0, 0]), O.to_f64(k[0, 0]), O.to_f64(v[0, 0])
    rng = np.random.default_rng(0)
    blocks = rng.permutation(wl.Qb)
    done, t_attn = 0, 0.0
    while done < len(blocks) and (done < 1 or t_attn < budget_s):
        t1 = time.perf_counter()
        O.attention_rows(qh, kh, vh, mask[0, 0, blocks[done]], int(blocks[done]))
        t_attn += time.perf_counter() - t1
        done += 1
    heads = wl.B * wl.H
    est = t_sel * heads + (t_attn / done) * heads * wl.Qb
    desc = (f"fp64 oracle: selection of 1 of {heads} heads ({t_sel:.2f} s) + attention of {done} of "
            f"{heads * wl.Qb} query blocks ({t_attn:.2f} s), extrapolated to the full call")
    return est, desc, t_sel + t_attn


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def run_reference(args, world, rank):
    """The oracle, as it stands, on a bounded sample of the bench's workload.  Each
    timed step runs the sample (one head's selection plus attention for some of
    its query blocks); the line's value is the extrapolation of that sample to
    the full call, flagged as such."""
    if rank != 0:
        return 0
    wl = W.WORKLOADS[args.workload]
    q, k, v = W.make_qkv(wl)
    if args.steps is None:
        args.steps = 10
    per_step = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(q, k, v, wl, args.topk, per_step)
    ests, desc, wall = [], "", 0.0
    for _ in range(args.steps):
        est, desc, w = oracle_sample(q, k, v, wl, args.topk, per_step)
        ests.append(est)
        wall += w
    est = statistics.median(ests)
    value = wl.dense_flops() / est / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": wall / max(1, args.steps) * 1e3,
        "extrapolated": True, "extrapolated_ms_per_call": est * 1e3,
        "step_is": "one bounded sample of the call (see cpu_baseline.sample); value is that sample "
                   "extrapolated to the full call",
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(wl, "topk", args.topk, False, wl.H),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": desc, "extrapolated": True},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


CALL_NAMES = {"topk": "sparse_attn_select + block_sparse_attn_apply (= sparse_attn_topk)",
              "mask": "block_sparse_attn_plan + block_sparse_attn_apply (= block_sparse_attn_fwd, caller mask)",
              "cdf": "sparse_attn_select_cdf + block_sparse_attn_apply (= sparse_attn_cdf)"}


def workload_config(wl, call, param, causal, H, plan_reuse=1):
    knob = {"topk": "topk", "mask": "density", "cdf": "threshold"}[call]
    cfg = {"workload": f"{wl.name}: {wl.note}", "B": wl.B, "H": H, "N": wl.N, "d": wl.d,
           "grid_thw": list(wl.grid), knob: param, "causal": bool(causal), "call": CALL_NAMES[call],
           "l2": "inputs larger than L2 (q/k/v/out 4 x %.0f MB); no flush" % (wl.B * H * wl.N * wl.d * 2 / 1e6)
           if 4 * wl.B * H * wl.N * wl.d * 2 > 126e6 else "inputs fit in L2 (launch-bound parity case)",
           "parallelism": "replicas (one independent call per GPU)"}
    if plan_reuse > 1:
        cfg["plan_reuse"] = plan_reuse
    return cfg


def metric_name(wl, call, param, causal, plan_reuse=1):
    if (wl.name, call, param, causal, plan_reuse) == ("wan14b", "topk", 0.5, False, 1):
        return METRIC
    knob = {"topk": "topk", "mask": "caller mask p", "cdf": "cdfthreshd"}[call]
    extra = (" causal" if causal else "") + (f" plan reused x{plan_reuse}" if plan_reuse > 1 else "")
    return f"ms/call and dense-equiv TFLOPS, {wl.name} {knob}={param}{extra}, % of bf16 TC peak"


def dense_flops(wl, H, causal):
    """Dense-attention FLOPs of the call: 4 B H N^2 d, or for causal attention the
    4 B H d N (N + 1) / 2 of the lower triangle."""
    N = float(wl.N)
    return 4.0 * wl.B * H * wl.d * (N * (N + 1) / 2 if causal else N * N)


# ------------------------------------------------------------------- GPU arm
class Case:
    """One timed configuration: the selection-or-compaction call followed by
    `plan_reuse` applies of its plan, on device-resident inputs."""

    def __init__(self, bsa, wl, H, qkv, call, param, causal, plan_reuse=1):
        self.bsa, self.wl, self.H = bsa, wl, H
        self.q, self.k, self.v = qkv
        self.call, self.param, self.causal, self.R = call, param, bool(causal), max(1, plan_reuse)
        B, N, d = wl.B, wl.N, wl.d
        self.out = torch.empty_like(self.q)
        self.ws = bsa.make_workspace(B, H, N, d)
        self.mask = torch.empty(B, H, wl.Qb, wl.Kb, dtype=torch.uint8, device="cuda")
        if call == "mask":
            self.mask.copy_(W.make_random_mask(W.Workload(wl.name, B=B, H=H, d=d, grid=wl.grid,
                                                          text=wl.text, seed=wl.seed), param))

    def select(self):
        b, c = self.bsa, self.causal
        if self.call == "topk":
            b.sparse_attn_select(self.q, self.k, self.param, c, mask_out=self.mask, workspace=self.ws)
        elif self.call == "cdf":
            b.sparse_attn_select_cdf(self.q, self.k, self.param, mask_out=self.mask, workspace=self.ws)
        else:
            b.block_sparse_attn_plan(self.q, self.mask, c, workspace=self.ws)

    def apply(self):
        self.bsa.block_sparse_attn_apply(self.q, self.k, self.v, self.ws, self.causal, out=self.out)

    def fused(self):
        b, c = self.bsa, self.causal
        if self.call == "topk":
            b.sparse_attn_topk(self.q, self.k, self.v, self.param, c, out=self.out, workspace=self.ws)
        elif self.call == "cdf":
            b.sparse_attn_cdf(self.q, self.k, self.v, self.param, c, out=self.out, workspace=self.ws)
        else:
            b.block_sparse_attn_fwd(self.q, self.k, self.v, self.mask, c, out=self.out, workspace=self.ws)

    def launches_per_step(self):
        # pool + dots + row kernel for a selection, one compaction kernel for a
        # caller mask; one attention kernel per apply
        return (1 if self.call == "mask" else 3) + self.R

    def time(self, K, Wm, world, local, fused=True):
        stream = torch.cuda.current_stream()
        clocks = ClockSampler(local)
        clocks.start()
        for _ in range(Wm):
            self.select()
            for _ in range(self.R):
                self.apply()
        self.bsa.last_device_status(self.ws)
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
        barrier(world)
        torch.cuda.synchronize()
        t_begin = time.time()
        for i in range(K):
            ev[i][0].record(stream)
            self.select()
            ev[i][1].record(stream)
            for _ in range(self.R):
                self.apply()
            ev[i][2].record(stream)
        torch.cuda.synchronize()
        t_end = time.time()
        barrier(world)
        clk = clocks.stop(t_begin, t_end)
        self.bsa.last_device_status(self.ws)
        step_s = ev[0][0].elapsed_time(ev[K - 1][2]) / 1e3 / K
        sel_s = statistics.mean(e[0].elapsed_time(e[1]) for e in ev) / 1e3
        attn_s = statistics.mean(e[1].elapsed_time(e[2]) for e in ev) / 1e3 / self.R
        res = {"step_s": step_s, "call_s": step_s / self.R, "sel_s": sel_s, "attn_s": attn_s, "clocks": clk,
               "density": float(self.mask.float().mean().item()) if not self.causal or self.call != "mask"
               else None}
        if self.call == "mask" and self.causal:
            # the caller mask's entries past block 2i+1 are ignored under causal attention
            Qb, Kb = self.wl.Qb, self.wl.Kb
            elig = torch.arange(Kb, device="cuda")[None, :] <= 2 * torch.arange(Qb, device="cuda")[:, None] + 1
            res["density"] = float((self.mask.bool() & elig).float().mean().item())
        res["kept"] = int(self.mask.sum().item()) if self.call != "mask" else None
        if fused:
            for _ in range(2):
                self.fused()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(stream)
            for _ in range(K):
                self.fused()
            e1.record(stream)
            torch.cuda.synchronize()
            self.bsa.last_device_status(self.ws)
            res["fused_s"] = max_over_ranks(e0.elapsed_time(e1) / 1e3 / K, world)
        res["step_max_s"] = max_over_ranks(step_s, world)
        return res


def rooflines(case, res, peaks, kind, traffic):
    wl, H = case.wl, case.H
    B, N, d = wl.B, wl.N, wl.d
    kept_flops = 4.0 * B * H * N * N * d * res["density"]
    achieved = kept_flops / res["attn_s"] / 1e12
    # d = 64 runs the two-CTA-per-SM kernel, d = 128 the two-warpgroup one
    roofline = {"bound": "tensor", "kernel": "bsa_fwd1_kernel" if d == 64 else "bsa_fwd_kernel",
                "achieved": achieved,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                "traffic": traffic, "peak_kind": f"bf16 dense burst, of {kind}",
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                "algorithmic_flops_per_launch": kept_flops, "avg_launch_ms": res["attn_s"] * 1e3}
    rows = B * H * wl.Qb
    if case.call == "mask":
        sel_bytes = rows * wl.Kb + 2 * int(case.mask.sum().item()) + 4 * rows
        kern = "compact_kernel"
    else:
        sel_bytes = 2 * B * H * N * d * 2 + rows * wl.Kb + 2 * res["kept"]
        kern = "pool_kernel + dots_tc_kernel + " + ("select_cdf_kernel" if case.call == "cdf" else "select_kernel")
    roofline_select = {"bound": "hbm", "kernel": kern, "achieved": sel_bytes / res["sel_s"] / 1e9,
                       "peak": peaks["hbm_gbs"], "unit": "GB/s",
                       "frac": sel_bytes / res["sel_s"] / 1e9 / peaks["hbm_gbs"],
                       "algorithmic_bytes_per_call": sel_bytes, "avg_call_ms": res["sel_s"] * 1e3}
    if case.call != "mask":
        # The block dot products (2 B H Qb Kb d FLOPs) run after the pooling, on
        # the tensor cores as three TF32 products each (hi*hi + hi*lo + lo*hi): the
        # selection's floor is the HBM time plus their tensor time at the TF32
        # peak, taken as the measured bf16 peak x the nominal TF32 / bf16 ratio
        # (1.1 / 2.25 PFLOP/s dense).
        dots_flops = 2.0 * B * H * wl.Qb * wl.Kb * d
        tf32_peak = peaks["bf16_tflops"] * 1e12 * TF32_PER_BF16
        floor_s = sel_bytes / (peaks["hbm_gbs"] * 1e9) + 3.0 * dots_flops / tf32_peak
        roofline_select.update({"dots_flops": dots_flops, "dots_tensor_flops": 3.0 * dots_flops,
                                "tf32_peak_tflops_derived": tf32_peak / 1e12,
                                "sequential_floor_ms": floor_s * 1e3,
                                "frac_of_sequential_floor": floor_s / res["sel_s"]})
    return roofline, kept_flops, roofline_select


def case_line(case, res, world, K, Wm, peaks, kind, traffic):
    wl, H = case.wl, case.H
    dflops = dense_flops(wl, H, case.causal)
    roofline, kept_flops, roofline_select = rooflines(case, res, peaks, kind, traffic)
    call_max = res["step_max_s"] / case.R
    line = {
        "metric": metric_name(wl, case.call, case.param, case.causal, case.R),
        "value": whole_job_value(dflops, call_max, world), "unit": UNIT,
        "n_gpus": world, "steps": K, "warmup": Wm, "ms_per_step": res["step_max_s"] * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": workload_config(wl, case.call, case.param, case.causal, H, case.R),
        "roofline": roofline, "roofline_select": roofline_select,
        "gpu_launches": case.launches_per_step() * K, "clocks": res["clocks"],
        "breakdown": {"select_ms": res["sel_s"] * 1e3, "attention_ms": res["attn_s"] * 1e3,
                      "ms_per_call": call_max * 1e3, "fused_call_ms": res.get("fused_s", 0) * 1e3 or None,
                      "density": res["density"], "kept_tflop": kept_flops / 1e12,
                      "dense_tflop": dflops / 1e12},
    }
    if case.R > 1:
        line["breakdown"]["plan_reuse"] = {"applies_per_selection": case.R,
                                           "amortised_ms_per_call": call_max * 1e3,
                                           "select_ms": res["sel_s"] * 1e3, "apply_ms": res["attn_s"] * 1e3}
    return line


# Rows of the workload table: (workload, call, knob value, causal, plan reuse).
SWEEP = [
    ("tiny", "topk", 0.5, False, 1),
    ("cogvideox2b", "topk", 0.5, False, 1),
    ("cogvideox2b", "topk", 0.5, True, 1),
    ("wan13b", "topk", 1.0, False, 1),
    ("wan13b", "topk", 0.5, False, 1),
    ("wan13b", "topk", 0.3, False, 1),
    ("wan13b", "topk", 0.1, False, 1),
    ("wan13b", "cdf", 0.9, False, 1),
    ("wan13b", "cdf", 0.5, False, 1),
    ("wan14b", "mask", 0.5, False, 1),
    ("wan14b", "mask", 0.1, False, 1),
    ("wan14b", "topk", 0.5, False, 1),
    ("wan14b", "topk", 0.5, True, 1),
    ("wan14b", "topk", 0.5, False, 4),
    ("hunyuan13b", "topk", 0.1, False, 1),
]


def knob(args):
    return {"topk": args.topk, "mask": args.density, "cdf": args.threshold}[args.call]


def default_steps(case, world) -> int:
    """Steps for ~1 s of timed work (at least 10, at most 500), from the second of
    two untimed steps (the first pays one-time setup), so that short calls still
    get clock samples.  Every rank takes the largest count, so all ranks time the
    same number of steps."""
    for rep in range(2):
        torch.cuda.synchronize()
        t0 = time.time()
        case.select()
        for _ in range(case.R):
            case.apply()
        torch.cuda.synchronize()
    step_est = max(time.time() - t0, 1e-4)
    k = min(500, max(10, int(math.ceil(1.0 / step_est))))
    if world > 1:
        import torch.distributed as dist

        t = torch.tensor([k], dtype=torch.int64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        k = int(t.item())
    return k


def run_b200(args, world, rank, local):
    import block_sparse_attention_14_b200 as bsa

    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    peaks, kind = load_peaks()
    K, Wm = args.steps, args.warmup

    def inputs(name):
        base = W.WORKLOADS[name]
        H = args.heads or base.H
        wl = W.Workload(base.name, B=base.B, H=H, d=base.d, grid=base.grid, text=base.text,
                        topk=base.topk, seed=base.seed + rank, note=base.note)
        q_h, k_h, v_h = W.make_qkv(wl)
        return wl, H, (q_h, k_h, v_h), (q_h.cuda(), k_h.cuda(), v_h.cuda())

    if args.sweep:
        cur = None
        for name, call, param, causal, reuse in SWEEP:
            if cur is None or cur[0].name != name:
                cur = None
                torch.cuda.empty_cache()
                cur = inputs(name)
            wl, H, _, qkv = cur
            case = Case(bsa, wl, H, qkv, call, param, causal, reuse)
            # At least ~1 s of timed steps per row, so that short calls still get
            # clock samples (nvidia-smi samples every 50 ms); at most 500 steps.
            K_row = default_steps(case, world) if K is None else min(500, max(K, default_steps(case, world)))
            res = case.time(K_row, Wm, world, local, fused=reuse == 1)
            K_used = K_row
            traffic = recorded_traffic(wl.name) if (call, param, causal) == ("topk", 0.5, False) else None
            line = case_line(case, res, world, K_used, Wm, peaks, kind, traffic)
            line["sweep"] = True
            if rank == 0:
                print(json.dumps(line), flush=True)
            del case
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
        return 0

    wl, H, (q_h, k_h, v_h), qkv = inputs(args.workload)
    case = Case(bsa, wl, H, qkv, args.call, knob(args), args.causal, args.plan_reuse)
    if K is None:
        K = default_steps(case, world)
    res = case.time(K, Wm, world, local, fused=not args.no_fused)
    plain = (args.call, knob(args), args.causal) == ("topk", 0.5, False)
    traffic = recorded_traffic(wl.name if not args.heads else f"{wl.name}-h{H}") if plain else None
    line = case_line(case, res, world, K, Wm, peaks, kind, traffic)

    e2e = None
    if not args.no_e2e and args.call == "topk" and args.plan_reuse == 1:
        q, k, v = qkv
        qp, kp, vp = (t.pin_memory() for t in (q_h, k_h, v_h))
        op = torch.empty(q_h.shape, dtype=torch.bfloat16).pin_memory()
        qd, kd, vd = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        stream = torch.cuda.current_stream()

        def e2e_step():
            # One C-ABI call on the pinned host buffers: head chunks are copied in,
            # computed and copied out as a pipeline; it returns when out is on the host.
            bsa.sparse_attn_topk_host(qp, kp, vp, args.topk, args.causal, out_host=op,
                                      device_buffers=(qd, kd, vd, case.out), workspace=case.ws)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        bsa.last_device_status(case.ws)
        t_e2e = max_over_ranks(e0.elapsed_time(e1) / 1e3 / K, world)
        nbytes = q.numel() * 2
        e2e = {"value": world * dense_flops(wl, H, args.causal) / t_e2e / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes,
               "ms_per_step": t_e2e * 1e3,
               "api": "sparse_attn_topk_host (pinned host q/k/v/out; copies pipelined over head chunks)"}
    line["e2e"] = e2e

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.call == "topk" and not args.causal:
        est, desc, _ = oracle_sample(q_h, k_h, v_h, wl, args.topk, budget_s=15.0)
        cpu = {"value": dense_flops(wl, H, False) / est / 1e12, "unit": UNIT, "cores": blas_threads(),
               "kind": "oracle", "sample": desc, "extrapolated": True}
    line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


def sweep_table(path: str) -> str:
    """Markdown table of the JSON lines a --sweep run printed."""
    out = ["| Config | Call | Density | Select ms | Attention ms | ms per call | Dense-eq TFLOPS | "
           "Kept TFLOP/s | % of burst peak | % of sustained | SM MHz (median) |",
           "|---|---|---|---|---|---|---|---|---|---|---|"]
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line.startswith("{"):
                continue
            d = json.loads(line)
            c, bd, r = d["config"], d["breakdown"], d["roofline"]
            knob = next(k for k in ("topk", "density", "threshold") if k in c)
            call = {"topk": "top-k", "density": "caller mask p", "threshold": "cdfthreshd"}[knob]
            call = f"{call} {c[knob]}" + (" causal" if c.get("causal") else "")
            if c.get("plan_reuse"):
                call += f", plan reused x{c['plan_reuse']} (amortised)"
            clk = d.get("clocks") or {}
            out.append(f"| {c['workload'].split(':')[0]} (B{c['B']} H{c['H']} N{c['N']} d{c['d']}) | {call} | "
                       f"{bd['density']:.3f} | {bd['select_ms']:.3f} | {bd['attention_ms']:.3f} | "
                       f"{bd['ms_per_call']:.3f} | {d['value']:.0f} | {r['achieved']:.0f} | "
                       f"{100 * r['frac']:.1f} | {100 * r['frac_of_sustained']:.1f} | {clk.get('sm_mhz')} |")
    return "\n".join(out)


def main():
    args = parse_args()
    if args.table:
        print(sweep_table(args.table))
        return 0
    world, rank, local = dist_setup()
    if args.impl == "reference":
        return run_reference(args, world, rank)
    return run_b200(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
