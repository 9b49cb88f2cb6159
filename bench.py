#!/usr/bin/env python
"""Benchmark of the block-sparse attention hot path on B200.

One step = one pass of the whole path on the Wan2.1-14B-shaped self-attention
call (B=1, H=40, N=75600 = 21x45x80 tokens, d=128, bf16, topk=0.5): mean
pooling, block scores + top-k selection, and block-sparse attention over the
kept 128x64 tiles.  The timed step issues sparse_attn_select and then
block_sparse_attn_apply on one stream -- the same three kernels, in the same
order, that the fused sparse_attn_topk call launches -- so that the attention
kernel can be timed on its own with CUDA events; the fused call is timed too.

Prints one JSON line (rank 0).  Metric: dense-equivalent TFLOPS
(4*B*H*N^2*d / step time), plus ms/call and the fraction of the measured bf16
tensor-core peak reached by the attention kernel on its kept tiles.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {b200,reference}]

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
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ATTN_SRCS = [os.path.join(ROOT, "block_sparse_attention_14_b200", "csrc", f)
             for f in ("bsa_attn.cu", "bsa_common.cuh")]
TRAFFIC_GLOB = os.path.join(ROOT, "profiles", "bsa_fwd_kernel_*_ncu.md")


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["b200", "reference"], default="b200")
    p.add_argument("--workload", default="wan14b", choices=sorted(W.WORKLOADS))
    p.add_argument("--topk", type=float, default=0.5)
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
    (profiles/bsa_fwd_kernel_*_ncu.md), valid only if it was taken on the current
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
    if rank != 0:
        return 0
    wl = W.WORKLOADS[args.workload]
    q, k, v = W.make_qkv(wl)
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
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": est * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, args.topk, wl.H),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(wl, topk, H):
    return {"workload": f"{wl.name}: {wl.note}", "B": wl.B, "H": H, "N": wl.N, "d": wl.d,
            "grid_thw": list(wl.grid), "topk": topk, "call": "sparse_attn_topk (select + apply)",
            "l2": "inputs larger than L2 (q/k/v/out 4 x %.0f MB); no flush" % (wl.B * H * wl.N * wl.d * 2 / 1e6),
            "parallelism": "replicas (one independent call per GPU)"}


# ------------------------------------------------------------------- GPU arm
def run_b200(args, world, rank, local):
    import block_sparse_attention_14_b200 as bsa

    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    wl = W.WORKLOADS[args.workload]
    H = args.heads or wl.H
    wl = W.Workload(wl.name, B=wl.B, H=H, d=wl.d, grid=wl.grid, text=wl.text, topk=wl.topk,
                    seed=wl.seed + rank, note=wl.note)
    q_h, k_h, v_h = W.make_qkv(wl)
    q, k, v = q_h.cuda(), k_h.cuda(), v_h.cuda()
    B, N, d = wl.B, wl.N, wl.d
    out = torch.empty_like(q)
    ws = bsa.make_workspace(B, H, N, d)
    mask = torch.empty(B, H, wl.Qb, wl.Kb, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    K, Wm = args.steps, args.warmup

    def step():
        bsa.sparse_attn_select(q, k, args.topk, mask_out=mask, workspace=ws)
        bsa.block_sparse_attn_apply(q, k, v, ws, out=out)

    clocks = ClockSampler(local)
    clocks.start()
    for _ in range(Wm):
        step()
    bsa.last_device_status(ws)
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    t_begin = time.time()
    for i in range(K):
        ev[i][0].record(stream)
        bsa.sparse_attn_select(q, k, args.topk, mask_out=mask, workspace=ws)
        ev[i][1].record(stream)
        bsa.block_sparse_attn_apply(q, k, v, ws, out=out)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    t_end = time.time()
    barrier(world)
    clk = clocks.stop(t_begin, t_end)
    bsa.last_device_status(ws)
    step_s = ev[0][0].elapsed_time(ev[K - 1][2]) / 1e3 / K
    sel_s = statistics.mean(e[0].elapsed_time(e[1]) for e in ev) / 1e3
    attn_s = statistics.mean(e[1].elapsed_time(e[2]) for e in ev) / 1e3
    step_max = max_over_ranks(step_s, world)

    density = float(mask.float().mean().item())
    dense_flops = wl.dense_flops()
    kept_flops = dense_flops * density

    fused_ms = None
    if not args.no_fused:
        for _ in range(2):
            bsa.sparse_attn_topk(q, k, v, args.topk, out=out, workspace=ws)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(K):
            bsa.sparse_attn_topk(q, k, v, args.topk, out=out, workspace=ws)
        e1.record(stream)
        torch.cuda.synchronize()
        fused_ms = max_over_ranks(e0.elapsed_time(e1) / K, world)

    e2e = None
    if not args.no_e2e:
        qp, kp, vp = (t.pin_memory() for t in (q_h, k_h, v_h))
        op = torch.empty(q_h.shape, dtype=torch.bfloat16).pin_memory()
        qd, kd, vd = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

        def e2e_step():
            # One C-ABI call on the pinned host buffers: head chunks are copied in,
            # computed and copied out as a pipeline; it returns when out is on the host.
            bsa.sparse_attn_topk_host(qp, kp, vp, args.topk, out_host=op,
                                      device_buffers=(qd, kd, vd, out), workspace=ws)

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
        t_e2e = max_over_ranks(e0.elapsed_time(e1) / 1e3 / K, world)
        nbytes = q.numel() * 2
        e2e = {"value": world * dense_flops / t_e2e / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes,
               "ms_per_step": t_e2e * 1e3,
               "api": "sparse_attn_topk_host (pinned host q/k/v/out; copies pipelined over head chunks)"}

    peaks, kind = load_peaks()
    achieved = kept_flops / attn_s / 1e12
    sel_bytes = 2 * B * H * N * d * 2 + B * H * wl.Qb * wl.Kb + 2 * int(mask.sum().item())
    roofline = {"bound": "tensor", "kernel": "bsa_fwd_kernel", "achieved": achieved,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                "traffic": recorded_traffic(wl.name if not args.heads else f"{wl.name}-h{H}"),
                "peak_kind": f"bf16 dense burst, of {kind}",
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                "algorithmic_flops_per_launch": kept_flops, "avg_launch_ms": attn_s * 1e3}
    roofline_select = {"bound": "hbm", "kernel": "pool_kernel + dots_kernel + select_kernel",
                       "achieved": sel_bytes / sel_s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                       "frac": sel_bytes / sel_s / 1e9 / peaks["hbm_gbs"],
                       "algorithmic_bytes_per_call": sel_bytes, "avg_call_ms": sel_s * 1e3}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        est, desc, _ = oracle_sample(q_h, k_h, v_h, wl, args.topk, budget_s=15.0)
        cpu = {"value": dense_flops / est / 1e12, "unit": UNIT, "cores": blas_threads(),
               "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": whole_job_value(dense_flops, step_max, world), "unit": UNIT,
            "n_gpus": world, "steps": K, "warmup": Wm, "ms_per_step": step_max * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": workload_config(wl, args.topk, H),
            "roofline": roofline, "roofline_select": roofline_select, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": 4 * K, "clocks": clk,  # pool, dots, select, attention
            "breakdown": {"select_ms": sel_s * 1e3, "attention_ms": attn_s * 1e3,
                          "fused_call_ms": fused_ms, "density": density,
                          "kept_tflop": kept_flops / 1e12, "dense_tflop": dense_flops / 1e12},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    world, rank, local = dist_setup()
    if args.impl == "reference":
        return run_reference(args, world, rank)
    return run_b200(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
