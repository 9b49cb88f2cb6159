"""The benchmark's host logic on CPU: two gloo ranks, max-over-ranks timing,
weak-scaling throughput, the reference arm's rank-0-only rule, and the clock record's
restriction to the timed region."""
import json
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, _ = bench.dist_setup()
        assert (w, r) == (world, rank)
        step = 0.05 + 0.01 * rank              # rank 1 is the slowest
        bench.barrier(world)
        m = bench.max_over_ranks(step, world)
        v = bench.whole_job_value(1e12, m, world)
        q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_step_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, m, v in got:
        assert m == pytest.approx(0.06)
        assert v == pytest.approx(2 * 1e12 / 0.06 / 1e12)


def test_reference_arm_runs_only_on_rank_zero(monkeypatch):
    class A:
        workload, topk, steps, warmup, gpus = "tiny", 0.5, 1, 1, 2

    called = []
    monkeypatch.setattr(bench.W, "make_qkv", lambda wl: called.append(1))
    assert bench.run_reference(A(), world=2, rank=1) == 0
    assert not called


def test_single_rank_helpers():
    assert bench.max_over_ranks(0.123, 1) == 0.123
    assert bench.whole_job_value(2e12, 0.5, 1) == pytest.approx(4.0)


def _fake_smi(path, rows):
    with open(path, "w") as f:
        for ts, mhz, reasons in rows:
            stamp = ts.strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
            flags = ", ".join("Active" if r else "Not Active" for r in reasons)
            f.write(f"{stamp}, {mhz}, 1965, 900.00, 0x4, {flags}\n")


class _DoneProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        pass


def test_clock_sampler_keeps_only_the_timed_region(tmp_path):
    """Rows before and after the timed region (warm-up, teardown) are dropped; the
    median and the throttle reasons come from the rows inside it."""
    from datetime import datetime, timedelta

    t0 = datetime(2026, 1, 1, 12, 0, 0)
    cap = (False, False, False, True)
    thermal = (False, True, False, True)
    _fake_smi(tmp_path / "smi.csv", [
        (t0 - timedelta(seconds=1), 1965, thermal),   # warm-up, throttled: dropped
        (t0 + timedelta(milliseconds=100), 1500, cap),
        (t0 + timedelta(milliseconds=150), 1480, cap),
        (t0 + timedelta(milliseconds=200), 1520, cap),
        (t0 + timedelta(seconds=3), 900, thermal),    # after the region: dropped
    ])
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.proc, c.path = _DoneProc(), str(tmp_path / "smi.csv")
    rec = c.stop(t0.timestamp(), (t0 + timedelta(milliseconds=500)).timestamp())
    assert rec == {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                   "samples": 3, "window": "timed region"}


def test_clock_sampler_falls_back_to_the_whole_run(tmp_path):
    from datetime import datetime, timedelta

    t0 = datetime(2026, 1, 1, 12, 0, 0)
    _fake_smi(tmp_path / "smi.csv", [(t0 + timedelta(seconds=2), 1400, (False, False, False, True))])
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.proc, c.path = _DoneProc(), str(tmp_path / "smi.csv")
    rec = c.stop(t0.timestamp(), (t0 + timedelta(seconds=1)).timestamp())
    assert rec["window"] == "whole run" and rec["samples"] == 1 and rec["sm_mhz"] == 1400.0


def test_roofline_arithmetic_of_a_bench_line():
    """The bench line's rooflines for the Wan2.1-14B shape at density 0.5, worked by
    hand: kept FLOPs 4 B H N^2 d rho; selection bytes 2 B H N d 2 (q, k) + B H Qb Kb
    (mask) + 2 per kept block (idx); its sequential floor adds the dot products'
    three TF32 products of 2 B H Qb Kb d FLOPs at the bf16 peak x 1.1 / 2.25."""
    import types

    wl = bench.W.WORKLOADS["wan14b"]
    B, H, N, d, Qb, Kb = 1, 40, 75600, 128, 591, 1182
    kept = 40 * 591 * 591  # blocks kept at topk 0.5
    case = types.SimpleNamespace(wl=wl, H=H, call="topk", mask=None)
    res = {"density": 0.5, "attn_s": 0.05, "sel_s": 0.001, "kept": kept}
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1300.0, "sm_max_mhz": 2000.0}
    roof, kept_flops, sel = bench.rooflines(case, res, peaks, "measured", None)
    assert kept_flops == pytest.approx(4 * B * H * N * N * d * 0.5)
    assert roof["achieved"] == pytest.approx(kept_flops / 0.05 / 1e12)
    assert roof["frac"] == pytest.approx(kept_flops / 0.05 / 1e12 / 1600.0)
    sel_bytes = 2 * B * H * N * d * 2 + B * H * Qb * Kb + 2 * kept
    assert sel["algorithmic_bytes_per_call"] == sel_bytes
    assert sel["frac"] == pytest.approx(sel_bytes / 0.001 / 1e9 / 6000.0)
    floor = sel_bytes / 6000e9 + 3 * 2 * B * H * Qb * Kb * d / (1600e12 * 1.1 / 2.25)
    assert sel["sequential_floor_ms"] == pytest.approx(floor * 1e3)
    assert sel["frac_of_sequential_floor"] == pytest.approx(floor / 0.001)
    assert bench.dense_flops(wl, H, causal=True) == pytest.approx(4 * B * H * d * N * (N + 1) / 2)


def test_sweep_table_renders_a_line(tmp_path):
    line = {"config": {"workload": "wan14b: Wan2.1-14B-shaped", "B": 1, "H": 40, "N": 75600, "d": 128,
                       "topk": 0.5, "causal": True},
            "breakdown": {"density": 0.25, "select_ms": 0.7, "attention_ms": 27.5, "ms_per_call": 28.2},
            "value": 2074.4, "roofline": {"achieved": 1067.2, "frac": 0.663, "frac_of_sustained": 0.797},
            "clocks": {"sm_mhz": 1500.0}}
    p = tmp_path / "sweep.jsonl"
    p.write_text("not json\n" + json.dumps(line) + "\n")
    t = bench.sweep_table(str(p)).splitlines()
    assert len(t) == 3
    assert t[2] == ("| wan14b (B1 H40 N75600 d128) | top-k 0.5 causal | 0.250 | 0.700 | 27.500 | 28.200 | "
                    "2074 | 1067 | 66.3 | 79.7 | 1500.0 |")
