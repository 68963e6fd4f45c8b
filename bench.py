#!/usr/bin/env python
"""Throughput of windowed int8-state GDN decode on B200.

One step = initial quantization of the fp32 states + T decode steps (one kernel launch each, the
window flush fused into every W-th) over the whole batch of the serving-scale workload
(B=1024 sequences x H=32 heads, d=128, T=256, W=64, bf16 q/k/v/o, int8 state with per-row
scales). The metric is head-steps per second; one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
    torchrun --nproc-per-node N bench.py --gpus N ...     (one rank per GPU, weak scaling)
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import WORKLOADS, decode_inputs, outlier_scales, step_inputs, torch_dtype  # noqa: E402

METRIC = "GDN decode head-steps/s (int8 windowed state); achieved HBM GB/s vs B200 peak"
UNIT = "head-steps/s"
PROFILE = os.path.join(ROOT, "profiles", "window_step_gdn-serving.md")
KERNEL_SOURCES = ["bit_recurrent_state_gdn_b200/csrc/window_kernels.cuh",
                  "bit_recurrent_state_gdn_b200/csrc/window_mma.cuh",
                  "bit_recurrent_state_gdn_b200/csrc/window_dispatch.cuh",
                  "bit_recurrent_state_gdn_b200/csrc/device_util.cuh",
                  "bit_recurrent_state_gdn_b200/csrc/mma_util.cuh",
                  "bit_recurrent_state_gdn_b200/csrc/tc_util.cuh"]
PW_PROFILE = os.path.join(ROOT, "profiles", "pw_step_gdn-serving.md")
PW_KERNEL_SOURCES = ["bit_recurrent_state_gdn_b200/csrc/pw_kernels.cuh",
                     "bit_recurrent_state_gdn_b200/csrc/pw.cu",
                     "bit_recurrent_state_gdn_b200/csrc/device_util.cuh",
                     "bit_recurrent_state_gdn_b200/csrc/mma_util.cuh"]
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="gdnq", choices=["gdnq", "reference"])
    p.add_argument("--workload", default="gdn-serving")
    p.add_argument("--batch", type=int, default=None, help="override B (profiling captures)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-baselines", action="store_true")
    p.add_argument("--no-cpu", action="store_true")
    p.add_argument("--cpu-heads", type=int, default=8192)
    p.add_argument("--ref-heads", type=int, default=2048)
    p.add_argument("--pw-only", action="store_true",
                   help="run only the pure-write window legs (profiling captures)")
    p.add_argument("--prefill-only", action="store_true",
                   help="run only the chunkwise prefill leg (profiling captures)")
    p.add_argument("--prefill-batch", type=int, default=None, help="override the prefill B")
    return p.parse_args()


# ---------------------------------------------------------------------------------------------
# Algorithmic bytes (what the method must move; no re-reads)
# ---------------------------------------------------------------------------------------------
def step_bytes(wl, P: int) -> int:
    """HBM bytes one decode step of one head must move at window position P."""
    D, W, r = wl.D, wl.W, wl.r
    act = 4 if wl.act == "f32" else 2
    buf = 4 if wl.buf == "f32" else 2
    lbytes = 4 * D if wl.gate == "diag" else 4
    codes = D * D // 2 if wl.fmt == "int4_g32" else D * D
    scales = 4 * D * (D // 32 if wl.fmt == "int4_g32" else 1)
    scales += D if wl.smooth else 0  # residual smoothing: one exponent byte per key column
    comps = r * (4 + 4 * D) + (r * 4 * D if wl.comp_rule == "power" else 0)
    pair = D * act + D * buf + lbytes
    io_ = 4 * D * act + (4 * D if wl.gate == "diag" else 4) + 4 + 8  # q k v o, g, beta, pos r/w
    read = codes + scales + comps + P * pair
    write = pair if P + 1 < W else codes + scales + comps
    return read + write + io_


def avg_step_bytes(wl) -> float:
    return sum(step_bytes(wl, P) for P in range(wl.W)) / wl.W


def baseline_bytes(wl, state_bytes: int) -> int:
    act = 4 if wl.act == "f32" else 2
    return 2 * wl.D * wl.D * state_bytes + 4 * wl.D * act + 8


def peak_hbm():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def profiled_traffic(profile=PROFILE, sources=KERNEL_SOURCES, key="traffic_bytes_per_launch"):
    """Per-launch DRAM bytes of a kernel from its committed ncu summary, if the kernel source
    still matches the one profiled; else None."""
    try:
        text = open(profile).read()
    except OSError:
        return None, None
    m = re.search(key + r":\s*([0-9.eE+]+)", text)
    s = re.search(r"kernel_source_sha256:\s*([0-9a-f]{64})", text)
    if not m or not s or s.group(1) != kernel_sha(sources):
        return None, None
    return float(m.group(1)), os.path.relpath(profile, ROOT)


def kernel_sha(sources=KERNEL_SOURCES) -> str:
    h = hashlib.sha256()
    for p in sources:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


# ---------------------------------------------------------------------------------------------
# Sharding over ranks: every (sequence, head) is independent, so rank r runs its own sequences
# (the workload's recipe under its own seed) and nothing crosses ranks but the timing
# ---------------------------------------------------------------------------------------------
def shard_workload(wl, rank: int):
    return wl.with_(seed=wl.seed + 7919 * rank)


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time (all ranks take this collective in the same order)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist

    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, world: int, max_ms: float) -> float:
    """Units all ranks processed per second of the slowest rank's time."""
    return units_per_rank * world / (max_ms / 1e3)


# ---------------------------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------------------------
class ClockSampler:
    Q = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        import torch

        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", sel, f"--query-gpu={self.Q}", "--format=csv,noheader",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return []
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        return [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]

    @staticmethod
    def summarise(rows, t0: float, t1: float):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        mhz, maxmhz, reasons = [], None, set()
        for r in rows:
            try:
                ts = time.mktime(time.strptime(r[0].strip().split(".")[0], "%Y/%m/%d %H:%M:%S"))
            except ValueError:
                continue
            if ts < int(t0) or ts > t1 + 1:
                continue
            try:
                mhz.append(float(r[1].split()[0]))
                maxmhz = float(r[2].split()[0])
            except (ValueError, IndexError):
                continue
            for name, val in zip(names, r[5:9]):
                if "Active" in val and "Not" not in val:
                    reasons.add(name)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": maxmhz,
                "reasons": sorted(reasons), "samples": len(mhz)}


# ---------------------------------------------------------------------------------------------
# CPU oracle timing (the reported CPU baseline and the reference arm)
# ---------------------------------------------------------------------------------------------
def time_oracle(wl, q, k, v, g, beta, S0):
    """Head-steps/s of the oracle's buffered-window decode (storage roundings on) over the
    given inputs ([T][n][D] numpy) from fp32 states S0 [n][D][D]."""
    import oracle

    T, n = q.shape[0], q.shape[1]
    t0 = time.perf_counter()
    oracle.o2_run(q, k, v, g, beta, W=wl.W, r=wl.r, fmt=wl.fmt, S0=S0, round_storage=True,
                  buf_round=wl.buf)
    dt = time.perf_counter() - t0
    return n * T / dt, dt, oracle.num_threads()


def oracle_warm_state(wl, warm):
    import oracle

    if wl.warmup == 0:
        n = warm["q"].shape[1] if warm["q"].ndim == 3 else 0
        return __import__("numpy").zeros((n, wl.D, wl.D))
    _, S = oracle.plain_run(warm["q"], warm["k"], warm["v"], warm["g"], warm["beta"],
                            state_round="f32", want_o=False)
    return S


def cpu_inputs(wl, device="cpu"):
    """Warm-up and decode inputs of a (small) workload as float64 numpy [T][heads][D]."""
    import numpy as np

    def flat(t, x):
        return x.reshape(t, wl.heads, *x.shape[3:]).double().cpu().numpy()

    warm = decode_inputs(wl, device, T=wl.warmup, phase="warmup")
    dec = decode_inputs(wl, device)
    w = {n: flat(wl.warmup, x) for n, x in warm.items()}
    d = {n: flat(wl.T, x) for n, x in dec.items()}
    return w, d


def reference_arm(args, rank, world):
    """The oracle as the reference implementation, timed on this machine's host cores."""
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    sample = wl.with_(B=max(1, args.ref_heads // wl.H))
    w, d = cpu_inputs(sample)
    S0 = oracle_warm_state(sample, w)
    times, cores = [], 1
    for i in range(args.warmup + args.steps):
        hs, dt, cores = time_oracle(sample, d["q"], d["k"], d["v"], d["g"], d["beta"], S0)
        if i >= args.warmup:
            times.append(dt)
    per_step = statistics.mean(times)
    value = sample.heads * sample.T / per_step
    desc = (f"oracle buffered-window decode, {sample.heads} heads ({sample.B} sequences x "
            f"{sample.H}) x {sample.T} steps of the {wl.name} workload per step, inputs drawn on "
            f"the CPU with the workload's recipe")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": bench_config(wl, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def bench_config(wl, n):
    return {"workload": wl.name, "B": wl.B, "H": wl.H, "d_k": wl.D, "d_v": wl.D, "T": wl.T,
            "W": wl.W, "r": wl.r, "gate": wl.gate, "state": wl.fmt, "act": wl.act,
            "buf": wl.buf, "step": f"initial quantize + {wl.T} decode steps",
            "l2": "no flush: the per-step working set is larger than the 126 MB L2",
            "parallelism": f"dp{n} (disjoint sequences per GPU, no collective)"}


# ---------------------------------------------------------------------------------------------
# The GPU arm
# ---------------------------------------------------------------------------------------------
def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        reference_arm(args, rank, world)
        return
    if args.prefill_only:
        import torch

        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dev = torch.device("cuda")
        line = {"prefill": prefill_leg(args, dev), "prefill_kda": prefill_leg(args, dev, "kda-prefill")}
        if rank == 0:
            print(json.dumps(line), flush=True)
        return

    import numpy as np
    import torch
    import torch.distributed as dist

    import bit_recurrent_state_gdn_b200 as gdn

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    wl0 = WORKLOADS[args.workload]
    if args.batch:
        wl0 = wl0.with_(B=args.batch)
    wl = shard_workload(wl0, rank)
    cfg = gdn.make_config(wl.B, wl.H, wl.D, wl.W, wl.r, wl.gate, wl.fmt, wl.act, wl.buf)

    # ---- inputs resident in HBM: decode tokens and the fp32 warm-up states ------------------
    inp = decode_inputs(wl, dev)
    S0 = torch.zeros((wl.B, wl.H, wl.D, wl.D), dtype=torch.float32, device=dev)
    bcfg32 = gdn.make_config(wl.B, wl.H, wl.D, gate=wl.gate, fmt="fp32", act=wl.act)
    scales = outlier_scales(wl, dev)
    o_w = torch.empty((wl.B, wl.H, wl.D), dtype=torch_dtype(wl.act), device=dev)
    for t in range(wl.warmup):
        s = step_inputs(wl, "warmup", t, dev, scales)
        gdn.gdn_baseline_step(bcfg32, S0, s.q, s.k, s.v, s.g, s.beta, o_w)
    state = gdn.GdnState.allocate(cfg, dev)
    o = torch.empty_like(inp["q"])
    torch.cuda.synchronize()
    if args.pw_only:
        peak, _ = peak_hbm()
        pw = {f: pw_leg(wl.with_(fmt=f), 8, S0, inp, o, peak, cpu=not args.no_cpu)
              for f in ("int4_g32", "int8")}
        if rank == 0:
            print(json.dumps({"pure_write_s8": pw, "config": bench_config(wl0, world)}),
                  flush=True)
        if world > 1:
            dist.destroy_process_group()
        return

    def one_step(ev=None):
        if ev is not None:
            ev[0].record()
        gdn.gdn_state_quantize(cfg, S0, state)
        if ev is not None:
            ev[1].record()
        gdn.gdn_decode_window_steps(cfg, state, inp["q"], inp["k"], inp["v"], inp["g"],
                                    inp["beta"], o)
        if ev is not None:
            ev[2].record()

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for i in range(args.steps):
        one_step(evs[i])
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if world > 1:
        dist.barrier()
    clocks = ClockSampler.summarise(sampler.stop(), t_wall0, t_wall1)
    total_ms = evs[0][0].elapsed_time(evs[-1][2])
    decode_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    quant_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    total_ms = max_over_ranks(total_ms, world, dev)
    status = int(state.status[0].item())
    if status != 0:
        raise RuntimeError(f"device status word {status:#x} after the timed region")
    # the quality figure uses this step's outputs, before the legs below reuse the buffer
    quality = None
    if not args.no_cpu and world == 1 and rank == 0:
        quality = quality_figure(wl, inp, o, dev)

    value = whole_job_rate(wl.heads * wl.T * args.steps, world, total_ms)
    launches = args.steps * wl.T
    avg_launch_s = decode_ms / 1e3 / launches
    alg_bytes = avg_step_bytes(wl) * wl.heads
    peak, peak_kind = peak_hbm()
    achieved = alg_bytes / avg_launch_s / 1e9
    traffic, traffic_src = profiled_traffic()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "state_dtype": wl.fmt,
        "data": "synthetic (seeded; fp32 warm-up recurrence over 512 tokens makes the states)",
        "config": bench_config(wl0, world),
        "roofline": {
            "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "traffic": traffic,
            "kernel": "window_step_kernel (decode step + fused window flush)",
            "algorithmic_bytes_per_launch": alg_bytes,
            "avg_launch_us": avg_launch_s * 1e6, "peak_source": f"{peak_kind} hbm_gbs",
            "traffic_source": traffic_src,
        },
        "quantize_ms_per_step": quant_ms / args.steps,
        "gpu_launches": args.steps * (1 + wl.T),
        "clocks": clocks,
    }

    # ---- mixed per-head widths: every second head int4, the same inputs ---------------------
    if not args.no_baselines and wl.fmt == "int8" and wl.D == 128:
        line["mixed_half_int4"] = mixed_leg(wl, S0, inp, o, peak)

    # ---- residual smoothing at every quantization, the same inputs ---------------------------
    if not args.no_baselines and wl.fmt in ("int8", "int4_g32"):
        line["smoothing"] = smoothing_leg(wl, S0, inp, o, peak, dev,
                                          cpu=not args.no_cpu and world == 1 and rank == 0)

    # ---- pure-write sliding window (PW-S8) over int4 and int8 histories, the same inputs ----
    if not args.no_baselines and wl.D == 128:
        line["pure_write_s8"] = {
            f: pw_leg(wl.with_(fmt=f), 8, S0, inp, o, peak,
                      cpu=not args.no_cpu and world == 1 and rank == 0)
            for f in ("int4_g32", "int8")}

    # ---- the other decode workloads, each on its own inputs, and int4 at the serving size ----
    if not args.no_baselines and world == 1 and wl0.name == "gdn-serving":
        cpu = not args.no_cpu and rank == 0
        line["workloads"] = {
            "int4-serving": decode_leg(wl.with_(name="int4-serving", fmt="int4_g32"), dev, peak,
                                       cpu=False, inp=inp, S0=S0, o=o)}
        for name in ("kda", "gdn-mid", "gdn-long-int4"):
            line["workloads"][name] = decode_leg(WORKLOADS[name], dev, peak, cpu=cpu,
                                                 quality=cpu and name == "kda")
            torch.cuda.empty_cache()
        # compensator tokens on the KDA workload: power tokens against column tokens, int8 and
        # int4 (quality figures from each leg's own outputs)
        kda = WORKLOADS["kda"]
        for name, wk in (("kda-power", kda.with_(name="kda-power", comp_rule="power")),
                         ("kda-int4", kda.with_(name="kda-int4", fmt="int4_g32")),
                         ("kda-int4-power", kda.with_(name="kda-int4-power", fmt="int4_g32",
                                                      comp_rule="power"))):
            line["workloads"][name] = decode_leg(wk, dev, peak, cpu=False, quality=cpu)
            torch.cuda.empty_cache()

    # ---- chunkwise prefill of a prompt batch (its own workload) ----------------------------
    if not args.no_baselines and world == 1:
        line["prefill"] = prefill_leg(args, dev)
        line["prefill_kda"] = prefill_leg(args, dev, "kda-prefill")

    # ---- high-precision-state baselines on the same inputs ---------------------------------
    if not args.no_baselines:
        line["baselines"] = {}
        for fmt, sdt, sbytes in (("fp32", torch.float32, 4), ("bf16", torch.bfloat16, 2)):
            bcfg = gdn.make_config(wl.B, wl.H, wl.D, gate=wl.gate, fmt=fmt, act=wl.act)
            S = S0.to(sdt)
            for t in range(4):
                gdn.gdn_baseline_step(bcfg, S, inp["q"][t], inp["k"][t], inp["v"][t],
                                      inp["g"][t], inp["beta"][t], o[t])
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record()
            for t in range(wl.T):
                gdn.gdn_baseline_step(bcfg, S, inp["q"][t], inp["k"][t], inp["v"][t],
                                      inp["g"][t], inp["beta"][t], o[t])
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            hs = wl.heads * wl.T / (ms / 1e3)
            gbs = baseline_bytes(wl, sbytes) * wl.heads * wl.T / (ms / 1e3) / 1e9
            line["baselines"][f"{fmt}_state"] = {
                "value": hs * world, "unit": UNIT, "achieved_gbs": gbs, "frac": gbs / peak,
                "ms_per_run": ms, "int8_window_speedup": value / (hs * world)}
            del S

    # ---- end to end through the host-buffer entry point ------------------------------------
    if not args.no_e2e:
        line["e2e"] = e2e(args, wl, cfg, inp, S0, state, world, dev)

    # ---- the oracle on the host cores (rank 0, one GPU) ------------------------------------
    if not args.no_cpu and world == 1 and rank == 0:
        line["cpu_baseline"] = cpu_baseline(args, wl, inp, dev)
        line["quality"] = quality

    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


L2_BYTES = 126 * 2**20
LEG_PROFILES = {"kda": ("window_step_kda.md", "traffic_bytes_per_launch")}


def warm_states(wl, dev):
    """fp32 initial states: the workload's warm-up tokens through the fp32-state baseline
    kernel (zero states without warm-up)."""
    import torch

    import bit_recurrent_state_gdn_b200 as gdn

    S0 = torch.zeros((wl.B, wl.H, wl.D, wl.D), dtype=torch.float32, device=dev)
    cfg = gdn.make_config(wl.B, wl.H, wl.D, gate=wl.gate, fmt="fp32", act=wl.act)
    scales = outlier_scales(wl, dev)
    o = torch.empty((wl.B, wl.H, wl.D), dtype=torch_dtype(wl.act), device=dev)
    for t in range(wl.warmup):
        s = step_inputs(wl, "warmup", t, dev, scales)
        gdn.gdn_baseline_step(cfg, S0, s.q, s.k, s.v, s.g, s.beta, o)
    return S0


def decode_leg(wl, dev, peak, cpu: bool, inp=None, S0=None, o=None, cpu_heads: int = 256,
               quality: bool = False):
    """One decode workload on its own: its states quantized (untimed), then its T decode launches
    timed with CUDA events; the roofline of the average launch from the workload's algorithmic
    bytes; with cpu, the oracle on a bounded sample of its heads; with quality, the outputs'
    error against the unquantized fp64 recurrence on its first sequences."""
    import numpy as np
    import torch

    import bit_recurrent_state_gdn_b200 as gdn

    if inp is None:
        inp = decode_inputs(wl, dev)
        S0 = warm_states(wl, dev)
        o = torch.empty_like(inp["q"])
    cfg = gdn.make_config(wl.B, wl.H, wl.D, wl.W, wl.r, wl.gate, wl.fmt, wl.act, wl.buf,
                          comp_rule=wl.comp_rule)
    st = gdn.GdnState.allocate(cfg, dev)
    gdn.gdn_state_quantize(cfg, S0, st)
    n0 = min(4, wl.T)
    gdn.gdn_decode_window_steps(cfg, st, inp["q"][:n0], inp["k"][:n0], inp["v"][:n0],
                                inp["g"][:n0], inp["beta"][:n0], o[:n0])
    gdn.gdn_state_quantize(cfg, S0, st)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    gdn.gdn_decode_window_steps(cfg, st, inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], o)
    e1.record()
    torch.cuda.synchronize()
    if int(st.status[0].item()) != 0:
        raise RuntimeError(f"{wl.name}: device status word set")
    ms = e0.elapsed_time(e1)
    per_launch = avg_step_bytes(wl) * wl.heads
    avg_s = ms / 1e3 / wl.T
    gbs = per_launch / avg_s / 1e9
    resident = per_launch < L2_BYTES
    traffic, src = None, None
    if wl.name in LEG_PROFILES:
        f, key = LEG_PROFILES[wl.name]
        traffic, src = profiled_traffic(os.path.join(ROOT, "profiles", f), KERNEL_SOURCES, key)
    out = {"value": wl.heads * wl.T / (ms / 1e3), "unit": UNIT, "ms_per_run": ms,
           "config": {"workload": wl.name, "B": wl.B, "H": wl.H, "D": wl.D, "T": wl.T,
                      "W": wl.W, "r": wl.r, "gate": wl.gate, "state": wl.fmt, "act": wl.act,
                      "compensators": wl.comp_rule},
           "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                        "frac": gbs / peak, "traffic": traffic, "traffic_source": src,
                        "algorithmic_bytes_per_launch": per_launch,
                        "avg_launch_us": avg_s * 1e6,
                        "kernel": "window_step_kernel (decode step + fused window flush)"}}
    if resident:
        out["roofline"]["note"] = (
            "effective GB/s: one launch moves %.1f MB, under the 126 MB L2, so the state stays "
            "L2-resident between launches and the launch is latency-bound" % (per_launch / 1e6))
    if cpu:
        n_seq = max(1, min(wl.B, cpu_heads // wl.H))
        d, S0c = oracle_sample(wl, inp, n_seq, dev)
        hs, dt, cores = time_oracle(wl, d["q"], d["k"], d["v"], d["g"], d["beta"], S0c)
        out["cpu_baseline"] = {"value": hs, "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": f"{n_seq * wl.H} heads (sequences 0..{n_seq - 1}) x "
                                         f"{wl.T} steps of the same inputs, {dt:.1f} s"}
    if quality:
        out["quality"] = quality_figure(wl, inp, o, dev, n_seq=4)
    del st
    return out


def mixed_leg(wl, S0, inp, o, peak):
    """The same decode with every second head held as int4 (group 32) in one mixed-format
    launch; algorithmic bytes averaged over the two formats."""
    import torch

    import bit_recurrent_state_gdn_b200 as gdn

    cfg = gdn.make_config(wl.B, wl.H, wl.D, wl.W, wl.r, wl.gate, "mixed", wl.act, wl.buf)
    fmts = ["int8" if h % 2 == 0 else "int4_g32" for h in range(wl.heads)]
    st = gdn.GdnState.allocate(cfg, head_fmt=fmts)
    gdn.gdn_state_quantize(cfg, S0, st)
    for t in range(4):
        gdn.gdn_decode_window_step(cfg, st, inp["q"][t], inp["k"][t], inp["v"][t], inp["g"][t],
                                   inp["beta"][t], o[t])
    gdn.gdn_state_quantize(cfg, S0, st)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    gdn.gdn_decode_window_steps(cfg, st, inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], o)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    per_head = (avg_step_bytes(wl) + avg_step_bytes(wl.with_(fmt="int4_g32"))) / 2
    gbs = per_head * wl.heads * wl.T / (ms / 1e3) / 1e9
    return {"value": wl.heads * wl.T / (ms / 1e3), "unit": UNIT, "achieved_gbs": gbs,
            "frac": gbs / peak, "ms_per_run": ms,
            "note": "GDN_FMT_MIXED, heads alternately int8 / int4-g32, one launch per step"}


def smoothing_leg(wl, S0, inp, o, peak, dev, cpu: bool):
    """The same decode with residual smoothing at every quantization (per-key-column power-of-
    two factors), timed like the mixed leg; with cpu, its output error against the unquantized
    fp64 recurrence on the quality figure's sample."""
    import torch

    import bit_recurrent_state_gdn_b200 as gdn

    ws = wl.with_(smooth=True)
    cfg = gdn.make_config(ws.B, ws.H, ws.D, ws.W, ws.r, ws.gate, ws.fmt, ws.act, ws.buf,
                          smooth=True)
    st = gdn.GdnState.allocate(cfg)
    gdn.gdn_state_quantize(cfg, S0, st)
    for t in range(4):
        gdn.gdn_decode_window_step(cfg, st, inp["q"][t], inp["k"][t], inp["v"][t], inp["g"][t],
                                   inp["beta"][t], o[t])
    gdn.gdn_state_quantize(cfg, S0, st)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    gdn.gdn_decode_window_steps(cfg, st, inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], o)
    e1.record()
    torch.cuda.synchronize()
    if int(st.status[0].item()) != 0:
        raise RuntimeError("smoothing leg: device status word set")
    ms = e0.elapsed_time(e1)
    gbs = avg_step_bytes(ws) * ws.heads * ws.T / (ms / 1e3) / 1e9
    out = {"value": ws.heads * ws.T / (ms / 1e3), "unit": UNIT, "achieved_gbs": gbs,
           "frac": gbs / peak, "ms_per_run": ms,
           "note": "GDN_SMOOTH_POW2_COLUMNS: residual columns scaled by 2^-floor(E/2) before "
                   "the row quantizer, E the exponent of the column's max-abs"}
    if cpu:
        out["quality"] = quality_figure(ws, inp, o, dev)
    return out


def pw_step_bytes(wl, Wp: int) -> int:
    """Algorithmic bytes of one pure-write window step per head with a full window: the history
    (codes + scales) read and written, the Wp pairs (e4m3 x and y, fp32 scales) read, the Wp - 1
    carried keys and the new pair written with their scales, q / k / v / g / beta / count read,
    o and count written."""
    D = wl.D
    act = 4 if wl.act == "f32" else 2
    hist = (D * D // 2 + 4 * D * (D // 32)) if wl.fmt == "int4_g32" else (D * D + 4 * D)
    g = 4 * D if wl.gate == "diag" else 4
    read = hist + 2 * Wp * D + 8 * Wp + 3 * D * act + g + 4 + 4
    write = hist + ((Wp + 1) * D + 4 * (Wp + 1) if Wp else 0) + D * act + 4
    return read + write


def prefill_flops_per_chunk(C: int = 64, D: int = 128) -> int:
    """The UT-form products of one chunk with single-precision operands: K K^T, Q K^T (C x C x D),
    K S^T, Q S^T (C x D x D), T V', P U (C x C x D) and the state update U^T K (D x C x D)."""
    return 2 * (4 * C * C * D + 2 * C * D * D + D * C * D)


def peak_bf16():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured bf16_tflops (burst)"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback"


def prefill_leg(args, dev, name: str = "gdn-prefill", reps: int = 5):
    """gdn_prefill over a prompt workload (B x H heads, L-token prompts, zero initial state):
    the median of `reps` launches after two untimed ones, CUDA events."""
    import torch

    import bit_recurrent_state_gdn_b200 as gdn

    wl = WORKLOADS[name]
    if args.prefill_batch:
        wl = wl.with_(B=args.prefill_batch)
    L = wl.T
    inp = decode_inputs(wl, dev)
    hm = {n: t.permute(1, 2, 0, *range(3, t.dim())).contiguous() for n, t in inp.items()}
    cfg = gdn.make_config(wl.B, wl.H, wl.D, gate=wl.gate, act="bf16")
    o = torch.empty_like(hm["q"])
    S = torch.zeros((wl.B, wl.H, wl.D, wl.D), dtype=torch.float32, device=dev)
    ws = torch.empty(max(gdn.gdn_prefill_workspace_bytes(cfg, L), 16), dtype=torch.uint8,
                     device=dev)
    for _ in range(2):
        gdn.gdn_prefill(cfg, hm["q"], hm["k"], hm["v"], hm["g"], hm["beta"], o, S, ws)
    torch.cuda.synchronize()
    ms = []
    for _ in range(reps):
        S.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        gdn.gdn_prefill(cfg, hm["q"], hm["k"], hm["v"], hm["g"], hm["beta"], o, S, ws)
        e1.record()
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    t = sorted(ms)[len(ms) // 2]
    if not bool(torch.isfinite(S).all()):
        raise RuntimeError(f"prefill {wl.name}: non-finite state")
    C = 16 if wl.gate == "diag" else 64
    chunks = wl.heads * ((L + C - 1) // C)
    flops = chunks * prefill_flops_per_chunk(C)
    tf = flops / (t / 1e3) / 1e12
    peak, src = peak_bf16()
    cpu = None if args.no_cpu else prefill_cpu_baseline(wl, inp, dev)
    kernel = ("prefill_kda_kernel (one CTA per head, two per SM, 16-token chunks, mma.sync)"
              if wl.gate == "diag" else
              "prefill_chunk_kernel (every 64-token chunk in parallel: scores, inverse, T and P "
              "on tcgen05) + prefill_tc_kernel (one CTA per head: the state in TMEM, "
              "tcgen05.mma, TMA-staged tiles)")
    return {"value": wl.heads * L / (t / 1e3), "unit": "head-tokens/s", "ms_per_launch": t,
            "cpu_baseline": cpu,
            "config": {"workload": wl.name, "B": wl.B, "H": wl.H, "L": L, "D": wl.D,
                       "gate": wl.gate, "act": "bf16", "chunk": C},
            "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s",
                         "frac": tf / peak, "peak_source": src,
                         "flops_per_launch": flops,
                         "note": "UT-form products at single precision; the kernel issues "
                                 "up to three times that on the tensor cores (hi/lo bf16 "
                                 "splits)"},
            "kernel": kernel}


def pw_leg(wl, Wp, S0, inp, o, peak, cpu=False):
    """The pure-write sliding window decode on the same inputs: the history quantized from the
    same initial states, then the T steps, one launch each, timed with CUDA events."""
    import torch

    import bit_recurrent_state_gdn_b200 as gdn

    cfg = gdn.make_pw_config(wl.B, wl.H, wl.D, Wp, wl.gate, wl.fmt, wl.act)
    st = gdn.PwState.allocate(cfg)
    gdn.gdn_pw_quantize(cfg, S0, st)
    gdn.gdn_pw_decode_steps(cfg, st, inp["q"][:4], inp["k"][:4], inp["v"][:4], inp["g"][:4],
                            inp["beta"][:4], o[:4])
    gdn.gdn_pw_quantize(cfg, S0, st)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    gdn.gdn_pw_decode_steps(cfg, st, inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], o)
    e1.record()
    torch.cuda.synchronize()
    if int(st.status[0].item()) != 0:
        raise RuntimeError("pure-write window: device status word set")
    ms = e0.elapsed_time(e1)
    gbs = pw_step_bytes(wl, Wp) * wl.heads * wl.T / (ms / 1e3) / 1e9
    traffic, src = profiled_traffic(PW_PROFILE, PW_KERNEL_SOURCES,
                                    f"traffic_bytes_per_head_{wl.fmt}")
    return {"value": wl.heads * wl.T / (ms / 1e3), "unit": UNIT, "achieved_gbs": gbs,
            "cpu_baseline": pw_cpu_baseline(wl, Wp, inp, S0.device) if cpu else None,
            "frac": gbs / peak, "avg_launch_us": ms * 1e3 / wl.T, "ms_per_run": ms,
            "bytes_per_head_step": pw_step_bytes(wl, Wp), "Wp": Wp,
            "traffic": None if traffic is None else traffic * wl.heads, "traffic_source": src,
            "kernel": "pw_step_kernel (history requantised every step, FP8 pairs)"}


def e2e(args, wl, cfg, inp, S0, state, world, dev):
    import torch
    import torch.distributed as dist

    import bit_recurrent_state_gdn_b200 as gdn

    host = {n: t.cpu().pin_memory() for n, t in inp.items()}
    hS0 = S0.cpu().pin_memory()
    ho = torch.empty(inp["q"].shape, dtype=inp["q"].dtype).pin_memory()
    dS = torch.empty_like(S0)
    staging = torch.empty(gdn.gdn_host_staging_bytes(cfg), dtype=torch.uint8, device=dev)

    def step():
        dS.copy_(hS0, non_blocking=True)
        gdn.gdn_state_quantize(cfg, dS, state)
        gdn.gdn_decode_window_steps_host(cfg, state, host["q"], host["k"], host["v"], host["g"],
                                         host["beta"], ho, staging)

    step()
    torch.cuda.synchronize()
    n = max(1, min(args.steps, 3))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(n):
        step()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    ms = max_over_ranks(ms, world, dev)
    state_up = hS0.numel() * 4
    h2d = state_up + sum(t.numel() * t.element_size() for t in host.values())
    d2h = ho.numel() * ho.element_size()
    return {"value": whole_job_rate(wl.heads * wl.T * n, world, ms), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n,
            "link_gbs": (h2d + d2h) * n / (ms / 1e3) / 1e9,
            "state_upload_bytes_per_step": state_up,
            "state_upload_share": state_up / (h2d + d2h),
            "note": "each step uploads the fp32 initial states (to quantize them) and every "
                    "decode token's q / k / v / g / beta, and reads back every output: the "
                    "host link, not the kernels, bounds this figure",
            "api": "gdn_decode_window_steps_host (pinned host buffers, copies pipelined)"}


def oracle_sample(wl, inp, n_seq, dev):
    """The first n_seq sequences' inputs as float64 numpy ([T][n][...]) and their initial states
    made by the oracle's own fp32-storage warm-up recurrence (nothing from the GPU)."""
    import numpy as np
    import torch

    heads = np.arange(n_seq * wl.H)
    idx = torch.as_tensor(heads, device=dev)

    def pick(x, T):
        flat = x.reshape(T, wl.heads, *x.shape[3:])
        return flat.index_select(1, idx).double().cpu().numpy()

    d = {n: pick(x, x.shape[0]) for n, x in inp.items()}
    if wl.warmup == 0:
        return d, np.zeros((len(heads), wl.D, wl.D))
    scales = outlier_scales(wl, dev)
    warm = {n: [] for n in ("q", "k", "v", "g", "beta")}
    for t in range(wl.warmup):
        s = step_inputs(wl, "warmup", t, dev, scales)
        for n in warm:
            x = getattr(s, n)
            warm[n].append(x.reshape(wl.heads, *x.shape[2:]).index_select(0, idx).double()
                           .cpu().numpy())
    warm = {n: np.stack(v) for n, v in warm.items()}
    return d, oracle_warm_state(wl, warm)


def cpu_baseline(args, wl, inp, dev):
    n_seq = max(1, min(wl.B, args.cpu_heads // wl.H))
    d, S0 = oracle_sample(wl, inp, n_seq, dev)
    hs, dt, cores = time_oracle(wl, d["q"], d["k"], d["v"], d["g"], d["beta"], S0)
    return {"value": hs, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n_seq * wl.H} heads (sequences 0..{n_seq - 1}, all {wl.H} heads) x "
                      f"{wl.T} steps of the same inputs, {dt:.1f} s"}


def quality_figure(wl, inp, o, dev, n_seq: int = 8):
    """Output error of the windowed int8 decode against the unquantized fp64 recurrence (the
    oracle's plain run from the oracle's own warm-up states), on the first n_seq sequences: the
    cost of the low-bit state, not a parity bar."""
    import numpy as np

    import oracle

    d, S0 = oracle_sample(wl, inp, n_seq, dev)
    ref, _ = oracle.plain_run(d["q"], d["k"], d["v"], d["g"], d["beta"], S0=S0, want_o=True)
    n = n_seq * wl.H
    got = o.reshape(wl.T, wl.heads, wl.D)[:, :n].double().cpu().numpy()
    err = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    return {"o_rel_l2_vs_fp64_recurrence": err, "heads": n, "steps": wl.T,
            "note": "%s windowed state (W = %d, r = %d %s tokens%s) against the fp64 recurrence "
                    "with no quantization; GPU outputs in bf16"
                    % (wl.fmt, wl.W, wl.r, wl.comp_rule,
                       ", residual smoothing" if wl.smooth else "")}


def pw_cpu_baseline(wl, Wp, inp, dev, n_seq: int = 4):
    """The oracle's pure-write window (GPU storage roundings on) on the first n_seq sequences."""
    import oracle

    d, S0 = oracle_sample(wl, inp, n_seq, dev)
    T, n = d["q"].shape[0], d["q"].shape[1]
    t0 = time.perf_counter()
    oracle.pw_run(d["q"], d["k"], d["v"], d["g"], d["beta"], Wp=Wp, fmt=wl.fmt, S0=S0,
                  prec32=True)
    dt = time.perf_counter() - t0
    return {"value": n * T / dt, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} heads (sequences 0..{n_seq - 1}) x {T} steps, {dt:.1f} s"}


def prefill_cpu_baseline(wl, inp, dev, n_heads: int = 16):
    """The oracle's plain fp64 recurrence over the first n_heads heads' prompts."""
    import oracle
    import torch

    idx = torch.arange(n_heads, device=dev)
    d = {n: x.reshape(x.shape[0], wl.heads, *x.shape[3:]).index_select(1, idx).double().cpu()
         .numpy() for n, x in inp.items()}
    t0 = time.perf_counter()
    oracle.plain_run(d["q"], d["k"], d["v"], d["g"], d["beta"])
    dt = time.perf_counter() - t0
    L = d["q"].shape[0]
    return {"value": n_heads * L / dt, "unit": "head-tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle", "sample": f"{n_heads} heads x {L} tokens, {dt:.1f} s"}


if __name__ == "__main__":
    main()
