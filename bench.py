"""Benchmark: steady-state frame-steps of the Summaryformer frame memory on B200.

One step (one "frame") = wm_advance(t) (RAW -> SUM eviction in all 28 blocks)
followed, for each of the 28 blocks, by wm_write_attend: the frame's K/V
record written into its slot and the attention of its 1104 queries over the
6,528 keys (16 heads x 64), in one launch, at the served shape 24x42 + X=96,
Y=2, W=24, in steady state (t >= 31).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line on rank 0.  ``value`` = frame-steps/s over all ranks
(each rank runs its own independent session: weak scaling, no collective on
the data path), timed with CUDA events between a barrier + synchronize on
both sides, max over ranks.  ``--impl reference`` times the fp64 CPU oracle on
the host cores instead (rank 0 only).

One frame-step is one pass per frame (one record write and one attention
per block); the served pattern of four passes per frame (three denoising
passes and the clean rewrite) is timed as well, under ``extras``.

At N = 1 the line also carries ``long_run`` (median of 5 separate runs of 200
frame-steps) and ``extras`` (none of them enters ``value``): the frame-step
replayed from CUDA graphs, the four-pass served frame, the HBM throughput of
the eviction and record-write kernels, a batch of 8 sessions, and the scaled
memory (24 x 128, W = 48) against the dense full-history attention it
replaces.  On rank 0 at N = 1 the CPU-baseline leg times the fp64 oracle on
one block and, before the timed region, compares the GPU path with it on the
same inputs (every byte of the block's buffers, sampled attention rows); a
mismatch stops the run.

``--ncu-csv FILE --ncu-out FILE`` only summarises an ncu CSV capture (per
kernel: launches, total time, share, per-launch metrics, and the digest of
the attention kernel's sources) into JSON for ``profiles/``; it needs no GPU.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import seeded_inputs as si  # noqa: E402

METRIC = "steady-state frames/s (28 blocks attend+evict, 6528 keys); % bf16 TC peak"
UNIT = "frames/s"

# served shape (model card: 24x42 latent grid, X=96, Y=2, W=24 trained window,
# 28 blocks, heads of 64; the synthetic workload uses 16 heads)
BLOCKS, HEADS, D, GH, GW, X, Y, W = 28, 16, 64, 24, 42, 96, 2, 24
HW = GH * GW
R = HW + X
C = R * (Y + 2) + X * (W - Y)
T_STEADY = 31
ATTN_FLOP = 4 * R * C * D * HEADS                 # QK^T + PV, multiply-add = 2
EVICT_BYTES = 2 * 2 * X * HEADS * D * 2 * BLOCKS  # read + write, K and V, all blocks
WRITE_BYTES = 2 * 2 * R * HEADS * D * 2           # read + write, K and V, one block
WORKLOAD = (f"served frame-step: advance (evict) + {BLOCKS} x write_attend (record write + attend), "
            f"grid {GH}x{GW} + X={X}, Y={Y}, W={W}, {HEADS} heads x {D}, "
            f"{R} queries x {C} keys, steady state t>={T_STEADY}, one session per GPU")
CONFIG_ID = 3
# a timed region at least this long runs at the power-capped (sustained) clock
SUSTAINED_REGION_S = 2.0

PROFILES = os.path.join(ROOT, "profiles")
TRAFFIC_JSON = os.path.join(PROFILES, "attend_kernel_served.json")
LAUNCHES_JSON = os.path.join(PROFILES, "frame_step_launches_served.json")
CSRC = os.path.join(ROOT, "kv_memory_attention_b200", "csrc")
# the files each kernel is compiled from
ATTEND_SOURCES = ("attend_sm100.cu", "sm100_ptx.cuh", "wmkv_internal.h")
COPY_SOURCES = ("copy_kernels.cu", "sm100_ptx.cuh", "wmkv_internal.h")


# --kv-format e4m3: the same workload on the FP8 memory, one scale for every
# (block, head) of K and of V (N(0,1) values stay well inside E4M3's range)
FP8_SCALE = 1.0 / 64


def config_dict(world: int, kv_format: str = "bf16") -> dict:
    """The workload, identical for both arms."""
    c = {"workload": WORKLOAD, "blocks": BLOCKS, "heads": HEADS, "head_dim": D,
         "grid": f"{GH}x{GW}", "X": X, "Y": Y, "W": W, "queries": R, "keys": C,
         "passes_per_frame": 1,
         "parallelism": f"replicas x{world} (independent sessions)",
         "l2": "no flush: per step the 28 blocks touch 748 MB of K/V buffers + 190 MB of "
               "inputs, far above the 126 MB L2"}
    if kv_format != "bf16":
        c.update({"kv_format": kv_format, "kv_scale": FP8_SCALE,
                  "l2": "no flush: per step the 28 blocks touch 374 MB of FP8 K/V buffers + 190 MB "
                        "of inputs, far above the 126 MB L2"})
    return c


def make_memory(wm, kv_format: str, blocks=BLOCKS, heads=HEADS, d=D, gh=GH, gw=GW, x=X, y=Y, w=W):
    if kv_format == "e4m3":
        n = blocks * heads
        return wm.KVMemory(blocks, heads, d, gh, gw, x, y, w, kv_format="e4m3",
                           k_scale=[FP8_SCALE] * n, v_scale=[FP8_SCALE] * n)
    return wm.KVMemory(blocks, heads, d, gh, gw, x, y, w)


def peaks() -> dict:
    """Roofline denominators: the driver's measured peaks, else the recipe's fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"sustained": float(p["bf16_tflops_sustained"]), "burst": float(p["bf16_tflops"]),
                "hbm": float(p["hbm_gbs"]), "source": "measured"}
    except Exception:
        return {"sustained": 1400.0, "burst": 1590.0, "hbm": 6650.0, "source": "fallback"}


def source_digest(files=ATTEND_SOURCES) -> str:
    """sha256 prefix of a kernel's source files (in a fixed order)."""
    h = hashlib.sha256()
    for name in files:
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def file_digests() -> dict:
    """sha256 prefix of every library source file."""
    out = {}
    for name in sorted(os.listdir(CSRC)):
        with open(os.path.join(CSRC, name), "rb") as f:
            out[name] = hashlib.sha256(f.read()).hexdigest()[:16]
    return out


# ---------------------------------------------------------------- ncu summaries

_TIME_UNITS = {"nsecond": 1e-3, "usecond": 1.0, "msecond": 1e3, "second": 1e6,
               "ns": 1e-3, "us": 1.0, "ms": 1e3, "s": 1e6}
_BYTE_UNITS = {"byte": 1.0, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9,
               "kibyte": 1024.0, "mibyte": 1024.0 ** 2, "gibyte": 1024.0 ** 3,
               "b": 1.0, "kb": 1e3, "mb": 1e6, "gb": 1e9, "kib": 1024.0, "mib": 1024.0 ** 2,
               "gib": 1024.0 ** 3}


def _kernel_short_name(name: str) -> str:
    """'void ns::(anonymous namespace)::attend_kernel<64>(ns::P)' -> 'attend_kernel<64>'."""
    m = re.search(r"([A-Za-z_]\w*(?:<[^()]*>)?)\s*\(", name)
    return m.group(1) if m else name.strip()


def summarize_ncu_csv(path: str, command: str) -> dict:
    """Per-kernel summary of an ncu ``--csv`` capture (one row per launch and metric).

    Times are converted to microseconds and byte counts to bytes; every other
    metric is averaged per launch as printed."""
    with open(path, newline="") as f:
        lines = [ln for ln in f if not ln.startswith("==")]
    rows = list(csv.reader(lines))
    head = next(i for i, r in enumerate(rows) if "Kernel Name" in r and "Metric Name" in r)
    cols = {name: i for i, name in enumerate(rows[head])}
    launches = {}
    for r in rows[head + 1:]:
        if len(r) < len(cols):
            continue
        lid = r[cols["ID"]]
        kname = _kernel_short_name(r[cols["Kernel Name"]])
        metric = r[cols["Metric Name"]]
        unit = r[cols["Metric Unit"]].strip().lower()
        try:
            val = float(r[cols["Metric Value"]].replace(",", ""))
        except ValueError:
            continue
        if unit in _TIME_UNITS:
            val *= _TIME_UNITS[unit]
        elif unit in _BYTE_UNITS:
            val *= _BYTE_UNITS[unit]
        launches.setdefault(lid, {"kernel": kname, "metrics": {}})["metrics"][metric] = val
    per = {}
    for rec in launches.values():
        k = per.setdefault(rec["kernel"], {"launches": 0, "sums": {}})
        k["launches"] += 1
        for m, v in rec["metrics"].items():
            k["sums"][m] = k["sums"].get(m, 0.0) + v
    total_us = sum(k["sums"].get("gpu__time_duration.sum", 0.0) for k in per.values())
    kernels = []
    for name, k in sorted(per.items(), key=lambda kv: -kv[1]["sums"].get("gpu__time_duration.sum", 0)):
        n = k["launches"]
        entry = {"kernel": name, "launches": n}
        t = k["sums"].get("gpu__time_duration.sum")
        if t is not None:
            entry.update({"total_us": round(t, 3), "avg_us": round(t / n, 3),
                          "share": round(t / total_us, 4) if total_us else None})
        for m, v in sorted(k["sums"].items()):
            if m != "gpu__time_duration.sum":
                entry[m + " (per launch)"] = v / n
        rd = k["sums"].get("dram__bytes_read.sum")
        wr = k["sums"].get("dram__bytes_write.sum")
        if rd is not None and wr is not None:
            entry["dram_bytes_per_launch"] = int(round((rd + wr) / n))
        kernels.append(entry)
    return {"command": command, "source_sha256": source_digest(), "sources": file_digests(),
            "captured_launches": len(launches), "kernels": kernels,
            "note": "ncu replays each launch cold and serialised: compare shares, not absolute times"}


def _profile_entry(path: str, prefix: str, files=ATTEND_SOURCES):
    """The kernel entry whose name starts with ``prefix`` in a summary JSON
    captured from the current version of ``files``, else None."""
    try:
        with open(path) as f:
            j = json.load(f)
        now = file_digests()
        if any(j.get("sources", {}).get(name) != now[name] for name in files):
            return None
        for k in j["kernels"]:
            if k["kernel"].startswith(prefix):
                return k
    except Exception:
        return None
    return None


def load_traffic():
    """DRAM bytes (read + write) per attention launch from the committed ncu JSON,
    or None when the kernel sources changed since it was captured."""
    k = _profile_entry(TRAFFIC_JSON, "attend_kernel<64")
    return None if k is None else k.get("dram_bytes_per_launch")


def load_ncu_share():
    k = _profile_entry(LAUNCHES_JSON, "attend_kernel<64")
    return None if k is None else k.get("share")


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- distributed

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_pg(world, backend):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Largest value over all ranks (the slowest rank sets the job's time)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(steps_per_rank: int, elapsed_ms_max: float, world: int) -> float:
    """Whole-job frame-steps/s: all ranks' steps over the slowest rank's time."""
    return world * steps_per_rank / (elapsed_ms_max / 1e3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def attention_launch_time(step_ms_total: float, evict_ms_total: float, steps: int) -> float:
    """Average attention launch duration (ms) inside a run of frame-steps: the run's
    time minus its evictions, over its 28 launches per step."""
    return (step_ms_total - evict_ms_total) / (BLOCKS * steps)


def choose_peak(pk: dict, region_s: float):
    """The burst peak for a region shorter than SUSTAINED_REGION_S, else the sustained one."""
    if region_s >= SUSTAINED_REGION_S:
        return pk["sustained"], "bf16_tflops_sustained"
    return pk["burst"], "bf16_tflops"


# ---------------------------------------------------------------- our arm

def run_ours(args, world, rank, local):
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_pg(world, "nccl")
    import kv_memory_attention_b200 as wm

    # CPU baseline (rank 0, N = 1): the oracle timed on host cores, and the GPU
    # path checked against it on the same inputs before anything is timed
    fp8 = args.kv_format == "e4m3"
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_and_parity(args.cpu_seconds, torch, wm, args.kv_format)

    kv = make_memory(wm, args.kv_format)
    pool = torch.from_numpy(si._pool()["bf16"].view(np.int16)).to(device).view(torch.bfloat16)
    psize = pool.shape[0]
    n = R * HEADS * D

    def window(seed):
        s = seed % psize
        if s + n <= psize:
            return pool[s:s + n].view(R, HEADS, D).clone()
        return torch.cat([pool[s:], pool[:n - (psize - s)]]).view(R, HEADS, D)

    # distinct per-block inputs (28 x Q, K, V = 190 MB resident in HBM)
    Q = [window(si.seed_for(CONFIG_ID, rank, b, 0, 0, si.T_Q)) for b in range(BLOCKS)]
    K = [window(si.seed_for(CONFIG_ID, rank, b, 0, 0, si.T_K)) for b in range(BLOCKS)]
    V = [window(si.seed_for(CONFIG_ID, rank, b, 0, 0, si.T_V)) for b in range(BLOCKS)]
    O = [torch.empty(R, HEADS, D, dtype=torch.bfloat16, device=device) for _ in range(BLOCKS)]
    stream = torch.cuda.current_stream()

    # fill the memory up to steady state
    t = 0
    for t in range(T_STEADY):
        kv.advance(t)
        for b in range(BLOCKS):
            kv.write_record(b, t, K[b], V[b])
    t = T_STEADY

    def step(t, ev=None):
        # one launch per block: the record write and the attention are fused
        if ev is not None:
            ev[0].record(stream)
        kv.advance(t, stream)
        if ev is not None:
            ev[1].record(stream)
        for b in range(BLOCKS):
            kv.write_attend(b, t, Q[b], K[b], V[b], O[b], stream)

    for _ in range(args.warmup):
        step(t)
        t += 1
    torch.cuda.synchronize()
    kv.sync_status()

    # ------------------------------------------------ timed region (device-resident inputs)
    # Only the start/stop events sit in the stream here: an event between two
    # kernels would stop the next kernel's prologue from overlapping the
    # previous one (programmatic dependent launch).
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record(stream)
        for s in range(args.steps):
            step(t)
            t += 1
        stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    kv.sync_status()
    elapsed_ms = max_over_ranks(start.elapsed_time(stop), world, device)
    # per step: the eviction, then per block one launch (bf16: fused write and
    # attention) or two (FP8: record store + widening, attention)
    launches = args.steps * (1 + (2 if fp8 else 1) * BLOCKS)

    # ------------------------------------------------ attention launch time (roofline)
    # The same steps again with an event pair around each eviction only: the
    # attention launches keep overlapping each other, and their average
    # duration is the run's time minus the evictions, over 28 per step.
    n_rf = max(1, min(args.steps, 200))
    ev_evict = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(n_rf)]
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    r0.record(stream)
    for s in range(n_rf):
        step(t, ev_evict[s])
        t += 1
    r1.record(stream)
    torch.cuda.synchronize()
    kv.sync_status()
    rf_total_ms = r0.elapsed_time(r1)
    evict_ms = sum(a.elapsed_time(b) for a, b in ev_evict)
    attn_avg_ms = max_over_ranks(attention_launch_time(rf_total_ms, evict_ms, n_rf), world, device)

    # ------------------------------------------------ end to end: host buffers through the ABI
    e2e = run_e2e(args, torch, wm, kv, t, rank, world, device, Q, K, V)
    t = e2e.pop("_t")
    kv.sync_status()

    # ------------------------------------------------ longer runs and secondary measurements (N = 1)
    long_run, extras = None, None
    if world == 1 and not args.no_extras and not fp8:
        long_run, t = extra_runs(torch, kv, t, Q, K, V, O)
        extras, t = run_extras(torch, wm, device, kv, t, Q, K, V, O, window,
                               elapsed_ms / args.steps)

    value = aggregate_throughput(args.steps, elapsed_ms, world)
    pk = peaks()
    peak, peak_name = choose_peak(pk, rf_total_ms / 1e3)
    achieved_tflops = ATTN_FLOP / (attn_avg_ms * 1e-3) / 1e12
    step_tflops = BLOCKS * ATTN_FLOP * args.steps / (elapsed_ms / 1e3) / 1e12
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(elapsed_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_dict(world, args.kv_format),
        "tflops_per_step": round(step_tflops, 1),
        "frac_of_bf16_peak_step": round(step_tflops / peak, 4),
        "roofline": {"kernel": ("per block: store_widen_pair_kernel + attend_kernel<64>"
                                if fp8 else "attend_kernel<64> (fused record write)"),
                     "bound": "tensor",
                     "achieved": round(achieved_tflops, 1), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved_tflops / peak, 4),
                     "peak_source": f"{peak_name} ({pk['source']}); timed region "
                                    f"{rf_total_ms:.1f} ms",
                     "frac_of_sustained": round(achieved_tflops / pk["sustained"], 4),
                     "avg_launch_us": round(attn_avg_ms * 1e3, 2),
                     "how": f"{n_rf} frame-steps with events around each eviction only: "
                            f"(run time - evictions) / ({BLOCKS} x {n_rf}) launches",
                     "run_ms": round(rf_total_ms, 3), "evict_ms": round(evict_ms, 3),
                     "share_from_events": round(1.0 - evict_ms / rf_total_ms, 4),
                     "ncu_share": None if fp8 else load_ncu_share(),
                     "flop_per_launch": ATTN_FLOP, "traffic": None if fp8 else load_traffic()},
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }
    if long_run is not None:
        line["long_run"] = long_run
    if extras is not None:
        line["extras"] = extras
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    kv.close()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def run_e2e(args, torch, wm, kv, t, rank, world, device, Qd, Kd, Vd):
    """Same steps with inputs in pinned host memory: H2D of Q/K/V and D2H of O every step.

    Each block's Q, K and V sit back to back in one pinned host buffer and in
    one device buffer, so a block's inputs cross the host link as one copy."""
    hqkv = [torch.stack([q.cpu(), k.cpu(), v.cpu()]).pin_memory() for q, k, v in zip(Qd, Kd, Vd)]
    ho = [torch.empty(R, HEADS, D, dtype=torch.bfloat16).pin_memory() for _ in range(BLOCKS)]
    dqkv = [torch.empty_like(x, device=device) for x in hqkv]
    dq = [x[0] for x in dqkv]
    dk = [x[1] for x in dqkv]
    dv = [x[2] for x in dqkv]
    do = [torch.empty(R, HEADS, D, dtype=torch.bfloat16, device=device) for _ in range(BLOCKS)]
    comp = torch.cuda.current_stream()
    s_in = torch.cuda.Stream()
    s_out = torch.cuda.Stream()
    used = [torch.cuda.Event() for _ in range(BLOCKS)]     # staging inputs consumed, O written
    landed = [torch.cuda.Event() for _ in range(BLOCKS)]   # H2D of the block's inputs finished
    copied = [torch.cuda.Event() for _ in range(BLOCKS)]   # D2H of the block's O finished
    for b in range(BLOCKS):
        used[b].record(comp)
        copied[b].record(s_out)

    def step(t):
        for b in range(BLOCKS):
            s_in.wait_event(used[b])
            with torch.cuda.stream(s_in):
                dqkv[b].copy_(hqkv[b], non_blocking=True)
            landed[b].record(s_in)
        wm.wm_advance(kv.h, t, comp)
        for b in range(BLOCKS):
            comp.wait_event(landed[b])
            comp.wait_event(copied[b])
            wm.wm_write_attend(kv.h, b, t, dq[b], dk[b], dv[b], do[b], comp)
            used[b].record(comp)
            s_out.wait_event(used[b])
            with torch.cuda.stream(s_out):
                ho[b].copy_(do[b], non_blocking=True)
            copied[b].record(s_out)

    for _ in range(max(1, args.warmup)):
        step(t)
        t += 1
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record(comp)
    s_in.wait_event(start)
    s_out.wait_event(start)
    for _ in range(args.steps):
        step(t)
        t += 1
    comp.wait_stream(s_out)
    stop.record(comp)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(start.elapsed_time(stop), world, device)
    nbytes = R * HEADS * D * 2
    h2d = 3 * BLOCKS * nbytes
    # the host link alone: the step's own input copies (the same pinned buffers,
    # the same stream), with no kernels running; the fastest of 5 passes
    link_ms = []
    for _ in range(5):
        l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        l0.record(s_in)
        with torch.cuda.stream(s_in):
            for b in range(BLOCKS):
                dqkv[b].copy_(hqkv[b], non_blocking=True)
        l1.record(s_in)
        torch.cuda.synchronize()
        link_ms.append(l0.elapsed_time(l1))
    link_gbs = h2d / (min(link_ms) * 1e-3) / 1e9
    return {"value": round(world * args.steps / (ms / 1e3), 3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": BLOCKS * nbytes,
            "ms_per_step": round(ms / args.steps, 4),
            "h2d_link_GB_per_s": round(link_gbs, 1),
            "h2d_bound_ms_per_step": round(h2d / (link_gbs * 1e9) * 1e3, 4),
            "how": "pinned host Q/K/V (one buffer per block) copied in on a copy stream, O copied "
                   "out on another, overlapped with the kernels block by block; the link figure is "
                   "the fastest of 5 passes of the same input copies with no kernels running", "_t": t}


# ---------------------------------------------------------------- secondary measurements
# Reported under "long_run" / "extras" at N = 1; none of them enters `value`.

GRAPH_PERIOD = 66   # lcm(Y + 1, W - Y): the served slot pattern repeats every 66 frames


def _timed(torch, fn, n):
    """CUDA-event time of n calls of fn on the current stream, in ms per call."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(n):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / n


def extra_graph(torch, kv, t, Q, K, V, O):
    """The served frame-step replayed from CUDA graphs.

    One graph per frame for GRAPH_PERIOD consecutive frames: the slots a frame
    writes and evicts repeat with that period, so replaying the graphs in
    order continues the rollout exactly.  Returns (result, next t).
    """
    cap = torch.cuda.Stream()
    graphs = []
    torch.cuda.synchronize()
    for _ in range(GRAPH_PERIOD):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            s = torch.cuda.current_stream()
            kv.advance(t, s)
            for b in range(BLOCKS):
                kv.write_attend(b, t, Q[b], K[b], V[b], O[b], s)
        graphs.append(g)
        t += 1

    def cycle():
        for g in graphs:
            g.replay()

    cycle()                                   # warm-up cycle
    cycles = 3
    ms = _timed(torch, cycle, cycles) / GRAPH_PERIOD
    kv.sync_status()
    del graphs
    return {"value": round(1e3 / ms, 3), "unit": UNIT, "ms_per_step": round(ms, 4),
            "steps": cycles * GRAPH_PERIOD,
            "how": f"{GRAPH_PERIOD} frame-steps captured as one CUDA graph each "
                   f"(29 launches), replayed in order {cycles} times after one warm-up cycle"}, t


def extra_runs(torch, kv, t, Q, K, V, O, runs=5, steps=200):
    """The served frame-step timed as `runs` separate runs of `steps` steps
    (CUDA events per run); median, min and max frame-steps/s."""
    vals = []
    for _ in range(runs):
        def one():
            nonlocal t
            kv.advance(t)
            for b in range(BLOCKS):
                kv.write_attend(b, t, Q[b], K[b], V[b], O[b])
            t += 1
        vals.append(1e3 / _timed(torch, one, steps))
    kv.sync_status()
    return {"runs": runs, "steps_each": steps, "median": round(statistics.median(vals), 3),
            "min": round(min(vals), 3), "max": round(max(vals), 3), "unit": UNIT,
            "tflops_per_step_median": round(BLOCKS * ATTN_FLOP * statistics.median(vals) / 1e12, 1)}, t


def extra_four_pass(torch, kv, t, Q, K, V, O, frames=50):
    """The served frame as the model runs it: one advance, then four passes
    (three denoising passes and the clean rewrite), each writing every block's
    record into the same slot and attending; frames per second measured."""
    def frame():
        nonlocal t
        kv.advance(t)
        for _ in range(4):
            for b in range(BLOCKS):
                kv.write_attend(b, t, Q[b], K[b], V[b], O[b])
        t += 1
    frame()
    ms = _timed(torch, frame, frames)
    kv.sync_status()
    return {"value": round(1e3 / ms, 3), "unit": "frames/s (4 passes each)", "ms_per_frame": round(ms, 4),
            "frames": frames, "launches_per_frame": 1 + 4 * BLOCKS}, t


def extra_copies(torch, kv, t, K, V, hbm_gbs):
    """HBM throughput of the eviction (wm_advance) and the record write
    (wm_write_record), each launch timed alone after reading a 512 MB buffer
    (clean lines: the L2 holds none of the copy's data and nothing dirty).
    The rollout stays valid: every block gets its record every frame."""
    flush = torch.empty(128 * 2 ** 20, dtype=torch.float32, device=K[0].device).fill_(1.0)
    ev, wr = [], []
    n = 10
    for _ in range(n):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        flush.sum()
        e[0].record()
        kv.advance(t)
        e[1].record()
        for b in range(BLOCKS):
            if b == 0:
                flush.sum()
                e[2].record()
            kv.write_record(b, t, K[b], V[b])
            if b == 0:
                e[3].record()
        ev.append(e)
        t += 1
    torch.cuda.synchronize()
    kv.sync_status()
    evict_us = statistics.median(x[0].elapsed_time(x[1]) for x in ev) * 1e3
    write_us = statistics.median(x[2].elapsed_time(x[3]) for x in ev) * 1e3
    del flush

    def entry(kernel, nbytes, us):
        gbs = nbytes / (us * 1e-6) / 1e9
        return {"kernel": kernel, "bytes": nbytes, "us": round(us, 2), "GB_per_s": round(gbs, 1),
                "frac_of_hbm": round(gbs / hbm_gbs, 3)}

    out = {"evict": entry("evict_kernel (28 blocks, one launch)", EVICT_BYTES, evict_us),
           "record_write": entry("copy_pair_kernel (one block)", WRITE_BYTES, write_us),
           "how": f"median of {n} launches, each after a 512 MB read (L2 holds no copy data); "
                  "bytes = algorithmic read + write; CUDA events around one launch, so launch "
                  "and event overhead are included (an upper bound on the kernel's time)"}
    ev = _profile_entry(LAUNCHES_JSON, "evict_kernel", COPY_SOURCES)
    if ev is not None:
        out["evict_ncu"] = entry("evict_kernel, ncu gpu__time_duration in the frame-step launch list",
                                 EVICT_BYTES, ev["avg_us"])
    return out, t


def extra_batch(torch, wm, window, device, sessions=8, steps=20):
    """Eight independent served sessions on one stream, interleaved block by
    block (each session: its own memory and inputs, K rows scaled per token by
    U(0.5, 2)); aggregate frame-steps/s."""
    gen = torch.Generator(device=device)
    gen.manual_seed(0x5EED + 4)
    mems, ins = [], []
    for s in range(sessions):
        mems.append(wm.KVMemory(BLOCKS, HEADS, D, GH, GW, X, Y, W))
        q = [window(si.seed_for(4, s, b, 0, 0, si.T_Q)) for b in range(BLOCKS)]
        k = [window(si.seed_for(4, s, b, 0, 0, si.T_K)) for b in range(BLOCKS)]
        v = [window(si.seed_for(4, s, b, 0, 0, si.T_V)) for b in range(BLOCKS)]
        for b in range(BLOCKS):
            scale = torch.rand(R, 1, 1, generator=gen, device=device) * 1.5 + 0.5
            k[b] = (k[b].float() * scale).to(torch.bfloat16)
        o = [torch.empty(R, HEADS, D, dtype=torch.bfloat16, device=device) for _ in range(BLOCKS)]
        ins.append((q, k, v, o))
    for t in range(T_STEADY):
        for s, m in enumerate(mems):
            m.advance(t)
            for b in range(BLOCKS):
                m.write_record(b, t, ins[s][1][b], ins[s][2][b])
    t = T_STEADY

    def step():
        nonlocal t
        for m in mems:
            m.advance(t)
        for b in range(BLOCKS):
            for s, m in enumerate(mems):
                q, k, v, o = ins[s]
                m.write_attend(b, t, q[b], k[b], v[b], o[b])
        t += 1

    for _ in range(3):
        step()
    ms = _timed(torch, step, steps)
    for m in mems:
        m.sync_status()
        m.close()
    return {"sessions": sessions, "value": round(sessions * 1e3 / ms, 3), "unit": UNIT,
            "ms_per_step": round(ms, 4), "steps": steps,
            "how": "8 served sessions on one stream: each frame-step advances all 8, then for "
                   "each block runs write_attend of every session"}


def extra_scaled(torch, wm, device, pk, steps=10):
    """The scaled memory (24 heads x 128, 45x80 + X=256, Y=2, W=48: 3856 queries
    x 27,200 keys) at steady state, and the dense full-history baseline it
    replaces (3600 queries x 180,000 keys, wm_attend_dense), 28 blocks each.
    Every block has its own inputs: windows at different offsets of one random
    pool per tensor (4,096 rows apart for the dense keys and values)."""
    B, H, d, gh, gw, x, y, w = 28, 24, 128, 45, 80, 256, 2, 48
    hw = gh * gw
    r = hw + x
    c = r * (y + 2) + x * (w - y)
    gen = torch.Generator(device=device)
    gen.manual_seed(0x5EED + 5)

    def randn(*shape):
        return torch.randn(*shape, generator=gen, device=device).to(torch.bfloat16)

    def windows(pool, rows, step):
        return [pool[b * step:b * step + rows] for b in range(B)]

    kv2 = wm.KVMemory(B, H, d, gh, gw, x, y, w)
    qp, kp, vp = (randn(r + (B - 1) * 64, H, d) for _ in range(3))
    q, k, v = windows(qp, r, 64), windows(kp, r, 64), windows(vp, r, 64)
    o = torch.empty(r, H, d, dtype=torch.bfloat16, device=device)
    t_steady = 60
    for t in range(t_steady):
        kv2.advance(t)
        for b in range(B):
            kv2.write_record(b, t, k[b], v[b])
    t = t_steady

    # the copy kernels at this size (one eviction: 28 blocks x 256 rows of K and
    # V; one record write: 3856 rows of K and V), each launch timed alone after
    # a 512 MB read that leaves no copy data in L2
    flush = torch.empty(128 * 2 ** 20, dtype=torch.float32, device=device).fill_(1.0)
    ev = []
    for _ in range(5):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        flush.sum()
        e[0].record()
        kv2.advance(t)
        e[1].record()
        flush.sum()
        e[2].record()
        kv2.write_record(0, t, k[0], v[0])
        e[3].record()
        for b in range(1, B):
            kv2.write_record(b, t, k[b], v[b])
        ev.append(e)
        t += 1
    torch.cuda.synchronize()
    del flush
    evict_us = statistics.median(e[0].elapsed_time(e[1]) for e in ev) * 1e3
    write_us = statistics.median(e[2].elapsed_time(e[3]) for e in ev) * 1e3
    evict_bytes = 2 * 2 * x * H * d * 2 * B
    write_bytes = 2 * 2 * r * H * d * 2

    def step():
        nonlocal t
        kv2.advance(t)
        for b in range(B):
            kv2.write_attend(b, t, q[b], k[b], v[b], o)
        t += 1

    step()
    ms_s = _timed(torch, step, steps)
    kv2.sync_status()
    kv2.close()
    del q, k, v, o, qp, kp, vp

    lk = (w + 2) * hw
    qdp, kdp, vdp = randn(hw + (B - 1) * 64, H, d), randn(lk + (B - 1) * 4096, H, d), \
        randn(lk + (B - 1) * 4096, H, d)
    qd, kd, vd = windows(qdp, hw, 64), windows(kdp, lk, 4096), windows(vdp, lk, 4096)
    od = torch.empty(hw, H, d, dtype=torch.bfloat16, device=device)
    st = torch.zeros(1, dtype=torch.int32, device=device)

    def dense_step():
        for b in range(B):
            wm.wm_attend_dense(qd[b], kd[b], vd[b], od, hw, lk, H, d, st)

    wm.wm_attend_dense(qd[0], kd[0], vd[0], od, hw, lk, H, d, st)
    ms_d = _timed(torch, dense_step, 1)
    if int(st.item()) != 0:
        raise RuntimeError("dense attention reported a device timeout")
    del qd, kd, vd, od, qdp, kdp, vdp

    def entry(ms, flop, n):
        tf = flop / (ms * 1e-3) / 1e12
        peak, name = choose_peak(pk, ms * n / 1e3)
        return {"ms_per_step": round(ms, 3), "frame_steps_per_s": round(1e3 / ms, 3),
                "tflops": round(tf, 1), "frac_of_bf16_peak": round(tf / peak, 4),
                "peak": f"{name} ({pk['source']})", "steps": n}

    scaled = entry(ms_s, B * 4 * r * c * d * H, steps)
    scaled.update({"queries": r, "keys": c, "heads": H, "head_dim": d})
    dense = entry(ms_d, B * 4 * hw * lk * d * H, 1)
    dense.update({"queries": hw, "keys": lk, "heads": H, "head_dim": d})
    copies = {}
    for name, kern, nbytes, us in (("evict", "evict_kernel (28 blocks, one launch)", evict_bytes, evict_us),
                                   ("record_write", "copy_pair_kernel (one block)", write_bytes, write_us)):
        gbs = nbytes / (us * 1e-6) / 1e9
        copies[name] = {"kernel": kern, "bytes": nbytes, "us": round(us, 2), "GB_per_s": round(gbs, 1),
                        "frac_of_hbm": round(gbs / pk["hbm"], 3)}
    return {"scaled": scaled, "dense_baseline": dense, "copy_kernels_scaled": copies,
            "speedup_vs_dense": round(ms_d / ms_s, 2),
            "how": "frame-step = advance + 28 x write_attend (scaled) vs 28 x wm_attend_dense over "
                   "the full history; per-block inputs are windows of one random pool per tensor"}


def extra_fp8(torch, wm, Q, K, V, O, steps=50):
    """The served frame-step on an FP8 (E4M3) memory: same inputs, one scale of
    1/64 for every (block, head) of K and V; each write_attend is three launches
    (quantise the record into its slot, widen the block's codes to bf16, attend)."""
    n = BLOCKS * HEADS
    kv8 = wm.KVMemory(BLOCKS, HEADS, D, GH, GW, X, Y, W, kv_format="e4m3",
                      k_scale=[1 / 64] * n, v_scale=[1 / 64] * n)
    for t in range(T_STEADY):
        kv8.advance(t)
        for b in range(BLOCKS):
            kv8.write_record(b, t, K[b], V[b])
    t = T_STEADY

    def step():
        nonlocal t
        kv8.advance(t)
        for b in range(BLOCKS):
            kv8.write_attend(b, t, Q[b], K[b], V[b], O[b])
        t += 1

    for _ in range(3):
        step()
    ms = _timed(torch, step, steps)
    kv8.sync_status()

    # the widening pass: dense FP8 attention minus dense bf16 attention over the
    # same 6,528 keys (the K/V codes of block 0's buffer, widened by the call)
    k8, v8 = kv8.kv_views(0)
    dev = K[0].device
    scale = torch.full((HEADS,), 1 / 64, dtype=torch.float32, device=dev)
    nbytes = wm.wm_attend_dense_fp8_scratch_bytes(C, HEADS, D)
    scratch = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    kb = torch.zeros(C, HEADS, D, dtype=torch.bfloat16, device=dev)
    vb = torch.zeros_like(kb)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    n = 20
    ms8 = _timed(torch, lambda: wm.wm_attend_dense_fp8(Q[0], k8, v8, scale, scale, O[0], R, C, HEADS, D,
                                                       scratch, nbytes, st), n)
    ms16 = _timed(torch, lambda: wm.wm_attend_dense(Q[0], kb, vb, O[0], R, C,
                                                    HEADS, D, st), n)
    kv8.close()
    widen_us = (ms8 - ms16) * 1e3
    widen_bytes = 2 * C * HEADS * D * (1 + 2)         # codes read, bf16 written, K and V
    return {"value": round(1e3 / ms, 3), "unit": UNIT, "ms_per_step": round(ms, 4), "steps": steps,
            "launches_per_step": 1 + 2 * BLOCKS,
            "buffer_bytes": 2 * BLOCKS * C * HEADS * D,
            "tflops_per_step": round(BLOCKS * ATTN_FLOP / (ms * 1e-3) / 1e12, 1),
            "widen": {"us": round(widen_us, 2), "bytes": widen_bytes,
                      "GB_per_s": round(widen_bytes / max(widen_us, 1e-3) / 1e3, 1),
                      "how": f"wm_attend_dense_fp8 minus wm_attend_dense over {C} keys x {HEADS} x {D}, "
                             f"{n} calls each, back to back"},
            "how": "advance + 28 x write_attend on an E4M3 memory (store and widen, attend)"}


def extra_served_dense(torch, wm, device, ms_step, pk, steps=3):
    """The page's comparison at the served shape: the same span kept at full
    resolution, (W + 2) x 1008 = 26,208 keys, attended by the frame's 1008 raw
    queries in every block (wm_attend_dense, per-block windows of one random
    pool per tensor), against the memory's frame-step measured above."""
    gen = torch.Generator(device=device)
    gen.manual_seed(0x5EED + 6)
    lk = (W + 2) * HW
    assert lk == 26208

    def randn(*shape):
        return torch.randn(*shape, generator=gen, device=device).to(torch.bfloat16)

    qp, kp, vp = randn(HW + (BLOCKS - 1) * 64, HEADS, D), randn(lk + (BLOCKS - 1) * 512, HEADS, D), \
        randn(lk + (BLOCKS - 1) * 512, HEADS, D)
    q = [qp[b * 64:b * 64 + HW] for b in range(BLOCKS)]
    k = [kp[b * 512:b * 512 + lk] for b in range(BLOCKS)]
    v = [vp[b * 512:b * 512 + lk] for b in range(BLOCKS)]
    o = torch.empty(HW, HEADS, D, dtype=torch.bfloat16, device=device)
    st = torch.zeros(1, dtype=torch.int32, device=device)

    def step():
        for b in range(BLOCKS):
            wm.wm_attend_dense(q[b], k[b], v[b], o, HW, lk, HEADS, D, st)

    step()
    ms = _timed(torch, step, steps)
    if int(st.item()) != 0:
        raise RuntimeError("dense attention reported a device timeout")
    flop = BLOCKS * 4 * HW * lk * D * HEADS
    tf = flop / (ms * 1e-3) / 1e12
    peak, name = choose_peak(pk, ms * steps / 1e3)
    return {"ms_per_step": round(ms, 4), "frame_steps_per_s": round(1e3 / ms, 3), "tflops": round(tf, 1),
            "frac_of_bf16_peak": round(tf / peak, 4), "peak": f"{name} ({pk['source']})",
            "queries": HW, "keys": lk, "steps": steps,
            "memory_speedup": round(ms / ms_step, 2),
            "how": "28 x wm_attend_dense over (W+2) x 1008 keys against the timed frame-step "
                   "(advance + 28 x write_attend over 6,528 keys)"}


def run_extras(torch, wm, device, kv, t, Q, K, V, O, window, ms_step):
    """All secondary measurements; a section that fails reports its error."""
    pk = peaks()
    out = {}
    for name, fn in (("graph", lambda: extra_graph(torch, kv, t, Q, K, V, O)),
                     ("four_pass_frame", lambda: extra_four_pass(torch, kv, t, Q, K, V, O)),
                     ("copy_kernels", lambda: extra_copies(torch, kv, t, K, V, pk["hbm"])),
                     ("batch8", lambda: (extra_batch(torch, wm, window, device), t)),
                     ("fp8_buffer", lambda: (extra_fp8(torch, wm, Q, K, V, O), t)),
                     ("served_vs_dense", lambda: (extra_served_dense(torch, wm, device, ms_step, pk), t)),
                     ("scaled_vs_dense", lambda: (extra_scaled(torch, wm, device, pk), t))):
        try:
            out[name], t = fn()
        except Exception as e:  # reported, not hidden: the main line stands on its own
            out[name] = {"error": f"{type(e).__name__}: {e}"}
            torch.cuda.synchronize()
    return out, t


# ---------------------------------------------------------------- CPU oracle

def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        if info:
            return max(i.get("num_threads", 1) for i in info)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


class OracleStepper:
    """The fp64 oracle stepping one block through steady-state frames.

    Each ``step(budget)`` advances the oracle's memory one frame (eviction),
    writes the block's record and runs attention for query rows (all heads,
    all keys of the filled prefix) until ``budget`` seconds of attention have
    been spent; the time is extrapolated to a full frame-step of 28 blocks x
    all query rows.  Default: the served shape (16 x 64, 1104 queries x 6,528
    keys).
    """

    def __init__(self, layout=None, config_id=CONFIG_ID, t_steady=T_STEADY, kv_format="bf16"):
        from oracle import FrameMemory, Layout
        self.L = layout if layout is not None else Layout(GH, GW, X, Y, W, heads=HEADS, d=D)
        self.config_id = config_id
        self.kv_format = kv_format
        if kv_format == "e4m3":
            sc = np.full((1, self.L.heads), FP8_SCALE, np.float32)
            self.mem = FrameMemory(self.L, 1, track_records=False, kv_format="e4m3", k_scale=sc,
                                   v_scale=sc)
        else:
            self.mem = FrameMemory(self.L, 1, track_records=False)
        L = self.L
        for t in range(t_steady):
            self.mem.advance(t)
            _, k, v = si.record_inputs(config_id, 0, 0, t, 0, L.R, L.heads, L.d)
            self.mem.write_record(0, t, k, v)
        self.t = t_steady
        self.next_row = 0

    def inputs(self, t):
        L = self.L
        return si.record_inputs(self.config_id, 0, 0, t, 0, L.R, L.heads, L.d)

    def step(self, budget_s: float):
        from oracle import attend_memory
        L = self.L
        R_ = L.R
        q, k, v = self.inputs(self.t)
        t0 = time.perf_counter()
        self.mem.advance(self.t)
        t_evict = time.perf_counter() - t0
        t0 = time.perf_counter()
        self.mem.write_record(0, self.t, k, v)
        t_write = time.perf_counter() - t0
        rows_done, t_attn = 0, 0.0
        while True:
            rows = (np.arange(self.next_row, self.next_row + 128)) % R_
            self.next_row = (self.next_row + 128) % R_
            t0 = time.perf_counter()
            attend_memory(self.mem, 0, q, rows=rows)
            t_attn += time.perf_counter() - t0
            rows_done += 128
            if t_attn >= budget_s:
                break
        self.t += 1
        per_step = BLOCKS * (R_ * t_attn / rows_done + t_write) + t_evict
        spent = t_evict + t_write + t_attn
        return per_step, rows_done, t_attn, spent


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.lower().startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def gpu_parity_on_stepper(stepper, torch, wm):
    """The GPU path (wm_write_attend, the call the bench times) on the inputs
    the oracle stepper is about to use for its next frame, compared with the
    oracle: every byte of the block's K/V buffers, and sampled attention rows
    (all heads) within max-abs 2e-2 and relative L2 5e-3.  Raises on a mismatch."""
    from oracle import attend_memory
    L = stepper.L
    kv = make_memory(wm, stepper.kv_format, 1, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W)

    def dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)

    for t in range(stepper.t):
        kv.advance(t)
        _, k, v = stepper.inputs(t)
        kv.write_record(0, t, dev(k), dev(v))
    t = stepper.t
    q, k, v = stepper.inputs(t)
    kv.advance(t)
    o = torch.full((L.R, L.heads, L.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    kv.write_attend(0, t, dev(q), dev(k), dev(v), o)
    torch.cuda.synchronize()
    kv.sync_status()
    kd, vd = kv.kv_views(0)
    if stepper.kv_format == "e4m3":
        kb, vb = kd.contiguous().cpu().numpy(), vd.contiguous().cpu().numpy()
    else:
        kb = kd.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        vb = vd.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    ob = o.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    kv.close()
    # the oracle's memory after the same frame (a copy: the stepper's own
    # memory advances when it is timed)
    import copy
    mem = copy.deepcopy(stepper.mem)
    mem.advance(t)
    mem.write_record(0, t, k, v)
    if not (np.array_equal(kb, mem.K[0]) and np.array_equal(vb, mem.V[0])):
        raise RuntimeError("parity: the GPU buffers differ from the oracle's")
    rng = np.random.default_rng(0x5EED)
    rows = np.unique(np.concatenate([[0, L.HW - 1, L.HW, L.R - 1], rng.choice(L.R, 60, replace=False)]))
    ref = attend_memory(mem, 0, q, rows=rows)
    got = si.bf16_bits_to_f64(ob[rows])
    if not np.isfinite(got).all():
        raise RuntimeError("parity: non-finite attention output")
    max_abs = float(np.abs(got - ref).max())
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    if max_abs > 2e-2 or rel > 5e-3:
        raise RuntimeError(f"parity: attention max_abs {max_abs:.3e} rel_l2 {rel:.3e}")
    return {"buffers": "bit-exact", "rows": int(len(rows)), "heads": L.heads,
            "max_abs": round(max_abs, 6), "rel_l2": round(rel, 7), "frame": t,
            "call": "wm_write_attend", "kv_format": stepper.kv_format}


def cpu_baseline_and_parity(budget_s: float, torch=None, wm=None, kv_format="bf16"):
    """The oracle timed on the host cores (served block, extrapolated to a
    frame-step), one thread and the scaled memory as well; with ``wm`` given,
    the GPU path is first checked against the oracle on the same inputs."""
    stepper = OracleStepper(kv_format=kv_format)
    parity = gpu_parity_on_stepper(stepper, torch, wm) if wm is not None else None
    per_step, rows, t_attn, _ = stepper.step(budget_s)
    out = {"value": round(1.0 / per_step, 6), "unit": UNIT, "cores": _oracle_threads(),
           "kind": "oracle",
           "sample": f"{rows} query rows x 16 heads x 6528 keys of one block ({t_attn:.1f} s fp64 numpy), "
                     f"plus one eviction and one record write of that block's memory, "
                     f"extrapolated to 28 blocks x 1104 rows",
           "host_cpus": len(os.sched_getaffinity(0)), "cpu_model": _cpu_model()}
    if parity is not None:
        out["gpu_parity"] = parity
    small = max(0.5, budget_s / 4)
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            per1, rows1, t1, _ = OracleStepper().step(small)
        out["one_thread"] = {"value": round(1.0 / per1, 6), "unit": UNIT, "cores": 1,
                             "sample": f"{rows1} query rows of one served block ({t1:.1f} s), "
                                       f"extrapolated the same way"}
    except Exception as e:  # reported, not hidden
        out["one_thread"] = {"error": f"{type(e).__name__}: {e}"}
    try:
        from oracle import Layout
        scaled = Layout(45, 80, 256, 2, 48, heads=24, d=128)
        per_s, rows_s, t_s, _ = OracleStepper(scaled, config_id=5, t_steady=60).step(small)
        out["scaled"] = {"value": round(1.0 / per_s, 6), "unit": UNIT, "cores": _oracle_threads(),
                         "sample": f"{rows_s} query rows x 24 heads x {scaled.end(60)} keys of one "
                                   f"scaled block ({t_s:.1f} s), plus one eviction and one record "
                                   f"write, extrapolated to 28 blocks x {scaled.R} rows"}
    except Exception as e:
        out["scaled"] = {"error": f"{type(e).__name__}: {e}"}
    return out


def cpu_baseline(budget_s: float):
    """The CPU baseline without the GPU parity check."""
    return cpu_baseline_and_parity(budget_s)


def run_reference(args, world, rank):
    if rank != 0:
        return
    # size each step so the whole run stays within ~2 minutes
    n_steps = args.warmup + args.steps
    budget = max(0.05, min(2.0, 120.0 / max(1, n_steps)))
    stepper = OracleStepper(kv_format=args.kv_format)
    for _ in range(args.warmup):
        stepper.step(budget)
    per = []
    rows_total, spent_total = 0, 0.0
    for _ in range(args.steps):
        s, rows, _, spent = stepper.step(budget)
        per.append(s)
        rows_total += rows
        spent_total += spent
    total = sum(per)
    value = args.steps / total
    cores = _oracle_threads()
    line = {"metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": config_dict(world, args.kv_format),
            "extrapolated": True,
            "seconds_spent": round(spent_total, 2),
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
                             "cpu_model": _cpu_model(),
                             "sample": f"per step about {budget:.2f} s of query rows of one block "
                                       f"({rows_total} rows in all) plus one eviction and one record "
                                       f"write, extrapolated to a full 28-block frame-step; "
                                       f"ms_per_step is that extrapolation, the timed steps took "
                                       f"{spent_total:.1f} s of host time"},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_dense_case(spec: str, calls: int):
    """``LQ,LK,HEADS,D``: ``calls`` back-to-back dense attention calls of that
    shape on synthetic N(0,1) bf16 inputs, timed with CUDA events (a small,
    fixed case for kernel captures: one launch per call).  Prints one line."""
    import torch
    import kv_memory_attention_b200 as wm
    lq, lk, heads, d = (int(x) for x in spec.split(","))
    g = torch.Generator(device="cuda").manual_seed(11)
    q, k, v = (torch.randn(n, heads, d, device="cuda", dtype=torch.bfloat16, generator=g)
               for n in (lq, lk, lk))
    o = torch.empty(lq, heads, d, device="cuda", dtype=torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(3):
        wm.wm_attend_dense(q, k, v, o, lq, lk, heads, d, status)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(calls):
        wm.wm_attend_dense(q, k, v, o, lq, lk, heads, d, status)
    e1.record()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "a bounded wait ran out"
    us = e0.elapsed_time(e1) * 1e3 / calls
    flop = 4.0 * lq * lk * heads * d
    print(json.dumps({"dense": {"lq": lq, "lk": lk, "heads": heads, "d": d, "calls": calls,
                                "us_per_call": round(us, 2), "tflops": round(flop / us / 1e6, 1)}}),
          flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kv-format", choices=["bf16", "e4m3"], default="bf16",
                    help="storage of the frame memory: bf16 (the default workload) or FP8 E4M3 codes "
                         "with one scale per (block, head); e4m3 runs no extras")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the long runs and the secondary measurements (CUDA graphs, four-pass "
                         "frame, copy kernels' HBM throughput, batch of 8, scaled memory vs dense)")
    ap.add_argument("--ncu-csv", help="summarise this ncu --csv capture and exit (no GPU)")
    ap.add_argument("--ncu-out", help="JSON file the summary is written to")
    ap.add_argument("--ncu-cmd", default="", help="the ncu command line, recorded in the summary")
    ap.add_argument("--dense", metavar="LQ,LK,HEADS,D",
                    help="time only dense attention calls of this shape (a fixed case for kernel "
                         "captures; --steps calls) and exit")
    args = ap.parse_args()
    if args.dense:
        run_dense_case(args.dense, args.steps)
        return
    if args.ncu_csv:
        summary = summarize_ncu_csv(args.ncu_csv, args.ncu_cmd)
        with open(args.ncu_out, "w") as f:
            json.dump(summary, f, indent=1)
            f.write("\n")
        return
    args.warmup = max(3, args.warmup)      # at least 3 untimed warm-up steps
    world, rank, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
