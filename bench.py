#!/usr/bin/env python
"""Benchmark of the selective-scan hot path on B200.

One step = one prompt scan of the Mamba-2.8B-layer-shaped long workload
(batch 1, channels 5120, state_dim 16, seq 16384, bf16 storage, z gate, fp32 state)
followed by one decode update of the 2.8B-shaped decode workload (batch 256,
channels 5120, state_dim 16, fp32 state in place).  The metric is scan elements
(batch * seq * channels * state_dim) per second over both calls.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torch.distributed.run) every rank runs the same per-GPU
workload on its own problems (weak scaling, no data-path collective); the time is
the maximum over ranks of the device-timed region.  Rank 0 prints one JSON line.

    python bench.py --seq-shard [--emulate-ranks R] ...

times the prompt scan alone with its one sequence cut into a segment per rank
(strong scaling; one NCCL all-gather of segment composites per step).

    python bench.py --form {scan-130m,scan-packed,states,conv,conv-decode,gated,
                            segment-decay,two-level,single-pass-small} [--steps K]

times one kernel form on its own workload (one GPU) and prints its own JSON line.
"""
from __future__ import annotations

import argparse
import gc
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from selective_state_space_18_b200.inputs import WORKLOADS, make_workload  # noqa: E402

METRIC = "scan elems/s (B·L·D·N) and HBM GB/s vs roofline, 2.8B-shape prompt + decode"
PROMPT = WORKLOADS["mamba2p8b_layer_long"]
DECODE = WORKLOADS["decode_2p8b"]
SM_COUNT_NOMINAL = 148
MUFU_PER_CLK_PER_SM = 16           # ex2 results per clock per SM (sm_100)
FALLBACK_HBM_GBS = 6650.0
CSRC = os.path.join(ROOT, "selective_state_space_18_b200", "csrc")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")


# ---------------------------------------------------------------------------------------
# work accounting (algorithmic, per launch)
# ---------------------------------------------------------------------------------------

def prompt_work(w=PROMPT):
    """Algorithmic bytes and exponentials of one prompt-scan launch.

    Bytes: x, dt_raw, z read and y written once ([b,c,L] each, storage dtype);
    B, C read once per batch row; A, D, dt_bias read once; h_last written once.
    Exponentials: N decays per (b,t,c), plus one for softplus and one for silu."""
    es = 2 if w.dtype == "bf16" else 4
    rows = w.batch * w.channels
    bytes_ = (4 if w.z else 3) * rows * w.seq * es + 2 * w.batch * w.state_dim * w.seq * es
    bytes_ += w.channels * w.state_dim * 4 + 2 * w.channels * 4 + rows * w.state_dim * 4
    exps = rows * w.seq * (w.state_dim + 1 + (1 if w.z else 0))
    return {"elems": w.elems, "bytes": bytes_, "exps": exps}


def decode_work(w=DECODE):
    """One decode launch: the fp32 state read and written once, x/dt/z read and y
    written once ([b,c]), B/C once per batch row, A/D/dt_bias once."""
    es = 2 if w.dtype == "bf16" else 4
    rows = w.batch * w.channels
    bytes_ = 2 * rows * w.state_dim * 4 + (4 if w.z else 3) * rows * es
    bytes_ += 2 * w.batch * w.state_dim * es + w.channels * w.state_dim * 4 + 2 * w.channels * 4
    exps = rows * (w.state_dim + 1 + (1 if w.z else 0))
    return {"elems": w.batch * w.channels * w.state_dim, "bytes": bytes_, "exps": exps}


# the sources each kernel's device code is compiled from
KERNEL_SOURCES = {
    "ss_scan_fwd_kernel": ("ss_scan_fwd.cuh", "ss_device.cuh", "ss_sync.cuh"),
    "ss_state_update_stream_kernel": ("ss_state_update.cuh", "ss_device.cuh", "ss_sync.cuh"),
    "ss_gated_tc_kernel": ("ss_gated_tc.cuh", "ss_device.cuh", "ss_sync.cuh"),
}


def _kernel_source_hash(kernel):
    """Hash of the sources of `kernel`'s device code (its own header and the shared
    device headers)."""
    h = hashlib.sha256()
    for name in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def _measured_traffic(kernel, launch=None):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current device code of that kernel and, where the entry records one, with the same
    launch plan (else None)."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    entry = rec.get(kernel)
    if not entry or entry.get("source_hash") != _kernel_source_hash(kernel):
        return None
    if "launch" in entry and launch is not None and entry["launch"] != launch:
        return None
    return entry.get("dram_bytes_per_launch")


def _measured_peak(key):
    """A figure of MEASURED_PEAKS.json as a positive float: the value itself, or the
    "value" of an object.  None when the file, the key or a usable number is missing."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            v = json.load(f)[key]
        if isinstance(v, dict):
            v = v["value"]
        v = float(v)
        return v if v > 0 and math.isfinite(v) else None
    except (OSError, ValueError, KeyError, TypeError):
        return None


def _tensor_peak_tflops():
    """Dense bf16 tensor throughput (TFLOP/s): the measured burst figure when present,
    else the pool's earlier measurement."""
    v = _measured_peak("bf16_tflops")
    return 1590.0 if v is None else v


def _peaks():
    """(HBM GB/s, SM max MHz, basis): the measured copy bandwidth when present, else the
    pool's earlier measurement."""
    hbm = _measured_peak("hbm_gbs")
    if hbm is None:
        return FALLBACK_HBM_GBS, 1965.0, "fallback"
    mhz = _measured_peak("sm_max_mhz")
    return hbm, 1965.0 if mhz is None else mhz, "measured"


# ---------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------

class ClockSampler:
    """SM clock and clock-event reasons of one GPU, sampled every `period` seconds by a
    background thread over NVML (nvidia-smi polling if NVML is unavailable), each
    sample stamped with time.perf_counter().  summary(t0, t1) keeps only the samples
    taken inside [t0, t1], so the record describes the timed region itself."""

    NAMES = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
             ("sw_power_cap", 0x4), ("hw_power_brake", 0x80))

    def __init__(self, device_index, period=0.002):
        import threading
        self.period = period
        self.samples = []          # (t, sm_mhz, reasons bitmask)
        self.max_mhz = None
        self.source = None
        self._stop = threading.Event()
        self._thread = None
        self._handle = None
        self._smi = None
        try:
            self.uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            self.uuid = str(device_index)
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._handle = pynvml.nvmlDeviceGetHandleByUUID(self.uuid.encode())
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self._handle, pynvml.NVML_CLOCK_SM))
            self.source = "nvml"
        except Exception:
            self._handle = None
            self.source = "nvidia-smi"

    def _poll_nvml(self):
        nv, h = self._nvml, self._handle
        getr = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                rs = int(getr(h))
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def _poll_smi(self):
        fields = "clocks.sm,clocks.max.sm,clocks_event_reasons.active"
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", "-i", self.uuid, f"--query-gpu={fields}",
                                      "--format=csv,noheader,nounits"], capture_output=True, text=True,
                                     timeout=5).stdout.strip().split(",")
                t = time.perf_counter()
                self.max_mhz = float(out[1])
                self.samples.append((t, float(out[0]), int(out[2].strip(), 16)))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        import threading
        target = self._poll_nvml if self._handle is not None else self._poll_smi
        self._thread = threading.Thread(target=target, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=10)

    def summary(self, t0, t1):
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside:  # a region shorter than the sampling period: the nearest sample
            near = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:1]
            inside = near
        if not inside:
            return None
        mhz = [s[1] for s in inside]
        mask = 0
        for s in inside:
            mask |= s[2]
        return {"sm_mhz": statistics.median(mhz), "sm_min_mhz": min(mhz), "sm_max_mhz": self.max_mhz,
                "reasons": [n for n, bit in self.NAMES if mask & bit], "samples": len(inside),
                "source": self.source, "window": "timed region only"}


def wait_event(ev):
    """Wait for a recorded CUDA event without holding the GIL (so the clock sampler
    thread keeps sampling), then synchronise on it."""
    while not ev.query():
        time.sleep(0.0002)
    ev.synchronize()


# ---------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------

def _dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Maximum of a per-rank number over all ranks (identity on one rank)."""
    if world <= 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int, device=None) -> float:
    if world <= 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _inputs_on(dev, seed_offset):
    p = make_workload(PROMPT, seed=PROMPT.seed + 1000 * seed_offset)
    u = make_workload(DECODE, seed=DECODE.seed + 1000 * seed_offset)
    return p, u


def run_ours(args):
    from selective_state_space_18_b200 import ssscan

    world, rank, local = _dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    ssscan.load_library()

    # two rotating input sets per workload: every timed step reads data not in L2
    # (the host copies are dropped here: freeing 0.7 GB of host tensors later, when a
    # name that still held them is rebound inside the timed loop, stalls the host for
    # about 12 ms, long enough for the GPU to drain its queue)
    sets = [tuple({k: (None if v is None else v.to(dev)) for k, v in d.items()} for d in _inputs_on(dev, rank * 2 + s))
            for s in range(args.sets)]
    gc.collect()
    p0, u0 = sets[0]
    y_scan = [torch.empty_like(p0["x"]) for _ in range(2)]
    h_last = [torch.empty(PROMPT.batch, PROMPT.channels, PROMPT.state_dim, device=dev) for _ in range(2)]
    y_dec = [torch.empty(DECODE.batch, DECODE.channels, device=dev, dtype=u0["x"].dtype) for _ in range(2)]
    stream = torch.cuda.current_stream(dev)

    nsets = len(sets)

    def step(i):
        p, u = sets[i % nsets]
        ssscan.ss_scan_fwd(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["z"], p["dt_bias"],
                           None, None, y=y_scan[i & 1], h_last=h_last[i & 1], stream=stream)
        ssscan.ss_state_update(u["state"], u["x"], u["dt"], u["A"], u["B"], u["C"], u["D"], u["z"],
                               u["dt_bias"], y=y_dec[i & 1], stream=stream)

    sampler = ClockSampler(local)
    sampler.start()
    # W declared warm-up steps, then a time-based pre-roll of the same steps until
    # prewarm_s seconds have passed, so the timed steps run at the steady-state SM
    # clock (a GPU that was idle starts at a low clock and ramps up under load).  The
    # host stays at most 8 steps ahead of the GPU, and no idle gap separates the
    # pre-roll from the timed region.
    done = []
    i = 0
    gc.collect()
    gc.disable()  # no collector pauses from here to the end of the timed region
    t_pre = time.perf_counter()
    while i < args.warmup or time.perf_counter() - t_pre < args.prewarm_s:
        if len(done) >= 8:
            done.pop(0).synchronize()
        step(i)
        e = torch.cuda.Event()
        e.record(stream)
        done.append(e)
        i += 1
    torch.cuda.synchronize(dev)
    prewarm_steps = i - args.warmup
    prewarm_s = time.perf_counter() - t_pre
    step_s = prewarm_s / max(1, i)  # (an upper bound on the GPU's time per step)

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    _barrier(world)
    torch.cuda.synchronize(dev)
    # The host must never let the GPU's queue run dry inside a timed interval (a host
    # stall between a step's first event and its launch would be timed as GPU work), and
    # the GPU must not idle or run light right before it: untimed steps worth about
    # 10 ms of GPU work go first, so the GPU is busy with the step's own work while the
    # host enqueues the timed steps (garbage collection stays off throughout).
    head = max(3, min(64, int(10e-3 / max(step_s, 1e-5)) + 1))
    for h in range(head):
        step(i + h)
    t0 = time.perf_counter()
    start.record(stream)
    for i in range(K):
        e0, e1, e2 = ev[i]
        e0.record(stream)
        p, u = sets[i % nsets]
        ssscan.ss_scan_fwd(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["z"], p["dt_bias"],
                           None, None, y=y_scan[i & 1], h_last=h_last[i & 1], stream=stream)
        e1.record(stream)
        ssscan.ss_state_update(u["state"], u["x"], u["dt"], u["A"], u["B"], u["C"], u["D"], u["z"],
                               u["dt_bias"], y=y_dec[i & 1], stream=stream)
        e2.record(stream)
    end.record(stream)
    t_enq = time.perf_counter()
    wait_event(end)
    torch.cuda.synchronize(dev)
    t1 = time.perf_counter()
    gc.enable()
    _barrier(world)
    sampler.stop()
    clocks = sampler.summary(t0, t1)

    total_ms = start.elapsed_time(end)
    scan_list = [e[0].elapsed_time(e[1]) for e in ev]
    dec_list = [e[1].elapsed_time(e[2]) for e in ev]
    scan_ms = sum(scan_list) / K
    dec_ms = sum(dec_list) / K
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / K

    pw, dw = prompt_work(), decode_work()
    elems_step = pw["elems"] + dw["elems"]
    value = world * elems_step * K / (total_ms * 1e-3)

    dec_b2b_ms = decode_back_to_back(sets, y_dec, stream, ssscan)

    # end to end: pinned host inputs -> device -> scan + decode -> results back to host
    if args.no_e2e:
        e2e = {"ms_per_step": float("nan"), "h2d": 0, "d2h": 0, "steps": 0}
    else:
        e2e = run_e2e(args, dev, stream, sets[0], ssscan)
    e2e_ms = max_over_ranks(e2e["ms_per_step"], world, dev)

    plan = ssscan.ss_scan_plan(PROMPT.batch, PROMPT.channels, PROMPT.state_dim, PROMPT.seq,
                               torch.bfloat16, has_reset=False, workspace=True, device=dev)
    hbm_gbs, sm_max_mhz, peak_kind = _peaks()
    # the special-function unit's rate, measured on this GPU after the timed region
    # (results per SM clock; the peak takes it at the maximum SM clock)
    ex2_rate, ex2_rates = ssscan.mufu_rate("ex2", device=dev)
    tanh_rate, _ = ssscan.mufu_rate("tanh", device=dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    sfu_peak = sms * ex2_rate * sm_max_mhz * 1e6  # ex2/s
    scan_s = scan_ms * 1e-3
    dec_s = dec_ms * 1e-3
    scan_exps_rate = pw["exps"] / scan_s
    scan_hbm = pw["bytes"] / scan_s / 1e9
    t_roof_scan = max(pw["bytes"] / (hbm_gbs * 1e9), pw["exps"] / sfu_peak)
    t_roof_dec = max(dw["bytes"] / (hbm_gbs * 1e9), dw["exps"] / sfu_peak)
    sm_clk = (clocks or {}).get("sm_mhz")
    roofline = {
        "kernel": "ss_scan_fwd_kernel (prompt scan)",
        "bound": "alu",
        "alu_unit": "MUFU ex2 (SFU)",
        "achieved": round(scan_exps_rate / 1e9, 2),
        "peak": round(sfu_peak / 1e9, 2),
        "unit": "Gexp/s",
        "frac": round(scan_exps_rate / sfu_peak, 4),
        "peak_basis": (f"{sms} SMs x {ex2_rate:.2f} ex2/clk/SM (measured: ss_debug_mufu_probe, median over SMs) "
                       f"x {sm_max_mhz:.0f} MHz (max SM clock)"),
        "sfu_probe": {"ex2_per_clk_per_sm": round(ex2_rate, 3), "ex2_min": round(ex2_rates[0], 3),
                      "ex2_max": round(ex2_rates[-1], 3), "tanh_per_clk_per_sm": round(tanh_rate, 3),
                      "nominal": MUFU_PER_CLK_PER_SM},
        "frac_at_measured_clock": (round(scan_exps_rate / (sms * ex2_rate * sm_clk * 1e6), 4)
                                   if sm_clk else None),
        "exps_per_launch": pw["exps"],
        # every MUFU op the kernel issues, per (b, t, c) of this bf16 workload: the N decays,
        # the softplus's exponential (its log1p is a polynomial on the FMA pipe) and the
        # gate's tanh (sigmoid(z) = (1 + tanh(z/2)) / 2): no MUFU log or reciprocal
        "mufu_ops_per_launch": pw["exps"] if PROMPT.dtype == "bf16" else None,
        "algorithmic_bytes_per_launch": pw["bytes"],
        "hbm_achieved_gbs": round(scan_hbm, 1),
        "hbm_peak_gbs": hbm_gbs,
        "hbm_frac": round(scan_hbm / hbm_gbs, 4),
        "roofline_frac": round(t_roof_scan / scan_s, 4),
        "traffic": _measured_traffic("ss_scan_fwd_kernel", {k: plan[k] for k in ("grid", "segments", "seg_len")}),
        "peak_source": (f"HBM {'measured (MEASURED_PEAKS.json)' if peak_kind == 'measured' else 'fallback'} "
                        f"{hbm_gbs:.0f} GB/s; SFU measured per clock, at the max clock"),
    }
    kernels = {
        "scan": {"ms": round(scan_ms, 5), "ms_min": round(min(scan_list), 5),
                 "ms_median": round(statistics.median(scan_list), 5), "ms_max": round(max(scan_list), 5),
                 "max_step": scan_list.index(max(scan_list)),
                 "kcycles_at_median_clock": (round(scan_ms * sm_clk, 1) if sm_clk else None),
                 "elems_per_s": pw["elems"] / scan_s,
                 "hbm_gbs": round(scan_hbm, 1), "roofline_frac": round(t_roof_scan / scan_s, 4),
                 "t_roof_ms": round(t_roof_scan * 1e3, 5), "launch": plan},
        "decode": {"kernel": "ss_state_update_stream_kernel (decode update)",
                   "ms": round(dec_ms, 5), "ms_min": round(min(dec_list), 5),
                   "ms_median": round(statistics.median(dec_list), 5), "ms_max": round(max(dec_list), 5),
                   "elems_per_s": dw["elems"] / dec_s,
                   "hbm_gbs": round(dw["bytes"] / dec_s / 1e9, 1),
                   "hbm_frac": round(dw["bytes"] / dec_s / 1e9 / hbm_gbs, 4),
                   "roofline_frac": round(t_roof_dec / dec_s, 4),
                   "t_roof_ms": round(t_roof_dec * 1e3, 5),
                   "traffic": _measured_traffic("ss_state_update_stream_kernel"),
                   "back_to_back": {
                       "ms": round(dec_b2b_ms, 5),
                       "hbm_frac": round(dw["bytes"] / (dec_b2b_ms * 1e-3) / 1e9 / hbm_gbs, 4),
                       "what": "decode calls one after another, outside the step: each pays the write-back "
                               "of the state the previous call left dirty in L2, which within the step "
                               "drains during the next prompt scan"}},
    }

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.cpu_seconds)

    line = {
        "metric": METRIC,
        "value": value,
        "unit": "elems/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": "mamba2p8b_layer_long prompt scan (batch 1, channels 5120, state_dim 16, "
                        "seq 16384, bf16 x/dt/z/B/C/y, z gate, dt_bias, fp32 state) + decode_2p8b "
                        "update (batch 256, channels 5120, state_dim 16, bf16 I/O, fp32 state in place)",
            "storage": "bf16 x/dt/z/B/C/y; fp32 A, D, dt_bias, state and all arithmetic",
            "elems_per_step": elems_step,
            "l2": "inputs larger than L2 (scan 673 MB + decode 179 MB per step), two rotating input sets",
            "parallelism": f"replicas x{world} (independent problems per rank, no collective)",
        },
        "roofline": roofline,
        "kernels": kernels,
        "cpu_baseline": cpu,
        "e2e": {"value": world * elems_step / (e2e_ms * 1e-3), "unit": "elems/s",
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "steps": e2e["steps"]},
        "clocks": clocks,
        "prewarm_s": round(prewarm_s, 3),
        "head_start_steps": head,
        "host_enqueue_ms": round((t_enq - t0) * 1e3, 2),
        "prewarm_steps": prewarm_steps,
        "gpu_launches": 2 * K,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def decode_back_to_back(sets, y_dec, stream, ssscan, n=200):
    """Per-call time (ms) of decode updates run one after another with no other kernel
    between them: an untimed head start of the same calls, then a burst of n calls timed
    by one pair of events (no event between calls)."""
    def call(i):
        u = sets[i % len(sets)][1]
        ssscan.ss_state_update(u["state"], u["x"], u["dt"], u["A"], u["B"], u["C"], u["D"], u["z"],
                               u["dt_bias"], y=y_dec[i & 1], stream=stream)
    for i in range(32):
        call(i)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n):
        call(i)
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / n


def run_e2e(args, dev, stream, inputs, ssscan):
    """Same step through the public API with the per-step inputs in pinned host memory:
    H2D copies of x, dt_raw, z, B, C (both calls), the two kernels, and D2H of y,
    h_last and the decode output, all inside the timed region.  A, D, dt_bias and the
    decode state (the cache) stay resident on the device.

    The steps are pipelined the way a serving loop would run them: step i's inputs go up
    on a copy stream while step i-1's kernels run on `stream` and step i-2's results come
    down on a third stream (PCIe is full duplex, and the copy engines are not the SMs).
    Device input and output buffers are double-buffered; events order each buffer's
    reuse, so no copy overwrites data a kernel still reads and no kernel overwrites a
    result before it has reached the host.  The timed region runs from the first H2D
    copy of the first timed step to the last D2H copy of the last one."""
    p, u = inputs
    per_step = {"p": ("x", "dt", "z", "B", "C"), "u": ("x", "dt", "z", "B", "C")}
    host = {("p", k): p[k].cpu().pin_memory() for k in per_step["p"]}
    host.update({("u", k): u[k].cpu().pin_memory() for k in per_step["u"]})
    devb = [{key: torch.empty_like(t, device=dev) for key, t in host.items()} for _ in range(2)]
    y = [torch.empty_like(p["x"]) for _ in range(2)]
    hl = [torch.empty(PROMPT.batch, PROMPT.channels, PROMPT.state_dim, device=dev) for _ in range(2)]
    yd = [torch.empty(DECODE.batch, DECODE.channels, device=dev, dtype=u["x"].dtype) for _ in range(2)]
    out_host = [[torch.empty_like(t, device="cpu").pin_memory() for t in (y[b], hl[b], yd[b])] for b in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in out_host[0])
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: [torch.cuda.Event() for _ in range(2)]  # noqa: E731
    uploaded, computed, downloaded = ev(), ev(), ev()
    used = [False, False]

    def one(i):
        b = i & 1
        with torch.cuda.stream(up):
            if used[b]:
                up.wait_event(computed[b])          # step i-2's kernels are done with devb[b]
            for key, t in host.items():
                devb[b][key].copy_(t, non_blocking=True)
            uploaded[b].record(up)
        stream.wait_event(uploaded[b])
        if used[b]:
            stream.wait_event(downloaded[b])        # step i-2's results have left y[b] ...
        d = devb[b]
        ssscan.ss_scan_fwd(d[("p", "x")], d[("p", "dt")], p["A"], d[("p", "B")], d[("p", "C")],
                           p["D"], d[("p", "z")], p["dt_bias"], None, None, y=y[b], h_last=hl[b], stream=stream)
        ssscan.ss_state_update(u["state"], d[("u", "x")], d[("u", "dt")], u["A"], d[("u", "B")],
                               d[("u", "C")], u["D"], d[("u", "z")], u["dt_bias"], y=yd[b], stream=stream)
        computed[b].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(computed[b])
            for h, t in zip(out_host[b], (y[b], hl[b], yd[b])):
                h.copy_(t, non_blocking=True)
            downloaded[b].record(down)
        used[b] = True

    for i in range(2):
        one(i)
    torch.cuda.synchronize(dev)
    steps = max(3, min(args.steps, args.e2e_steps))
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(up)
    for i in range(steps):
        one(i)
    e.record(down)
    torch.cuda.synchronize(dev)
    return {"ms_per_step": s.elapsed_time(e) / steps, "h2d": h2d, "d2h": d2h, "steps": steps}


# ---------------------------------------------------------------------------------------
# CPU oracle legs (cpu_baseline and --impl reference)
# ---------------------------------------------------------------------------------------

class OracleSampler:
    """The float64 oracle, as it stands, timed on bounded samples of both calls of
    the step: the first R channels of the prompt workload (all tokens) and the first
    U batch rows of the decode workload, with R and U sized to a time budget.  The
    per-element times are scaled to one full step."""

    def __init__(self):
        from oracle import oracle
        self.oracle = oracle
        self.p = make_workload(PROMPT)
        self.u = make_workload(DECODE)
        self.cores = oracle.num_threads()
        self.s_row = None
        self.s_dec_row = None

    def _prompt(self, R):
        p = self.p
        sub = {k: p[k][:, :R] for k in ("x", "dt", "z")}
        sub.update({k: p[k][:R] for k in ("A", "D", "dt_bias")})
        sub.update({"B": p["B"], "C": p["C"]})
        t = time.perf_counter()
        self.oracle.scan(**sub)
        return time.perf_counter() - t

    def _decode(self, U):
        u = self.u
        sub = {k: u[k][:U] for k in ("state", "x", "dt", "z", "B", "C")}
        sub.update({k: u[k] for k in ("A", "D", "dt_bias")})
        t = time.perf_counter()
        self.oracle.update(**sub)
        return time.perf_counter() - t

    def sample(self, budget_s):
        """One timed sample of about budget_s seconds.  Returns (seconds per full
        step, sample description, seconds spent)."""
        if self.s_row is None:  # calibration
            r0 = min(PROMPT.channels, max(self.cores, 8))
            self.s_row = self._prompt(r0) / r0
            self.s_dec_row = self._decode(1)
        R = int(max(1, min(PROMPT.channels, 0.85 * budget_s / max(self.s_row, 1e-9))))
        U = int(max(1, min(DECODE.batch, 0.15 * budget_s / max(self.s_dec_row, 1e-9))))
        tp, td = self._prompt(R), self._decode(U)
        pw, dw = prompt_work(), decode_work()
        t_step = tp / (R * PROMPT.seq * PROMPT.state_dim) * pw["elems"] + \
            td / (U * DECODE.channels * DECODE.state_dim) * dw["elems"]
        desc = (f"float64 oracle (C, OpenMP over rows) on channels 0..{R - 1} of the prompt "
                f"workload (all {PROMPT.seq} tokens) and batch rows 0..{U - 1} of the decode "
                f"workload, per-element times scaled to one full step")
        return t_step, desc, tp + td


def cpu_baseline(target_s):
    smp = OracleSampler()
    t_step, desc, spent = smp.sample(target_s)
    pw, dw = prompt_work(), decode_work()
    return {"value": (pw["elems"] + dw["elems"]) / t_step, "unit": "elems/s", "cores": smp.cores,
            "kind": "oracle", "sample": desc, "seconds": round(spent, 2)}


def run_reference(args):
    world, rank, _ = _dist_env()
    if rank != 0:
        return
    smp = OracleSampler()
    per = max(0.05, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    times, desc = [], None
    for i in range(args.warmup + args.steps):
        t_step, desc, _ = smp.sample(per)
        if i >= args.warmup:
            times.append(t_step)
    t = statistics.median(times)
    pw, dw = prompt_work(), decode_work()
    value = (pw["elems"] + dw["elems"]) / t
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "elems/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": t * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "same step as our arm (mamba2p8b_layer_long prompt scan + decode_2p8b "
                               "update); each step a bounded sample of it on the host cores",
                   "storage": "bf16 values widened exactly to float64"},
        "cpu_baseline": {"value": value, "unit": "elems/s", "cores": smp.cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "elems/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_seq_shard(args):
    """The 2.8B-layer prompt cut into sequence segments, one per rank (strong scaling):
    each rank scans its segment, the segments' composites are all-gathered (NCCL), and
    every rank but 0 rescans from its joined entering state.  With one process and
    --emulate-ranks R, the R segments run one after another on this GPU and each
    emulated rank's own work is timed separately (the all-gather is not emulated)."""
    from selective_state_space_18_b200 import seqshard, ssscan

    world, rank, local = _dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    ssscan.load_library()
    emulate = args.emulate_ranks if world == 1 else 1
    segs = max(world, emulate)
    full = make_workload(PROMPT, seed=PROMPT.seed)
    L = full["x"].shape[-1]
    bounds = seqshard.shard_bounds(L, segs)
    seq_keys = ("x", "dt", "z", "B", "C")

    def part(r):
        a, b = bounds[r]
        q = {k: (None if v is None else (v[..., a:b].contiguous() if k in seq_keys else v).to(dev))
             for k, v in full.items() if k not in ("reset", "h0")}
        q["dt_softplus"] = True
        return q

    mine = [part(r) for r in range(segs)] if emulate > 1 else [part(rank)]
    del full
    stream = torch.cuda.current_stream(dev)

    if emulate > 1:
        K = args.steps
        ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
                torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(segs)] for _ in range(K + args.warmup)]

        def step(i):
            ys, comps = [], []
            for r, q in enumerate(mine):
                ev[i][r][0].record(stream)
                y, comp = seqshard.local_pass(q, r)
                ev[i][r][1].record(stream)
                ys.append(y)
                comps.append(comp)
            gathered = torch.stack(comps)
            for r, q in enumerate(mine):
                ev[i][r][2].record(stream)
                seqshard.finish_pass(q, r, gathered, ys[r])
                ev[i][r][3].record(stream)

        for i in range(args.warmup):
            step(i)
        torch.cuda.synchronize(dev)
        sampler = ClockSampler(local)
        sampler.start()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        start.record(stream)
        for i in range(args.warmup, args.warmup + K):
            step(i)
        end.record(stream)
        wait_event(end)
        torch.cuda.synchronize(dev)
        t1 = time.perf_counter()
        sampler.stop()
        clocks = sampler.summary(t0, t1)
        serial_ms = start.elapsed_time(end) / K
        per_rank = []
        for r in range(segs):
            loc = sum(ev[i][r][0].elapsed_time(ev[i][r][1]) for i in range(args.warmup, args.warmup + K)) / K
            fin = sum(ev[i][r][2].elapsed_time(ev[i][r][3]) for i in range(args.warmup, args.warmup + K)) / K
            per_rank.append({"rank": r, "tokens": bounds[r][1] - bounds[r][0], "local_pass_ms": round(loc, 5),
                             "finish_pass_ms": round(fin, 5)})
        worst = max(p["local_pass_ms"] + p["finish_pass_ms"] for p in per_rank)
        ms = serial_ms
        launches = K * (1 + 4 * (segs - 1))
        extra = {"emulated": {"ranks": segs, "per_rank": per_rank, "max_rank_compute_ms": round(worst, 5),
                              "note": "all segments on one GPU in turn; the value is that serial time. "
                                      "max_rank_compute_ms is the slowest emulated rank's own kernels, "
                                      "without the all-gather of composites"}}
    else:
        q = mine[0]
        K = args.steps
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # 256 MB > L2
        for _ in range(args.warmup):
            seqshard.seq_sharded_scan(q["x"], q["dt"], q["A"], q["B"], q["C"], q["D"], q["z"], q["dt_bias"])
        torch.cuda.synchronize(dev)
        sampler = ClockSampler(local)
        sampler.start()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        _barrier(world)
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        for i in range(K):
            flush.zero_()                      # L2 flushed between steps, outside the timed events
            ev[i][0].record(stream)
            seqshard.seq_sharded_scan(q["x"], q["dt"], q["A"], q["B"], q["C"], q["D"], q["z"], q["dt_bias"])
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        t1 = time.perf_counter()
        _barrier(world)
        sampler.stop()
        clocks = sampler.summary(t0, t1)
        ms = max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in ev) / K, world, dev)
        launches = K * (1 if world == 1 else 4)
        extra = {}

    elems = PROMPT.batch * PROMPT.channels * PROMPT.state_dim * L
    line = {
        "metric": "scan elems/s (B·L·D·N), 2.8B-shape prompt cut into sequence segments",
        "value": elems / (ms * 1e-3),
        "unit": "elems/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "strong",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {
            "workload": "mamba2p8b_layer_long prompt scan (batch 1, channels 5120, state_dim 16, seq 16384, "
                        "bf16 x/dt/z/B/C/y, z gate, dt_bias, fp32 state), one sequence cut into segments",
            "segments": bounds,
            "parallelism": (f"sequence segments x{world}: NCCL all-gather of segment composites" if world > 1
                            else f"{segs} segments emulated on one GPU" if segs > 1 else "one segment"),
            "l2": ("all segments' inputs (673 MB) per step" if emulate > 1
                   else "256 MB buffer written between steps, outside the timed events"),
        },
        **extra,
        "clocks": clocks,
        "gpu_launches": launches,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------------------------------
# the next rows' kernels, one at a time (--form)
# ---------------------------------------------------------------------------------------

FORMS = ("scan-130m", "scan-packed", "states", "betas", "conv", "conv-decode", "gated", "gated-recurrent",
         "segment-decay", "two-level", "single-pass-small")


def run_form(args):
    """Time one kernel form on its workload with the protocol of the headline step
    (pre-roll, GPU-side head start, clocks sampled inside the timed region) and print one
    JSON line with its own roofline.  The time per call ("ms") comes from one pair of
    CUDA events around a burst of K calls; a pass with events around every call gives
    the spread ("per_call_events_ms")."""
    from selective_state_space_18_b200 import ssscan
    from selective_state_space_18_b200.inputs import make_gated_inputs, make_scan_inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    ssscan.load_library()
    form = args.form
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    hbm_gbs, sm_max_mhz, peak_kind = _peaks()
    bf16 = torch.bfloat16
    nsets = 2
    g = torch.Generator().manual_seed(4242)

    def to_dev(d):
        return {k: (None if v is None else v.to(dev)) for k, v in d.items()}

    if form in ("scan-130m", "scan-packed", "states", "betas", "conv", "two-level", "single-pass-small"):
        wname = {"scan-130m": "mamba130m_layer", "scan-packed": "packed_resets"}.get(form, "mamba2p8b_layer_long")
        w = WORKLOADS[wname]
        if form in ("two-level", "single-pass-small"):
            shape = (1, 1024, 16, 65536)
            mk = lambda sd: make_scan_inputs(*shape, "bf16", seed=sd, a_perturb=True)
            desc = "batch 1, channels 1024, state_dim 16, seq 65536, bf16, z gate, dt_bias"
        else:
            shape = (w.batch, w.channels, w.state_dim, w.seq)
            mk = lambda sd: make_workload(w, seed=sd)
            desc = f"{wname}: batch {w.batch}, channels {w.channels}, state_dim {w.state_dim}, seq {w.seq}, bf16"
        if form == "states":
            nsets = 1  # 5.4 GB of states per call: one set already far exceeds L2
        sets = [to_dev(mk(w.seed + 1000 * i)) for i in range(nsets)]
        bt, ch, n, L = shape
        rows, elems = bt * ch, bt * ch * n * L
        keys = ("x", "dt", "A", "B", "C", "D", "z", "dt_bias", "reset", "h0")
        y = torch.empty(bt, ch, L, device=dev, dtype=bf16)
        hl = torch.empty(bt, ch, n, device=dev)
        if form == "states":
            hall = torch.empty(bt, ch, L, n, device=dev)
        if form == "betas":
            betas = torch.empty(bt, ch, L, device=dev)
        if form == "conv":
            cw = (torch.randn(ch, 4, generator=g) * 0.5).to(dev)
            cb = (torch.randn(ch, generator=g) * 0.1).to(dev)
        if form == "single-pass-small":
            ssscan.ss_debug_set_scan_two_level(1)

        def call(i):
            d = sets[i % nsets]
            a = [d[k] for k in keys]
            if form == "states":
                ssscan.ss_scan_fwd(*a, y=y, h_last=hl, h_all=hall)
            elif form == "betas":
                ssscan.ss_scan_fwd(*a, y=y, h_last=hl, betas=betas)
            elif form == "conv":
                ssscan.ss_scan_fwd_conv(d["x"], cw, d["dt"], d["A"], d["B"], d["C"], d["D"], d["z"], d["dt_bias"],
                                        conv_b=cb, return_conv_state=False)
            else:
                ssscan.ss_scan_fwd(*a, y=y, h_last=hl)
        # N decays, the softplus and the gate per (b, t, c); the fused conv form adds its SiLU
        exps = rows * L * (n + 3 if form == "conv" else n + 2)
        byts = 4 * rows * L * 2 + 2 * bt * n * L * 2 + rows * n * 4
        if form == "states":
            byts += rows * L * n * 4
        if form == "betas":
            byts += rows * L * 4
        kernel = {"states": "ss_scan_fwd_kernel (states form)", "conv": "ss_scan_fwd_kernel (fused conv form)",
                  "betas": "ss_scan_fwd_kernel (emitting form, step sizes only)",
                  "two-level": "ss_scan_fwd_kernel x2 + ss_segment_decay_kernel + ss_join_all_kernel (two-level)",
                  "single-pass-small": "ss_scan_fwd_kernel (single pass, chained segments)"}.get(form, "ss_scan_fwd_kernel")
        bound = "hbm" if form == "states" else "alu"
        metric_elems = elems
    elif form == "conv-decode":
        w = DECODE
        sets = [to_dev(make_workload(w, seed=w.seed + 1000 * i)) for i in range(nsets)]
        cw = (torch.randn(w.channels, 4, generator=g) * 0.5).to(dev)
        cs = [torch.randn(w.batch, w.channels, 3, generator=g).to(dev) for _ in range(nsets)]
        y = torch.empty(w.batch, w.channels, device=dev, dtype=bf16)

        def call(i):
            u = sets[i % nsets]
            ssscan.ss_state_update_conv(u["state"], cs[i % nsets], cw, u["x"], u["dt"], u["A"], u["B"], u["C"],
                                        u["D"], u["z"], u["dt_bias"])
        rows = w.batch * w.channels
        byts = decode_work()["bytes"] + 2 * rows * 3 * 4 + w.channels * 4 * 4
        exps, bound, kernel = rows * (w.state_dim + 3), "hbm", "ss_state_update_stream_kernel (fused conv form)"
        metric_elems = rows * w.state_dim
        desc = "decode_2p8b with the conv form (conv_k 4, fp32 conv state in place)"
    elif form in ("gated", "gated-recurrent"):
        B_, S_, dk, dv = 512, 2048, 128, 64
        sets = [to_dev(make_gated_inputs(B_, S_, dk, dv, "bf16", seed=77 + i)) for i in range(nsets)]
        if form == "gated-recurrent":
            ssscan.ss_debug_set_gated_path(1)

        def call(i):
            d = sets[i % nsets]
            ssscan.ss_gated_scan(d["q"], d["k"], d["v"], d["gamma"])
        metric_elems = B_ * S_ * dk * dv
        lane_ops = 3 * metric_elems
        byts = B_ * S_ * (2 * dk + 2 * dv) * 2 + B_ * S_ * 4 + B_ * dk * dv * 2
        if form == "gated":
            # the chunked form's matrix products per 128-token chunk: Q K^T, (L o S) V, Q H
            # and K^T (w o V)
            C_ = 128
            flops = 2 * B_ * (S_ // C_) * (C_ * C_ * dk + C_ * C_ * dv + C_ * dk * dv + dk * C_ * dv)
            exps, bound, kernel = 0, "tensor", "ss_gated_tc_kernel (chunked, tcgen05)"
        else:
            exps, bound, kernel = 0, "fp32-pipe", "ss_gated_scan_kernel (token by token)"
        desc = f"gated state scan: batch {B_}, seq {S_}, dk {dk}, dv {dv}, bf16"
    elif form == "segment-decay":
        w = PROMPT
        Ls = 1816  # one segment of the 2.8B-layer prompt cut into 8
        full = make_workload(w, seed=w.seed)
        sets = [{"dt": full["dt"][..., i * Ls:(i + 1) * Ls].contiguous().to(dev), "A": full["A"].to(dev),
                 "dt_bias": full["dt_bias"].to(dev)} for i in range(nsets)]
        out = torch.empty(w.batch, w.channels, w.state_dim, device=dev)

        def call(i):
            d = sets[i % nsets]
            ssscan.ss_segment_decay(d["dt"], d["A"], d["dt_bias"], out=out)
        rows = w.batch * w.channels
        byts = rows * Ls * 2 + rows * w.state_dim * 4 * 2 + w.channels * 4
        exps, bound, kernel = rows * Ls, "hbm", "ss_segment_decay_kernel"
        metric_elems = rows * Ls
        desc = "segment decay: batch 1, channels 5120, one 1816-token segment of the 2.8B-layer prompt, bf16"
    else:
        raise SystemExit(f"unknown form {form}")

    stream = torch.cuda.current_stream(dev)
    sampler = ClockSampler(0)
    sampler.start()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    gc.collect()
    gc.disable()
    t_pre, i = time.perf_counter(), 0
    while i < args.warmup or time.perf_counter() - t_pre < args.prewarm_s:
        call(i)
        i += 1
        if i % 8 == 0:
            torch.cuda.synchronize(dev)
    torch.cuda.synchronize(dev)
    call_s = (time.perf_counter() - t_pre) / max(1, i)
    for h in range(max(3, min(64, int(10e-3 / max(call_s, 1e-5)) + 1))):  # head start, untimed
        call(i + h)
    # Two timed passes over the same K calls, each behind its own head start: per-call
    # events (the spread), then one pair of events around the whole burst (the time per
    # call: an event between two short kernels adds an idle gap of a few microseconds).
    t0 = time.perf_counter()
    for k in range(K):
        ev[k][0].record(stream)
        call(k)
        ev[k][1].record(stream)
    wait_event(ev[-1][1])
    for h in range(max(3, min(64, int(10e-3 / max(call_s, 1e-5)) + 1))):
        call(K + h)
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b0.record(stream)
    for k in range(K):
        call(k)
    b1.record(stream)
    wait_event(b1)
    torch.cuda.synchronize(dev)
    t1 = time.perf_counter()
    gc.enable()
    sampler.stop()
    clocks = sampler.summary(t0, t1)
    ssscan.ss_debug_set_scan_two_level(0)
    ssscan.ss_debug_set_gated_path(0)
    ts = [a.elapsed_time(b) for a, b in ev]
    ms = b0.elapsed_time(b1) / K
    sec = ms * 1e-3
    ex2_rate, _ = ssscan.mufu_rate("ex2", device=dev)
    sfu_peak = sms * ex2_rate * sm_max_mhz * 1e6
    roof = {"bound": bound, "algorithmic_bytes_per_launch": byts, "hbm_achieved_gbs": round(byts / sec / 1e9, 1),
            "hbm_frac": round(byts / sec / 1e9 / hbm_gbs, 4), "hbm_peak_gbs": hbm_gbs}
    if bound == "alu":
        roof.update({"unit_peak": "MUFU ex2", "exps_per_launch": exps, "achieved_gexp_s": round(exps / sec / 1e9, 2),
                     "peak_gexp_s": round(sfu_peak / 1e9, 2), "frac": round(exps / sec / sfu_peak, 4)})
    elif bound == "hbm":
        roof["frac"] = roof["hbm_frac"]
    elif bound == "tensor":
        peak_tf = _tensor_peak_tflops()
        roof.update({"flops_per_launch": flops, "achieved_tflops": round(flops / sec / 1e12, 2),
                     "peak_tflops": peak_tf, "frac": round(flops / sec / 1e12 / peak_tf, 4),
                     "fp32_pipe_equivalent": round(lane_ops / sec / (sms * 128 * sm_max_mhz * 1e6), 4)})
    else:
        peak_ops = sms * 128 * sm_max_mhz * 1e6
        roof.update({"lane_ops_per_launch": lane_ops, "peak_lane_ops_s": peak_ops,
                     "frac": round(lane_ops / sec / peak_ops, 4)})
    line = {"form": form, "kernel": kernel, "workload": desc, "ms": round(ms, 5),
            "per_call_events_ms": {"mean": round(sum(ts) / K, 5), "median": round(statistics.median(ts), 5),
                                   "min": round(min(ts), 5), "max": round(max(ts), 5)},
            "elems_per_s": metric_elems / sec, "steps": K, "warmup": args.warmup, "sets": nsets,
            "roofline": roof, "clocks": clocks, "peaks": f"HBM {peak_kind}; SFU {ex2_rate:.2f} ex2/clk/SM measured"}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--prewarm-s", type=float, default=1.0,
                    help="seconds of untimed steps after the warm-up steps (clock ramp-up)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--sets", type=int, default=2, choices=[1, 2],
                    help="rotating input sets (1 for small profiler captures)")
    ap.add_argument("--seq-shard", action="store_true",
                    help="time the prompt scan with its sequence cut into one segment per rank (strong scaling)")
    ap.add_argument("--emulate-ranks", type=int, default=1,
                    help="with --seq-shard on one process: run this many segments on the one GPU")
    ap.add_argument("--form", choices=FORMS, default=None,
                    help="time one kernel form of the next rows on its own workload instead of the step")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.form:
        run_form(args)
    elif args.impl == "reference":
        run_reference(args)
    elif args.seq_shard:
        run_seq_shard(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
