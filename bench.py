#!/usr/bin/env python
"""Benchmark of libssq's quantized state update on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

A step is one pass of the decode hot path -- read the packed state, decode,
recurrence, refit, requantize, write back, readout -- over one batch of
synthetic input.  The default workload is the Mamba-2 130M-shaped decode
step: 24 layers x batch 256 in one launch, 24 heads x 64 x 128 per layer,
int8 asymmetric state, N(0, 1) initial state.  Other workloads (--workload)
are the 8B-shaped decode, the serving-scale format sweep and the 370M-shaped
per-token scan.

Timing: W untimed warm-up steps, then exactly K steps between a barrier and a
device synchronize, timed with CUDA events on the launching stream; the max
over ranks is taken; the kernel time of the roofline is the median launch.
A step whose footprint (state, inputs, output) is under 4x the L2 rotates
over enough copies of them that every step reads from HBM; the line says
which.  --gpus N starts N ranks (one per GPU, torch.distributed.run on
127.0.0.1) when no launcher did; they are independent replicas (weak
scaling, no collective on the data path).  --impl reference times the CPU
oracle on every host core of rank 0 on a bounded sample of the same
workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import glob
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_recurrent_state_mamba_b200 import workloads as W  # noqa: E402

METRIC = "quantized state-update HBM GB/s (% of B200 peak) and request-steps/s/layer"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
SM_MAX_MHZ = 1965.0        # B200 maximum SM clock, used when NVML is unavailable
SCAN_FP32_OPS = 6          # algorithmic fp32 operations per element-token of the scan
PREFILL_FP32_OPS = 3       # ... of the prefill hand-off: w = dtx*B, the fma, C*s
DAMP_PROTECTED = 16        # DAMP layout: key channels per head kept in FP16


# ---------------------------------------------------------------------------
# Workloads and their algorithmic bytes
# ---------------------------------------------------------------------------

def workload(name):
    table = {
        "tiny": lambda: W.tiny(),
        "decode_130m": lambda: W.decode_130m("i8a"),
        "decode_130m_f32": lambda: W.decode_130m("f32"),
        "decode_130m_sr": lambda: W.decode_130m("i8a"),
        "decode_8b_b1_i8a": lambda: W.decode_8b("i8a", 1),
        "decode_8b_b16_i8a": lambda: W.decode_8b("i8a", 16),
        "decode_8b_b64_i8a": lambda: W.decode_8b("i8a", 64),
        "decode_8b_b256_i8a": lambda: W.decode_8b("i8a", 256),
        "decode_8b_b1_i8s": lambda: W.decode_8b("i8s", 1),
        "decode_8b_b16_i8s": lambda: W.decode_8b("i8s", 16),
        "decode_8b_b64_i8s": lambda: W.decode_8b("i8s", 64),
        "decode_8b_b256_i8s": lambda: W.decode_8b("i8s", 256),
        "decode_8b_b1_f32": lambda: W.decode_8b("f32", 1),
        "decode_8b_b16_f32": lambda: W.decode_8b("f32", 16),
        "decode_8b_b64_f32": lambda: W.decode_8b("f32", 64),
        "decode_8b_b256_f32": lambda: W.decode_8b("f32", 256),
        "sweep_f32": lambda: W.sweep_serving("f32"),
        "sweep_bf16": lambda: W.sweep_serving("bf16"),
        "sweep_i8a": lambda: W.sweep_serving("i8a"),
        "sweep_i4a": lambda: W.sweep_serving("i4a"),
        "scan_370m_all": lambda: W.scan_370m("all"),
        "scan_370m_b64": lambda: W.scan_370m("all", batch=64),
        "scan_370m_mid": lambda: W.scan_370m("mid"),
        "prefill_370m_all": lambda: W.scan_370m("all"),
        "prefill_370m_mid": lambda: W.scan_370m("mid"),
        "decode_130m_damp": lambda: W.decode_130m_damp(),
        "diag_130m": lambda: dataclasses.replace(
            W.decode_130m("i8a"), name="mamba2-130m step diagnostics L24 b256 H24 P64 N128 i8a"),
    }
    if name not in table:
        raise SystemExit(f"unknown workload {name}; choose from {sorted(table)}")
    return table[name]()


def row_state_bytes(fmt, N):
    """Bytes one stored row occupies (codes + metadata, or fp values)."""
    return {"f32": 4 * N, "bf16": 2 * N, "i8s": N + 4, "i8a": N + 8,
            "i4s": N // 2 + 4, "i4a": N // 2 + 8}[fmt]


def decode_bytes(wl):
    """Algorithmic bytes of one decode step: every stored row read and written
    once (codes + metadata), x / B / C / dt read and y written once.  A and D
    (per layer and head) are left out."""
    rows = wl.nl * wl.batch * wl.nheads * wl.headdim
    mask = wl.head_mask
    if mask is not None and wl.fmt not in ("f32", "bf16"):
        qfrac = float(np.mean(np.asarray(mask) != 0))
    else:
        qfrac = 1.0
    state = rows * (qfrac * row_state_bytes(wl.fmt, wl.d_state)
                    + (1 - qfrac) * row_state_bytes("f32", wl.d_state))
    io = rows * 4 * 2 + wl.nl * wl.batch * (2 * wl.ngroups * wl.d_state + wl.nheads) * 4
    return int(round(2 * state + io))


def damp_bytes(wl, K=DAMP_PROTECTED):
    """Algorithmic bytes of one DAMP decode step: every head block (FP16
    tier, INT8 codes, {step, zero point} per INT8 channel) read and written
    once, x / B / C / dt read and y written once, the channel map of the
    layers read once."""
    P, N = wl.headdim, wl.d_state
    head = 2 * K * P + (N - K) * P + 8 * (N - K)
    units = wl.nl * wl.batch * wl.nheads
    io = units * P * 4 * 2 + wl.nl * wl.batch * (2 * wl.ngroups * N + wl.nheads) * 4
    return int(2 * units * head + io + wl.nl * wl.nheads * N * 4)


def diag_bytes(wl):
    """Algorithmic bytes of one diagnostics pass (read-only): every stored
    row read once, x / B / C / dt read once, four fp32 results per row
    written."""
    rows = wl.nl * wl.batch * wl.nheads * wl.headdim
    io = rows * 4 + wl.nl * wl.batch * (2 * wl.ngroups * wl.d_state + wl.nheads) * 4
    return int(rows * row_state_bytes(wl.fmt, wl.d_state) + io + rows * 16)


def scan_bytes(wl):
    """Algorithmic bytes of one scan call: inputs x / B / C / dt read and y
    written once per token, the state read and written once."""
    per_tok = wl.batch * (2 * wl.nheads * wl.headdim + 2 * wl.ngroups * wl.d_state
                          + wl.nheads) * 4
    rows = wl.batch * wl.nheads * wl.headdim
    return int(per_tok * wl.T + 2 * rows * row_state_bytes(wl.fmt, wl.d_state))


def footprint_bytes(wl, name):
    """Distinct bytes one step touches: the stored state it reads and writes
    in place (one copy), its inputs and its output."""
    if isinstance(wl, W.Scan):
        rows = wl.batch * wl.nheads * wl.headdim
        return scan_bytes(wl) - rows * row_state_bytes(wl.fmt, wl.d_state)
    if name.startswith("diag"):
        return diag_bytes(wl)
    if name.endswith("_damp"):
        P, N, K = wl.headdim, wl.d_state, DAMP_PROTECTED
        units = wl.nl * wl.batch * wl.nheads
        return damp_bytes(wl) - units * (2 * K * P + (N - K) * P + 8 * (N - K))
    rows = wl.nl * wl.batch * wl.nheads * wl.headdim
    qfrac = 1.0
    if wl.head_mask is not None and wl.fmt not in ("f32", "bf16"):
        qfrac = float(np.mean(np.asarray(wl.head_mask) != 0))
    state = rows * (qfrac * row_state_bytes(wl.fmt, wl.d_state)
                    + (1 - qfrac) * row_state_bytes("f32", wl.d_state))
    return int(decode_bytes(wl) - state)


L2_FALLBACK_BYTES = 126 * 1024 * 1024


def l2_bytes(device):
    import torch
    try:
        return int(torch.cuda.get_device_properties(device).L2_cache_size)
    except Exception:
        return L2_FALLBACK_BYTES


def elem_steps(wl):
    if isinstance(wl, W.Scan):
        return wl.batch * wl.T * wl.nheads * wl.headdim * wl.d_state
    return wl.nl * wl.batch * wl.nheads * wl.headdim * wl.d_state


# ---------------------------------------------------------------------------
# Measured peaks, clocks, ncu traffic
# ---------------------------------------------------------------------------

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d.get("hbm_gbs", FALLBACK_HBM_GBS)), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def _code_only(src):
    """C / CUDA source with comments and blank space removed, so that an
    edit of comments alone keeps the hash (and the counters taken on the
    kernels stay attached to them)."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


# The sources each workload's dominant kernel is built from (with the host
# code that sizes its launch).
_COMMON_SOURCES = ("ssq_common.cuh", "ssq_params.h", "ssq_api.cu")
_DECODE_SOURCES = ("ssq_decode.cu", "ssq_decode_impl.cuh", "ssq_pipe.cuh",
                   "ssq_decode_f32.cu", "ssq_decode_bf16.cu", "ssq_decode_i8s.cu",
                   "ssq_decode_i8a.cu", "ssq_decode_i4s.cu", "ssq_decode_i4a.cu")
_KERNEL_SOURCES = {
    "decode": _DECODE_SOURCES,
    "damp": ("ssq_damp.cu", "ssq_pipe.cuh"),
    "scan": ("ssq_scan.cu",),
    "diag": _DECODE_SOURCES,
}


def _kernel_family(workload_name):
    if workload_name.endswith("_damp"):
        return "damp"
    if workload_name.startswith(("scan", "prefill")):
        return "scan"
    if workload_name.startswith("diag"):
        return "diag"
    return "decode"


def kernel_source_hash(workload_name="decode_130m"):
    """Hash of the code (comments and blank space removed) of the sources
    the workload's dominant kernel is built from."""
    h = hashlib.sha256()
    pkg = os.path.join(ROOT, "quantized_recurrent_state_mamba_b200", "csrc")
    names = sorted(_COMMON_SOURCES + _KERNEL_SOURCES[_kernel_family(workload_name)])
    files = [os.path.join(pkg, n) for n in names] + [os.path.join(ROOT, "include", "ssq.h")]
    for p in files:
        with open(p, encoding="utf-8") as f:
            h.update(os.path.basename(p).encode())
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(workload_name):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary for this workload, if it was captured on the current kernel
    sources (else None)."""
    src = kernel_source_hash(workload_name)
    for p in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        kv = {}
        with open(p) as f:
            for line in f:
                line = line.strip()
                if line.startswith("- ") and ":" in line:
                    k, v = line[2:].split(":", 1)
                    kv[k.strip()] = v.strip().strip("`")
        if kv.get("bench_workload") == workload_name and kv.get("source_hash") == src:
            try:
                return float(kv["dram_bytes_per_launch"])
            except (KeyError, ValueError):
                return None
    return None


class ClockSampler:
    """Samples the SM clock and the clock-event reasons through NVML in a
    background thread (every ~5 ms) and keeps the samples taken inside a
    marked window."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index):
        self.samples = []
        self.window = None
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = None
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            except Exception:
                uuid = None
            h = None
            if uuid:
                u = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID(u)
                except Exception:
                    h = None
            if h is None:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES")
                idx = int(vis.split(",")[device_index]) if vis else device_index
                h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.nv, self.h = pynvml, h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that clocks were not sampled
            self.err = str(e)

    def _run(self):
        nv, h = self.nv, self.h
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(0.005)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "note": "NVML unavailable: " + getattr(self, "err", "")}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        note = "samples inside the timed region"
        if not inside:
            # the region is shorter than the sampling period: take the
            # samples nearest to it
            near = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))
            inside = near[:3]
            note = "timed region shorter than the sampling period; nearest samples"
        reasons = set()
        for _, _, rs in inside:
            for bit, name in self.REASONS.items():
                if rs & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[1] for s in inside) if inside else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(inside), "note": note}


# ---------------------------------------------------------------------------
# Distributed plumbing
# ---------------------------------------------------------------------------

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(ms, world, device):
    """The slowest rank's time: every rank contributes its own device-timed
    milliseconds and gets the maximum back (a no-op on one rank)."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_step, steps, world, ms):
    """Whole-job GB/s: every rank runs its own replica of the step, so the
    job moves world x steps x bytes in the slowest rank's time."""
    return bytes_per_step * steps * world / (ms / 1e3) / 1e9


# ---------------------------------------------------------------------------
# The CPU oracle leg (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------

def oracle_decode_sample(wl, budget_s):
    """Time the CPU oracle on the first pairs of the decode workload until
    about budget_s seconds of work; returns (seconds, bytes, pairs)."""
    import oracle as O
    fmt = O.FORMATS[wl.fmt]
    H, P, N, G = wl.nheads, wl.headdim, wl.d_state, wl.ngroups
    ocfg = O.Cfg(fmt, H, P, N, G, wl.head_mask)
    inp = wl.inputs()
    per_pair = decode_bytes(wl) / (wl.nl * wl.batch)
    # calibrate on one pair
    st = O.state_from_f32(ocfg, wl.state_pair(0, 0).reshape(1, H, P, N))
    t = time.perf_counter()
    O.step(ocfg, st, 0, inp["x"][0, 0], inp["B"][0, 0], inp["C"][0, 0], inp["dt"][0, 0],
           inp["A"][0], inp["D"][0])
    one = max(time.perf_counter() - t, 1e-6)
    npairs = int(max(1, min(wl.nl * wl.batch, budget_s / one)))
    pairs = [(i // wl.batch, i % wl.batch) for i in range(npairs)]
    S0 = np.stack([wl.state_pair(l, b).reshape(H, P, N) for (l, b) in pairs])
    st = O.state_from_f32(ocfg, S0)
    t = time.perf_counter()
    for i, (l, b) in enumerate(pairs):
        O.step(ocfg, st, i, inp["x"][l, b], inp["B"][l, b], inp["C"][l, b], inp["dt"][l, b],
               inp["A"][l], inp["D"][l])
    sec = time.perf_counter() - t
    return sec, per_pair * npairs, npairs


def oracle_damp_sample(wl, budget_s, K=DAMP_PROTECTED):
    """Time the oracle's DAMP step on the first (layer, request) pairs."""
    import oracle as O
    H, P, N, G = wl.nheads, wl.headdim, wl.d_state, wl.ngroups
    chan = W.damp_channels(wl.seed, wl.nl, H, N)
    inp = wl.inputs()
    per_pair = damp_bytes(wl, K) / (wl.nl * wl.batch)
    ocs = [O.DampCfg(H, P, N, G, K, chan[l]) for l in range(wl.nl)]
    st = O.damp_from_f32(ocs[0], wl.state_pair(0, 0).reshape(H, P, N))
    t = time.perf_counter()
    O.damp_step(ocs[0], st, 0, inp["x"][0, 0], inp["B"][0, 0], inp["C"][0, 0],
                inp["dt"][0, 0], inp["A"][0], inp["D"][0])
    one = max(time.perf_counter() - t, 1e-6)
    npairs = int(max(1, min(wl.nl * wl.batch, budget_s / one)))
    pairs = [(i // wl.batch, i % wl.batch) for i in range(npairs)]
    sts = [O.damp_from_f32(ocs[l], wl.state_pair(l, b).reshape(H, P, N)) for (l, b) in pairs]
    t = time.perf_counter()
    for st, (l, b) in zip(sts, pairs):
        O.damp_step(ocs[l], st, 0, inp["x"][l, b], inp["B"][l, b], inp["C"][l, b],
                    inp["dt"][l, b], inp["A"][l], inp["D"][l])
    sec = time.perf_counter() - t
    return sec, per_pair * npairs, npairs


def oracle_diag_sample(wl, budget_s):
    """Time the oracle's step diagnostics on the first (layer, request)
    pairs."""
    import oracle as O
    H, P, N, G = wl.nheads, wl.headdim, wl.d_state, wl.ngroups
    ocfg = O.Cfg(O.FORMATS[wl.fmt], H, P, N, G, wl.head_mask)
    inp = wl.inputs()
    per_pair = diag_bytes(wl) / (wl.nl * wl.batch)
    st = O.state_from_f32(ocfg, wl.state_pair(0, 0).reshape(1, H, P, N))
    t = time.perf_counter()
    O.step_diag(ocfg, st, 0, inp["x"][0, 0], inp["B"][0, 0], inp["C"][0, 0], inp["dt"][0, 0],
                inp["A"][0], inp["D"][0])
    one = max(time.perf_counter() - t, 1e-6)
    npairs = int(max(1, min(wl.nl * wl.batch, budget_s / one)))
    pairs = [(i // wl.batch, i % wl.batch) for i in range(npairs)]
    st = O.state_from_f32(ocfg, np.stack([wl.state_pair(l, b).reshape(H, P, N)
                                          for (l, b) in pairs]))
    t = time.perf_counter()
    for i, (l, b) in enumerate(pairs):
        O.step_diag(ocfg, st, i, inp["x"][l, b], inp["B"][l, b], inp["C"][l, b],
                    inp["dt"][l, b], inp["A"][l], inp["D"][l])
    sec = time.perf_counter() - t
    return sec, per_pair * npairs, npairs


def oracle_scan_sample(wl, budget_s, prefill=False):
    import oracle as O
    H, P, N = wl.nheads, wl.headdim, wl.d_state
    inp = wl.inputs()
    ocfg = O.Cfg(O.FORMATS[wl.fmt], H, P, N, wl.ngroups, wl.head_mask)
    t = time.perf_counter()
    st = O.State(ocfg, 1)
    run = O.prefill if prefill else O.scan
    T1 = min(wl.T, 8)
    run(ocfg, st, 0, inp["x"][0, :T1], inp["B"][0, :T1], inp["C"][0, :T1],
        inp["dt"][0, :T1], inp["A"], inp["D"])
    per_tok = max((time.perf_counter() - t) / T1, 1e-6)
    ntok = int(max(1, min(wl.T * wl.batch, budget_s / per_tok)))
    st = O.State(ocfg, 1)
    b, done = 0, 0
    t = time.perf_counter()
    while done < ntok:
        n = min(wl.T, ntok - done)
        run(ocfg, st, 0, inp["x"][b, :n], inp["B"][b, :n], inp["C"][b, :n],
            inp["dt"][b, :n], inp["A"], inp["D"])
        done += n
        b = (b + 1) % wl.batch
    sec = time.perf_counter() - t
    frac = ntok / (wl.T * wl.batch)
    return sec, scan_bytes(wl) * frac, ntok


def cpu_leg(wl, budget_s, name=""):
    """The oracle, single thread, on a bounded sample of the workload."""
    if isinstance(wl, W.Scan):
        pf = name.startswith("prefill")
        sec, nbytes, n = oracle_scan_sample(wl, budget_s, prefill=pf)
        sample = (f"{n} request-tokens of the {'prefill' if pf else 'scan'} "
                  f"(request 0 onward), single thread")
        rsps = n / sec
    else:
        damp = name.endswith("_damp")
        diag = name.startswith("diag")
        sample_fn = (oracle_damp_sample if damp else
                     oracle_diag_sample if diag else oracle_decode_sample)
        sec, nbytes, n = sample_fn(wl, budget_s)
        what = "DAMP decode step" if damp else ("step diagnostics pass" if diag
                                                else "decode step")
        sample = (f"{n} of {wl.nl * wl.batch} (layer, request) pairs of one {what} "
                  f"(layer-major from pair 0), single thread")
        rsps = n / sec
    return {"value": nbytes / sec / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": sample, "seconds": round(sec, 3),
            "request_steps_per_s_per_layer": rsps}


# ---- the oracle on every host core ------------------------------------------
# One worker process per core (spawn start method: this process may already
# hold a CUDA context).  Each worker receives its share of the sample's
# inputs and builds its states untimed ("load"), then steps them ("run"); the
# parent times the run phase on the wall clock from the first "run" message
# to the last answer.

def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _oracle_worker(conn):
    import oracle as O
    job = None
    while True:
        msg = conn.recv()
        if msg[0] == "stop":
            break
        if msg[0] == "load":
            job = _worker_load(O, msg[1])
            conn.send("ready")
        elif msg[0] == "run":
            t = time.perf_counter()
            _worker_run(O, job)
            conn.send(time.perf_counter() - t)


def _worker_load(O, task):
    kind = task["kind"]
    H, P, N, G = task["shape"]
    if kind == "damp":
        cfgs = [O.DampCfg(H, P, N, G, task["K"], c) for c in task["chan"]]
        sts = [O.damp_from_f32(cfgs[i], S) for i, S in enumerate(task["S0"])]
        return dict(task, cfgs=cfgs, sts=sts)
    cfg = O.Cfg(task["fmt"], H, P, N, G, task["mask"])
    if kind == "scan":
        return dict(task, cfg=cfg, st=O.State(cfg, len(task["x"])))
    st = O.state_from_f32(cfg, np.stack(task["S0"]))
    return dict(task, cfg=cfg, st=st)


def _worker_run(O, job):
    kind = job["kind"]
    if kind == "scan":
        run = O.prefill if job["prefill"] else O.scan
        for i in range(len(job["x"])):
            run(job["cfg"], job["st"], i, job["x"][i], job["B"][i], job["C"][i], job["dt"][i],
                job["A"], job["D"])
        return
    for i in range(len(job["x"])):
        args = (job["x"][i], job["B"][i], job["C"][i], job["dt"][i], job["A"][i], job["D"][i])
        if kind == "damp":
            O.damp_step(job["cfgs"][i], job["sts"][i], 0, *args)
        elif kind == "diag":
            O.step_diag(job["cfg"], job["st"], i, *args[:5], job["D"][i])
        else:
            O.step(job["cfg"], job["st"], i, *args)


def _pair_tasks(wl, name, pairs, workers):
    """Split the (layer, request) pairs over the workers; each task carries
    its pairs' inputs and initial states."""
    import oracle as O
    inp = wl.inputs()
    H, P, N = wl.nheads, wl.headdim, wl.d_state
    damp = name.endswith("_damp")
    kind = "damp" if damp else ("diag" if name.startswith("diag") else "decode")
    chan = W.damp_channels(wl.seed, wl.nl, H, N) if damp else None
    tasks = []
    for w in range(workers):
        mine = pairs[w::workers]
        t = {"kind": kind, "shape": (H, P, N, wl.ngroups), "fmt": O.FORMATS[wl.fmt],
             "mask": wl.head_mask, "K": DAMP_PROTECTED,
             "S0": [wl.state_pair(l, b).reshape(H, P, N) for (l, b) in mine],
             "x": [inp["x"][l, b] for (l, b) in mine], "B": [inp["B"][l, b] for (l, b) in mine],
             "C": [inp["C"][l, b] for (l, b) in mine], "dt": [inp["dt"][l, b] for (l, b) in mine],
             "A": [inp["A"][l] for (l, b) in mine], "D": [inp["D"][l] for (l, b) in mine]}
        if damp:
            t["chan"] = [chan[l] for (l, b) in mine]
        tasks.append(t)
    return tasks


def _scan_tasks(wl, name, ntok, workers):
    """One request per worker (the scan is sequential in t), each running
    its first ntok tokens."""
    import oracle as O
    inp = wl.inputs()
    tasks = []
    for w in range(workers):
        b = w % wl.batch
        tasks.append({"kind": "scan", "prefill": name.startswith("prefill"),
                      "shape": (wl.nheads, wl.headdim, wl.d_state, wl.ngroups),
                      "fmt": O.FORMATS[wl.fmt], "mask": wl.head_mask,
                      "x": [inp["x"][b, :ntok]], "B": [inp["B"][b, :ntok]],
                      "C": [inp["C"][b, :ntok]], "dt": [inp["dt"][b, :ntok]],
                      "A": inp["A"], "D": inp["D"]})
    return tasks


def cpu_leg_all_cores(wl, budget_s, name="", max_workers=None):
    """The oracle, as it stands, on every host core: one process per core,
    each stepping its share of a bounded sample of the workload (about
    budget_s seconds of wall time).  Returns the cpu_baseline record, with
    the single-thread figure of cpu_leg beside it."""
    import multiprocessing as mp
    single = cpu_leg(wl, max(1.0, budget_s / 4), name)
    cores = host_cores()
    is_scan = isinstance(wl, W.Scan)
    units_total = wl.batch if is_scan else wl.nl * wl.batch
    workers = max(1, min(cores, max_workers or cores, units_total))
    if is_scan:
        # tokens per request so the run lasts about budget_s
        per_tok = single["seconds"] / max(1, int(single["request_steps_per_s_per_layer"]
                                                 * single["seconds"]))
        ntok = int(max(1, min(wl.T, budget_s / max(per_tok, 1e-9))))
        tasks = _scan_tasks(wl, name, ntok, workers)
        units = workers * ntok
        nbytes = scan_bytes(wl) * units / (wl.T * wl.batch)
        what = (f"{workers} requests x {ntok} tokens of the "
                f"{'prefill' if name.startswith('prefill') else 'scan'}, one request per process")
    else:
        per_pair = single["seconds"] / max(1, int(single["request_steps_per_s_per_layer"]
                                                  * single["seconds"]))
        npairs = int(max(workers, min(units_total,
                                      workers * budget_s / max(per_pair, 1e-9))))
        pairs = [(i // wl.batch, i % wl.batch) for i in range(npairs)]
        tasks = _pair_tasks(wl, name, pairs, workers)
        units = npairs
        per_bytes = (damp_bytes(wl) if name.endswith("_damp") else
                     diag_bytes(wl) if name.startswith("diag") else decode_bytes(wl))
        nbytes = per_bytes * npairs / (wl.nl * wl.batch)
        what = (f"{npairs} of {units_total} (layer, request) pairs (layer-major from pair 0), "
                f"split over {workers} processes")
    ctx = mp.get_context("spawn")
    conns, procs = [], []
    try:
        for _ in range(workers):
            a, b = ctx.Pipe()
            pr = ctx.Process(target=_oracle_worker, args=(b,), daemon=True)
            pr.start()
            conns.append(a)
            procs.append(pr)
        for c, t in zip(conns, tasks):
            c.send(("load", t))
        for c in conns:
            assert c.recv() == "ready"
        t0 = time.perf_counter()
        for c in conns:
            c.send(("run",))
        busy = [c.recv() for c in conns]
        wall = time.perf_counter() - t0
    finally:
        for c in conns:
            try:
                c.send(("stop",))
            except (BrokenPipeError, OSError):
                pass
        for pr in procs:
            pr.join(timeout=30)
    return {"value": nbytes / wall / 1e9, "unit": "GB/s", "cores": workers, "kind": "oracle",
            "sample": what, "seconds": round(wall, 3),
            "request_steps_per_s_per_layer": units / wall,
            "host_cores": cores, "worker_busy_s_max": round(max(busy), 3),
            "single_thread": {"value": single["value"], "unit": "GB/s",
                              "sample": single["sample"], "seconds": single["seconds"]}}


def run_reference(args, wl, name):
    """The reference arm: the CPU oracle, as it stands, on every host core of
    rank 0 (other ranks exit at once); each step a bounded sample of the
    workload, so the whole --steps K --warmup W run ends within minutes."""
    world, rank, _ = dist_setup()
    if rank != 0:
        return 0
    steps, warm = args.steps, args.warmup
    budget = max(0.5, min(20.0, 150.0 / max(1, steps + warm)))
    for _ in range(warm):
        cpu_leg_all_cores(wl, budget, name, args.cpu_workers)
    vals, secs, rec = [], 0.0, None
    for _ in range(steps):
        rec = cpu_leg_all_cores(wl, budget, name, args.cpu_workers)
        vals.append(rec["value"])
        secs += rec["seconds"]
    value = statistics.median(vals)
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
           "n_gpus": world, "steps": steps, "warmup": warm,
           "ms_per_step": 1000 * secs / max(1, steps), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
           "config": {"workload": wl.name, "bench_workload": name},
           "cpu_baseline": {"value": value, "unit": "GB/s", "cores": rec["cores"],
                            "kind": "oracle", "sample": rec["sample"] + " per step",
                            "host_cores": rec["host_cores"],
                            "single_thread": rec["single_thread"]},
           "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out))
    return 0


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------

def run_ours(args, wl, name):
    import torch
    import torch.distributed as dist
    from quantized_recurrent_state_mamba_b200 import ssq

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    is_scan = isinstance(wl, W.Scan)
    damp = name.endswith("_damp")
    fmt = f"damp-k{DAMP_PROTECTED}" if damp else wl.fmt
    H, P, N, G = wl.nheads, wl.headdim, wl.d_state, wl.ngroups
    n_layers = 1 if is_scan else wl.nl
    inp = wl.inputs()
    d = {k: torch.from_numpy(np.ascontiguousarray(v)).to(dev) for k, v in inp.items()}
    if damp:
        cfg = ssq.DampConfig(n_layers=n_layers, n_slots=wl.batch, nheads=H, headdim=P,
                             d_state=N, ngroups=G, n_protected=DAMP_PROTECTED)
        pool = ssq.damp_alloc_pool(cfg, dev)
        chan = torch.from_numpy(W.damp_channels(wl.seed, n_layers, H, N)).to(dev)
        pool_error = lambda pl: ssq.ssq_damp_pool_error(cfg, pl)  # noqa: E731
    else:
        cfg = ssq.Config(n_layers=n_layers, n_slots=wl.batch, nheads=H, headdim=P, d_state=N,
                         ngroups=G, fmt=fmt, head_mask=wl.head_mask)
        pool = ssq.alloc_pool(cfg, dev)
        pool_error = lambda pl: ssq.ssq_pool_error(cfg, pl)  # noqa: E731

    # initial state
    if damp:
        for l in range(wl.nl):
            S = np.empty((wl.batch, wl.rows, N), np.float32)
            for b in range(wl.batch):
                S[b] = wl.state_pair(l, b)
            ssq.ssq_damp_quantize(cfg, pool, chan, None, wl.batch, l, 1,
                                  torch.from_numpy(S).to(dev))
        torch.cuda.synchronize()
    elif not is_scan and wl.init != "zero":
        for l in range(wl.nl):
            S = np.empty((wl.batch, wl.rows, N), np.float32)
            for b in range(wl.batch):
                S[b] = wl.state_pair(l, b)
            ssq.ssq_quantize_rows(cfg, pool, None, wl.batch, l, 1,
                                  torch.from_numpy(S).to(dev))
        torch.cuda.synchronize()

    # L2: below 4x the L2, the timed steps rotate over enough copies of the
    # pool, the inputs and the output that each step finds its state and
    # inputs evicted by the copies stepped since its last turn.
    l2 = l2_bytes(dev)
    foot = footprint_bytes(wl, name)
    copies = 1 if foot >= 4 * l2 else int(math.ceil(4 * l2 / foot))
    pools = [pool] + [pool.clone() for _ in range(copies - 1)]
    ds = [d] + [{k: v.clone() for k, v in d.items()} for _ in range(copies - 1)]
    if copies == 1:
        l2_note = (f"step footprint {foot / 1e6:.0f} MB >= 4x the {l2 / 1e6:.0f} MB L2; "
                   f"no rotation, no flush")
    else:
        l2_note = (f"step footprint {foot / 1e6:.1f} MB < 4x the {l2 / 1e6:.0f} MB L2: "
                   f"timed steps rotate over {copies} copies of pool, inputs and output "
                   f"({copies * foot / 1e6:.0f} MB)")

    # the prefill hand-off runs the scan's shape with the state in fp32
    # between tokens and one quantization at the end
    scan_fn = ssq.ssq_prefill if name.startswith("prefill") else ssq.ssq_scan
    sr = name.endswith("_sr")
    if is_scan:
        yshape = (wl.batch, wl.T, H, P)
        nbytes = scan_bytes(wl)
        units = wl.batch * wl.T          # request-tokens
    elif name.startswith("diag"):
        # the diagnostics pass reads the state and writes four numbers per
        # row; y stands for its output in the end-to-end leg
        yshape = (wl.nl, wl.batch, H, P, 4)
        nbytes = diag_bytes(wl)
        units = wl.batch * wl.nl
    else:
        yshape = (wl.nl, wl.batch, H, P)
        nbytes = damp_bytes(wl) if damp else decode_bytes(wl)
        units = wl.batch * wl.nl         # request-layer steps
    y = torch.empty(yshape, device=dev)
    ys = [y] + [torch.empty_like(y) for _ in range(copies - 1)]
    nstep = [0]

    def launch(pool_i, t, y_i, stream=None):
        """One step of the workload's call on the given pool, inputs and
        output (the stochastic-rounding variant draws fresh randomness each
        step)."""
        if is_scan:
            scan_fn(cfg, pool_i, None, wl.batch, 0, wl.T, t["x"], t["B"], t["C"], t["dt"],
                    d["A"], d["D"], y_i, stream=stream)
        elif name.startswith("diag"):
            ssq.ssq_decode_diag(cfg, pool_i, None, wl.batch, 0, wl.nl, t["x"], t["B"], t["C"],
                                t["dt"], d["A"], y_i, stream=stream)
        elif damp:
            ssq.ssq_damp_decode_step(cfg, pool_i, chan, None, wl.batch, 0, wl.nl, t["x"],
                                     t["B"], t["C"], t["dt"], d["A"], d["D"], y_i,
                                     stream=stream)
        elif sr:
            nstep[0] += 1
            ssq.ssq_decode_step_sr(cfg, pool_i, None, wl.batch, 0, wl.nl, t["x"], t["B"],
                                   t["C"], t["dt"], d["A"], d["D"], y_i, 12345, nstep[0],
                                   stream=stream)
        else:
            ssq.ssq_decode_step(cfg, pool_i, None, wl.batch, 0, wl.nl, t["x"], t["B"], t["C"],
                                t["dt"], d["A"], d["D"], y_i, stream=stream)

    def step(i):
        k = i % copies
        launch(pools[k], ds[k], ys[k])

    stream = torch.cuda.current_stream(dev)
    # The clock sampler starts before the warm-up, so that its first NVML
    # queries (the slow ones) do not fall inside the timed region.
    sampler = ClockSampler(local)
    sampler.start()
    t_wait = time.perf_counter()
    while sampler.ok and len(sampler.samples) < 3 and time.perf_counter() - t_wait < 2.0:
        time.sleep(0.005)
    for i in range(max(args.warmup, copies)):
        step(i)
    torch.cuda.synchronize()
    if any(pool_error(pl) != 0 for pl in pools):
        raise SystemExit("device error word set during warm-up")
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(K):
        ev[i][0].record(stream)
        step(i)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    barrier()
    sampler.stop()
    region_ms = ev[0][0].elapsed_time(ev[-1][1])
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    kern_ms = statistics.median(launch_ms)
    # device time between steps (the host enqueueing late), for the record
    host_gap_ms = max(0.0, region_ms - sum(launch_ms))
    region_ms = max_over_ranks(region_ms, world, dev)
    value = job_throughput(nbytes, K, world, region_ms)
    ms_per_step = region_ms / K

    # End to end through the public API: every step copies that step's inputs
    # from pinned host memory and reads its result y back.  Copies in, the
    # kernel and the copy out run on three streams with double-buffered
    # device inputs and outputs, so step i's copies overlap steps i-1 and
    # i+1's work, as a serving loop would run them.
    keys = ("x", "B", "C", "dt")
    h = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).pin_memory() for k in keys}
    din = [{k: torch.empty_like(d[k]) for k in keys} for _ in range(2)]
    yb = [torch.empty_like(y) for _ in range(2)]
    yh = [torch.empty(y.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    s_in, s_c, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    h2d = sum(t.numel() * 4 for t in h.values())
    d2h = y.numel() * 4

    def e2e_step(i):
        kk = i & 1
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_c[kk])
            for k2 in keys:
                din[kk][k2].copy_(h[k2], non_blocking=True)
            ev_in[kk].record(s_in)
        s_c.wait_event(ev_in[kk])
        if i >= 2:
            s_c.wait_event(ev_out[kk])
        t = din[kk]
        launch(pools[i % copies], t, yb[kk], stream=s_c)
        ev_c[kk].record(s_c)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_c[kk])
            yh[kk].copy_(yb[kk], non_blocking=True)
            ev_out[kk].record(s_out)

    for i in range(max(3, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    s_c.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(K):
        e2e_step(i)
    e1.record(s_out)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    e2e_value = job_throughput(nbytes, K, world, e2e_ms)
    e2e_launches = K
    err = 0
    for pl in pools:
        err |= pool_error(pl)

    peak, peak_kind = measured_peaks()
    achieved = nbytes / (kern_ms / 1e3) / 1e9
    traffic = ncu_traffic(name)
    clocks = sampler.summary(t0, t1)
    if is_scan:
        # The scan reads each input once and keeps the state on chip: its
        # bound is the FP32 pipe, not HBM.  Algorithmic fp32 operations per
        # element-token (each add / mul / fma one): w = dtx*B, s' = fma,
        # fma(s', inv, M) and -M (round the exact product to nearest),
        # r*Delta, C*r = 6.
        # Peak: 148 SMs x 128 FP32 lanes x the maximum SM clock.
        ops = (PREFILL_FP32_OPS if name.startswith("prefill") else SCAN_FP32_OPS) \
            * elem_steps(wl)
        sm_max = clocks.get("sm_max_mhz") or SM_MAX_MHZ
        alu_peak = 148 * 128 * sm_max * 1e6 / 1e12
        alu_ach = ops / (kern_ms / 1e3) / 1e12
        roofline = {"bound": "alu", "achieved": round(alu_ach, 3), "peak": round(alu_peak, 2),
                    "unit": "Top/s (fp32 pipe operations)", "frac": round(alu_ach / alu_peak, 4),
                    "traffic": traffic, "peak_source": "148 SMs x 128 fp32 lanes x max SM clock",
                    "kernel_ms_per_launch": round(kern_ms, 5),
                    "kernel_ms_stat": f"median of {K} launches (CUDA events)",
                    "hbm_achieved_gbs": round(achieved, 2)}
    else:
        roofline = {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                    "unit": "GB/s", "frac": round(achieved / peak, 4),
                    "traffic": traffic, "peak_source": peak_kind,
                    "kernel_ms_per_launch": round(kern_ms, 5),
                    "kernel_ms_stat": f"median of {K} launches (CUDA events)"}

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl.name, "bench_workload": name, "format": fmt,
                   "layers_per_launch": n_layers, "batch_per_gpu": wl.batch,
                   "nheads": H, "headdim": P, "d_state": N, "ngroups": G,
                   "T": getattr(wl, "T", 1),
                   "algorithmic_bytes_per_step": nbytes,
                   "l2": l2_note, "pool_copies": copies,
                   "parallelism": f"replicas x{world}"},
        "request_steps_per_s_per_layer": round(units * K * world / (region_ms / 1e3), 1),
        "pct_of_measured_hbm": round(100 * value / world / peak, 2),
        "pct_of_8tbs": round(100 * value / world / NOMINAL_HBM_GBS, 2),
        "roofline": roofline,
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms / K, 5),
                "note": "pinned host inputs in and y out every step; copies overlap "
                        "neighbouring steps' kernels (three streams, double buffers)"},
        "gpu_launches": K,
        "idle_between_steps_ms": round(host_gap_ms, 4),
        "clocks": clocks,
        "device_error_word": err,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_leg_all_cores(wl, args.cpu_budget, name,
                                                args.cpu_workers)
    if rank == 0:
        print(json.dumps(out))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def spawn_ranks(n):
    """Run this command as n ranks on this node (torch.distributed.run,
    rendezvous on 127.0.0.1) and return its exit code."""
    import socket
    import subprocess
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1",
           "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode_130m")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle work for the cpu_baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-workers", type=int, default=None,
                    help="cap on the oracle worker processes (default: every host core)")
    ap.add_argument("--nl", type=int, default=None,
                    help="layers per decode launch (a smaller case of the same shape, "
                         "for profiler captures; the bench lines use the workload's own)")
    args = ap.parse_args()
    if args.gpus < 1:
        raise SystemExit("--gpus must be >= 1")
    world_env = os.environ.get("WORLD_SIZE")
    if world_env is None and args.gpus > 1:
        # one process per GPU: start the ranks here when no launcher did
        return spawn_ranks(args.gpus)
    if world_env is not None and int(world_env) != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but the launcher started "
                         f"WORLD_SIZE={world_env} ranks")
    wl = workload(args.workload)
    if args.nl is not None:
        if not isinstance(wl, W.Decode):
            raise SystemExit("--nl applies to decode workloads")
        wl = dataclasses.replace(wl, nl=args.nl,
                                 name=wl.name.replace(f"L{wl.nl} ", f"L{args.nl} "))
    if args.impl == "reference":
        # the oracle on the host cores: no device timing, so no warm-up rule
        return run_reference(args, wl, args.workload)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    return run_ours(args, wl, args.workload)


if __name__ == "__main__":
    sys.exit(main())
