#!/usr/bin/env python3
"""Benchmark of the B200 Ulysses 4D all-to-all re-layout.

One step = one pass of the whole hot path over one batch of synthetic input:
mode 0 (scatter heads, gather sequence) on the w input slabs, then mode 1 (the
inverse) on its result, each through the C ABI (host checks, descriptor table,
tile scheduler, copy kernel). Headline workload: w=8, B=2, S_local=4725 (a
ragged last tile), H=40, D=128, bf16, N(0,1) values: a payload P of 774.1 MB
per call.

Metric: payload GB/s (P per call / device time, 1 GB = 1e9 B) and the fraction
of the HBM roofline counting 2P bytes moved per call, against the measured copy
bandwidth of this B200 (MEASURED_PEAKS.json) and against the nominal 8 TB/s of
B200 HBM3e. The K steps run back to back between two CUDA events on the
launching stream; every call's input (774 MB) is larger than the 126 MB L2 and
mode 1 reads its own input slabs rather than mode 0's fresh output, so no kernel
reads what the kernel before it touched.

The same line carries, on one GPU:
  per_mode        each mode of the headline workload, back to back (>= 1 s each);
  isolated_call   one call at a time after an L2 flush that READS a buffer twice
                  the L2 (leaving only clean lines), for the headline workload
                  and w4_S8192_H24_D128: median device time per call;
  workloads       w4_S8192_H24_D128 per mode, and w4_B4_S16384_H32_D64 unchunked,
                  chunked per plane and chunked through the staging window;
  sweep           payloads of 1 MiB, 64 MiB, 512 MiB and 2 GiB at w = 2/4/8
                  (H = 8w, D = 128, B = 1), bf16 and fp32 U[-1,1), both modes;
                  the 512 MiB bf16 points (w_sweep_512MiB) run >= 1 s per mode;
  vec_shapes      shapes only the vector path takes: 200-byte and 6/12-byte
                  rows, slab bases 8 and 2 bytes off a 16-byte boundary (both sides,
                  or the [B, S, H, D] side only), w = 16;
  e2e             the step through the host-buffer entry point (pinned slabs);
  cpu_baseline    the CPU oracle on a sample of the headline workload: the
                  OpenMP build on every host core, and the single-threaded one.
Each timed section carries its own clock record (SM MHz sampled every ~2 ms by
NVML during that section, and the clock-event reasons seen).

Multi-GPU (torchrun, one process per GPU): every rank runs its own independent
instance of the headline workload (the w logical ranks all live in one GPU's
memory), and `value` = payload of all ranks / the slowest rank's time ("weak"
scaling). The line then adds the Ulysses all-to-all ACROSS the GPUs (w = the
number of GPUs, one rank slab of the headline's per-rank shape per GPU):
exchange_peer_gbs (this library's PeerExchange: windows, peer loads) and
exchange_nccl_gbs (a library all-to-all baseline), with the barrier share of a
PeerExchange step.

`--impl reference` times the CPU oracle (the plain nested-loop definition) on
the host cores, on a bounded sample of the same workload, as a baseline only.

Other modes, each printing its own line:
  --sweep          the full 128 KiB..2 GiB bandwidth sweep (w = 2/4/8, bf16/fp32);
  --packed         q, k, v in one head-packed launch vs three per-tensor launches;
  --peer-one-gpu   the cross-GPU exchange's publish and pull kernels, with the
                   ranks as contexts on one GPU;
  --tuning-sweep   the schedule knobs one at a time (the measurements behind the
                   default schedule);
  --exchange X     the Ulysses all-to-all across the GPUs of a torchrun job (one
                   rank slab per GPU): X = nccl (a library all-to-all baseline)
                   or peer (PeerExchange).
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "payload GB/s and % of HBM roofline (2x bytes) per mode at w=2/4/8, 1xB200"
# The benchmark workloads (bf16, N(0,1) values), named by their sizes:
#   w2_S64_H4_D64          a tiny round trip (B = 1);
#   w4_S8192_H24_D128      192 MiB per call (B = 1);
#   w8_B2_S4725_H40_D128   the default: w = 8, a ragged sequence tail
#                          (4725 = 787 x 6 + 3), 774 MB per call;
#   w4_B4_S16384_H32_D64   four planes, for the chunked per-plane variant, 1 GiB.
DEFAULT_WORKLOAD = "w8_B2_S4725_H40_D128"
WORKLOADS = {
    "w2_S64_H4_D64": dict(w=2, B=1, S_local=64, H=4, D=64),
    "w4_S8192_H24_D128": dict(w=4, B=1, S_local=8192, H=24, D=128),
    "w8_B2_S4725_H40_D128": dict(w=8, B=2, S_local=4725, H=40, D=128),
    "w4_B4_S16384_H32_D64": dict(w=4, B=4, S_local=16384, H=32, D=64),
}
WORKLOAD = WORKLOADS[DEFAULT_WORKLOAD]
# Shapes only the vector path takes (bf16 unless noted): name -> (w, B, S, H, D,
# element bytes, byte offset of every slab base from a 16-byte boundary).
VEC_SHAPES = {
    "rows200B_w8_S41943_H8_D100": (8, 1, 41943, 8, 100, 2, 0),     # 200-byte runs
    "rows12B_w4_S1398101_H4_D3_fp32": (4, 1, 1398101, 4, 3, 4, 0),  # 12-byte runs
    "rows6B_w4_S2796202_H4_D3": (4, 1, 2796202, 4, 3, 2, 0),        # 6-byte runs
    "base8_w4_S8192_H24_D128": (4, 1, 8192, 24, 128, 2, 8),         # bases 8 B off
    "base2_w4_S8192_H24_D128": (4, 1, 8192, 24, 128, 2, 2),         # bases 2 B off
    # [B, S, H, D] slabs 2 B off, the [B, S*w, H/w, D] slabs aligned
    "base2in_w4_S8192_H24_D128": (4, 1, 8192, 24, 128, 2, 2, 0),
    "w16_S4096_H32_D128": (16, 1, 4096, 32, 128, 2, 0),             # w above the TMA limit
}
# Dense shapes with runs off 16 bytes (about 256 MiB each; bf16 unless noted):
# name -> (w, B, S, H, D, element bytes). --staged-forms times each on the
# staged path's two forms, and on the vector path; the first ten have
# pieces of 4 bytes or less, the others 8 bytes.
STAGED_FORM_SHAPES = {
    "w4_S2796202_H4_D3": (4, 1, 2796202, 4, 3, 2),             # 6-byte runs, 4 regions
    "w8_S699050_H8_D3": (8, 1, 699050, 8, 3, 2),                # 6-byte runs, 8 regions
    "w16_S174762_H16_D3": (16, 1, 174762, 16, 3, 2),            # 6-byte runs, 16 regions
    "w3_S2982616_H3_D5": (3, 1, 2982616, 3, 5, 2),              # 10-byte runs
    "w4_S1398101_H4_D3_fp32": (4, 1, 1398101, 4, 3, 4),         # 12-byte runs
    "w2_S13421772_H2_D5_u8": (2, 1, 13421772, 2, 5, 1),         # 5-byte runs, 1-byte pieces
    "w4_S838860_H8_D5": (4, 1, 838860, 8, 5, 2),                # 20-byte runs
    "w8_S116508_H8_D9_fp32": (8, 1, 116508, 8, 9, 4),           # 36-byte runs
    "w27_S36822_H27_D5": (27, 1, 36822, 27, 5, 2),              # 10-byte runs, 135 movers
    "w35_S43826_H35_D5_u8": (35, 1, 43826, 35, 5, 1),           # 5-byte runs, 175 movers
    "w4_S2097152_H4_D4": (4, 1, 2097152, 4, 4, 2),              # 8-byte runs
    "w4_S2796202_H4_D6_fp32": (4, 1, 2796202, 4, 6, 4),         # 24-byte runs
    "w4_S419430_H4_D20": (4, 1, 419430, 4, 20, 2),              # 40-byte runs
    "w4_S233016_H4_D36": (4, 1, 233016, 4, 36, 2),              # 72-byte runs
    "w4_S161319_H4_D52": (4, 1, 161319, 4, 52, 2),              # 104-byte runs
    "w4_S123361_H4_D68": (4, 1, 123361, 4, 68, 2),              # 136-byte runs
    "w8_S41943_H8_D100": (8, 1, 41943, 8, 100, 2),              # 200-byte runs
}


# Every workload --workload accepts: the table above, and the vector-path shapes
# (element size and base offset as listed there).
# off: the [B, S, H, D] slabs' bytes past a 16-byte boundary; goff: the
# [B, S*w, H/w, D] slabs' (the same unless a shape gives an eighth field).
ALL_WORKLOADS = {**{n: dict(v, E=2, off=0, goff=0) for n, v in WORKLOADS.items()},
                 **{n: dict(w=v[0], B=v[1], S_local=v[2], H=v[3], D=v[4], E=v[5], off=v[6],
                            goff=v[7] if len(v) > 7 else v[6])
                    for n, v in VEC_SHAPES.items()}}
DTYPE_OF = {1: "u8", 2: "bf16", 4: "fp32"}
INT_OF = {2: torch.int16, 4: torch.int32}


def workload_key(w, B, S, H, D, path, E=2, off=0, goff=None):
    goff = off if goff is None else goff
    tail = (f"_base{off}" if off else "") if goff == off else f"_base{off}_gathered{goff}"
    return f"{path}:w{w}_B{B}_S{S}_H{H}_D{D}_{DTYPE_OF[E]}" + tail


def workload_name(w, B, S, H, D, chunked, E=2, off=0, goff=None):
    how = {0: "", 1: ", chunked per plane", 2: ", chunked through the staging window"}[chunked]
    goff = off if goff is None else goff
    if goff != off:
        base = (f", [B, S, H, D] slab bases {off} bytes and the others {goff} bytes past a "
                "16-byte boundary")
    else:
        base = f", slab bases {off} bytes past a 16-byte boundary" if off else ""
    return (f"ulysses_a2a w={w} B={B} S_local={S} H={H} D={D} {DTYPE_OF[E]}{base}, "
            f"step = mode 0 + mode 1{how}")


FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0        # B200 HBM3e, nominal
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------- helpers
def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def max_over_ranks(value: float, dist=None, device="cpu") -> float:
    """The largest of every rank's `value` (the slowest rank's time); identity on one rank."""
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(world: int, bytes_per_step: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: every rank's bytes over the slowest rank's time (GB = 1e9 B)."""
    return world * bytes_per_step * steps / (max_ms / 1e3) / 1e9


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs: torch copy, 1 Gi bf16)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s copy bandwidth, an earlier B200 measurement)"


def fracs(payload_bytes: int, ms: float, peak: float) -> dict:
    """Payload GB/s of one call of `ms`, and 2 x payload against the measured and
    the nominal HBM bandwidth."""
    gbs = payload_bytes / (ms / 1e3) / 1e9
    return {"gbs": round(gbs, 1), "frac": round(2 * gbs / peak, 4),
            "frac_nominal": round(2 * gbs / NOMINAL_HBM_GBS, 4)}


def _code_only(text: str) -> str:
    """C/C++/CUDA source with comments removed and whitespace collapsed."""
    import re

    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


KERNEL_FILES = {"tma": "kernels_tma.cuh", "vec": "kernels_vec.cuh", "peel": "kernels_peel.cuh",
                "staged": "kernels_stage.cuh", "phase": "kernels_phase.cuh"}
PATH_NAMES = {1: "tma", 2: "vec", 3: "staged"}
LAUNCH_FIELDS = ("path", "rows_per_tile", "producers", "stages", "lookahead", "chunk_units",
                 "order", "grid", "block", "smem_bytes", "vec_bytes", "peeled", "fixed_phase")


def kernel_source_hash(path):
    """Hash of one kernel file's device code (comments and layout ignored):
    ncu counters taken on one hash stay valid until that code changes."""
    name = KERNEL_FILES[path]
    h = hashlib.sha256()
    with open(os.path.join(ROOT, "sequence_all_re_b200", "csrc", name), encoding="utf-8") as f:
        h.update(name.encode())
        h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(key, plan, chunked):
    """DRAM bytes per launch from the committed ncu summary, while the capture
    matches this kernel's code and this launch shape; else (None, why)."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            entry = json.load(f).get("workloads", {}).get(key)
    except Exception:
        return None, "no ncu traffic summary"
    if not entry:
        return None, "no ncu capture of this kernel and workload"
    # the vector path's peeled and shifted kernels, and the staged path's
    # fixed-phase kernel, live in files of their own
    kernel = ("peel" if plan.get("peeled") else
              "phase" if plan.get("fixed_phase") else key.split(":")[0])
    if entry.get("kernel_hash") != kernel_source_hash(kernel):
        return None, "kernel changed since the ncu counters were taken"
    launch = entry.get("launch", {})
    if chunked or any(launch.get(f) != plan[f] for f in LAUNCH_FIELDS):
        return None, "the capture was taken with another launch shape"
    return entry.get("dram_bytes_per_launch"), "ncu"


class ClockSampler:
    """SM clock and clock-event reasons of one GPU, sampled every ~2 ms by a
    background thread for as long as it runs (NVML; nvidia-smi every 100 ms
    when NVML is unavailable). `window(t0, t1)` summarises the samples taken
    between two time.perf_counter() stamps, i.e. during one timed region."""

    # NVML clock-event reason bits that matter for a bandwidth number
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}
    SMI_FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index, period_s=0.002):
        self.period = period_s
        self.samples = []            # (t, sm_mhz, reason names)
        self.source = None
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._proc = None
        try:
            p = torch.cuda.get_device_properties(device_index)
            self.bus = "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
        except Exception:
            self.bus = None

    def _nvml_loop(self, nv, h):
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            except Exception:
                break
            names = tuple(n for b, n in self.REASONS.items() if bits & b)
            self.samples.append((time.perf_counter(), float(mhz), names))
            time.sleep(self.period)

    def _smi_loop(self):
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in self._proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 6:
                continue
            try:
                mhz, mx = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            self.max_mhz = mx
            act = tuple(n for n, v in zip(names, parts[2:6]) if v.lower() == "active")
            self.samples.append((time.perf_counter(), mhz, act))

    def start(self):
        if self.bus is None:
            return self
        try:
            import pynvml as nv

            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByPciBusId(self.bus)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.source = "nvml"
            self._thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
        except Exception:
            try:
                self._proc = subprocess.Popen(
                    ["nvidia-smi", "-i", self.bus, f"--query-gpu={self.SMI_FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.source = "nvidia-smi"
                self._thread = threading.Thread(target=self._smi_loop, daemon=True)
            except Exception:
                return self
        self._thread.start()
        return self

    def stop(self):
        self._stop.set()
        if self._proc is not None:
            self._proc.terminate()
        if self._thread is not None:
            self._thread.join(timeout=5)

    def window(self, t0, t1):
        """Median SM MHz and the reasons seen between t0 and t1 (None if no sample)."""
        sel = [s for s in self.samples if t0 <= s[0] <= t1]
        if not sel:
            return None
        reasons = sorted({n for s in sel for n in s[2]})
        return {"sm_mhz": statistics.median(s[1] for s in sel), "sm_max_mhz": self.max_mhz,
                "samples": len(sel), "reasons": reasons, "source": self.source}


# ---------------------------------------------------------------- our arm
def make_inputs(w, B, S, H, D, dtype, device, seed0=1234, offset_bytes=0):
    """Seeded N(0,1) slabs (uniform bytes for "u8") drawn on the device
    generator (values do not affect timing); with offset_bytes each slab starts
    that many bytes past the start of its own allocation (a base off the 16-byte
    boundary)."""
    dt = {"bf16": torch.bfloat16, "fp32": torch.float32, "u8": torch.uint8}[dtype]
    xs = []
    for k in range(w):
        g = torch.Generator(device=device)
        g.manual_seed(seed0 + k)
        if dt == torch.uint8:
            v = torch.randint(0, 256, (B, S, H, D), generator=g, device=device, dtype=dt)
        else:
            v = torch.randn((B, S, H, D), generator=g, device=device, dtype=torch.float32).to(dt)
        if offset_bytes:
            n = v.numel() * v.element_size()
            raw = torch.empty(n + offset_bytes, dtype=torch.uint8, device=device)
            t = raw[offset_bytes:].view(dt).view(B, S, H, D)
            t.copy_(v)
            v = t
        xs.append(v)
    return xs


def empty_slabs(w, shape, dt, device, offset_bytes=0):
    if not offset_bytes:
        return [torch.empty(shape, dtype=dt, device=device) for _ in range(w)]
    E = torch.empty((), dtype=dt).element_size()
    n = math.prod(shape) * E
    return [torch.empty(n + offset_bytes, dtype=torch.uint8, device=device)[offset_bytes:]
            .view(dt).view(shape) for _ in range(w)]


def timed_steps(a2a, x, y, y2, z, steps, warmup, stream, chunked=0):
    """K back-to-back steps (mode 0: x -> y, mode 1: y2 -> z) between one pair of events.

    Returns (total ms, launches of our kernels in the timed region, t0, t1)."""
    for _ in range(warmup):
        a2a.run(x, 0, out=y, stream=stream, chunked=chunked)
        a2a.run(y2, 1, out=z, stream=stream, chunked=chunked)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    launches0 = a2a.launch_count
    t0 = time.perf_counter()
    e0.record(stream)
    for _ in range(steps):
        a2a.run(x, 0, out=y, stream=stream, chunked=chunked)
        a2a.run(y2, 1, out=z, stream=stream, chunked=chunked)
    e1.record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    return e0.elapsed_time(e1), a2a.launch_count - launches0, t0, t1


def timed_loop(fn, stream, min_seconds, sampler=None, warmup=3):
    """Back-to-back calls of fn (each enqueues one call on `stream`) for at least
    min_seconds of device time, between one pair of events.

    Returns (ms per call, calls timed, clock record of the timed region)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(3):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    per = max(e0.elapsed_time(e1) / 3, 1e-3)
    reps = max(3, int(math.ceil(min_seconds * 1e3 / per)))
    t0 = time.perf_counter()
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    clocks = sampler.window(t0, t1) if sampler else None
    return e0.elapsed_time(e1) / reps, reps, clocks


def graph_ms_per_call(a2a, src, dst, mode, calls, reps, stream):
    """Device time per call of `calls` back-to-back calls captured in one CUDA graph."""
    with torch.cuda.stream(stream):
        a2a.run(src, mode, out=dst, stream=stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(calls):
            a2a.run(src, mode, out=dst, stream=stream)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    # replay() launches on the current stream: make it the timed stream
    with torch.cuda.stream(stream):
        g.replay()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (reps * calls)
    del g
    return ms


def isolated_call(a2a, src, dst, mode, stream, reps, flush, acc, sampler=None):
    """Median device time (ms) of one call at a time, each after an L2 flush that
    reads `flush` (twice the L2): the flush leaves only clean lines in L2, so no
    write-back of earlier data falls inside the timed call."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps + 2)]
    with torch.cuda.stream(stream):
        t0 = time.perf_counter()
        for a, b in ev:
            acc.add_(flush.sum())
            a.record(stream)
            a2a.run(src, mode, out=dst, stream=stream)
            b.record(stream)
        torch.cuda.synchronize()
        t1 = time.perf_counter()
    times = [a.elapsed_time(b) for a, b in ev[2:]]
    return statistics.median(times), min(times), sampler.window(t0, t1) if sampler else None


def bandwidth_sweep(device, peak, payload_exps=range(17, 32), dtypes=(("bf16", 2), ("fp32", 4)),
                    ws=(2, 4, 8), sampler=None, long_payload=None, long_seconds=1.0):
    """Payloads 2^e bytes (e in payload_exps), w = 2/4/8, H = 8w, D = 128, B = 1,
    U[-1,1) values, both modes. Payloads up to 64 MiB: device time per call from
    CUDA-graph replays of back-to-back calls (a call issued from Python can take
    longer on the host than its kernel on the device); larger: back-to-back
    loops of at least 0.25 s (long_seconds for the long_payload bf16 points)."""
    from sequence_all_re_b200 import UlyssesA2A

    stream = torch.cuda.Stream(device)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    rows = []
    for dtype, E in dtypes:
        a2a = UlyssesA2A(device.index or 0, E)
        for w in ws:
            H, D = 8 * w, 128
            for k in payload_exps:
                P = 1 << k
                S = P // (w * H * D * E)
                if S < 1:
                    rows.append({"dtype": dtype, "w": w, "payload_bytes": P, "S_local": None,
                                 "note": "n/a: one sequence row across all ranks exceeds the payload"})
                    continue
                dt = torch.bfloat16 if E == 2 else torch.float32
                x = []
                for r in range(w):
                    gen = torch.Generator(device=device)
                    gen.manual_seed(1234 + r)
                    x.append((torch.rand((1, S, H, D), generator=gen, device=device) * 2 - 1).to(dt))
                y = [torch.empty((1, S * w, H // w, D), dtype=dt, device=device) for _ in range(w)]
                row = {"dtype": dtype, "w": w, "payload_bytes": P, "S_local": S,
                       "l2_assisted": 2 * P <= l2}
                for mode, (src, dst) in ((0, (x, y)), (1, (y, x))):
                    if P <= (64 << 20):         # a host-side call can take longer than the kernel
                        calls = max(1, min(64, (256 << 20) // P))
                        reps = max(3, min(50, (8 << 30) // (P * calls)))
                        ms = graph_ms_per_call(a2a, src, dst, mode, calls, reps, stream)
                        clk = None
                    else:
                        secs = long_seconds if (P == long_payload and dtype == "bf16") else 0.25
                        ms, _, clk = timed_loop(
                            lambda: a2a.run(src, mode, out=dst, stream=stream), stream, secs,
                            sampler)
                    f = fracs(P, ms, peak)
                    row[f"mode{mode}_gbs"] = f["gbs"]
                    row[f"mode{mode}_frac"] = f["frac"]
                    row[f"mode{mode}_frac_nominal"] = f["frac_nominal"]
                    if clk:
                        row[f"mode{mode}_clocks"] = clk
                rows.append(row)
                del x, y
        a2a.close()
    torch.cuda.empty_cache()
    return rows


def per_mode_block(a2a, ins, outs, back, P, stream, peak, sampler, seconds, chunked=0):
    """Mode 0 (ins -> outs) and mode 1 (outs -> back), each back to back for at
    least `seconds`: payload GB/s, fractions and the clock record per mode."""
    res = {}
    for mode, (src, dst) in ((0, (ins, outs)), (1, (outs, back))):
        ms, reps, clk = timed_loop(
            lambda: a2a.run(src, mode, out=dst, stream=stream, chunked=chunked), stream,
            seconds, sampler)
        res[f"mode{mode}"] = dict(fracs(P, ms, peak), us_per_call=round(ms * 1e3, 2), calls=reps,
                                  clocks=clk)
    return res


def vec_shape_block(device, peak, sampler, seconds=0.5):
    """The shapes TMA cannot take: each mode back to back, on the path AUTO picks
    (the staged path where 16-byte vectors cannot be used directly) and on the
    vector path forced; plan, GB/s and fractions."""
    from sequence_all_re_b200 import UlyssesA2A

    stream = torch.cuda.Stream(device)
    out = {}
    for name, shape in VEC_SHAPES.items():
        w, B, S, H, D, E, off = shape[:7]
        goff = shape[7] if len(shape) > 7 else off
        dt = {2: "bf16", 4: "fp32"}[E]
        a2a = UlyssesA2A(device.index or 0, E)
        x = make_inputs(w, B, S, H, D, dt, device, offset_bytes=off)
        y = empty_slabs(w, (B, S * w, H // w, D), x[0].dtype, device, goff)
        z = empty_slabs(w, (B, S, H, D), x[0].dtype, device, off)
        p = a2a.plan(x, 0, out=y)
        P = w * B * S * H * D * E
        res = per_mode_block(a2a, x, y, z, P, stream, peak, sampler, seconds)
        torch.cuda.synchronize()
        if not all(torch.equal(z[k], x[k]) for k in range(w)):
            raise SystemExit(f"vector-path shape {name}: round trip mismatch")
        p1 = a2a.plan(y, 1, out=z)
        out[name] = {"payload_bytes": P, "path": PATH_NAMES[p["path"]],
                     "vec_bytes": p["vec_bytes"], "peeled": p["peeled"],
                     "fixed_phase": p["fixed_phase"], "mode1_path": PATH_NAMES[p1["path"]],
                     "row_bytes": p["row_bytes"], "base_offset_bytes": off,
                     "gathered_base_offset_bytes": goff, **res}
        # the other of the two paths, forced: the vector kernel where AUTO
        # re-aligns, the staged kernel where AUTO moves narrow vectors or
        # 16-byte vectors between peeled heads and tails
        other = {3: 2, 2: 3 if (p["vec_bytes"] < 16 or p["peeled"]) else None}.get(p["path"])
        if other is not None:
            a2a.set_path(other)
            po = a2a.plan(x, 0, out=y)
            for t in z:
                t.zero_()
            forced = per_mode_block(a2a, x, y, z, P, stream, peak, sampler, seconds)
            torch.cuda.synchronize()
            if not all(torch.equal(z[k], x[k]) for k in range(w)):
                raise SystemExit(f"shape {name}: round trip mismatch ({PATH_NAMES[other]} forced)")
            out[name][f"{PATH_NAMES[other]}_forced"] = {
                "vec_bytes": po["vec_bytes"], "peeled": po["peeled"],
                **{m: {k: v for k, v in forced[m].items() if k != "clocks"} for m in forced}}
        a2a.close()
        del x, y, z
        torch.cuda.empty_cache()
    return out


def staged_forms_block(device, peak, sampler, seconds=0.5):
    """STAGED_FORM_SHAPES on the path AUTO picks, on the staged path's
    fixed-phase and per-piece forms, and on the vector path: fractions per mode."""
    from sequence_all_re_b200 import UlyssesA2A

    stream = torch.cuda.Stream(device)
    out = {}
    for name, (w, B, S, H, D, E) in STAGED_FORM_SHAPES.items():
        a2a = UlyssesA2A(device.index or 0, E)
        x = make_inputs(w, B, S, H, D, DTYPE_OF[E], device)
        y = empty_slabs(w, (B, S * w, H // w, D), x[0].dtype, device)
        z = empty_slabs(w, (B, S, H, D), x[0].dtype, device)
        P = w * B * S * H * D * E
        row = {"payload_bytes": P, "row_bytes": (H // w) * D * E}
        for label, path, knobs in (("auto", 0, {}), ("fixed_phase", 3, {}),
                                   ("per_piece", 3, {"staged_form": 1}), ("vec", 2, {})):
            a2a.set_path(path)
            a2a.set_tuning(**knobs)
            p, p1 = a2a.plan(x, 0, out=y), a2a.plan(y, 1, out=z)
            for t in z:
                t.zero_()
            res = per_mode_block(a2a, x, y, z, P, stream, peak, sampler, seconds)
            torch.cuda.synchronize()
            if not all(torch.equal(z[k], x[k]) for k in range(w)):
                raise SystemExit(f"shape {name}: round trip mismatch ({label})")
            row[label] = {"path": PATH_NAMES[p["path"]], "vec_bytes": p["vec_bytes"],
                          "fixed_phase": p["fixed_phase"], "mode1_path": PATH_NAMES[p1["path"]],
                          "mode1_fixed_phase": p1["fixed_phase"],
                          "mode0": res["mode0"]["frac"], "mode1": res["mode1"]["frac"],
                          "sm_mhz": (res["mode0"]["clocks"] or {}).get("sm_mhz")}
        out[name] = row
        a2a.close()
        del x, y, z
        torch.cuda.empty_cache()
    return out


def run_staged_forms(args):
    """The staged path's two forms and the vector path on STAGED_FORM_SHAPES
    (each mode back to back for >= 0.5 s); prints its own line."""
    if args.gpus != 1:
        raise SystemExit("--staged-forms runs on one GPU")
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    peak, peak_src = hbm_peak()
    sampler = ClockSampler(0).start()
    res = staged_forms_block(device, peak, sampler)
    sampler.stop()
    print(json.dumps({"metric": "fraction of the measured copy bandwidth per form, back to "
                                "back, 2 x payload per call",
                      "peak": peak, "peak_source": peak_src, "shapes": res}), flush=True)


def cpu_oracle_baseline(w, B, S, H, D, budget_s=12.0, E=2):
    """The oracle, as it stands, on the host cores: the OpenMP build (the outer
    (r, b) loops over every core) and the single-threaded build, each on whole
    mode 0 + mode 1 steps of a sample of the workload for about budget_s / 2."""
    import oracle
    from synth import normal_slabs

    dt = DTYPE_OF[E]
    cores_on_box = os.cpu_count() or 1
    threads = oracle.omp_threads()
    res = {}
    for kind, lib in (("openmp", oracle.omp_lib()), ("single", oracle._get_lib())):
        # size the sample from a small probe: about 1 s per step
        probe_S = min(S, 64)
        xs = normal_slabs((B, probe_S, H, D), w, dt)
        t = time.perf_counter()
        oracle.ulysses_a2a(oracle.ulysses_a2a(xs, 0, lib=lib), 1, lib=lib)
        per_row = (time.perf_counter() - t) / probe_S
        S_sample = int(max(1, min(S, 1.0 / max(per_row, 1e-9))))
        xs = normal_slabs((B, S_sample, H, D), w, dt)
        done, t_start = 0, time.perf_counter()
        while True:
            oracle.ulysses_a2a(oracle.ulysses_a2a(xs, 0, lib=lib), 1, lib=lib)
            done += 1
            if time.perf_counter() - t_start > budget_s / 2:
                break
        el = time.perf_counter() - t_start
        P = w * B * S_sample * H * D * E
        res[kind] = {"value": round(2 * P * done / el / 1e9, 4), "threads": threads if kind == "openmp" else 1,
                     "sample": f"{done} steps (mode 0 + mode 1) on S_local={S_sample} of {S} rows "
                               f"(w={w},B={B},H={H},D={D} {dt}) in {el:.1f} s"}
    return {"value": res["openmp"]["value"], "unit": "GB/s", "cores": threads, "kind": "oracle",
            "threads": threads, "cores_on_box": cores_on_box,
            "sample": "OpenMP build, outer (r, b) loops over every core: " + res["openmp"]["sample"],
            "single_thread": {"value": res["single"]["value"], "unit": "GB/s", "cores": 1,
                              "sample": res["single"]["sample"]}}


def exchange_arms(dist, device, rank, world, steps, warmup, wl, native=None):
    """The Ulysses all-to-all across the job's GPUs (w = world, one rank slab of
    the workload's per-rank shape per GPU), a step being mode 0 then mode 1:
    this library's PeerExchange and a library all-to-all (NCCL) baseline. Every
    rank takes the same steps in the same order; times are the max over ranks,
    from CUDA events on the launching stream (host timing between barriers when
    the group runs on CPU tensors, as the tests do; `native` then stands in for
    the peer object)."""
    from sequence_all_re_b200.peer import PeerExchange

    B, S, H, D = (wl[k] for k in ("B", "S_local", "H", "D"))
    if H % world:
        return {"skipped": f"H={H} is not divisible by {world} GPUs"}
    x = make_inputs(1, B, S, H, D, "bf16", device, seed0=1234 + rank)[0]
    slab = B * S * H * D * 2
    cuda = device.type == "cuda"
    stream = torch.cuda.current_stream(device) if cuda else None
    res = {"workload": f"one rank slab per GPU, w = {world}: B={B} S_local={S} H={H} D={D} bf16",
           "steps": steps}

    def sync():
        if cuda:
            torch.cuda.synchronize()

    def clock_ms(fn, n):
        """ms for n back-to-back calls of fn, the slowest rank's."""
        dist.barrier()
        sync()
        if cuda:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n):
                fn()
            e1.record(stream)
            sync()
            ms = e0.elapsed_time(e1)
        else:
            t0 = time.perf_counter()
            for _ in range(n):
                fn()
            ms = (time.perf_counter() - t0) * 1e3
        return max_over_ranks(ms, dist, device)

    def timed(step):
        for _ in range(warmup):
            z = step()
        sync()
        if not torch.equal(z, x):
            raise SystemExit("round trip mismatch across GPUs")
        return clock_ms(step, steps) / steps

    ex = (PeerExchange(device=device.index, elem_bytes=2) if native is None
          else PeerExchange(native=native, elem_bytes=2))
    ms = timed(lambda: ex.all_to_all_4d(ex.all_to_all_4d(x, 0), 1))
    # the barrier alone (on NCCL a one-element all-reduce on the stream), one per
    # exchange: 2 per step
    nb = 50
    bar_ms = clock_ms(lambda: ex._barrier(ex.native.current_stream()), nb) / nb
    ex.shutdown()
    res["peer"] = {"ms_per_step": round(ms, 4), "gbs": round(job_gbs(world, 2 * slab, 1, ms), 1),
                   "barrier_us": round(bar_ms * 1e3, 2), "barriers_per_step": 2,
                   "barrier_share": round(2 * bar_ms / ms, 4)}
    ms = timed(lambda: nccl_all_to_all_4d(nccl_all_to_all_4d(x, 0), 1))
    res["nccl"] = {"ms_per_step": round(ms, 4), "gbs": round(job_gbs(world, 2 * slab, 1, ms), 1)}
    return res


def exchange_keys(exchange):
    """The bench line's cross-GPU keys from exchange_arms' result."""
    return {"exchange_peer_gbs": exchange.get("peer", {}).get("gbs"),
            "exchange_nccl_gbs": exchange.get("nccl", {}).get("gbs"),
            "exchange": exchange}


def run_ours(args):
    rank, local_rank, world = env_rank()
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch N>1 with torchrun")
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", device_id=device, timeout=datetime.timedelta(seconds=120))

    from sequence_all_re_b200 import UlyssesA2A

    sampler = ClockSampler(local_rank).start()
    wl = ALL_WORKLOADS[args.workload]
    w, B, S, H, D, E, off, goff = (wl[k] for k in ("w", "B", "S_local", "H", "D", "E", "off",
                                                   "goff"))
    P = w * B * S * H * D * E
    a2a = UlyssesA2A(local_rank, E)
    a2a.set_path({"auto": 0, "tma": 1, "vec": 2, "staged": 3}[args.path])
    chunked = args.chunked
    stream = torch.cuda.Stream(device)
    x = make_inputs(w, B, S, H, D, DTYPE_OF[E], device, offset_bytes=off)
    y = empty_slabs(w, (B, S * w, H // w, D), x[0].dtype, device, goff)
    z = empty_slabs(w, (B, S, H, D), x[0].dtype, device, off)
    # mode 1 reads its own slabs (a seeded copy of mode 0's result), not y
    with torch.cuda.stream(stream):
        a2a.run(x, 0, out=y, stream=stream)
    torch.cuda.synchronize()
    y2 = empty_slabs(w, (B, S * w, H // w, D), x[0].dtype, device, goff)
    for a, b in zip(y2, y):
        a.copy_(b)
    plan = a2a.plan(x, 0, chunked=chunked, out=y)

    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    total_ms, launches, t0, t1 = timed_steps(a2a, x, y, y2, z, args.steps, args.warmup, stream,
                                             chunked)
    clocks = sampler.window(t0, t1)
    a2a.status(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    # the round trip must reproduce the input bit for bit (y2 holds mode 0's output)
    for k in range(w):
        if not torch.equal(z[k].view(INT_OF[E]), x[k].view(INT_OF[E])):
            raise SystemExit("round trip mismatch: mode1(mode0(x)) != x")
    total_ms = max_over_ranks(total_ms, dist, device)
    ms_per_step = total_ms / args.steps
    value = job_gbs(world, 2 * P, args.steps, total_ms)

    peak, peak_src = hbm_peak()
    avg_launch_ms = total_ms / launches
    bytes_per_launch = 2 * P * 2 * args.steps // launches       # 2 calls of 2P per step
    achieved = bytes_per_launch / (avg_launch_ms / 1e3) / 1e9
    key = workload_key(w, B, S, H, D, PATH_NAMES[plan["path"]], E, off, goff)
    traffic_bytes, traffic_src = ncu_traffic(key, plan, chunked)

    extras = {}
    if world == 1 and not args.no_extras and args.workload in WORKLOADS:
        # each mode of the headline workload, back to back for >= 1 s
        extras["per_mode"] = per_mode_block(a2a, x, y2, z, P, stream, peak, sampler, 1.0, chunked)
        # one call at a time after a clean L2 flush
        flush = torch.ones(2 * L2_BYTES // 4, dtype=torch.int32, device=device)
        acc = torch.zeros((), dtype=torch.int64, device=device)
        iso = {args.workload: {}}
        for mode, (src, dst) in ((0, (x, y)), (1, (y, z))):
            med, mn, clk = isolated_call(a2a, src, dst, mode, stream, 40, flush, acc, sampler)
            iso[args.workload][f"mode{mode}"] = dict(fracs(P, med, peak),
                                                     us_median=round(med * 1e3, 2),
                                                     us_min=round(mn * 1e3, 2), clocks=clk)
        del y2, z
        torch.cuda.empty_cache()
        # the other single-GPU workloads
        wls = {}
        for name, variants in (("w4_S8192_H24_D128", ((0, 1.0),)),
                               ("w4_B4_S16384_H32_D64", ((0, 0.5), (1, 0.5), (2, 0.5)))):
            v = WORKLOADS[name]
            ww, BB, SS, HH, DD = (v[k] for k in ("w", "B", "S_local", "H", "D"))
            PP = ww * BB * SS * HH * DD * E
            xa = make_inputs(ww, BB, SS, HH, DD, "bf16", device)
            ya = [torch.empty((BB, SS * ww, HH // ww, DD), dtype=torch.bfloat16, device=device)
                  for _ in range(ww)]
            za = [torch.empty_like(t) for t in xa]
            entry = {"payload_bytes": PP}
            for ch, secs in variants:
                entry[{0: "unchunked", 1: "chunked_per_plane", 2: "chunked_window"}[ch]] = \
                    per_mode_block(a2a, xa, ya, za, PP, stream, peak, sampler, secs, ch)
            torch.cuda.synchronize()
            if not all(torch.equal(za[k], xa[k]) for k in range(ww)):
                raise SystemExit(f"{name}: round trip mismatch")
            if name == "w4_S8192_H24_D128":
                iso[name] = {}
                for mode, (src, dst) in ((0, (xa, ya)), (1, (ya, za))):
                    med, mn, clk = isolated_call(a2a, src, dst, mode, stream, 40, flush, acc,
                                                 sampler)
                    iso[name][f"mode{mode}"] = dict(fracs(PP, med, peak),
                                                    us_median=round(med * 1e3, 2),
                                                    us_min=round(mn * 1e3, 2), clocks=clk)
            wls[name] = entry
            del xa, ya, za
            torch.cuda.empty_cache()
        del flush
        extras["isolated_call"] = iso
        extras["workloads"] = wls
        # compact bandwidth sweep: 1 MiB, 64 MiB, 512 MiB, 2 GiB
        if not args.no_sweep:
            sweep = bandwidth_sweep(device, peak, payload_exps=(20, 26, 29, 31), sampler=sampler,
                                    long_payload=512 << 20, long_seconds=1.0)
            extras["sweep"] = sweep
            extras["w_sweep_512MiB"] = {
                f"w{r['w']}": {k: r[k] for k in r if k.startswith("mode") or k == "payload_bytes"}
                for r in sweep if r["dtype"] == "bf16" and r["payload_bytes"] == 512 << 20}
        extras["vec_shapes"] = vec_shape_block(device, peak, sampler)

    # e2e: the same step through the host-buffer entry point (pinned host slabs)
    e2e = None
    if not args.no_e2e:
        hx = [t.cpu().pin_memory() for t in x]
        hy = [torch.empty((B, S * w, H // w, D), dtype=x[0].dtype).pin_memory() for _ in range(w)]
        hz = [torch.empty_like(t).pin_memory() for t in hx]
        for _ in range(2):
            a2a.run_host(hx, 0, out=hy, stream=stream)
            a2a.run_host(hy, 1, out=hz, stream=stream)
        e_steps = max(3, min(args.e2e_steps, args.steps))
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        ea = torch.cuda.Event(enable_timing=True)
        eb = torch.cuda.Event(enable_timing=True)
        ta = time.perf_counter()
        ea.record(stream)
        for _ in range(e_steps):
            a2a.run_host(hx, 0, out=hy, stream=stream)
            a2a.run_host(hy, 1, out=hz, stream=stream)
        eb.record(stream)
        torch.cuda.synchronize()
        tb = time.perf_counter()
        e_ms = max_over_ranks(ea.elapsed_time(eb), dist, device)
        for k in range(w):
            if not torch.equal(hz[k].view(INT_OF[E]), hx[k].view(INT_OF[E])):
                raise SystemExit("host-path round trip mismatch")
        e2e = {"value": round(job_gbs(world, 2 * P, e_steps, e_ms), 3), "unit": "GB/s",
               "h2d_bytes_per_step": 2 * P, "d2h_bytes_per_step": 2 * P,
               "steps": e_steps, "via": "ulysses_a2a_run_host, pinned host slabs",
               "clocks": sampler.window(ta, tb)}
        del hx, hy, hz

    exchange = None
    if world > 1 and not args.no_exchange:
        # the exchange arms run after `value` is taken; an error that every rank
        # meets (a window that cannot be mapped, say) is recorded in the line
        # instead of losing it
        try:
            exchange = exchange_arms(dist, device, rank, world, min(args.steps, 200),
                                     max(3, args.warmup), wl)
        except Exception as e:          # noqa: BLE001 (reported in the line)
            exchange = {"error": f"{type(e).__name__}: {e}"[:300]}

    full_sweep = None
    if args.sweep and rank == 0:
        full_sweep = bandwidth_sweep(device, peak, sampler=sampler)

    sampler.stop()
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_baseline(w, B, S, H, D, budget_s=args.cpu_budget, E=E)

    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": DTYPE_OF[E],
        "data": "synthetic",
        "config": {
            "workload": workload_name(w, B, S, H, D, chunked, E, off, goff),
            "name": args.workload,
            "w": w, "B": B, "S_local": S, "H": H, "D": D,
            "payload_bytes_per_call": P,
            "path": PATH_NAMES[plan["path"]],
            "rows_per_tile": plan["rows_per_tile"], "producers": plan["producers"],
            "stages": plan["stages"], "chunk_units": plan["chunk_units"], "grid": plan["grid"],
            "l2": (f"inputs larger than L2 ({P / 2**20:.0f} MiB per call vs 126 MB); no kernel "
                   "reads data the previous kernel touched; no flush in the timed region")
                  if P > L2_BYTES else
                  "L2-assisted: the inputs fit in L2 (below 126 MB); no flush",
            "parallelism": f"{world} independent instance(s), one per GPU",
        },
        "roofline": {
            "bound": "hbm",
            "kernel": {1: "ua2a_tma_kernel<0>/<1>", 2: "ua2a_vec_kernel",
                       3: "ua2a_stage_kernel"}[plan["path"]],
            "achieved": round(achieved, 1),
            "peak": peak,
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "frac_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
            "peak_source": peak_src,
            "algorithmic_bytes_per_launch": bytes_per_launch,
            "avg_launch_us": round(avg_launch_ms * 1e3, 3),
            "traffic": traffic_bytes,
            "traffic_source": traffic_src,
            **({"note": "chunked = 2 also copies every plane into the staging window: the "
                        "bytes actually moved are twice the algorithmic bytes"}
               if chunked == 2 else {}),
        },
        "gpu_launches": launches,
        "e2e": e2e,
        "clocks": clocks,
        **extras,
        "cpu_baseline": cpu,
    }
    if exchange is not None:
        line.update(exchange_keys(exchange))
    if full_sweep is not None:
        line["bandwidth_sweep"] = full_sweep
    if rank == 0:
        print(json.dumps(line), flush=True)
    a2a.close()
    if dist:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------- cross-GPU exchange kernels, one GPU
def run_peer_one_gpu(args):
    """The multi-GPU exchange's kernels with the w ranks as contexts on one GPU.

    Each step is, for mode 0 and then mode 1: every rank publishes its slab into
    its window, then every rank pulls its output slab from all windows (stream
    order stands in for the barriers). On one GPU the pulls' "peer" loads are
    local, so this times the two kernels against HBM, not NVLink.
    """
    from sequence_all_re_b200 import UlyssesA2A, _lib

    if args.gpus != 1:
        raise SystemExit("--peer-one-gpu runs on one GPU")
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    wl = WORKLOADS[args.workload]
    w, B, S, H, D = (wl[k] for k in ("w", "B", "S_local", "H", "D"))
    E = 2
    slab = B * S * H * D * E
    P = w * slab
    ctxs = [UlyssesA2A(0, E) for _ in range(w)]
    peers, recs = [], []
    for k in range(w):
        rc, h, rec = _lib.ulysses_a2a_peer_create(ctxs[k]._ctx, k, w, slab)
        if rc != _lib.OK:
            raise SystemExit("peer_create: " + ctxs[k].last_error())
        peers.append(h)
        recs.append(rec)
    for k in range(w):
        if _lib.ulysses_a2a_peer_open(peers[k], recs) != _lib.OK:
            raise SystemExit("peer_open: " + ctxs[k].last_error())
    x = make_inputs(w, B, S, H, D, "bf16", device)
    y = [torch.empty((B, S * w, H // w, D), dtype=torch.bfloat16, device=device) for _ in range(w)]
    z = [torch.empty_like(t) for t in x]
    stream = torch.cuda.Stream(device)
    st = stream.cuda_stream

    def publish(src, mode):
        for k in range(w):
            if _lib.ulysses_a2a_peer_publish(peers[k], src[k].data_ptr(), B, S, H, D, mode, 0,
                                             st) != _lib.OK:
                raise SystemExit("peer_publish: " + ctxs[k].last_error())

    def pull(dst, mode):
        for k in range(w):
            if _lib.ulysses_a2a_peer_pull(peers[k], dst[k].data_ptr(), B, S, H, D, mode, 0,
                                          st) != _lib.OK:
                raise SystemExit("peer_pull: " + ctxs[k].last_error())

    def step():
        publish(x, 0)
        pull(y, 0)
        publish(y, 1)
        pull(z, 1)

    def timed(fn, reps):
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                fn()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                fn()
            b.record(stream)
            b.synchronize()
        return a.elapsed_time(b) / reps

    steps = min(args.steps, 500)
    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    if not all(torch.equal(z[k], x[k]) for k in range(w)):
        raise SystemExit("round trip mismatch through the peer windows")
    n0 = sum(c.launch_count for c in ctxs)
    with torch.cuda.stream(stream):
        step()
    per_step = sum(c.launch_count for c in ctxs) - n0      # kernel launches of one step
    sampler = ClockSampler(0)
    sampler.start()
    ms_step = timed(step, steps)
    clocks = sampler.stop()
    launches = per_step * steps
    ms_pub = timed(lambda: publish(x, 0), steps)
    ms_pull0 = timed(lambda: pull(y, 0), steps)
    ms_pull1 = timed(lambda: pull(z, 1), steps)
    peak, peak_src = hbm_peak()

    def roof(ms_group):
        # w launches per group, each reading and writing one slab
        us = ms_group * 1e3 / w
        ach = 2 * slab / (us / 1e6) / 1e9
        return {"bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
                "frac": round(ach / peak, 4), "avg_launch_us": round(us, 3),
                "algorithmic_bytes_per_launch": 2 * slab}

    line = {
        "metric": "Ulysses all-to-all payload throughput through the peer-window exchange "
                  "(w ranks as contexts on one GPU)",
        "value": round(2 * P / (ms_step / 1e3) / 1e9, 1), "unit": "GB/s", "n_gpus": 1,
        "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_name(w, B, S, H, D, 0) + "; publish + pull per rank",
                   "l2": "inputs larger than L2 (back to back)"},
        "gpu_launches": launches,
        # inputs written into the windows in place (PeerExchange.input_buffer):
        # the step is the two pull groups alone, timed above
        "in_place_value": round(2 * P / ((ms_pull0 + ms_pull1) / 1e3) / 1e9, 1),
        "kernels": {"publish (one-rank re-layout into the own window)": roof(ms_pub),
                    "pull mode 0 (VEC, one output slab)": roof(ms_pull0),
                    "pull mode 1 (VEC, one output slab)": roof(ms_pull1)},
        "peak_source": peak_src,
        "clocks": clocks,
        "note": "each step moves every byte twice (publish + pull) per mode; value counts "
                "the payload 2P once per mode, as the main bench line does",
    }
    for h in peers:
        _lib.ulysses_a2a_peer_close(h)
    for h in peers:
        _lib.ulysses_a2a_peer_destroy(h)
    for c in ctxs:
        c.close()
    print(json.dumps(line), flush=True)


# --------------------------------------------- head-packed q, k, v in one launch
def run_packed(args):
    """q, k and v of the chosen workload's shape, packed [B, S_local, 3, H, D] per
    rank: one packed launch (run_packed) against three launches on the
    row-pitched per-tensor views (run), back to back."""
    from sequence_all_re_b200 import UlyssesA2A

    if args.gpus != 1:
        raise SystemExit("--packed runs on one GPU")
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    wl = WORKLOADS[args.workload]
    w, B, S, H, D = (wl[k] for k in ("w", "B", "S_local", "H", "D"))
    T, E = 3, 2
    P = T * w * B * S * H * D * E
    a2a = UlyssesA2A(0, E)
    stream = torch.cuda.Stream(device)
    g = torch.Generator(device=device)
    g.manual_seed(1234)
    packed = [torch.randn((B, S, T, H, D), generator=g, device=device).to(torch.bfloat16)
              for _ in range(w)]
    outs = [[torch.empty((B, S * w, H // w, D), dtype=torch.bfloat16, device=device)
             for _ in range(w)] for _ in range(T)]
    ref = [[torch.empty_like(o) for o in per_t] for per_t in outs]

    def one():
        a2a.run_packed(packed, 0, out=outs, stream=stream)

    def three():
        for t in range(T):
            a2a.run([x[:, :, t] for x in packed], 0, out=ref[t], stream=stream)

    def timed(fn, reps):
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                fn()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                fn()
            e1.record(stream)
            e1.synchronize()
        return e0.elapsed_time(e1) / reps

    reps = min(args.steps, 500)
    n0 = a2a.launch_count
    with torch.cuda.stream(stream):
        one()
    per_call = a2a.launch_count - n0          # kernel launches of one packed call
    ms_one = timed(one, reps)
    ms_three = timed(three, reps)
    torch.cuda.synchronize()
    if not all(torch.equal(outs[t][r], ref[t][r]) for t in range(T) for r in range(w)):
        raise SystemExit("packed launch differs from the per-tensor launches")
    peak, peak_src = hbm_peak()
    line = {
        "metric": "q, k, v Ulysses re-layout (mode 0) payload throughput: one packed launch",
        "value": round(P / (ms_one / 1e3) / 1e9, 1), "unit": "GB/s", "n_gpus": 1,
        "steps": reps, "warmup": args.warmup, "ms_per_step": round(ms_one, 4),
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"q, k, v packed [B, S_local, 3, H, D]: w={w} B={B} "
                               f"S_local={S} H={H} D={D} bf16, mode 0",
                   "l2": "inputs larger than L2 (back to back)"},
        "gpu_launches": per_call * reps,
        "frac_of_copy": round(2 * P / (ms_one / 1e3) / 1e9 / peak, 4),
        "three_launches": {"ms": round(ms_three, 4),
                           "value": round(P / (ms_three / 1e3) / 1e9, 1),
                           "frac_of_copy": round(2 * P / (ms_three / 1e3) / 1e9 / peak, 4)},
        "peak_source": peak_src,
    }
    a2a.close()
    print(json.dumps(line), flush=True)


# ------------------------------------- cross-GPU exchange arms (torchrun, N > 1)
def nccl_all_to_all_4d(x, mode, group=None):
    """The comparison arm: the same element map as a library all-to-all.

    mode 0: this rank's x [B, S_local, H, D] -> [B, S_local*w, H/w, D]; mode 1
    the inverse. Head group r is packed contiguous for rank r, exchanged with
    torch.distributed.all_to_all_single, and the received blocks are laid out
    rank-major. Plain torch ops and one collective: a baseline, not this
    library's path."""
    import torch.distributed as dist

    w = dist.get_world_size(group)
    if mode == 0:
        B, S, H, D = x.shape
        send = x.reshape(B, S, w, H // w, D).permute(2, 0, 1, 3, 4).contiguous()   # [r, b, s, h', d]
        recv = torch.empty_like(send)                                               # [j, b, s, h', d]
        dist.all_to_all_single(recv, send, group=group)
        return recv.permute(1, 0, 2, 3, 4).reshape(B, w * S, H // w, D)
    B, Sg, Hw, D = x.shape
    S = Sg // w
    send = x.reshape(B, w, S, Hw, D).permute(1, 0, 2, 3, 4).contiguous()           # [j, b, s, h', d]
    recv = torch.empty_like(send)                                                   # [r, b, s, h', d]
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 2, 0, 3, 4).reshape(B, S, w * Hw, D)


def run_exchange(args):
    """Time the Ulysses all-to-all across the GPUs of a torchrun job: each rank
    holds one rank slab of the workload (w = the number of GPUs); a step is
    mode 0 then mode 1. --exchange nccl times the library all-to-all above,
    --exchange peer this library's PeerExchange (windows, peer loads)."""
    import datetime
    import torch.distributed as dist

    rank, local_rank, world = env_rank()
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch N>1 with torchrun")
    if world == 1:          # a one-rank group without torchrun (the exchange is then a copy)
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29511")
        os.environ.setdefault("RANK", "0")
        os.environ.setdefault("WORLD_SIZE", "1")
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist.init_process_group("nccl", device_id=device, timeout=datetime.timedelta(seconds=120))
    wl = WORKLOADS[args.workload]
    B, S, H, D = (wl[k] for k in ("B", "S_local", "H", "D"))
    if H % world:
        raise SystemExit(f"H={H} is not divisible by {world} GPUs")
    x = make_inputs(1, B, S, H, D, "bf16", device, seed0=1234 + rank)[0]
    ex = None
    if args.exchange == "peer":
        from sequence_all_re_b200.peer import PeerExchange
        ex = PeerExchange(device=local_rank, elem_bytes=2)

        def step():
            return ex.all_to_all_4d(ex.all_to_all_4d(x, 0), 1)
    else:
        def step():
            return nccl_all_to_all_4d(nccl_all_to_all_4d(x, 0), 1)

    stream = torch.cuda.current_stream(device)
    for _ in range(args.warmup):
        z = step()
    if not torch.equal(z, x):
        raise SystemExit("round trip mismatch across GPUs")
    steps = min(args.steps, 200)
    dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), dist, device)
    slab = B * S * H * D * 2
    if rank == 0:
        print(json.dumps({
            "metric": "Ulysses all-to-all across GPUs: payload GB/s per step (mode 0 + mode 1)",
            "value": round(job_gbs(world, 2 * slab, steps, ms), 1), "unit": "GB/s",
            "n_gpus": world, "steps": steps, "warmup": args.warmup,
            "ms_per_step": round(ms / steps, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "exchange": args.exchange,
            "config": {"workload": f"one rank slab per GPU, w = {world}: B={B} S_local={S} H={H} "
                                   f"D={D} bf16", "parallelism": f"ulysses sp{world}"}}),
            flush=True)
    if ex is not None:
        ex.shutdown()
    dist.barrier()
    dist.destroy_process_group()




# ------------------------------------------------------------ schedule sweep
TUNING_SWEEP = [
    # (label, path, knobs): the default schedule, then one knob changed at a time
    ("default", "auto", {}),
    ("persistent grid, 4 producers x 4 stages", "tma", dict(chunk_units=0)),
    ("persistent grid, 1 producer x 4 stages", "tma", dict(chunk_units=0, producers=1, stages=4)),
    ("persistent grid, 8 producers x 2 stages", "tma", dict(chunk_units=0, producers=8, stages=16)),
    ("destination rank outermost", "tma", dict(order=0)),
    ("residency cap 8 CTAs/SM", "tma", dict(ctas_per_sm=8)),
    ("residency cap 11 CTAs/SM", "tma", dict(ctas_per_sm=11)),
    ("residency cap 16 CTAs/SM", "tma", dict(ctas_per_sm=16)),
    ("residency cap 20 CTAs/SM", "tma", dict(ctas_per_sm=20)),
    ("2 producers per CTA, cap 7", "tma", dict(producers=2, chunk_units=2, ctas_per_sm=7)),
    ("12 KB tiles (8 rows of 1.5 KB), cap 9", "tma", dict(rows_per_tile=8, ctas_per_sm=9)),
    ("vector path, 12 KB units", "vec", {}),
    ("vector path, grid-stride 16 CTAs/SM", "vec", dict(ctas_per_sm=16)),
    ("vector path, 4 KB units", "vec", dict(rows_per_tile=3)),
]


def run_tuning_sweep(args):
    """Each schedule of TUNING_SWEEP on w4_S8192_H24_D128 and the headline
    workload, both modes back to back (>= 0.5 s each): the measurements behind
    the default schedule, re-run from one command."""
    from sequence_all_re_b200 import UlyssesA2A

    if args.gpus != 1:
        raise SystemExit("--tuning-sweep runs on one GPU")
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    peak, peak_src = hbm_peak()
    sampler = ClockSampler(0).start()
    stream = torch.cuda.Stream(device)
    res = {}
    for name in ("w4_S8192_H24_D128", DEFAULT_WORKLOAD):
        v = WORKLOADS[name]
        w, B, S, H, D = (v[k] for k in ("w", "B", "S_local", "H", "D"))
        P = w * B * S * H * D * 2
        x = make_inputs(w, B, S, H, D, "bf16", device)
        y = [torch.empty((B, S * w, H // w, D), dtype=torch.bfloat16, device=device)
             for _ in range(w)]
        z = [torch.empty_like(t) for t in x]
        a2a = UlyssesA2A(0, 2)
        rows = []
        for label, path, knobs in TUNING_SWEEP:
            a2a.set_path({"auto": 0, "tma": 1, "vec": 2}[path])
            a2a.set_tuning(**knobs)
            p = a2a.plan(x, 0, out=y)
            pm = per_mode_block(a2a, x, y, z, P, stream, peak, sampler, 0.5)
            rows.append({"schedule": label, "knobs": knobs, "path": PATH_NAMES[p["path"]],
                         "grid": p["grid"], "block": p["block"], "rows_per_tile": p["rows_per_tile"],
                         "smem_bytes": p["smem_bytes"],
                         "mode0_frac": pm["mode0"]["frac"], "mode1_frac": pm["mode1"]["frac"],
                         "sm_mhz": (pm["mode0"]["clocks"] or {}).get("sm_mhz"),
                         "reasons": (pm["mode0"]["clocks"] or {}).get("reasons")})
        torch.cuda.synchronize()
        if not all(torch.equal(z[k], x[k]) for k in range(w)):
            raise SystemExit(f"{name}: round trip mismatch")
        res[name] = rows
        a2a.close()
        del x, y, z
        torch.cuda.empty_cache()
    sampler.stop()
    print(json.dumps({"metric": "fraction of the measured copy bandwidth per schedule, "
                                "back to back, 2 x payload per call",
                      "peak": peak, "peak_source": peak_src, "workloads": res}), flush=True)


# ---------------------------------------------------------------- reference arm
def run_reference(args):
    """The CPU oracle, as it stands, on the host cores: the OpenMP build over
    every core, each step mode 0 + mode 1 on a sample of the workload sized so
    that warm-up and timed steps end in about two minutes; the single-threaded
    build is timed on a short sample beside it."""
    rank, _, world = env_rank()
    if rank != 0:
        return
    import oracle
    from synth import normal_slabs

    wl = ALL_WORKLOADS[args.workload]
    w, B, S, H, D, E = (wl[k] for k in ("w", "B", "S_local", "H", "D", "E"))
    dt = DTYPE_OF[E]
    lib = oracle.omp_lib()
    threads = oracle.omp_threads()

    def step(xs, which):
        return oracle.ulysses_a2a(oracle.ulysses_a2a(xs, 0, lib=which), 1, lib=which)

    def per_row(which):
        probe_S = min(S, 64)
        xs = normal_slabs((B, probe_S, H, D), w, dt)
        t = time.perf_counter()
        step(xs, which)
        return (time.perf_counter() - t) / probe_S

    budget = min(4.0, 120.0 / max(1, args.steps + args.warmup))
    S_sample = int(max(1, min(S, budget / max(per_row(lib), 1e-9))))
    xs = normal_slabs((B, S_sample, H, D), w, dt)
    for _ in range(args.warmup):
        step(xs, lib)
    times = []
    for _ in range(args.steps):
        t = time.perf_counter()
        step(xs, lib)
        times.append(time.perf_counter() - t)
    P = w * B * S_sample * H * D * E
    total = sum(times)
    value = 2 * P * args.steps / total / 1e9
    # the single-threaded build, on a sample of about 4 s
    single = oracle._get_lib()
    S1 = int(max(1, min(S, 4.0 / max(per_row(single), 1e-9))))
    xs1 = normal_slabs((B, S1, H, D), w, dt)
    t = time.perf_counter()
    step(xs1, single)
    t1 = time.perf_counter() - t
    single_value = 2 * (w * B * S1 * H * D * E) / t1 / 1e9
    sample = (f"each step: mode 0 + mode 1 on S_local={S_sample} of {S} rows "
              f"(w={w},B={B},H={H},D={D} {dt}), OpenMP build of the C nested loops, outer "
              f"(r, b) loops over {threads} threads")
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total / args.steps * 1e3 * (S / S_sample), 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": dt,
        "data": "synthetic",
        "config": {"workload": workload_name(w, B, S, H, D, 0, E, wl["off"], wl["goff"]),
                   "name": args.workload,
                   "w": w, "B": B, "S_local": S, "H": H, "D": D},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                         "kind": "oracle", "sample": sample, "threads": threads,
                         "cores_on_box": os.cpu_count() or 1,
                         "single_thread": {"value": round(single_value, 4), "unit": "GB/s",
                                           "cores": 1,
                                           "sample": f"one step on S_local={S1} of {S} rows"}},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "note": "ms_per_step is scaled from the sample to the full workload",
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget", type=float, default=16.0,
                    help="seconds of CPU oracle timing, split over its two builds")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="only the headline step (no per-mode, isolated-call, other-workload, "
                         "sweep or vector-shape sections)")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the compact bandwidth sweep of the extra sections")
    ap.add_argument("--no-exchange", action="store_true",
                    help="with N > 1 GPUs, skip the cross-GPU exchange arms")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=sorted(ALL_WORKLOADS), default=DEFAULT_WORKLOAD,
                    help="benchmark workload, named by its sizes (default %(default)s)")
    ap.add_argument("--path", choices=["auto", "tma", "vec", "staged"], default="auto")
    ap.add_argument("--chunked", type=int, choices=[0, 1, 2], default=0)
    ap.add_argument("--sweep", action="store_true",
                    help="also run the full 128 KiB..2 GiB bandwidth sweep (w=2/4/8, bf16/fp32)")
    ap.add_argument("--exchange", choices=["nccl", "peer"], default=None,
                    help="multi-GPU Ulysses exchange (one rank slab per GPU, under torchrun): "
                         "nccl = a library all-to-all baseline, peer = this library's "
                         "PeerExchange (prints its own line)")
    ap.add_argument("--packed", action="store_true",
                    help="time q, k, v in one packed launch against three per-tensor launches "
                         "(prints its own line)")
    ap.add_argument("--tuning-sweep", action="store_true",
                    help="time the schedule knobs one at a time on two workloads (prints its "
                         "own line)")
    ap.add_argument("--staged-forms", action="store_true",
                    help="time the staged path's fixed-phase and per-piece forms and the "
                         "vector path on dense narrow-run shapes (prints its own line)")
    ap.add_argument("--peer-one-gpu", action="store_true",
                    help="time the multi-GPU exchange's publish and pull kernels with the w "
                         "ranks as contexts on one GPU (prints its own line)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("note: warm-up raised to 3 steps", file=sys.stderr)
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.exchange:
        run_exchange(args)
    elif args.peer_one_gpu:
        run_peer_one_gpu(args)
    elif args.packed:
        run_packed(args)
    elif args.tuning_sweep:
        run_tuning_sweep(args)
    elif args.staged_forms:
        run_staged_forms(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
