#!/usr/bin/env python
"""Throughput of the DART layer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dart|reference]

Headline workload: the bf16 layer forward at training length (B=2, L=8192,
H=32, P=64, N=128, S=256; 16384 tokens per step), inputs resident in HBM.  A
step is one `dart_ssd_chunk_scan` + one `dart_sma_forward` (scan, chunk
memories, state-memory attention, gated residual).  Beside it the decode
workload (64 sequences x 128 cached chunk memories, 256 consecutive steps with
the append on the last) is timed as its own region and reported under
"decode".  Rank 0 prints one JSON line.

Timing: CUDA events on the launching stream, W untimed warm-up steps, K timed
steps between a barrier + device synchronisation on both sides, max over
ranks.  Per-step inputs (272 MiB) exceed the 126 MB L2, so no flush is needed
between steps.  The roofline fraction is the SMA kernel's algorithmic rate
over the measured peak in MEASURED_PEAKS.json.

--impl reference times the fp64 CPU oracle (the only reference there is) on
a bounded sample of the same workload, on this host's cores.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from mamba_ssd_state_b200 import synth  # noqa: E402

FWD = synth.TRAIN_L8K
DEC = synth.DECODE_64x32K
METRIC = "DART layer fwd tokens/s at L=8K (% BF16 peak); decode tokens/s (% HBM BW)"


def fwd_config(world: int) -> dict:
    """The headline workload's `config`, the same object on both arms."""
    return {"workload": "dart_layer_fwd_L8k", "batch": FWD.batch, "seqlen": FWD.seqlen, "nheads": FWD.nheads,
            "headdim": FWD.headdim, "dstate": FWD.dstate, "chunk": FWD.chunk, "ngroups": 1,
            "parallelism": f"dp{world}", "l2": "inputs larger than L2 (272 MiB per step)"}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
SMS = 148
FP32_LANES_PER_SM = 128


def parse():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=("dart", "reference"), default="dart")
    p.add_argument("--no-decode", action="store_true", help="skip the decode region")
    p.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end region")
    p.add_argument("--no-cpu-baseline", action="store_true", help="skip timing the oracle")
    p.add_argument("--no-partial", action="store_true",
                   help="skip the forward with a partial last chunk (L = 8092)")
    p.add_argument("--no-decayed", action="store_true",
                   help="skip the forward with decayed memories (dart_sma_forward_decayed)")
    p.add_argument("--no-e4m3", action="store_true", help="skip the decode with an E4M3 cache")
    p.add_argument("--decode-steps", type=int, default=DEC.nsteps)
    p.add_argument("--decode-nseq", type=int, default=DEC.nseq,
                   help="sequences in the decode batch (a smaller cache for profiling)")
    p.add_argument("--no-configs", action="store_true",
                   help="skip the other forward workloads (B=4, L=2048 and B=1, L=65536)")
    p.add_argument("--no-backward", action="store_true", help="skip the backward region")
    p.add_argument("--backward-heads", type=int, default=0,
                   help="heads of the backward region (0: the forward's); a smaller case for profiling")
    p.add_argument("--reference-heads", type=int, default=0,
                   help="heads per reference-arm step (default: one per host core, at most 32)")
    return p.parse_args()


def captured_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from profiles/traffic.txt, or None if
    absent or if its source files changed since the capture."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    for line in open(path):
        if line.startswith("#") or "|" not in line:
            continue
        name, files, sha, nbytes = [f.strip() for f in line.split("|")[:4]]
        if name != kernel:
            continue
        m = hashlib.sha256()
        try:
            for f in files.split(","):
                with open(os.path.join(ROOT, f), "rb") as fh:
                    m.update(fh.read())
        except OSError:
            return None
        return float(nbytes) if m.hexdigest()[:16] == sha else None
    return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# algorithmic work (only what the method needs: masked pairs excluded)
# ---------------------------------------------------------------------------
def sma_flops(s: synth.LayerShape) -> float:
    """4*N*P per valid (token, earlier chunk) pair per head: 2NP for Q^T dH and
    2NP for C^T dH.  A token of chunk k pairs with k memories (S C(C-1)/2
    pairs per (b, h) when L = C S)."""
    pairs = sum(min(s.chunk, s.seqlen - k * s.chunk) * k for k in range(s.nchunks))
    return 4.0 * s.dstate * s.headdim * pairs * s.batch * s.nheads


def ssd_flops(s: synth.LayerShape) -> float:
    """Lower-triangular C B^T once per chunk (ngroups = 1), the causal intra
    block per (chunk, head), the chunk memory per (chunk, head) and the
    inter-chunk output per (chunk >= 1, head)."""
    S, N, P, C, H, B = s.chunk, s.dstate, s.headdim, s.nchunks, s.nheads, s.batch
    per_b = C * S * (S + 1) * N + C * H * S * (S + 1) * P + C * H * 2 * S * N * P + (C - 1) * H * 2 * S * N * P
    return float(B * per_b)


def decode_bytes(d: synth.DecodeShape, n: int, append: bool, e4m3: bool = False) -> float:
    """Bytes one decode step must move: every cached memory once, the float32
    state and running contribution read and written, the token inputs, the
    output, and the appended memory when the step closes a chunk.  An E4M3
    cache holds 1 byte per element plus 1 exponent byte per row."""
    esz = 2 if d.dtype == "bf16" else 4
    mem = d.dstate * d.headdim * esz if not e4m3 else d.dstate * (d.headdim + 1)
    per_sh = n * mem + 4 * d.dstate * d.headdim * 4
    per_sh += (2 * d.headdim + d.dstate) * esz + 4 + d.headdim * 4
    per_seq = d.nheads * per_sh + 2 * d.dstate * esz
    total = d.nseq * per_seq
    if append:
        total += d.nseq * d.nheads * mem
    return float(total)


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU.

    Two sources: `nvidia-smi -lms 100` over the whole window (start .. stop),
    and an NVML poll every millisecond from a thread that keeps only the
    samples taken between begin() and end(), the timed region (a region of
    a few milliseconds falls between two nvidia-smi samples).  The median
    clock is taken from the in-region NVML samples when there are any; the
    reasons are the union of both sources.  The GPU is found by its UUID."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits, in the order of the names reported
    REASON_BITS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
                   ("sw_power_cap", 0x4))

    def __init__(self, index: int, uuid: str | None = None, nvml=None):
        self.index = index
        self.uuid = uuid
        self.proc = None
        self.path = None
        self.nvml = nvml
        self.handle = None
        self.thread = None
        self.active = False
        self.running = False
        self.samples = []     # (sm MHz, reason bits, power W) inside the region

    @staticmethod
    def device_uuid(dev: torch.device) -> str | None:
        try:
            u = str(torch.cuda.get_device_properties(dev).uuid)
            return u if u.startswith("GPU-") else "GPU-" + u
        except (AttributeError, RuntimeError):
            return None

    def _open_nvml(self):
        try:
            if self.nvml is None:
                import pynvml
                self.nvml = pynvml
            self.nvml.nvmlInit()
            try:
                self.handle = self.nvml.nvmlDeviceGetHandleByUUID(self.uuid) if self.uuid else None
            except Exception:
                self.handle = None
            if self.handle is None:
                self.uuid = None
                self.handle = self.nvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = float(self.nvml.nvmlDeviceGetMaxClockInfo(self.handle, self.nvml.NVML_CLOCK_SM))
        except Exception:   # no NVML: nvidia-smi alone
            self.handle = None

    def _poll(self):
        nv, h = self.nvml, self.handle
        while self.running:
            if self.active:
                try:
                    self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                         int(nv.nvmlDeviceGetCurrentClocksEventReasons(h)),
                                         nv.nvmlDeviceGetPowerUsage(h) / 1000.0))
                except Exception:
                    self.running = False
                    break
            time.sleep(0.001)

    def start(self):
        self._open_nvml()
        # the UUID names the GPU for nvidia-smi too, once NVML has accepted it
        target = self.uuid if (self.handle is not None and self.uuid) else str(self.index)
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", target, f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        if self.handle is not None:
            import threading
            self.running = True
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()

    def begin(self):
        self.active = True

    def end(self):
        self.active = False

    def stop(self) -> dict:
        self.active = False
        if self.thread is not None:
            self.running = False
            self.thread.join(timeout=5)
        rows = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
            os.unlink(self.path)
        if not rows and not self.samples:
            why = "nvidia-smi unavailable" if self.proc is None else "no samples"
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [why]}
        names = [n for n, _ in self.REASON_BITS]
        reasons = {names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"}
        reasons |= {n for (_, bits, _) in self.samples for n, b in self.REASON_BITS if bits & b}
        sm_smi = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        sm_in = [c for c, _, _ in self.samples]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        if self.handle is not None:
            mx.append(self.max_mhz)
        power = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()] + [w for _, _, w in self.samples]
        sm = sm_in or sm_smi
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows) + len(self.samples),
                "region_samples": len(self.samples), "power_w_max": max(power, default=None)}


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU; weak scaling, no data-path collective)
# ---------------------------------------------------------------------------
class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import torch.distributed as dist
            backend = "nccl" if torch.cuda.is_available() else "gloo"
            if backend == "nccl":
                torch.cuda.set_device(self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg:
            if torch.cuda.is_available():
                self.pg.barrier(device_ids=[self.local])
            else:
                self.pg.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        dev = torch.device("cuda", self.local) if torch.cuda.is_available() else torch.device("cpu")
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ---------------------------------------------------------------------------
# GPU regions
# ---------------------------------------------------------------------------
def forward_region(args, dist, dart, shape=FWD, decayed=False):
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = synth.layer_inputs(shape, seed=dist.rank)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    B, L, H, P, N, S = shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate, shape.chunk
    C = -(-L // S)
    y = torch.empty((B, L, H, P), device=dev, dtype=torch.float32)
    dH = torch.empty((B, H, C, N, P), device=dev, dtype=torch.bfloat16)
    states = torch.empty((B, H, C, N, P), device=dev, dtype=torch.float32)
    ws = torch.empty(max(16, dart.scan_workspace_bytes(B, L, H, P, N, S, torch.bfloat16)), device=dev,
                     dtype=torch.uint8)
    sma_ws = torch.empty(max(16, dart.sma_decayed_workspace_bytes(B, L, H, P, N, S)), device=dev,
                         dtype=torch.uint8) if decayed else None
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        dart.dart_ssd_chunk_scan(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], S, y_ssd=y, dH=dH, states=states,
                                 workspace=ws)
        if ev:
            ev[1].record(stream)
        if decayed:
            dart.dart_sma_forward_decayed(d["Q"], d["E"], d["Cm"], dH, d["dt"], d["A"], S, d["g"], y, out=y,
                                          workspace=sma_ws)
        else:
            dart.dart_sma_forward(d["Q"], d["E"], d["Cm"], dH, S, d["g"], y, out=y)
        if ev:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    dart.dart_sync_status()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index, ClockSampler.device_uuid(dev))
    clocks.start()
    time.sleep(0.25)
    dist.barrier()
    torch.cuda.synchronize()
    n0 = dart.launch_count()
    clocks.begin()
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    clocks.end()
    n1 = dart.launch_count()
    dist.barrier()
    clk = clocks.stop()
    dart.dart_sync_status()
    ms = start.elapsed_time(end)
    scan_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    sma_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    return {"ms_total": ms, "scan_ms": scan_ms, "sma_ms": sma_ms, "launches": n1 - n0, "clocks": clk,
            "inputs": inp}


def backward_region(args, dist, dart, shape=FWD):
    """The training pass of the layer at the headline shape: SMA backward
    (dQ, dE, dC, memory and gate gradients) and scan backward (dx, ddt, dA,
    dB, dC) from the forward's memories and boundary states, timed per call
    with CUDA events."""
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = synth.layer_inputs(shape, seed=dist.rank)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    S = shape.chunk
    y, dH, states = dart.dart_ssd_chunk_scan(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], S)
    g = torch.Generator(device="cpu").manual_seed(7 + dist.rank)
    dy = torch.randn(y.shape, generator=g).to(dev)
    B, L, H, P, N = shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate
    sma_ws = torch.empty(max(16, dart.sma_backward_workspace_bytes(B, L, H, P, N, S)), device=dev,
                         dtype=torch.uint8)
    scan_ws = torch.empty(max(16, dart.scan_backward_workspace_bytes(B, L, H, P, N, S)), device=dev,
                          dtype=torch.uint8)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        sm = dart.dart_sma_backward(d["Q"], d["E"], d["Cm"], dH, S, d["g"], dy, workspace=sma_ws)
        if ev:
            ev[1].record(stream)
        dart.dart_ssd_scan_backward(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], S, states, dy, sm["ddH"],
                                    dCm_add=sm["dCm"], workspace=scan_ws)
        if ev:
            ev[2].record(stream)

    warm, steps = max(1, min(args.warmup, 2)), max(1, min(args.steps, 3))
    for _ in range(warm):
        step()
    dart.dart_sync_status()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    dist.barrier()
    torch.cuda.synchronize()
    n0 = dart.launch_count()
    for i in range(steps):
        step(evs[i])
    torch.cuda.synchronize()
    n1 = dart.launch_count()
    dist.barrier()
    dart.dart_sync_status()
    sma_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    scan_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    ms = dist.max(sma_ms + scan_ms)
    # algorithmic work of the SMA backward: per valid (t, c) pair and head,
    # 4 N P for U = Q dH and V = C dH, 5 N P for the row gradients (dQ, dE,
    # dC and the score gradient) and 4 N P for the memory gradient
    # sum_t ds Q E^T + p C do^T
    pairs = sum(min(S, L - k * S) * k for k in range(shape.nchunks)) * B * H
    sma_flop = 13.0 * N * P * pairs
    achieved = sma_flop / (sma_ms / 1e3) / 1e12
    # bf16 with N = 128, P = 64 and S a multiple of 128 runs on the tensor cores
    tc = shape.dtype == "bf16" and N == 128 and P == 64 and S % 128 == 0
    if tc:
        peaks, which = load_peaks()
        peak, bound, src = peaks["bf16_tflops"], "tensor", f"bf16_tflops ({which})"
    else:
        peak, bound = SMS * FP32_LANES_PER_SM * 2 * 1965e6 / 1e12, "alu"
        src = "fp32 FMA: 148 SMs x 128 lanes x 2 flop x 1965 MHz"
    return {"value": dist.world * B * L / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
            "warmup": warm, "sma_backward_ms": sma_ms, "scan_backward_ms": scan_ms, "launches": n1 - n0,
            "sma_backward_roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                                      "frac": achieved / peak, "flop_per_launch": sma_flop, "peak_source": src},
            "config": {"workload": "dart_layer_bwd_L8k", "batch": B, "seqlen": L, "nheads": H, "headdim": P,
                       "dstate": N, "chunk": S},
            "path": ("dart_sma_backward (tcgen05: sma_bwd_q_tc, sma_bwd_dh_tc)" if tc else
                     "dart_sma_backward (CUDA cores)")
                    + " + dart_ssd_scan_backward (chunk-parallel; intra-chunk products on tcgen05"
                      " for bf16, N = 128, P = 64) from the forward's memories"}


def e2e_region(args, dist, dart, inp):
    """Same workload through the public call with host (pinned) buffers: the
    inputs are copied host->device and y device->host inside every step."""
    dev = torch.device("cuda", torch.cuda.current_device())
    host = {k: (v.pin_memory() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    B, L, H, P, N, S = FWD.batch, FWD.seqlen, FWD.nheads, FWD.headdim, FWD.dstate, FWD.chunk
    C = -(-L // S)   # a partial last chunk counts
    bufs = {"y": torch.empty((B, L, H, P), device=dev, dtype=torch.float32),
            "dH": torch.empty((B, H, C, N, P), device=dev, dtype=torch.bfloat16),
            "states": torch.empty((B, H, C, N, P), device=dev, dtype=torch.float32),
            "workspace": torch.empty(max(16, dart.scan_workspace_bytes(B, L, H, P, N, S, torch.bfloat16)),
                                     device=dev, dtype=torch.uint8)}
    h2d = sum(v.numel() * v.element_size() for k, v in host.items() if isinstance(v, torch.Tensor))
    d2h = B * L * H * P * 4
    stream = torch.cuda.current_stream()

    def step():
        out = dart.layer_forward(host["x"], host["dt"], host["A"], host["Bm"], host["Cm"], host["Q"],
                                 host["E"], S, host["g"], outputs=("y",), buffers=bufs)
        return out["y"]

    for _ in range(max(1, min(args.warmup, 3))):
        step()
    torch.cuda.synchronize()
    k = max(1, min(args.steps, 10))
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(k):
        step()
    end.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    ms = dist.max(start.elapsed_time(end))
    return {"value": dist.world * B * L * k / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": k,
            "path": "dart.layer_forward on pinned host inputs, y returned to host"}


def decode_region(args, dist, dart, peaks, decayed=False, e4m3=False):
    dec = dataclasses.replace(DEC, nseq=args.decode_nseq)
    dev = torch.device("cuda", torch.cuda.current_device())
    init = synth.decode_initial(dec, seed=dist.rank)
    work = {k: v.to(dev) for k, v in init.items()}
    if e4m3:
        # the same memories in an E4M3 cache (codes + row exponents)
        cache8 = torch.empty(work["cache"].shape, device=dev, dtype=torch.uint8)
        cexp = torch.empty(work["cache"].shape[:-1], device=dev, dtype=torch.int8)
        dart.cache_quantize_e4m3(work["cache"], dec.ncached, cache8, cexp)
        del work["cache"]
        work["cache"], work["cache_exp"] = cache8, cexp
    if decayed:
        # log-decays of the cached memories (dart_decode_step_decayed), -U(0, 3)
        g = torch.Generator().manual_seed(1000 + dist.rank)
        work["memlog"] = (-3.0 * torch.rand((dec.nseq, dec.nheads, dec.cmax), generator=g)).to(dev)
    saved = {k: v.clone() for k, v in work.items()}
    A = synth.decode_A(dec, seed=dist.rank).to(dev)
    # the cache holds one free slot: at most S steps (one append) per run
    nsteps = max(1, min(args.decode_steps, dec.chunk * (dec.cmax - dec.ncached)))
    toks = [synth.decode_tokens(dec, s, seed=dist.rank) for s in range(nsteps)]
    toks = [{k: v.to(dev) for k, v in t.items()} for t in toks]
    y = torch.empty((dec.nseq, dec.nheads, dec.headdim), device=dev, dtype=torch.float32)
    ws = torch.empty(max(16, dart.decode_workspace_bytes(dec.nseq, dec.nheads, dec.headdim, dec.dstate,
                                                         dec.chunk, dec.cmax, torch.bfloat16)),
                     device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream()

    def step(s, ev=None):
        t = toks[s]
        if ev:
            ev[0].record(stream)
        dart.dart_decode_step(t["x"], t["dt"], A, t["Bm"], t["Cm"], t["Q"], t["E"], dec.g, work["state"],
                              work["dH_cur"], work["cache"], work["nchunks"], work["pos"], dec.chunk, y=y,
                              workspace=ws, memlog=work.get("memlog"), cache_exp=work.get("cache_exp"))
        if ev:
            ev[1].record(stream)

    for s in range(min(args.warmup, nsteps)):
        step(s)
    dart.dart_sync_status()
    for k in work:
        work[k].copy_(saved[k])
    del saved
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(nsteps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index, ClockSampler.device_uuid(dev))
    clocks.start()
    time.sleep(0.25)
    dist.barrier()
    torch.cuda.synchronize()
    n0 = dart.launch_count()
    clocks.begin()
    start.record(stream)
    for s in range(nsteps):
        step(s, evs[s])
    end.record(stream)
    torch.cuda.synchronize()
    clocks.end()
    n1 = dart.launch_count()
    dist.barrier()
    clk = clocks.stop()
    dart.dart_sync_status()
    ms = dist.max(start.elapsed_time(end))
    per = [e[0].elapsed_time(e[1]) for e in evs]
    # step s starts at pos = s % S with ncached + s // S memories; pos = S-1 appends
    total_bytes = sum(decode_bytes(dec, dec.ncached + s // dec.chunk, s % dec.chunk == dec.chunk - 1, e4m3)
                      for s in range(nsteps))
    if decayed:   # each cached memory's log-decay is read and written once per step
        total_bytes += sum(8 * dec.nseq * dec.nheads * (dec.ncached + s // dec.chunk) for s in range(nsteps))
    bytes_step = total_bytes / nsteps
    step_ms = statistics.mean(per)
    achieved = bytes_step / (step_ms / 1e3) / 1e9
    return {
        "value": dist.world * dec.nseq * nsteps / (ms / 1e3), "unit": "tokens/s",
        "ms_per_step": ms / nsteps, "steps": nsteps, "launches": n1 - n0, "clocks": clk,
        "config": {"workload": f"decode_{dec.nseq}seq_128mem", "nseq": dec.nseq, "nheads": dec.nheads,
                   "headdim": dec.headdim, "dstate": dec.dstate, "chunk": dec.chunk,
                   "cached_chunks": dec.ncached, "context": dec.ncached * dec.chunk,
                   "l2": "cache 4.3 GB per step >> 126 MB L2"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": captured_traffic("decode_step"),
                     "kernel": "dart_decode_step (decode_partial + decode_combine + decode_advance)",
                     "bytes_per_step": bytes_step},
    }


# ---------------------------------------------------------------------------
# CPU oracle
# ---------------------------------------------------------------------------
def oracle_sample(inp, heads, nthreads):
    from oracle import dart_oracle

    orc = dart_oracle.Oracle(nthreads=nthreads)
    f = {}
    for k, v in inp.items():
        if not isinstance(v, torch.Tensor):
            f[k] = v
            continue
        a = v.float().numpy()
        if k in ("x", "dt", "Q", "E"):
            a = a[:1][:, :, heads]
        elif k in ("Bm", "Cm"):
            a = a[:1]
        elif k == "A":
            a = a[heads]
        f[k] = np.ascontiguousarray(a)
    t0 = time.perf_counter()
    orc.layer_forward(f["x"], f["dt"], f["A"], f["Bm"], f["Cm"], f["Q"], f["E"], FWD.chunk, f["g"])
    sec = time.perf_counter() - t0
    tokens = FWD.seqlen * len(heads) / FWD.nheads  # full-layer token equivalents
    return tokens / sec, sec


def cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(inp):
    nthreads = cores()
    nh = min(FWD.nheads, max(1, 3 * nthreads))
    heads = list(range(nh))
    value, sec = oracle_sample(inp, heads, nthreads)
    return {"value": value, "unit": "tokens/s", "cores": min(nthreads, nh), "kind": "oracle",
            "sample": f"batch 0 of 2, heads 0..{nh - 1} of {FWD.nheads}, all {FWD.seqlen} tokens "
                      f"(fp64 scan + SMA + gate, {sec:.1f} s); tokens/s counted as full-layer tokens "
                      f"({FWD.seqlen} x {nh}/{FWD.nheads})"}


def run_reference(args):
    """The reference arm: the fp64 oracle on this host's cores, one bounded
    sample of the forward workload per step.  CPU only; under torchrun rank
    0 alone runs it and the other ranks exit without work (no process group
    is created)."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    inp = synth.layer_inputs(FWD, seed=0)
    nthreads = cores()
    nh = args.reference_heads if args.reference_heads > 0 else nthreads
    heads = list(range(min(FWD.nheads, nh)))
    for _ in range(args.warmup):
        oracle_sample(inp, heads, nthreads)
    secs = []
    for _ in range(args.steps):
        _, s = oracle_sample(inp, heads, nthreads)
        secs.append(s)
    total = sum(secs)
    tokens = FWD.seqlen * len(heads) / FWD.nheads * args.steps
    value = tokens / total
    sample = (f"per step: batch 0, heads 0..{len(heads) - 1} of {FWD.nheads}, all {FWD.seqlen} tokens; "
              f"full-layer token equivalents")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": fwd_config(args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": min(nthreads, len(heads)),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    dist = Dist()
    try:
        from mamba_ssd_state_b200 import build as dart_build
        from mamba_ssd_state_b200 import dart

        if dist.rank == 0 or dist.world == 1:
            dart_build.build()
        dist.barrier()
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA device")
        torch.cuda.set_device(dist.local)
        peaks, peak_src = load_peaks()

        fwd = forward_region(args, dist, dart)
        ms = dist.max(fwd["ms_total"])
        tokens = FWD.batch * FWD.seqlen
        value = dist.world * tokens * args.steps / (ms / 1e3)
        impl = dart.sma_impl(FWD.dstate, FWD.headdim, FWD.chunk, torch.bfloat16)
        f_sma = sma_flops(FWD)
        f_ssd = ssd_flops(FWD)
        sma_tflops = f_sma / (fwd["sma_ms"] / 1e3) / 1e12
        if impl == "sma_tcgen05":
            roof = {"bound": "tensor", "achieved": sma_tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": sma_tflops / peaks["bf16_tflops"]}
            peak_note = f"bf16_tflops ({peak_src})"
        else:
            alu_peak = SMS * FP32_LANES_PER_SM * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12
            roof = {"bound": "alu", "achieved": sma_tflops, "peak": alu_peak, "unit": "TFLOP/s",
                    "frac": sma_tflops / alu_peak}
            peak_note = "fp32 FMA peak: 148 SMs x 128 lanes x 2 flop x sm_max_mhz"
        roof.update({"traffic": captured_traffic(impl), "traffic_unit": "bytes per launch",
                     "kernel": f"{impl} (the dominant kernel, state-memory attention alone; "
                               "the whole layer is under layer_roofline)",
                     "flop_per_launch": f_sma, "peak_source": peak_note})
        layer_tflops = (f_sma + f_ssd) / (ms / args.steps / 1e3) / 1e12
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": dist.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": fwd_config(dist.world),
            "gpu_launches": fwd["launches"],
            "clocks": fwd["clocks"],
            "roofline": roof,
            "layer_roofline": {"bound": "tensor", "achieved": layer_tflops, "peak": peaks["bf16_tflops"],
                               "unit": "TFLOP/s", "frac": layer_tflops / peaks["bf16_tflops"],
                               "flop_per_step": f_sma + f_ssd,
                               "what": "scan + state-memory attention per step (all algorithmic flops) "
                                       "over the measured dense bf16 peak",
                               "peak_source": peak_note},
            "fwd_breakdown": {"scan_ms": fwd["scan_ms"], "sma_ms": fwd["sma_ms"],
                              "sma_gflop": f_sma / 1e9, "ssd_gflop": f_ssd / 1e9,
                              "layer_tflops": (f_sma + f_ssd) / (ms / args.steps / 1e3) / 1e12,
                              "layer_frac_bf16_peak": (f_sma + f_ssd) / (ms / args.steps / 1e3) / 1e12
                              / peaks["bf16_tflops"]},
        }
        if not args.no_partial:
            # the same layer when the sequence ends inside its last chunk
            ps = synth.TRAIN_L8K_PARTIAL
            part = forward_region(args, dist, dart, ps)
            pms = dist.max(part["ms_total"])
            line["partial_last_chunk"] = {
                "value": dist.world * ps.batch * ps.seqlen * args.steps / (pms / 1e3), "unit": "tokens/s",
                "ms_per_step": pms / args.steps, "scan_ms": part["scan_ms"], "sma_ms": part["sma_ms"],
                "sma_tflops": sma_flops(ps) / (part["sma_ms"] / 1e3) / 1e12,
                "config": {"workload": "dart_layer_fwd_L8092_partial_last_chunk", "batch": ps.batch,
                           "seqlen": ps.seqlen, "nheads": ps.nheads, "chunk": ps.chunk,
                           "last_chunk_tokens": ps.seqlen - (ps.nchunks - 1) * ps.chunk}}
            line["gpu_launches"] += part["launches"]
        if not args.no_decayed:
            # the same layer with the decayed-memory SMA (two decay-prefix kernels + SMA)
            dec_f = forward_region(args, dist, dart, FWD, decayed=True)
            dms = dist.max(dec_f["ms_total"])
            line["decayed_memories"] = {
                "value": dist.world * FWD.batch * FWD.seqlen * args.steps / (dms / 1e3), "unit": "tokens/s",
                "ms_per_step": dms / args.steps, "scan_ms": dec_f["scan_ms"], "sma_ms": dec_f["sma_ms"],
                "sma_tflops": f_sma / (dec_f["sma_ms"] / 1e3) / 1e12,
                "sma_ms_raw_memories": fwd["sma_ms"],
                "config": {"workload": "dart_layer_fwd_L8k_decayed_memories", "batch": FWD.batch,
                           "seqlen": FWD.seqlen, "nheads": FWD.nheads, "chunk": FWD.chunk}}
            line["gpu_launches"] += dec_f["launches"]
        if not args.no_configs:
            # the other forward workloads at their own sizes: the 370M layer shape
            # and the long-context one (256 chunk memories per head)
            line["configs"] = {}
            sub = argparse.Namespace(**vars(args))
            sub.warmup, sub.steps = max(3, min(args.warmup, 3)), max(1, min(args.steps, 5))
            for name, shp in (("layer_L2k", synth.LAYER_L2K), ("long_L64k", synth.LONG_L64K)):
                r = forward_region(sub, dist, dart, shp)
                rms = dist.max(r["ms_total"])
                fs, fd = sma_flops(shp), ssd_flops(shp)
                lt = (fs + fd) / (rms / sub.steps / 1e3) / 1e12
                st = fs / (r["sma_ms"] / 1e3) / 1e12
                line["configs"][name] = {
                    "value": dist.world * shp.batch * shp.seqlen * sub.steps / (rms / 1e3), "unit": "tokens/s",
                    "ms_per_step": rms / sub.steps, "steps": sub.steps, "warmup": sub.warmup,
                    "scan_ms": r["scan_ms"], "sma_ms": r["sma_ms"], "sma_gflop": fs / 1e9, "ssd_gflop": fd / 1e9,
                    "roofline": {"bound": "tensor", "kernel": "sma_tcgen05", "achieved": st,
                                 "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                 "frac": st / peaks["bf16_tflops"]},
                    "layer_tflops": lt, "layer_frac_bf16_peak": lt / peaks["bf16_tflops"],
                    "config": {"workload": f"dart_layer_fwd_{name}", "batch": shp.batch, "seqlen": shp.seqlen,
                               "nheads": shp.nheads, "headdim": shp.headdim, "dstate": shp.dstate,
                               "chunk": shp.chunk}}
                line["gpu_launches"] += r["launches"]
                del r
        if not args.no_backward:
            bshape = FWD if args.backward_heads <= 0 else dataclasses.replace(FWD, nheads=args.backward_heads)
            bwd = backward_region(args, dist, dart, bshape)
            line["backward"] = bwd
            line["gpu_launches"] += bwd.pop("launches")
        if not args.no_e2e:
            line["e2e"] = e2e_region(args, dist, dart, fwd["inputs"])
        if not args.no_decode:
            dec = decode_region(args, dist, dart, peaks)
            line["decode"] = dec
            line["gpu_launches"] += dec["launches"]
            if not args.no_decayed:
                dd = decode_region(args, dist, dart, peaks, decayed=True)
                line["decode"]["decayed_memories"] = {
                    "value": dd["value"], "unit": "tokens/s", "ms_per_step": dd["ms_per_step"],
                    "roofline_frac": dd["roofline"]["frac"], "bytes_per_step": dd["roofline"]["bytes_per_step"],
                    "kernel": "dart_decode_step_decayed"}
                line["gpu_launches"] += dd["launches"]
            if not args.no_e4m3:
                de = decode_region(args, dist, dart, peaks, e4m3=True)
                line["decode"]["e4m3_cache"] = {
                    "value": de["value"], "unit": "tokens/s", "ms_per_step": de["ms_per_step"],
                    "roofline_frac": de["roofline"]["frac"], "bytes_per_step": de["roofline"]["bytes_per_step"],
                    "achieved_gbs": de["roofline"]["achieved"], "kernel": "dart_decode_step_e4m3",
                    "cache": "E4M3 codes + one int8 exponent per row (1.016 B per element)"}
                line["gpu_launches"] += de["launches"]
        if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(fwd["inputs"])
        if dist.rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
