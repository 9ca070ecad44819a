#!/usr/bin/env python
"""Benchmark of the Mamba-2 SSD hot path on B200: chunked prefill tokens/s (the
long-context workload: 1 x 65536 tokens, H=64, P=64, G=8, N=128, chunk 256, bf16)
plus decode steps/s (256 sequences with 2 MiB FP32 states), each with its HBM
roofline fraction, and the FP64 oracle timed on the host cores beside them.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
  torchrun --nproc-per-node N bench.py --gpus N ...   (one rank per GPU)

One JSON line is printed by rank 0. Multi-GPU runs are replicas: every rank runs
its own independent problem (different seed), there is no data-path collective,
`value` is the tokens all ranks processed divided by the slowest rank's time, and
scaling is weak.
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
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mamba_ssd_state_02_b200 import workloads as W  # noqa: E402

METRIC = "SSD prefill tokens/s & decode steps/s on 1 B200; % of HBM/tensor roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PREFILL_CONFIG = 2
DECODE_CONFIG = 4


# ------------------------------------------------------------------------------ ranks
def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def dist_setup(world: int, backend: str):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def max_over_ranks(v: float, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(v)
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        if device is not None and device.type == "cuda":
            torch.distributed.barrier(device_ids=[device.index])
        else:
            torch.distributed.barrier()


def rank_seed(base: int, rank: int) -> int:
    """Independent problem per rank: same recipe, different seed."""
    return base + 7919 * rank


# ------------------------------------------------------------------------------ peaks / bytes
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def path_bytes(w: W.Workload) -> int:
    """Algorithmic bytes of one prefill call: each input read once, each output
    written once (x, B, C, dt_raw, y, initial and final states, per-head params)."""
    T, H, P, G, N = w.total_tokens, w.nheads, w.headdim, w.ngroups, w.dstate
    e = 2 if w.dtype == torch.bfloat16 else 4
    b = T * H * P * e * 2 + T * G * N * e * 2 + T * H * 4 + w.nseq * H * P * N * 4 + 3 * H * 4
    if w.init != "zero":
        b += w.nseq * H * P * N * 4
    return b


def path_flops(w: W.Workload, tile: int | None = None) -> int:
    """Tensor-core flops of the chunked method (2 per multiply-add), with the masked
    causal half of each Q x Q block excluded. Per token-head: C.B^T shared by the
    group's H/G heads Q*N/(H/G), intra-chunk M.X Q*P, chunk state 2*N*P, C.h 2*N*P.
    Q is the chunk the kernels actually use: the tensor-core pipeline always works on
    128-token tiles (pass tile=128), the CUDA-core one on the call's chunk."""
    Q, H, P, G, N = tile or w.chunk, w.nheads, w.headdim, w.ngroups, w.dstate
    per = Q * N // (H // G) + Q * P + 4 * N * P
    return w.total_tokens * H * per


def kernel_bytes(name: str, w: W.Workload, nchunks: int, variant: str = "simt", nsegs: int = 0) -> int:
    """Algorithmic bytes one launch of each kernel must move for the prefill workload
    (inputs read once, outputs written once, intermediates of the pipeline counted
    where the kernel reads or writes them)."""
    T, H, P, G, N, Q = w.total_tokens, w.nheads, w.headdim, w.ngroups, w.dstate, w.chunk
    e = 2 if w.dtype == torch.bfloat16 else 4
    x = T * H * P * e
    bc = T * G * N * e
    dtq = nchunks * H * Q * 4
    st = nchunks * H * P * N * 4
    fin = w.nseq * H * P * N * 4
    if variant == "tc":
        sst = nsegs * H * P * N * 4           # segment states (fp32)
        dtr = T * H * 4
        return {
            "ssd_chunk_table": nsegs * 16,
            "ssd_chunk_state": x + bc + dtr + sst + nsegs * H * 4,
            "ssd_state_passing": 2 * sst + fin + nsegs * H * 4,
            "ssd_chunk_scan": 2 * x + 2 * bc + dtr + sst,
        }.get(name, 0)
    return {
        "ssd_chunk_table": nchunks * 16,
        "ssd_chunk_cumsum": T * H * 4 + 2 * dtq,
        "ssd_chunk_state": x + bc + 2 * dtq + st,
        "ssd_state_passing": 2 * st + fin + nchunks * H * 4,
        "ssd_chunk_scan": 2 * x + 2 * bc + 2 * dtq + st,
    }.get(name, 0)


def decode_step_bytes(nseq, H, P, G, N, e=2) -> int:
    return 2 * nseq * H * P * N * 4 + 2 * nseq * H * P * e + 2 * nseq * G * N * e + nseq * H * 4


# Sources that determine each kernel's code and launch (the plan, grid and segment length
# live in ssd_lib.cu), by the stage name the library reports.
_KERNEL_SOURCES = {
    "tc": ["ssd_lib.cu", "ssd_common.cuh", "ssd_scan_tc.cuh", "ssd_tc_ptx.cuh", "ssd_scan_simt.cuh"],
    "ssd_state_update": ["ssd_lib.cu", "ssd_common.cuh", "ssd_decode.cuh"],
    "strict": ["ssd_lib.cu", "ssd_common.cuh", "ssd_scan_simt.cuh", "ssd_strict.cuh"],
    "conv": ["ssd_lib.cu", "ssd_common.cuh", "ssd_tc_ptx.cuh", "ssd_conv.cuh"],
    "norm": ["ssd_lib.cu", "ssd_common.cuh", "ssd_norm.cuh"],
}


def kernel_sources(kernel: str) -> list:
    if kernel.startswith("ssd_strict"):
        return _KERNEL_SOURCES["strict"]
    if kernel.startswith("ssd_conv1d"):
        return _KERNEL_SOURCES["conv"]
    if kernel == "ssd_gated_rmsnorm":
        return _KERNEL_SOURCES["norm"]
    if kernel in _KERNEL_SOURCES:
        return _KERNEL_SOURCES[kernel]
    return _KERNEL_SOURCES["tc"]


def source_hash(kernel: str | None = None) -> str:
    """Hash of the kernel's sources (all of csrc when kernel is None)."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "mamba_ssd_state_02_b200", "csrc")
    names = sorted(os.listdir(d)) if kernel is None else sorted(kernel_sources(kernel))
    for f in names:
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    kernel's current sources; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload, {}).get(kernel)
    if not e or e.get("source_hash") != source_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock/throttle samples every 100 ms while running."""
    FIELDS = ["timestamp", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device):
        self.proc = None
        self.file = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.sel = str(device.index)

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.sel, "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, window=None):
        """Summary of the samples taken inside `window` = (t0, t1) host wall-clock
        seconds (all samples if None; the nearest later sample if none fall inside)."""
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.strip().split(", ") for r in self.file.read().splitlines() if r.strip()]
        os.unlink(self.file.name)
        import datetime
        parsed = []
        for r in rows:
            if len(r) < len(self.FIELDS):
                continue
            try:
                ts = datetime.datetime.strptime(r[0].strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
                parsed.append((ts, float(r[1]), float(r[2]), r[5:9]))
            except ValueError:
                continue
        sel = parsed
        if window is not None:
            sel = [p for p in parsed if window[0] <= p[0] <= window[1]]
            if not sel:
                later = [p for p in parsed if p[0] >= window[0]]
                sel = later[:1]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, a, b, rs in sel:
            sm.append(a)
            mx.append(b)
            for k, v in zip(names, rs):
                if v.strip().lower() == "active":
                    reasons.add(k)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


class NvmlSampler:
    """SM clock and clock-event reasons read through NVML (the library nvidia-smi
    reports from) every ~2 ms on a background thread, so that a timed region of a few
    milliseconds still gets several samples. Read-only: no setting is changed."""
    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}

    def __init__(self, device):
        self.samples, self.thread, self.ok = [], None, False
        try:
            import pynvml
            self.nv = pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self.nv
        while not self.stop_flag:
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.time(), mhz, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        if not self.ok:
            return
        import threading
        self.stop_flag = False
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def stop(self, window):
        if not self.ok or self.thread is None:
            return None
        self.stop_flag = True
        self.thread.join(timeout=2)
        sel = [x for x in self.samples if window[0] <= x[0] <= window[1]]
        if not sel:
            return None
        reasons = sorted({k for _, _, rs in sel for k, bit in self.REASONS.items() if rs & bit})
        return {"sm_mhz": statistics.median([m for _, m, _ in sel]), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sel), "source": "nvml"}


# ------------------------------------------------------------------------------ oracle baseline
def oracle_sample(w: W.Workload, tokens: int, heads: int, seed_rank: int = 0):
    """Time the FP64 oracle (as it stands) on the first `tokens` tokens of sequence 0
    for `heads` heads; returns (tokens/s of the full workload's width, threads, desc)."""
    from oracle import oracle as O
    tok = W.make_tokens(w, 0, tokens)
    par = W.make_params(w)
    threads = max(1, len(os.sched_getaffinity(0)))
    pairs = [(0, h) for h in range(heads)]
    O.build()
    t0 = time.perf_counter()
    O.ssd_scan(tok["x"], tok["dt_raw"], par["dt_bias"], par["A"], tok["B"], tok["C"], par["D"],
               pairs=pairs, nthreads=threads)
    dt = time.perf_counter() - t0
    tok_heads_per_s = tokens * heads / dt
    return tok_heads_per_s / w.nheads, threads, dt


# ------------------------------------------------------------------------------ our arm
def bench_ours(args, rank, world, local_rank):
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist_setup(world, "nccl")
    from mamba_ssd_state_02_b200 import build
    if rank == 0:
        build.build()
    barrier(dev)
    from mamba_ssd_state_02_b200 import ssd
    peaks, peak_src = load_peaks()
    hbm = float(peaks["hbm_gbs"])

    # ---- prefill (long-context workload)
    w = W.config(PREFILL_CONFIG, seed=rank_seed(1000 + PREFILL_CONFIG, rank))
    inp = W.make_all(w, device=dev)
    L = w.seqlens[0]
    r4 = lambda t: t.view(w.nseq, L, *t.shape[1:])
    x, dtr, Bm, Cm = r4(inp["x"]), r4(inp["dt_raw"]), r4(inp["B"]), r4(inp["C"])
    y = torch.empty_like(x)
    fin = torch.empty(w.nseq, w.nheads, w.headdim, w.dstate, dtype=torch.float32, device=dev)
    dims = ssd.make_dims(w.total_tokens, w.nheads, w.headdim, w.ngroups, w.dstate, ssd.SSD_DTYPE_BF16,
                         batch=w.nseq, seqlen=L)
    ws = torch.empty(ssd.workspace_size(dims, w.chunk), dtype=torch.uint8, device=dev)
    variant = ssd.scan_variant(dims, w.chunk)
    seg_tokens = ssd.segment_tokens(dims, w.chunk)

    def step():
        ssd.scan_fwd(x, dtr, inp["dt_bias"], inp["A"], Bm, Cm, inp["D"], init_state=inp["init_state"],
                     chunk=w.chunk, y=y, final_state=fin, workspace=ws)

    for _ in range(args.warmup):
        step()
    ssd.device_status()
    launches_per_call = ssd.last_launch_count()
    stream = torch.cuda.current_stream(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev)
    nvml_clocks = NvmlSampler(dev)
    clocks.start()
    nvml_clocks.start()
    time.sleep(0.3)
    # Headline: exactly K steps between events, nothing else enqueued in between (the
    # library's per-kernel events stay off here).
    barrier(dev)
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    barrier(dev)
    ms_total = ev0.elapsed_time(ev1)
    time.sleep(0.1)
    # Per-kernel breakdown: a second loop of K steps with the library's per-kernel
    # events on (each launch bracketed by two events on its stream).
    torch.cuda.synchronize(dev)
    ssd.profile_enable(True)
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize(dev)
    kprof = ssd.profile_read()
    ssd.profile_enable(False)
    clk_smi = dict(clocks.stop((t_wall0, t_wall1)), source="nvidia-smi")
    clk = nvml_clocks.stop((t_wall0, t_wall1)) or clk_smi
    ssd.device_status()
    ms_step = max_over_ranks(ms_total / args.steps, dev)
    value = world * w.total_tokens / (ms_step / 1e3)

    # Dominant kernel roofline (per-launch device time from events inside the timed region).
    nchunks = w.nseq * math.ceil(L / w.chunk)
    nsegs = w.nseq * math.ceil(L / seg_tokens) if seg_tokens else 0
    dom = max((k for k in kprof if not k.startswith("_")), key=lambda k: kprof[k][1])
    n_l, t_l = kprof[dom]
    kb = kernel_bytes(dom, w, nchunks, variant, nsegs)
    achieved = kb / (t_l / n_l / 1e3) / 1e9
    roofline = {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": hbm,
                "peak_source": peak_src, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                "bytes_per_launch": kb, "ms_per_launch": round(t_l / n_l, 4),
                "traffic": ncu_traffic(dom, w.name)}
    pb = path_bytes(w)
    pf = path_flops(w, 128 if variant == "tc" else None)
    t_bw = pb / (hbm * 1e9)
    t_tc = pf / (float(peaks["bf16_tflops"]) * 1e12)
    path_roof = {"bytes": pb, "flops": pf, "roofline_ms": round(max(t_bw, t_tc) * 1e3, 4),
                 "bound": "hbm" if t_bw >= t_tc else "tensor",
                 "frac": round(max(t_bw, t_tc) * 1e3 / ms_step, 4),
                 "frac_nominal_8tbs": round(pb / 8e12 * 1e3 / ms_step, 4)}
    # The whole prefill step against its roofline (the target the workload is held to:
    # at least 60% of max(bytes / HBM bandwidth, flops / bf16 peak)).
    path_target = {"workload": w.name, "path_frac": path_roof["frac"], "path_frac_required": 0.6,
                  "met": path_roof["frac"] >= 0.6,
                  "note": "roofline below is the dominant kernel alone; path_frac is the whole step"}
    kernels = {}
    for k, v in kprof.items():
        kms = v[1] / max(1, v[0])
        kbk = kernel_bytes(k, w, nchunks, variant, nsegs)
        kernels[k] = {"launches": v[0], "ms_per_launch": round(kms, 4),
                      "gbs": round(kbk / (kms / 1e3) / 1e9, 1) if kms > 0 and kbk else None}

    # ---- end to end through the public call with host buffers. Every step copies its own
    # inputs from pinned host memory and reads its own results back. Two device buffer sets
    # and two pinned result sets let step i+1's inputs cross PCIe (copy-in stream) while
    # step i's results come back (copy-out stream; the link is full duplex) and the scan
    # runs on the compute stream; events order the reuse of each set.
    host = {k: (None if v is None else v.cpu().pin_memory()) for k, v in inp.items()
            if k in ("x", "dt_raw", "B", "C", "dt_bias", "A", "D", "init_state")}
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    y_h = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
    f_h = [torch.empty(fin.shape, dtype=fin.dtype).pin_memory() for _ in range(2)]
    d2h = y_h[0].numel() * y_h[0].element_size() + f_h[0].numel() * f_h[0].element_size()
    dbuf = [{k: (None if v is None else torch.empty_like(v, device=dev)) for k, v in host.items()} for _ in range(2)]
    ybuf = [y, torch.empty_like(y)]
    fbuf = [fin, torch.empty_like(fin)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_used = [torch.cuda.Event() for _ in range(2)]      # scan of the set done (inputs free)
    ev_back = [torch.cuda.Event() for _ in range(2)]      # results of the set copied out
    for e_ in ev_used + ev_back:
        e_.record(stream)

    def e2e_step(i):
        b = i % 2
        d = dbuf[b]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_used[b])
            for k, v in host.items():
                if v is not None:
                    d[k].copy_(v, non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_back[b])
        ssd.scan_fwd(r4(d["x"]), r4(d["dt_raw"]), d["dt_bias"], d["A"], r4(d["B"]), r4(d["C"]), d["D"],
                     init_state=d["init_state"], chunk=w.chunk, y=ybuf[b], final_state=fbuf[b], workspace=ws)
        ev_used[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_used[b])
            y_h[b].copy_(ybuf[b], non_blocking=True)
            f_h[b].copy_(fbuf[b], non_blocking=True)
            ev_back[b].record(s_out)

    e2e_steps = max(2, min(args.steps, 6))
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier(dev)
    ev0.record(stream)
    s_in.wait_event(ev0)
    for i in range(e2e_steps):
        e2e_step(i)
    for b in range(2):
        stream.wait_event(ev_back[b])
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(ev0.elapsed_time(ev1) / e2e_steps, dev)
    e2e = {"value": world * w.total_tokens / (e2e_ms / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 3),
           "steps": e2e_steps,
           "pipelined": "two buffer sets: step i+1's host-to-device copy overlaps step i's "
                        "device-to-host copy (separate streams); every step copies its own inputs and results"}

    # ---- state snapshots every 2048 tokens on the same workload (prefix-cache reuse)
    snap_every = 2048
    n_snap = ssd.snapshot_count(dims, snap_every)
    snaps = torch.empty(n_snap, w.nheads, w.headdim, w.dstate, dtype=torch.float32, device=dev)
    ws_snap = torch.empty(ssd.snapshot_workspace_size(dims, w.chunk, snap_every), dtype=torch.uint8, device=dev)

    def snap_step():
        ssd.scan_fwd(x, dtr, inp["dt_bias"], inp["A"], Bm, Cm, inp["D"], init_state=inp["init_state"],
                     chunk=w.chunk, y=y, final_state=fin, workspace=ws_snap, snapshot_tokens=snap_every,
                     snapshots=snaps)

    for _ in range(args.warmup):
        snap_step()
    ssd.device_status()
    barrier(dev)
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(args.steps):
        snap_step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    snap_ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dev)
    snapshots = {"interval_tokens": snap_every, "snapshots_per_step": n_snap,
                 "snapshot_bytes_per_step": snaps.numel() * 4, "ms_per_step": round(snap_ms, 4),
                 "overhead_vs_plain": round(snap_ms / ms_step - 1.0, 4)}

    # ---- conv1d prologue (width 4) over the same tokens: xBC = H*P + 2*G*N channels
    K = 4
    ci = W.make_conv_inputs(w, K, init=True, device=dev)
    Dc = W.conv_channels(w)
    cx = ci["xbc"].view(w.nseq, L, Dc)
    cst_out = torch.empty_like(ci["conv_state"])
    cxo, cbo, cco = torch.empty_like(x), torch.empty_like(Bm), torch.empty_like(Cm)

    def conv_step():
        ssd.conv1d_fwd(cx, ci["weight"], ci["bias"], w.nheads, w.headdim, w.ngroups, w.dstate,
                       conv_state=ci["conv_state"], x=cxo, B=cbo, C=cco, conv_state_out=cst_out)

    for _ in range(args.warmup):
        conv_step()
    ssd.device_status()
    barrier(dev)
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(args.steps):
        conv_step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    conv_ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dev)
    esz = 2 if w.dtype == torch.bfloat16 else 4
    conv_bytes = (2 * w.total_tokens * Dc * esz + Dc * K * 4 + Dc * 4
                  + 2 * w.nseq * Dc * (K - 1) * esz)
    # decode step of the conv for 256 sequences
    nd = 256
    dst = torch.zeros(nd, Dc, K - 1, dtype=w.dtype, device=dev)
    dx = ci["xbc"][:nd].contiguous()
    xo = torch.empty(nd, w.nheads, w.headdim, dtype=w.dtype, device=dev)
    bo = torch.empty(nd, w.ngroups, w.dstate, dtype=w.dtype, device=dev)
    co = torch.empty_like(bo)
    for _ in range(args.warmup):
        ssd.conv1d_update(dst, dx, ci["weight"], ci["bias"], w.nheads, w.headdim, w.ngroups, w.dstate, x=xo, B=bo, C=co)
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    nrep = 100
    for _ in range(nrep):
        ssd.conv1d_update(dst, dx, ci["weight"], ci["bias"], w.nheads, w.headdim, w.ngroups, w.dstate, x=xo, B=bo, C=co)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    ssd.device_status()
    conv_upd_us = ev0.elapsed_time(ev1) / nrep * 1e3
    conv1d = {"workload": f"conv1d_width{K}_{w.total_tokens}tok_D{Dc}", "ms_per_call": round(conv_ms, 4),
              "bytes_per_call": conv_bytes, "achieved_gbs": round(conv_bytes / conv_ms / 1e6, 1),
              "peak_gbs": hbm, "frac": round(conv_bytes / conv_ms / 1e6 / hbm, 4),
              "traffic": ncu_traffic("ssd_conv1d", w.name),
              "decode_256seq_us_per_step": round(conv_upd_us, 2)}
    del ci, cx, cst_out, cxo, cbo, cco

    # ---- gated group RMSNorm (group 512) over the scan's output and a z branch
    HPc = w.nheads * w.headdim
    yz = y.view(w.total_tokens, HPc)
    zb = W.to_input_dtype(W.normal(w.seed, 30, w.total_tokens * HPc, device=dev), w.dtype).view(w.total_tokens, HPc)
    nw = (W.uniform(w.seed, 32, HPc, device=dev) + 0.5).to(torch.float32)
    nout = torch.empty_like(yz)
    for _ in range(args.warmup):
        ssd.gated_rmsnorm(yz, zb, nw, group_size=512, eps=1e-6, out=nout)
    ssd.device_status()
    barrier(dev)
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(args.steps):
        ssd.gated_rmsnorm(yz, zb, nw, group_size=512, eps=1e-6, out=nout)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    norm_ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dev)
    norm_bytes = 3 * yz.numel() * yz.element_size() + HPc * 4
    gated_norm = {"workload": f"gated_rmsnorm_group512_{w.total_tokens}tok_C{HPc}", "ms_per_call": round(norm_ms, 4),
                  "bytes_per_call": norm_bytes, "achieved_gbs": round(norm_bytes / norm_ms / 1e6, 1),
                  "peak_gbs": hbm, "frac": round(norm_bytes / norm_ms / 1e6 / hbm, 4)}
    del zb, nout, yz

    # ---- strict mode (bitwise split-invariant CUDA-core prefill) on the same workload
    scache = ssd.ChunkCache.empty(w.nseq, w.nheads, w.headdim, w.ngroups, w.dstate, w.chunk, w.dtype, dev)
    ws_strict = torch.empty(ssd.strict_workspace_size(dims, w.chunk), dtype=torch.uint8, device=dev)

    def strict_step():
        ssd.strict_scan_fwd(x, dtr, inp["dt_bias"], inp["A"], Bm, Cm, inp["D"], scache, y=y, final_state=fin,
                            workspace=ws_strict)

    strict_steps = max(3, min(args.steps, 5))
    for _ in range(2):
        strict_step()
    ssd.device_status()
    barrier(dev)
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(strict_steps):
        strict_step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    strict_ms = max_over_ranks(ev0.elapsed_time(ev1) / strict_steps, dev)
    ssd.profile_enable(True)                     # per-kernel breakdown from a second loop
    for _ in range(strict_steps):
        strict_step()
    torch.cuda.synchronize(dev)
    sprof = ssd.profile_read()
    ssd.profile_enable(False)
    strict = {"workload": w.name, "prefill_ms_per_step": round(strict_ms, 3),
              "prefill_tokens_per_s": world * w.total_tokens / (strict_ms / 1e3),
              "slowdown_vs_default_path": round(strict_ms / ms_step, 2), "steps_timed": strict_steps,
              "kernels_ms_per_launch": {k: round(v[1] / max(1, v[0]), 4) for k, v in sprof.items()
                                        if not k.startswith("_")}}
    del scache, ws_strict
    del host, dbuf, inp, x, dtr, Bm, Cm, y, ws, snaps, ws_snap
    torch.cuda.empty_cache()

    # ---- the batched and packed-varlen prefill workloads (same protocol as the headline)
    other_prefill = {k: bench_prefill_config(args, ssd, dev, rank, world, k, hbm, float(peaks["bf16_tflops"]))
                     for k in (1, 3)}

    # ---- decode (256 sequences, FP32 states from a 2048-token prefill)
    decode = bench_decode(args, ssd, dev, rank, world, hbm, peak_src)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.nseq, "seq_len": L, "nheads": w.nheads,
                   "headdim": w.headdim, "ngroups": w.ngroups, "dstate": w.dstate, "chunk": w.chunk,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (%.2f GB per step vs 126 MB L2), no flush" % (pb / 1e9),
                   "variant": variant, "segment_tokens": seg_tokens},
        "roofline": roofline, "path_roofline": path_roof, "path_target": path_target, "kernels": kernels,
        "prefill_other": other_prefill,
        "clocks": clk, "e2e": e2e, "gpu_launches": launches_per_call * args.steps,
        "decode": decode,
        "snapshots": snapshots,
        "conv1d": conv1d,
        "gated_rmsnorm": gated_norm,
        "strict": strict,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, threads, secs = oracle_sample(w, w.total_tokens, w.nheads)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                "sample": f"the whole step: all {w.nheads} heads of all {w.total_tokens} tokens "
                                          f"({secs:.1f} s wall on {threads} threads)"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def bench_prefill_config(args, ssd, dev, rank, world, k, hbm, tflops):
    """Prefill of workload k (1: batched 4 x 4096, random initial states; 3: 16 packed
    sequences of 512-8192 tokens): W warm-up calls, then K calls between events; tokens/s
    and the whole call against its roofline, bytes and flops as for the headline."""
    w = W.config(k, seed=rank_seed(1000 + k, rank))
    inp = W.make_all(w, device=dev)
    H, P, G, N = w.nheads, w.headdim, w.ngroups, w.dstate
    if w.varlen:
        xs, ds, bs, cs = inp["x"], inp["dt_raw"], inp["B"], inp["C"]
        dims = ssd.make_dims(w.total_tokens, H, P, G, N, ssd.SSD_DTYPE_BF16, nseq=w.nseq)
    else:
        L = w.seqlens[0]
        r4 = lambda t: t.view(w.nseq, L, *t.shape[1:])
        xs, ds, bs, cs = r4(inp["x"]), r4(inp["dt_raw"]), r4(inp["B"]), r4(inp["C"])
        dims = ssd.make_dims(w.total_tokens, H, P, G, N, ssd.SSD_DTYPE_BF16, batch=w.nseq, seqlen=L)
    y = torch.empty_like(xs)
    fin = torch.empty(w.nseq, H, P, N, dtype=torch.float32, device=dev)
    ws = torch.empty(ssd.workspace_size(dims, w.chunk), dtype=torch.uint8, device=dev)

    def step():
        ssd.scan_fwd(xs, ds, inp["dt_bias"], inp["A"], bs, cs, inp["D"], init_state=inp["init_state"],
                     cu_seqlens=inp["cu_seqlens"], chunk=w.chunk, y=y, final_state=fin, workspace=ws)

    for _ in range(max(3, args.warmup)):
        step()
    ssd.device_status()
    stream = torch.cuda.current_stream(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    ssd.device_status()
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dev)
    pb, pf = path_bytes(w), path_flops(w, 128 if ssd.scan_variant(dims, w.chunk) == "tc" else None)
    t_bw, t_tc = pb / (hbm * 1e9), pf / (tflops * 1e12)
    out = {"workload": w.name, "tokens": w.total_tokens, "ms_per_step": round(ms, 4),
           "tokens_per_s": world * w.total_tokens / (ms / 1e3), "steps": args.steps,
           "segment_tokens": ssd.segment_tokens(dims, w.chunk),
           "path_roofline": {"bytes": pb, "flops": pf, "roofline_ms": round(max(t_bw, t_tc) * 1e3, 4),
                             "bound": "hbm" if t_bw >= t_tc else "tensor",
                             "frac": round(max(t_bw, t_tc) * 1e3 / ms, 4)},
           "l2": "inputs larger than L2 (%.2f GB per call vs 126 MB L2), no flush" % (pb / 1e9)}
    del inp, xs, ds, bs, cs, y, fin, ws
    torch.cuda.empty_cache()
    return out


def bench_decode(args, ssd, dev, rank, world, hbm, peak_src):
    w = W.config(DECODE_CONFIG, seed=rank_seed(1000 + DECODE_CONFIG, rank))
    nseq, H, P, G, N, prefix = w.nseq, w.nheads, w.headdim, w.ngroups, w.dstate, w.seqlens[0]
    steps_timed = max(args.steps, 64)
    Ltot = prefix + w.decode_steps
    par = W.make_params(w, device=dev)
    b_idx = torch.arange(nseq, device=dev, dtype=torch.int64)
    pre_rows = (b_idx[:, None] * Ltot + torch.arange(prefix, device=dev)[None, :]).reshape(-1)
    pre = W.make_tokens(w, 0, 0, rows=pre_rows)
    rs = lambda t: t.reshape(nseq, prefix, *t.shape[1:])
    _, state = ssd.scan_fwd(rs(pre["x"]), rs(pre["dt_raw"]), par["dt_bias"], par["A"], rs(pre["B"]),
                            rs(pre["C"]), par["D"], chunk=w.chunk)
    del pre
    torch.cuda.empty_cache()
    nstep_inputs = min(w.decode_steps, steps_timed + args.warmup)
    step_rows = (torch.arange(nstep_inputs, device=dev)[:, None] + prefix + b_idx[None, :] * Ltot).reshape(-1)
    stp = W.make_tokens(w, 0, 0, rows=step_rows)
    xs = stp["x"].view(-1, nseq, H, P)
    dts = stp["dt_raw"].view(-1, nseq, H)
    Bs = stp["B"].view(-1, nseq, G, N)
    Cs = stp["C"].view(-1, nseq, G, N)
    y = torch.empty(nseq, H, P, dtype=w.dtype, device=dev)
    k = [0]

    def step():
        i = k[0] % nstep_inputs
        ssd.state_update(state, xs[i], dts[i], par["dt_bias"], par["A"], Bs[i], Cs[i], par["D"], y=y)
        k[0] += 1

    for _ in range(max(3, args.warmup)):
        step()
    ssd.device_status()
    stream = torch.cuda.current_stream(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(steps_timed):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / steps_timed, dev)
    sb = decode_step_bytes(nseq, H, P, G, N)
    achieved = sb / (ms / 1e3) / 1e9

    # Chunk-emulating (strict) decode from the same state: whole chunk cycles, so the
    # steps that fold a full chunk into the state are included at their share.
    scache = ssd.ChunkCache.empty(nseq, H, P, G, N, w.chunk, w.dtype, dev)
    scache.set_state(state)

    def sstep():
        i = k[0] % nstep_inputs
        ssd.strict_state_update(scache, xs[i], dts[i], par["dt_bias"], par["A"], Bs[i], Cs[i], par["D"], y=y)
        k[0] += 1

    for _ in range(w.chunk):
        sstep()
    ssd.device_status()
    barrier(dev)
    torch.cuda.synchronize(dev)
    s_steps = 2 * w.chunk
    ev0.record(stream)
    for _ in range(s_steps):
        sstep()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    s_ms = max_over_ranks(ev0.elapsed_time(ev1) / s_steps, dev)
    ssd.profile_enable(True)                     # per-kernel breakdown from a second loop
    for _ in range(s_steps):
        sstep()
    torch.cuda.synchronize(dev)
    sprof = ssd.profile_read()
    ssd.profile_enable(False)
    ssd.device_status()
    strict = {"ms_per_step": round(s_ms, 4), "steps_timed": s_steps, "fold_every_steps": w.chunk,
              "overhead_vs_plain_decode": round(s_ms / ms - 1.0, 4),
              "kernels_ms_per_launch": {k: round(v[1] / max(1, v[0]), 4) for k, v in sprof.items()
                                        if not k.startswith("_")}}
    del scache
    return {"workload": w.name, "steps_per_s": 1e3 / ms, "replicas": world,
            "tokens_per_s": world * nseq * 1e3 / ms, "ms_per_step": round(ms, 4),
            "steps_timed": steps_timed,
            "roofline": {"bound": "hbm", "kernel": "ssd_state_update", "achieved": round(achieved, 1),
                         "peak": hbm, "peak_source": peak_src, "unit": "GB/s",
                         "frac": round(achieved / hbm, 4), "bytes_per_launch": sb,
                         "traffic": ncu_traffic("ssd_state_update", w.name)},
            "strict_chunk_emulating": strict}


# ------------------------------------------------------------------------------ reference arm
def bench_reference(args, rank, world):
    """The FP64 oracle on the host cores as the reference arm: same workload, metric
    and unit; each step a bounded sample (all heads of the first 4096 tokens)."""
    if rank != 0:
        return
    w = W.config(PREFILL_CONFIG)
    tokens = 4096
    for _ in range(args.warmup):
        oracle_sample(w, tokens, w.nheads)
    times, threads = [], 1
    for _ in range(args.steps):
        v, threads, secs = oracle_sample(w, tokens, w.nheads)
        times.append(secs)
    sec = statistics.mean(times)
    value = tokens / sec
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sec * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.nseq, "seq_len": w.seqlens[0], "nheads": w.nheads,
                   "headdim": w.headdim, "ngroups": w.ngroups, "dstate": w.dstate, "chunk": w.chunk},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"per step: all {w.nheads} heads of the first {tokens} tokens"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def ncu_case(args):
    """Small fixed workloads for ncu captures (no timing, no JSON): `decode` runs
    W + K decode steps of 256 sequences on a random 512 MiB FP32 state; `prefill`
    runs W + K prefill calls of the long-context workload; `strict` runs W + K strict
    prefill calls of the long-context workload, then W + K chunk-emulating decode
    steps of 256 sequences with half-full open chunks; `fold` runs W + K chunk-emulating
    decode steps of 256 sequences whose open chunks are one token short of full, so every
    step folds every (sequence, head) chunk; `conv` runs W + K conv1d prologue calls over
    the long-context workload's tokens."""
    from mamba_ssd_state_02_b200 import build
    build.build()
    from mamba_ssd_state_02_b200 import ssd
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if args.ncu_case == "decode":
        w = W.config(DECODE_CONFIG)
        nseq, H, P, G, N = w.nseq, w.nheads, w.headdim, w.ngroups, w.dstate
        par = W.make_params(w, device=dev)
        state = (W.normal(w.seed, W.STREAM["init_state"], nseq * H * P * N, 0, dev) * 0.1).float()
        state = state.view(nseq, H, P, N)
        rows = torch.arange(nseq, device=dev, dtype=torch.int64)
        tok = W.make_tokens(w, 0, 0, rows=rows)
        y = torch.empty(nseq, H, P, dtype=w.dtype, device=dev)
        for _ in range(args.warmup + args.steps):
            ssd.state_update(state, tok["x"], tok["dt_raw"], par["dt_bias"], par["A"], tok["B"], tok["C"],
                             par["D"], y=y)
    elif args.ncu_case == "conv":
        # conv1d prologue (width 4) over the long-context workload's tokens
        w = W.config(PREFILL_CONFIG)
        K = 4
        ci = W.make_conv_inputs(w, K, init=True, device=dev)
        L = w.seqlens[0]
        Dc = W.conv_channels(w)
        cx = ci["xbc"].view(w.nseq, L, Dc)
        xo = torch.empty(w.nseq, L, w.nheads, w.headdim, dtype=w.dtype, device=dev)
        bo = torch.empty(w.nseq, L, w.ngroups, w.dstate, dtype=w.dtype, device=dev)
        co = torch.empty_like(bo)
        so = torch.empty_like(ci["conv_state"])
        for _ in range(args.warmup + args.steps):
            ssd.conv1d_fwd(cx, ci["weight"], ci["bias"], w.nheads, w.headdim, w.ngroups, w.dstate,
                           conv_state=ci["conv_state"], x=xo, B=bo, C=co, conv_state_out=so)
    elif args.ncu_case in ("strict", "fold"):
        # strict: the strict prefill of the long-context workload, then chunk-emulating
        # decode steps of 256 sequences whose open chunks hold 64 tokens; fold: the decode
        # steps only, every open chunk one token short of full
        if args.ncu_case == "strict":
            w = W.config(PREFILL_CONFIG)
            inp = W.make_all(w, device=dev)
            L = w.seqlens[0]
            r4 = lambda t: t.view(w.nseq, L, *t.shape[1:])
            y = torch.empty_like(r4(inp["x"]))
            cache = ssd.ChunkCache.empty(w.nseq, w.nheads, w.headdim, w.ngroups, w.dstate, w.chunk, w.dtype, dev)
            for _ in range(args.warmup + args.steps):
                ssd.strict_scan_fwd(r4(inp["x"]), r4(inp["dt_raw"]), inp["dt_bias"], inp["A"], r4(inp["B"]),
                                    r4(inp["C"]), inp["D"], cache, y=y)
            del inp, y, cache
        wd = W.config(DECODE_CONFIG)
        nseq, H, P, G, N, Q = wd.nseq, wd.nheads, wd.headdim, wd.ngroups, wd.dstate, wd.chunk
        par = W.make_params(wd, device=dev)
        dc = ssd.ChunkCache.empty(nseq, H, P, G, N, Q, wd.dtype, dev)
        dc.set_state((W.normal(wd.seed, W.STREAM["init_state"], nseq * H * P * N, 0, dev) * 0.1)
                     .float().view(nseq, H, P, N))
        open_rows = torch.arange(nseq * Q, device=dev, dtype=torch.int64)
        tk = W.make_tokens(wd, 0, 0, rows=open_rows)
        dc.x.copy_(tk["x"].view(nseq, Q, H, P).transpose(1, 2))
        dc.B.copy_(tk["B"].view(nseq, Q, G, N).transpose(1, 2))
        dc.dt.fill_(0.01)
        dc.acum.copy_(-0.01 * torch.arange(1, Q + 1, device=dev, dtype=torch.float32).expand(nseq, H, Q))
        dc.len.fill_(Q - 1 if args.ncu_case == "fold" else Q // 2)
        rows = torch.arange(nseq, device=dev, dtype=torch.int64)
        tok = W.make_tokens(wd, 0, 0, rows=rows)
        yd = torch.empty(nseq, H, P, dtype=wd.dtype, device=dev)
        for _ in range(args.warmup + args.steps):
            if args.ncu_case == "fold":
                dc.len.fill_(Q - 1)
            ssd.strict_state_update(dc, tok["x"], tok["dt_raw"], par["dt_bias"], par["A"], tok["B"], tok["C"],
                                    par["D"], y=yd)
    else:
        w = W.config(PREFILL_CONFIG)
        inp = W.make_all(w, device=dev)
        L = w.seqlens[0]
        r4 = lambda t: t.view(w.nseq, L, *t.shape[1:])
        y = torch.empty_like(r4(inp["x"]))
        for _ in range(args.warmup + args.steps):
            ssd.scan_fwd(r4(inp["x"]), r4(inp["dt_raw"]), inp["dt_bias"], inp["A"], r4(inp["B"]),
                         r4(inp["C"]), inp["D"], chunk=w.chunk, y=y)
    ssd.device_status()
    torch.cuda.synchronize(dev)
    print(f"ncu case {args.ncu_case}: {args.warmup + args.steps} calls ok", flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ncu-case", choices=["decode", "prefill", "strict", "fold", "conv"], default=None,
                    help="run a small fixed workload for an ncu capture instead of the benchmark")
    args = ap.parse_args(argv)
    if args.ncu_case:
        ncu_case(args)
        return
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    rank, world, local_rank = dist_env()
    if args.impl == "reference":
        bench_reference(args, rank, world)
        return
    try:
        bench_ours(args, rank, world, local_rank)
    finally:
        if torch.distributed.is_available() and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
