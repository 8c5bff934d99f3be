#!/usr/bin/env python
"""Benchmark of the Mamba-3 recurrence on B200: prefill Mtokens/s and decode-step us.

One JSON line on rank 0.  `value` is the chunked-prefill throughput on the
SISO workload (batch 8, seqlen 2048, 64 heads, P 64, N 128, bf16 inputs, fp32
state) summed over all ranks (weak scaling: every rank runs the full batch,
no data-path collective).  A step is one `mamba3_scan_fwd` call over the
batch, exporting the final state.  The decode step (batch 128, SISO and MIMO
R=4, 1024 consecutive steps in one CUDA graph) is reported in the same line
under "decode".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_recurrent_scan_b200 import workloads as wl  # noqa: E402

PREFILL = wl.CONFIGS["siso_prefill_b8_l2048"]
DECODE = [wl.CONFIGS["siso_decode_b128"], wl.CONFIGS["mimo4_decode_b128"]]
# further prefill shapes of the benchmark table (reported beside the headline)
PREFILL_MORE = [wl.CONFIGS["mimo4_prefill_b4_l8192"], wl.CONFIGS["mimo4_long_b1_l65536"]]
# batch-1 decode after the 65536-token MIMO prefill: latency-bound (2.5 MB per step)
DECODE_LONG = wl.CONFIGS["mimo4_long_b1_l65536"].with_(prefill_tokens=65536)
FALLBACK_HBM_GBS = 6650.0
BACKWARD_KERNEL = "bwd_state_kernel + bwd_chunk_kernel (tcgen05, TMA)"

# DRAM bytes (read + write) per launch from ncu captures of the kernels as they
# stand: (kernel source files, sha256 of their concatenation, bytes per launch,
# capture).  A kernel whose sources no longer hash to the recorded value gets
# traffic null, since its counters are out of date.
TRAFFIC = {
    "prefill": (('scan_tc.cu', 'sm100_ptx.cuh', 'common.cuh'), "448664d301f10051f82172c25f0f7e4448a777edacd6cfbf54b425df8bab2511",
                813574656 + 137644800, "profiles/scan_tc_prefill_traffic_and_counters.txt"),
    "mimo4_prefill_b4_l8192": (('scan_tc.cu', 'sm100_ptx.cuh', 'common.cuh'), "448664d301f10051f82172c25f0f7e4448a777edacd6cfbf54b425df8bab2511",
                               5653950464 + 1070973184, "profiles/scan_tc_prefill_traffic_and_counters.txt"),
    # the segmented prefill: seg_state_kernel + seg_combine_kernel + scan_tc_kernel of one call
    "mimo4_long_b1_l65536": (('seg_state.cu', 'scan_seg.cu', 'scan_tc.cu', 'sm100_ptx.cuh', 'common.cuh'), "887c8a24ebd2ffc028fa17604efd17f2226f4deff7eb31d43698c2c8b2f2e9ee",
                             4590757632 + 36491776 + 38109696 + 322304 + 6772821504 + 2121624832,
                             "profiles/segmented_prefill_mimo4_b1_l65536.txt"),
    "siso_decode_b128": (('decode.cu', 'sm100_ptx.cuh', 'common.cuh'), "9209a603433cf2acc54a602e33acfa286eefb362ab1303717af46b2effb2b96c",
                         283177728 + 219681280, "profiles/decode_stream_b128_traffic_and_counters.txt"),
    "mimo4_decode_b128": (('decode.cu', 'sm100_ptx.cuh', 'common.cuh'), "9209a603433cf2acc54a602e33acfa286eefb362ab1303717af46b2effb2b96c",
                          317789952 + 241042432, "profiles/decode_stream_b128_traffic_and_counters.txt"),
    "grouped_prefill": (('scan_tc.cu', 'sm100_ptx.cuh', 'common.cuh'), "448664d301f10051f82172c25f0f7e4448a777edacd6cfbf54b425df8bab2511",
                        284654080 + 121231616, "profiles/grouped_bc_prefill_decode_traffic.txt"),
    "grouped_decode": (('decode.cu', 'sm100_ptx.cuh', 'common.cuh'), "9209a603433cf2acc54a602e33acfa286eefb362ab1303717af46b2effb2b96c",
                       279047936 + 219645952, "profiles/grouped_bc_prefill_decode_traffic.txt"),
    "backward": (('scan_bwd_tc.cu', 'sm100_ptx.cuh', 'common.cuh'), "58bdeb0f1b41cb82988d2c19c9a1ca646f603380d204215b052a7ef1a9d4bf3b",
                 541811456 + 241067776 + 1223138304 + 785098240,
                 "profiles/scan_bwd_tc_siso_b8_l2048_traffic_and_counters.txt"),
    "mimo_proj_up": (('mimo_proj.cu', 'sm100_ptx.cuh', 'common.cuh'), "c2a412f8cf230533471e6093ea6ca476f1bedd003f0d0f0a07475de750bfd4e2",
                     406625280 + 1016199424, "profiles/mimo_proj_b4_l8192_traffic.txt"),
    "mimo_proj_down_gated": (('mimo_proj.cu', 'sm100_ptx.cuh', 'common.cuh'), "c2a412f8cf230533471e6093ea6ca476f1bedd003f0d0f0a07475de750bfd4e2",
                             1480475392 + 247016704, "profiles/mimo_proj_b4_l8192_traffic.txt"),
    "gated_norm_per_head": (('gated_norm.cu', 'common.cuh'), "eb90ad7d72a2607cc062684461d599cc86e5eea7058c9d970afd24eac530e380",
                            268478976 + 101627392, "profiles/gated_norm_b8_l2048_traffic_and_counters.txt"),
}


def sources_sha(files) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "linear_recurrent_scan_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def traffic(key):
    files, sha, nbytes, _ = TRAFFIC[key]
    if sha is None or nbytes is None:
        return None
    try:
        return nbytes if sources_sha(files) == sha else None
    except OSError:
        return None


def esize(dt):
    return torch.tensor([], dtype=dt).element_size()


def prefill_bytes(w: wl.Workload, export_state=True, groups=0) -> int:
    """Algorithmic bytes of one prefill: every input read once, y written once,
    the final state written once (A, D included).  groups > 0: B and C hold
    `groups` rows per token instead of one per head."""
    s = esize(w.dtype)
    th = w.token_heads
    per_th = s * (2 * w.rank * w.headdim + w.dstate // 2 + 2)
    bc = s * 2 * w.rank * w.dstate * w.batch * w.seqlen * (groups or w.nheads)
    units = w.batch * w.nheads
    state = 4 * units * (w.dstate * w.headdim + w.rank * w.dstate + w.rank * w.headdim + w.dstate // 2)
    return th * per_th + bc + (state if export_state else 0) + 8 * w.nheads


def decode_bytes(w: wl.Workload, groups=0) -> int:
    """Algorithmic bytes of one decode step: the fp32 state read and written once,
    the per-token inputs read once, y written once (groups as in prefill_bytes)."""
    s = esize(w.dtype)
    units = w.batch * w.nheads
    state = 4 * (w.dstate * w.headdim + w.rank * w.dstate + w.rank * w.headdim + w.dstate // 2)
    io = s * (2 * w.rank * w.headdim + w.dstate // 2 + 2)
    bc = s * 2 * w.rank * w.dstate * w.batch * (groups or w.nheads)
    return units * (2 * state + io) + bc + 8 * w.nheads


def backward_bytes(w: wl.Workload) -> int:
    """Algorithmic bytes of one backward pass: the forward's inputs and dy read
    once, the gradients of x, B, C, theta, dt, lam written once, A, D and their
    gradients (zero initial state, no exported-state gradient)."""
    s = esize(w.dtype)
    per_th = s * (w.rank * w.headdim + 2 * w.rank * w.dstate + w.dstate // 2 + 2)  # x, B, C, theta, dt, lam
    return w.token_heads * (2 * per_th + s * w.rank * w.headdim) + 16 * w.nheads


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int, period_ms: int = 50):
        self.device = device
        self.period_ms = period_ms
        self.proc = None

    def start(self):
        ident = []
        try:
            ident = [f"--id=GPU-{torch.cuda.get_device_properties(self.device).uuid}"]
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", *ident, f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", str(self.period_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __enter__(self):
        return self.start()

    def stop(self):
        self.__exit__(None, None, None)

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": len(sm)}


def rl(nbytes: int, ms: float, peak: float, traffic_bytes=None) -> dict:
    """Compact roofline of one side measurement: GB/s achieved on the algorithmic
    bytes and its fraction of the HBM peak of the headline line."""
    gbs = nbytes / (ms * 1e-3) / 1e9
    d = {"bytes": nbytes, "gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}
    if traffic_bytes is not None:
        d["traffic"] = traffic_bytes
    return d


def bench_config(world: int) -> dict:
    """The workload of the headline line (the same dict in both arms)."""
    w = PREFILL
    return {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "nheads": w.nheads, "headdim": w.headdim,
            "dstate": w.dstate, "rank": w.rank, "state_dtype": "fp32", "parallelism": f"batch-sharded x{world} (weak)",
            "l2": "inputs (%.0f MB) larger than L2 (126 MB); no flush" % (prefill_bytes(w) / 1e6)}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# --------------------------------------------------------------------------- ranks
def setup_dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    from linear_recurrent_scan_b200.shard import max_over_ranks as _max
    return v if world == 1 else _max(v, device="cuda")


# --------------------------------------------------------------------------- our arm
NAMES = ("x", "B", "C", "theta", "dt", "lam")


def run_prefill(m3, args, world, rank, clk):
    w = PREFILL
    dev = torch.device("cuda")
    inp = wl.make_inputs(w, seed=wl.BASE_SEED + rank, device=dev)
    ins = [inp[n] for n in NAMES]
    y = torch.empty_like(inp["x"])
    fin = m3.State.zeros(w.batch, w.nheads, w.headdim, w.dstate, w.rank, device=dev)
    dims = m3.make_dims(inp["x"], inp["B"])
    ws = torch.zeros(m3.mamba3_scan_fwd_workspace_bytes(dims), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        m3.mamba3_scan_fwd(*ins, inp["A"], inp["D"], y=y, final_state=fin, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = m3.mamba3_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status after warm-up: {m3.mamba3_status_string(status)}")

    # timed region: events around every call (kernel duration) and around the whole loop
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    clk.start()
    t0.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    total_ms = max_over_ranks(t0.elapsed_time(t1), world)
    launch_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    launch_ms = max_over_ranks(launch_ms, world)
    status = m3.mamba3_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status after timing: {m3.mamba3_status_string(status)}")

    # end to end through the public host-buffer call: every step copies the inputs
    # in from pinned host memory and y back out (the library overlaps the copies of
    # one sub-batch with the prefill of another); the stage is allocated once
    host = {n: inp[n].cpu().pin_memory() for n in NAMES}
    yh = torch.empty(y.shape, dtype=y.dtype, pin_memory=True)
    stage = torch.zeros(m3.mamba3_scan_fwd_host_stage_bytes(dims), dtype=torch.uint8, device=dev)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = yh.numel() * yh.element_size()

    def e2e_step():
        m3.mamba3_scan_fwd_host(*(host[n] for n in NAMES), inp["A"], inp["D"], y=yh, final_state=fin, stage=stage,
                                stream=stream)

    e2e_steps = max(3, min(args.steps, 10))
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    status = m3.mamba3_device_status(stage)
    if status != 0:
        raise RuntimeError(f"device status after the end-to-end steps: {m3.mamba3_status_string(status)}")
    del host, stage
    return dict(total_ms=total_ms, launch_ms=launch_ms, e2e_ms=e2e_ms, h2d=h2d, d2h=d2h,
                tokens=w.batch * w.seqlen, bytes=prefill_bytes(w))


def run_prefill_plain(m3, w: wl.Workload, rank, steps, warmup, fused_norm=False, time_varying_a=False, groups=0):
    """Median per-launch time (ms) of one prefill launch of workload `w`, inputs
    resident on the device (larger than L2), final state exported.  With
    fused_norm the launch takes raw B, C and normalises them in the kernel; with
    time_varying_a it takes a decay rate per token (A_t) instead of A per head;
    with groups > 0, B and C are shared by groups of nheads / groups heads."""
    dev = torch.device("cuda")
    inp = wl.make_inputs(w, seed=wl.BASE_SEED + rank, device=dev)
    if groups:
        inp.update(wl.grouped_bc(inp, groups, seed=wl.BASE_SEED + 6 + rank))
    norm = None
    if fused_norm:
        raw = wl.raw_bc_inputs(inp, seed=wl.BASE_SEED + 2 + rank)
        inp["B"], inp["C"] = raw["B_raw"], raw["C_raw"]
        norm = m3.BCNorm(raw["w_B"], raw["w_C"], raw["bias_B"], raw["bias_C"], 1e-6)
    A_t = wl.decay_rates(inp["dt"], seed=wl.BASE_SEED + 4 + rank) if time_varying_a else None
    ins = [inp[n] for n in NAMES]
    y = torch.empty_like(inp["x"])
    fin = m3.State.zeros(w.batch, w.nheads, w.headdim, w.dstate, w.rank, device=dev)
    dims = m3.make_dims(inp["x"], inp["B"])
    # the workspace of the library's best schedule (segments for a long sequence over
    # few units, else the split last wave)
    ws = torch.zeros(m3.mamba3_scan_fwd_workspace_bytes(dims), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def launch():
        if time_varying_a:
            m3.mamba3_scan_fwd_at(*ins, A_t, inp["D"], y=y, final_state=fin, workspace=ws, stream=stream)
        elif fused_norm:
            m3.mamba3_scan_fwd_bcnorm(*ins, inp["A"], inp["D"], norm=norm, y=y, final_state=fin, workspace=ws,
                                      stream=stream)
        else:
            m3.mamba3_scan_fwd(*ins, inp["A"], inp["D"], y=y, final_state=fin, workspace=ws, stream=stream)

    for _ in range(warmup):
        launch()
    times = []
    for _ in range(steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        launch()
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    status = m3.mamba3_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status after {w.name}: {m3.mamba3_status_string(status)}")
    del inp, ins, y, fin, ws
    torch.cuda.empty_cache()
    return statistics.median(times)


def run_backward(m3, w: wl.Workload, rank, steps, warmup):
    """Median per-launch time (ms) of the prefill's backward pass on workload w
    (dy drawn N(0, 1); inputs and outputs resident on the device)."""
    dev = torch.device("cuda")
    inp = wl.make_inputs(w, seed=wl.BASE_SEED + rank, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(wl.BASE_SEED + 8 + rank)
    dy = torch.randn(inp["x"].shape, generator=g, device=dev).to(w.dtype)
    ins = [inp[n] for n in NAMES]
    dims = m3.make_dims(inp["x"], inp["B"])
    ws = torch.zeros(m3.mamba3_scan_bwd_workspace_bytes(dims), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    grads = m3.mamba3_scan_bwd(*ins, inp["A"], inp["D"], dy, workspace=ws, stream=stream)
    for _ in range(warmup):
        m3.mamba3_scan_bwd(*ins, inp["A"], inp["D"], dy, grads=grads, workspace=ws, stream=stream)
    # read 256 MB before each timed pass (outside the events): no step starts on what the
    # previous one left in L2; the state kernel's data is still there for the chunk kernel
    flush = torch.ones(256 << 20, dtype=torch.uint8, device=dev)
    times = []
    for _ in range(steps):
        flush.sum()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        m3.mamba3_scan_bwd(*ins, inp["A"], inp["D"], dy, grads=grads, workspace=ws, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    del inp, ins, dy, grads, ws, flush
    torch.cuda.empty_cache()
    return statistics.median(times)


def run_mimo_proj(m3, w: wl.Workload, rank, steps, warmup):
    """Median per-launch times (ms) of the MIMO rank-R projections on workload w:
    up (u [b, L, H, P] -> x [b, L, H, R, P]) and down with the fused RMS norm and
    silu gate (y [b, L, H, R, P], z -> out [b, L, H, P]); bf16, weights per head."""
    dev = torch.device("cuda")
    g = torch.Generator(device=dev)
    g.manual_seed(wl.BASE_SEED + 12 + rank)
    H, R, P = w.nheads, w.rank, w.headdim
    u = torch.randn((w.batch, w.seqlen, H, P), generator=g, device=dev).to(w.dtype)
    Wx = (torch.randn((H, R * P, P), generator=g, device=dev) * P ** -0.5).to(w.dtype)
    Wy = (torch.randn((H, P, R * P), generator=g, device=dev) * (R * P) ** -0.5).to(w.dtype)
    z = torch.randn((w.batch, w.seqlen, H, P), generator=g, device=dev).to(w.dtype)
    wt = torch.rand((H, P), generator=g, device=dev) + 0.5
    x = torch.empty((w.batch, w.seqlen, H, R, P), dtype=w.dtype, device=dev)
    o = torch.empty_like(u)
    stream = torch.cuda.current_stream()
    res = {}
    for name, fn in (("up", lambda: m3.mamba3_mimo_up(u, Wx, out=x, stream=stream)),
                     ("down_gated", lambda: m3.mamba3_mimo_down(x, Wy, z=z, w=wt, out=o, stream=stream))):
        for _ in range(warmup):
            fn()
        times = []
        for _ in range(steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        res[name] = statistics.median(times)
    status = m3.mamba3_library_status()
    if status != 0:
        raise RuntimeError(f"library status after the projections: {m3.mamba3_status_string(status)}")
    del u, Wx, Wy, z, wt, x, o
    torch.cuda.empty_cache()
    return res


def mimo_proj_bytes(w: wl.Workload) -> dict:
    """Algorithmic bytes of the two projections: inputs read once, outputs written
    once, the per-head weights once (and the gate z and norm weight for down)."""
    s = esize(w.dtype)
    th, H, R, P = w.token_heads, w.nheads, w.rank, w.headdim
    wts = s * H * R * P * P
    return {"up": th * s * (P + R * P) + wts, "down_gated": th * s * (R * P + 2 * P) + wts + 4 * H * P}


def run_gated_norm(m3, w: wl.Workload, rank, groups, steps, warmup):
    """Median per-launch time (ms) of the output side (grouped RMS norm + gate) on
    a prefill output of workload w: y, z drawn N(0, 1), weights U(0.5, 1.5)."""
    dev = torch.device("cuda")
    g = torch.Generator(device=dev)
    g.manual_seed(wl.BASE_SEED + 10 + rank)
    shape = (w.batch, w.seqlen, w.nheads, w.rank, w.headdim)
    y = torch.randn(shape, generator=g, device=dev).to(w.dtype)
    z = torch.randn(shape, generator=g, device=dev).to(w.dtype)
    wt = torch.rand((w.nheads, w.rank, w.headdim), generator=g, device=dev) + 0.5
    out = torch.empty_like(y)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        m3.mamba3_gated_norm(y, z, wt, groups=groups, out=out, stream=stream)
    times = []
    for _ in range(steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        m3.mamba3_gated_norm(y, z, wt, groups=groups, out=out, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    del y, z, out
    torch.cuda.empty_cache()
    return statistics.median(times)


def run_decode(m3, w: wl.Workload, world, rank, steps, fused_norm=False, time_varying_a=False, groups=0):
    """Seed the state with a 512-token prefill, then time `steps` decode steps
    captured in one CUDA graph (per-step inputs pre-generated, larger than L2).
    With fused_norm each step takes raw B, C and normalises them in the kernel;
    with groups > 0 each step's B and C are shared by groups of heads."""
    dev = torch.device("cuda")
    pre = wl.make_inputs(w.with_(seqlen=w.prefill_tokens), seed=wl.BASE_SEED + rank, device=dev)
    st = m3.State.zeros(w.batch, w.nheads, w.headdim, w.dstate, w.rank, device=dev)
    m3.mamba3_scan_fwd(*(pre[n] for n in NAMES), pre["A"], pre["D"], final_state=st)
    A, D = pre["A"], pre["D"]
    del pre
    steps_in = wl.decode_inputs(w, steps, seed=wl.BASE_SEED + 1 + rank, device=dev)
    if groups:
        steps_in.update(wl.grouped_bc(steps_in, groups, seed=wl.BASE_SEED + 7 + rank))
    norm = None
    if fused_norm:
        raw = wl.raw_bc_inputs(steps_in, seed=wl.BASE_SEED + 3 + rank)
        steps_in["B"], steps_in["C"] = raw["B_raw"], raw["C_raw"]
        norm = m3.BCNorm(raw["w_B"], raw["w_C"], raw["bias_B"], raw["bias_C"], 1e-6)
    A_t = wl.decay_rates(steps_in["dt"], seed=wl.BASE_SEED + 5 + rank) if time_varying_a else None
    if time_varying_a:
        step_fn = lambda st_, i_, y_: m3.mamba3_decode_step_at(st_, *(steps_in[n][i_] for n in NAMES), A_t[i_], D,
                                                               y=y_, stream=s)
    elif fused_norm:
        step_fn = lambda st_, i_, y_: m3.mamba3_decode_step_bcnorm(st_, *(steps_in[n][i_] for n in NAMES), A, D,
                                                                   norm=norm, y=y_, stream=s)
    else:
        step_fn = lambda st_, i_, y_: m3.mamba3_decode_step(st_, *(steps_in[n][i_] for n in NAMES), A, D, y=y_,
                                                            stream=s)
    ys = torch.empty((steps,) + steps_in["x"].shape[1:], dtype=w.dtype, device=dev)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    saved = st.clone()
    with torch.cuda.stream(s):
        for i in range(3):  # warm-up outside the graph
            step_fn(st, i, ys[i])
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for i in range(steps):
                step_fn(st, i, ys[i])
    torch.cuda.synchronize()
    times = []
    for rep in range(3):
        st.h.copy_(saved.h); st.b_prev.copy_(saved.b_prev); st.x_prev.copy_(saved.x_prev); st.angle.copy_(saved.angle)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s):  # replay on the stream the events are recorded on
            e0.record(s)
            g.replay()
            e1.record(s)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    us = max_over_ranks(min(times), world) * 1000.0 / steps
    del g, steps_in, ys
    torch.cuda.empty_cache()
    return us


def ours(args):
    world, rank, local = setup_dist()
    import linear_recurrent_scan_b200 as m3
    m3.load_library()
    peak, peak_kind = measured_peaks()
    clk = ClockSampler(torch.cuda.current_device())
    r = run_prefill(m3, args, world, rank, clk)
    per_step_ms = r["total_ms"] / args.steps
    tokens_all = r["tokens"] * world
    value = tokens_all / (per_step_ms * 1e-3) / 1e6
    achieved = r["bytes"] / (r["launch_ms"] * 1e-3) / 1e9
    dec = {}
    for w in DECODE:
        us = run_decode(m3, w, world, rank, w.decode_steps)
        dec[w.name] = {"us_per_step": round(us, 2), "steps": w.decode_steps,
                       **rl(decode_bytes(w), us * 1e-3, peak, traffic(w.name))}
    us = run_decode(m3, DECODE_LONG, world, rank, DECODE_LONG.decode_steps)
    # after the 65536-token prefill; latency-bound (2.5 MB per step)
    dec["mimo4_long_decode_b1"] = {"us_per_step": round(us, 2), "steps": DECODE_LONG.decode_steps,
                                   "bytes": decode_bytes(DECODE_LONG)}
    side_steps = max(5, min(args.steps, 20))
    # the fused B/C norm variant of the headline prefill and of the SISO decode step
    ms = max_over_ranks(run_prefill_plain(m3, PREFILL, rank, steps=side_steps, warmup=3, fused_norm=True), world)
    fused = {"prefill": {"ms": round(ms, 4), **rl(prefill_bytes(PREFILL), ms, peak)}}
    us = run_decode(m3, DECODE[0], world, rank, DECODE[0].decode_steps, fused_norm=True)
    fused["decode_siso_b128"] = {"us": round(us, 2), **rl(decode_bytes(DECODE[0]), us * 1e-3, peak)}
    # the time-varying decay variant (A_t per token: 2 more bytes per token-head)
    ms = max_over_ranks(run_prefill_plain(m3, PREFILL, rank, steps=side_steps, warmup=3, time_varying_a=True), world)
    tva = {"prefill": {"ms": round(ms, 4), **rl(prefill_bytes(PREFILL) + 2 * PREFILL.token_heads, ms, peak)}}
    us = run_decode(m3, DECODE[0], world, rank, DECODE[0].decode_steps, time_varying_a=True)
    tva["decode_siso_b128"] = {"us": round(us, 2), **rl(decode_bytes(DECODE[0]) + 2 * DECODE[0].batch *
                                                        DECODE[0].nheads, us * 1e-3, peak)}
    # grouped B/C: one B and C row per token shared by all heads (ngroups 1)
    ms = max_over_ranks(run_prefill_plain(m3, PREFILL, rank, steps=side_steps, warmup=3, groups=1), world)
    grp = {"prefill": {"ngroups": 1, "ms": round(ms, 4),
                       **rl(prefill_bytes(PREFILL, groups=1), ms, peak, traffic("grouped_prefill"))}}
    us = run_decode(m3, DECODE[0], world, rank, DECODE[0].decode_steps, groups=1)
    grp["decode_siso_b128"] = {"ngroups": 1, "us": round(us, 2),
                               **rl(decode_bytes(DECODE[0], groups=1), us * 1e-3, peak, traffic("grouped_decode"))}
    # the backward pass of the headline prefill (dy given; zero initial state)
    ms = max_over_ranks(run_backward(m3, PREFILL, rank, steps=3, warmup=1), world)
    bwd = {"prefill_" + PREFILL.name: {"ms": round(ms, 3), "kernel": BACKWARD_KERNEL,
                                       "l2": "256 MB read before each pass, outside the events",
                                       **rl(backward_bytes(PREFILL), ms, peak, traffic("backward"))}}
    # the output side on the headline prefill's y: grouped RMS norm + gate
    gated = {}
    for ng in (PREFILL.nheads, 8):
        ms = max_over_ranks(run_gated_norm(m3, PREFILL, rank, ng, steps=side_steps, warmup=3), world)
        by = 3 * esize(PREFILL.dtype) * PREFILL.token_heads * PREFILL.rank * PREFILL.headdim + 4 * PREFILL.nheads * \
            PREFILL.rank * PREFILL.headdim
        gated["groups%d" % ng] = {"ms": round(ms, 4), **rl(by, ms, peak, traffic("gated_norm_per_head")
                                                         if ng == PREFILL.nheads else None)}
    # the MIMO rank-R projections around the recurrence (R 4 prefill shape)
    pw = PREFILL_MORE[0]
    pt = run_mimo_proj(m3, pw, rank, steps=side_steps, warmup=3)
    pb = mimo_proj_bytes(pw)
    proj = {k: {"ms": round(max_over_ranks(v, world), 4),
                **rl(pb[k], max_over_ranks(v, world), peak, traffic("mimo_proj_" + k))}
            for k, v in pt.items()}
    proj["workload"] = pw.name
    more = {}
    for w in PREFILL_MORE:
        ms = max_over_ranks(run_prefill_plain(m3, w, rank, steps=side_steps, warmup=3), world)
        dims = m3.Dims(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.rank, 0, m3.MAMBA3_BF16, 0)
        segmented = m3.mamba3_scan_segmented_workspace_bytes(dims) > m3.mamba3_scan_workspace_bytes(dims)
        more[w.name] = {"ms": round(ms, 4), "mtokens_s": round(w.batch * w.seqlen / (ms * 1e-3) / 1e6, 3),
                        "segmented": segmented,
                        **rl(prefill_bytes(w), ms, peak, traffic(w.name) if w.name in TRAFFIC else None)}
    clk.stop()
    clocks = clk.summary()
    clocks["window"] = "headline prefill timed steps through the last side measurement"
    e2e_value = tokens_all / (r["e2e_ms"] * 1e-3) / 1e6
    out = {
        "metric": "prefill Mtokens/s (SISO, batch 8, seqlen 2048) and decode step us at batch 128",
        "value": round(value, 3),
        "unit": "Mtokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(per_step_ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; distributions of the layer inputs, no dataset or weights)",
        "config": bench_config(world),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic("prefill"), "peak_kind": peak_kind,
                     "bytes_per_launch": r["bytes"], "launch_ms": round(r["launch_ms"], 4)},
        "e2e": {"value": round(e2e_value, 3), "unit": "Mtokens/s", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": args.steps,
        "nccl_world_size": world,
        "clocks": clocks,
        "side_units": "ms / us per launch or step; gbs and frac against the same HBM peak as roofline",
        "fused_bc_norm": fused,
        "time_varying_decay": tva,
        "grouped_bc": grp,
        "gated_norm": gated,
        "mimo_proj": proj,
        "backward": bwd,
    }
    if rank == 0:
        cpu = cpu_baseline(args)
        if cpu is not None:
            out["cpu_baseline"] = cpu
    # the other configurations last, where a reader of the line's tail finds them
    out["decode"] = dec
    out["prefill_more"] = more
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# --------------------------------------------------------------------------- oracle arms
def host_threads() -> int:
    """Host threads this process may use: its CPU affinity, capped by a cgroup
    CPU quota when one is set (a container's os.cpu_count() reports the host)."""
    n = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    try:
        with open("/sys/fs/cgroup/cpu.max") as f:
            q, per = f.read().split()[:2]
        if q != "max":
            n = min(n, max(1, int(math.ceil(int(q) / int(per)))))
    except (OSError, ValueError):
        pass
    return max(1, n)


class OracleSample:
    """The fp64 oracle (as it stands, on the host threads available) on whole
    (batch, head) units of the prefill workload, sized by a calibration round of
    one unit per thread run in parallel."""

    def __init__(self, target_s: float):
        import oracle
        self.oracle = oracle
        w = PREFILL
        self.threads = min(host_threads(), w.batch * w.nheads)
        cal_batch = -(-self.threads // w.nheads)
        cal = wl.to_f64(wl.make_inputs(w.with_(batch=cal_batch), device="cpu"))
        t = time.perf_counter()
        oracle.scan_complex(**cal, units=list(range(self.threads)), nthreads=self.threads)
        per_round = time.perf_counter() - t
        rounds = max(1, int(target_s / max(per_round, 1e-3)))
        self.units = max(1, min(self.threads * rounds, w.batch * w.nheads))
        batch = -(-self.units // w.nheads)
        self.f = wl.to_f64(wl.make_inputs(w.with_(batch=batch), device="cpu"))

    def run(self):
        t = time.perf_counter()
        self.oracle.scan_complex(**self.f, units=list(range(self.units)), nthreads=self.threads)
        sec = time.perf_counter() - t
        # tokens of the whole layer (all heads): units * L / H
        return self.units * PREFILL.seqlen / PREFILL.nheads / sec / 1e6, sec

    @property
    def cores(self):
        return min(self.threads, self.units)


def cpu_baseline(args):
    try:
        o = OracleSample(target_s=12.0)
        mtok, sec = o.run()
    except Exception as e:  # the baseline is a report, never a reason to lose the line
        return {"error": str(e)[:200]}
    return {"value": round(mtok, 6), "unit": "Mtokens/s", "cores": o.cores, "kind": "oracle", "cpu_model": cpu_model(),
            "sample": f"{o.units} of {PREFILL.batch * PREFILL.nheads} (batch, head) units of the prefill workload, "
                      f"all {PREFILL.seqlen} tokens each, {sec:.1f} s"}


def reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    times, vals = [], []
    # each step a bounded sample (~3 s) so that warm-up + steps end in minutes
    o = OracleSample(target_s=min(3.0, 150.0 / max(1, args.warmup + args.steps)))
    units, threads = o.units, o.cores
    for i in range(args.warmup + args.steps):
        mtok, sec = o.run()
        if i >= args.warmup:
            times.append(sec)
            vals.append(mtok)
    value = statistics.median(vals)
    out = {
        "impl": "reference",
        "metric": "prefill Mtokens/s (SISO, batch 8, seqlen 2048) and decode step us at batch 128",
        "value": round(value, 6),
        "unit": "Mtokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1000 * statistics.median(times), 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": bench_config(world),
        "cpu_baseline": {"value": round(value, 6), "unit": "Mtokens/s", "cores": threads, "kind": "oracle",
                         "cpu_model": cpu_model(),
                         "sample": f"each step: {units} (batch, head) units x {PREFILL.seqlen} tokens on host cores"},
        "e2e": {"value": round(value, 6), "unit": "Mtokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world_env = os.environ.get("WORLD_SIZE")
    if args.impl == "ours" and args.gpus > 1 and world_env is None:
        # one process per GPU: relaunch this script under torchrun with --gpus ranks
        import socket
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
               "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *sys.argv[1:]]
        sys.exit(subprocess.call(cmd))
    if args.impl == "ours" and world_env is not None and int(world_env) != args.gpus:
        sys.exit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world_env}: launch one rank per GPU")
    if args.impl == "reference":
        reference(args)
    else:
        ours(args)


if __name__ == "__main__":
    main()
