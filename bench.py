#!/usr/bin/env python
"""Benchmark of the selective-scan forward pass (and the decode step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload mamba2p8b] [--no-extras] [--no-cpu-baseline]

One step = one ss_fwd call over the whole workload (Δ softplus, discretise,
recurrence, readout + skip, gate, final state: every step of the path), with
inputs resident in HBM.  The default workload is the Mamba-2.8B-shaped layer
(batch 4, L 8192, d_inner 5120, N 16, bf16 I/O, fp32 state).  Its inputs
(1.34 GB) are larger than the 126 MB L2, so no flush is needed between steps.

Metric: effective HBM bandwidth = compulsory bytes of the step / step time
(u, Δ_raw, z read and y written once each, B, C, A, D, bias read, final state
written), in GB/s.  Under torchrun every rank runs its own copy of the
workload (independent problems, no data-path collective: weak scaling); the
value is all ranks' bytes over the slowest rank's time.

Rank 0 prints ONE JSON line.  `--impl reference` times the CPU oracle (the
plain sequential loop the GPU path is checked against) on a bounded sample of
the same workload instead.
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "selective-scan fwd effective HBM GB/s (% of B200 peak); decode steps/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
# device code of the forward kernel (the profile's traffic figure is used only
# while these files are unchanged)
KERNEL_SOURCES = ["selective_state_space_37_b200/csrc/fwd.cuh",
                  "selective_state_space_37_b200/csrc/common.cuh",
                  "selective_state_space_37_b200/csrc/selscan.cu"]   # launch shapes


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mamba2p8b")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--mode", choices=["fwd", "decode", "bwd", "block", "ssd"], default="fwd",
                    help="decode: time only the decode workload, --steps single-token steps; "
                         "bwd: time only ss_bwd on --workload")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """(burst, sustained) dense bf16 TFLOP/s from MEASURED_PEAKS.json, with its kind."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return "measured", float(pk["bf16_tflops"]), float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"]))
    except Exception:
        return "fallback", FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS


def kernel_source_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload):
    """DRAM bytes per launch from the committed ncu summary, when it was taken
    on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", f"ss_fwd_kernel_{workload}.md")
    try:
        src, val = None, None
        with open(path) as f:
            for line in f:
                if line.startswith("source_sha:"):
                    src = line.split(":", 1)[1].strip()
                if line.startswith("dram_bytes_per_launch:"):
                    val = float(line.split(":", 1)[1].strip())
        if src == kernel_source_hash() and val:
            return val
    except OSError:
        pass
    return None


def shard_seed(seed, rank):
    """Seed of this rank's copy of the workload: every rank scans its own,
    independent synthetic problem (weak scaling, no data-path collective)."""
    return seed + 1000 * rank


def reduce_max(dist, x, device):
    """Max of a float over all ranks (host plumbing for the timing only)."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(world, per_rank_bytes, steps, ms_max):
    """Whole-job effective GB/s: all ranks' compulsory bytes over the slowest
    rank's time."""
    return world * per_rank_bytes * steps / (ms_max * 1e-3) / 1e9


# FP32 lane operations the forward kernel issues per channel-timestep on the
# structured-A path, counted from its source (both threads of a channel pair):
# 3 decay-exponent arguments (λ·a once, by the thread that prepares the step;
# λa·(8p+1) in each thread), 16 ladder products for the 16 decays, 16 Δu·B
# products, 16 state FMAs, 16 readout products, 2 lane-pair sums of the
# readout (one per thread), and 9 scalar operations of the step's own
# (softplus argument, 1 + 2^y, Δu, D u, two for the gate, three for the
# output).  ncu's FMA-pipe activity on the 2.8B-shaped layer (48 %) agrees
# with this count.
FP32_OPS_PER_CH_TS = 78


def alu_roofline(torch, device, ch_ts_per_s, clock_summary):
    """The forward kernel against the FP32 pipe: 128 lanes per SM (sm_100)
    x SMs x the SM clock seen during the timed region (max clock if unsampled)."""
    props = torch.cuda.get_device_properties(device)
    mhz = (clock_summary or {}).get("sm_mhz") or (clock_summary or {}).get("sm_max_mhz") or 1965.0
    peak = 128 * props.multi_processor_count * mhz * 1e6 / 1e12
    achieved = ch_ts_per_s * FP32_OPS_PER_CH_TS / 1e12
    return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "T FP32 lane-ops/s",
            "frac": achieved / peak, "ops_per_ch_ts": FP32_OPS_PER_CH_TS,
            "peak_kind": f"128 FP32 lanes/SM x {props.multi_processor_count} SMs x {mhz:.0f} MHz"}


class ClockSampler:
    """Samples SM clock and throttle reasons via NVML in a background thread."""
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, index, period=0.002):
        self.ok = False
        self.samples = []
        self.reasons = set()
        self.period = period
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ----------------------------------------------------------------- our arm
def fwd_call(ss, inp, y, st, ws, stream):
    return ss.ss_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"], z=inp["z"],
                     delta_bias=inp["delta_bias"], y=y, last_state=st, workspace=ws, stream=stream)


def time_fwd(ss, torch, cfg, device, steps, warmup, seed_offset=0, dist=None, clocks=None):
    from ss_inputs import fwd_inputs
    inp = fwd_inputs(cfg.batch, cfg.seqlen, cfg.d_inner, cfg.d_state, cfg.dtype,
                     cfg.seed + seed_offset, device, gate=cfg.gate, D_kind=cfg.D_kind)
    y = torch.empty_like(inp["u"])
    st = torch.empty((cfg.batch, cfg.d_inner, cfg.d_state), dtype=torch.float32, device=device)
    nbytes = ss.fwd_workspace_bytes(cfg.batch, cfg.seqlen, cfg.d_inner, cfg.dtype == "bf16")
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    for _ in range(warmup):
        fwd_call(ss, inp, y, st, ws, stream)
    torch.cuda.synchronize(device)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    ctx = clocks if clocks is not None else _Null()
    with ctx:
        e0.record(stream)
        for _ in range(steps):
            fwd_call(ss, inp, y, st, ws, stream)
        e1.record(stream)
        torch.cuda.synchronize(device)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(device)
    ms = e0.elapsed_time(e1)
    status = ss.ss_check(ws, stream=stream)
    if status != 0:
        raise RuntimeError(f"device status {ss.status_string(status)}")
    return ms, inp, y, st, ws


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def time_e2e(ss, torch, cfg, device, inp, steps):
    """Public API with host buffers: ss_fwd_host on pinned host inputs and
    outputs -- every step uploads u, Δ, z, B, C, scans and downloads y (batch
    slices of one row, with the three overlapped on separate streams), all
    inside the timed region."""
    names = ["u", "delta", "z", "B", "C"]
    host = {k: torch.empty(inp[k].shape, dtype=inp[k].dtype, pin_memory=True) for k in names}
    for k in names:
        host[k].copy_(inp[k])
    y_host = torch.empty(inp["u"].shape, dtype=inp["u"].dtype, pin_memory=True)
    stream = torch.cuda.current_stream(device)
    ws = torch.empty(ss.fwd_host_workspace_bytes(cfg.batch, cfg.seqlen, cfg.d_inner, cfg.dtype == "bf16", 1),
                     dtype=torch.uint8, device=device)
    h2d = sum(host[k].numel() * host[k].element_size() for k in names)
    d2h = y_host.numel() * y_host.element_size()

    def one():
        ss.ss_fwd_host(host["u"], host["delta"], inp["A"], host["B"], host["C"], D=inp["D"], z=host["z"],
                       delta_bias=inp["delta_bias"], y=y_host, return_last_state=False, rows_per_slice=1,
                       workspace=ws, stream=stream)

    one()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize(device)
    ms = e0.elapsed_time(e1) / steps
    return ms, h2d, d2h


def time_fwd_conv(ss, torch, cfg, device, steps, warmup):
    """ss_fwd_conv (conv1d + SiLU prologue fused) on a forward workload, x in
    place of u, timed back to back with CUDA events."""
    from ss_inputs import conv_params, fwd_inputs
    inp = fwd_inputs(cfg.batch, cfg.seqlen, cfg.d_inner, cfg.d_state, cfg.dtype, cfg.seed, device,
                     gate=cfg.gate, D_kind=cfg.D_kind)
    w, cb = conv_params(cfg.d_inner, cfg.seed, device)
    y = torch.empty_like(inp["u"])
    st = torch.empty((cfg.batch, cfg.d_inner, cfg.d_state), dtype=torch.float32, device=device)
    ws = torch.empty(ss.fwd_workspace_bytes(cfg.batch, cfg.seqlen, cfg.d_inner, cfg.dtype == "bf16"),
                     dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def one():
        ss.ss_fwd_conv(inp["u"], w, inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"], z=inp["z"],
                       delta_bias=inp["delta_bias"], conv_b=cb, y=y, last_state=st, workspace=ws, stream=stream)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize(device)
    ms = e0.elapsed_time(e1) / steps
    del inp, y, st, ws
    torch.cuda.empty_cache()
    return ms


def time_fwd_general(ss, torch, cfg, device, steps, warmup):
    """The forward on the general-A path: the workload with A perturbed off
    the ladder A[d, n] = a_d (n + 1) (every entry scaled by 1 + 1e-3 N(0, 1),
    so the kernel's exact structure test fails and every decay is its own
    exponential), timed back to back with CUDA events."""
    from ss_inputs import fwd_inputs
    inp = fwd_inputs(cfg.batch, cfg.seqlen, cfg.d_inner, cfg.d_state, cfg.dtype, cfg.seed, device,
                     gate=cfg.gate, D_kind=cfg.D_kind)
    g = torch.Generator(device=device).manual_seed(cfg.seed + 7)
    A = inp["A"] * (1.0 + 1e-3 * torch.randn(inp["A"].shape, generator=g, device=device))
    y = torch.empty_like(inp["u"])
    st = torch.empty((cfg.batch, cfg.d_inner, cfg.d_state), dtype=torch.float32, device=device)
    ws = torch.empty(ss.fwd_workspace_bytes(cfg.batch, cfg.seqlen, cfg.d_inner, cfg.dtype == "bf16"),
                     dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def one():
        ss.ss_fwd(inp["u"], inp["delta"], A, inp["B"], inp["C"], D=inp["D"], z=inp["z"],
                  delta_bias=inp["delta_bias"], y=y, last_state=st, workspace=ws, stream=stream)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize(device)
    ms = e0.elapsed_time(e1) / steps
    status = ss.ss_check(ws, stream=stream)
    del inp, A, y, st, ws
    torch.cuda.empty_cache()
    if status != 0:
        raise RuntimeError(f"device status {ss.status_string(status)}")
    return ms


def launch_overhead(ss, torch, cfg, device, reps=200):
    """What a call costs beyond the scan on a short workload: (a) the host
    time to enqueue one ss_fwd call (binding + C ABI + header memset + kernel
    launch), averaged over `reps` calls issued without synchronization;
    (b) the device time per call of a minimal forward (batch 1, 32 steps, 128
    channels: one CTA, one tile), back to back; (c) the workload's device time
    per call back to back, and the same calls replayed from one CUDA graph,
    whose difference is the per-launch gap the graph removes."""
    from ss_inputs import fwd_inputs
    stream = torch.cuda.current_stream(device)
    out = {}

    def prepared(b, L, d):
        inp = fwd_inputs(b, L, d, 16, "bf16", cfg.seed, device, gate=True, D_kind="ones")
        y = torch.empty_like(inp["u"])
        st = torch.empty((b, d, 16), dtype=torch.float32, device=device)
        ws = torch.empty(ss.fwd_workspace_bytes(b, L, d, True), dtype=torch.uint8, device=device)
        # the stream current at call time (the capture stream inside the graph)
        return lambda: ss.ss_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"], z=inp["z"],
                                 delta_bias=inp["delta_bias"], y=y, last_state=st, workspace=ws,
                                 stream=torch.cuda.current_stream(device))

    def device_ms(fn, n):
        for _ in range(3):
            fn()
        torch.cuda.synchronize(device)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(device)
        return e0.elapsed_time(e1) / n

    tiny = prepared(1, 32, 128)
    device_ms(tiny, 10)
    t0 = time.perf_counter()
    for _ in range(reps):
        tiny()
    t1 = time.perf_counter()
    torch.cuda.synchronize(device)
    out["host_enqueue_us_per_call"] = (t1 - t0) / reps * 1e6
    out["tiny_call_device_us"] = device_ms(tiny, reps) * 1e3
    work = prepared(cfg.batch, cfg.seqlen, cfg.d_inner)
    direct = device_ms(work, 50)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for _ in range(2):
            work()
    torch.cuda.synchronize(device)
    with torch.cuda.graph(g, stream=side):
        for _ in range(10):
            work()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(5):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize(device)
    graphed = e0.elapsed_time(e1) / 50
    del g
    out.update({"workload": cfg.name, "direct_ms_per_call": direct, "graph_ms_per_call": graphed,
                "launch_gap_us": (direct - graphed) * 1e3,
                "note": "tiny = batch 1, L 32, d_inner 128 (one CTA, one tile); the graph holds 10 calls "
                        "(each a header memset and one kernel)"})
    torch.cuda.empty_cache()
    return out


BLOCK_SHAPES = {   # Mamba-block inner path: (batch, L, d_model), d_inner = 2 d_model
    "block_mamba130m": (8, 2048, 768),
    "block_mamba2p8b": (4, 8192, 2560),
}


def time_block(ss, torch, name, device, steps, warmup):
    """ss_block_fwd (projections on cuBLAS, conv, scan, out_proj) on random-init
    weights, timed back to back with CUDA events.  Returns (ms, tokens,
    projection FLOPs per call)."""
    from ss_inputs import block_inputs
    b, L, dm = BLOCK_SHAPES[name]
    hidden, w = block_inputs(b, L, dm, seed=9, device=device)
    out = torch.empty_like(hidden)
    scratch = torch.empty(ss.block_scratch_bytes(w, b, L), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    for _ in range(warmup):
        ss.ss_block_fwd(hidden, w, out=out, scratch=scratch, stream=stream)
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        ss.ss_block_fwd(hidden, w, out=out, scratch=scratch, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(device)
    ms = e0.elapsed_time(e1) / steps
    di, rk = 2 * dm, w["x_proj_dt"].shape[0]
    flops = 2 * b * L * (2 * di * dm + di * (rk + 32) + rk * di + dm * di)
    del hidden, w, out, scratch
    torch.cuda.empty_cache()
    return ms, b * L, flops


SSD_SHAPES = {   # multi-head scalar-decay scan: (batch, L, nheads, d_state), headdim 64
    "ssd_mamba2_2p7b": (4, 8192, 80, 128),    # d_model 2560, expand 2: 5120 = 80 heads x 64
    "ssd_mamba2_130m": (8, 2048, 24, 128),    # d_model 768: 1536 = 24 heads x 64
}


def ssd_useful_flops(b, L, H, N, Q=64, P=64):
    """Dense-equivalent FLOPs of the chunked form per call: the causal half of
    C Bᵀ (Q/2 · N per step) and of the masked product with x (Q/2 · P), the
    carried state into the outputs (N · P) and the state update (N · P)."""
    return 2 * (Q // 2 * N + Q // 2 * P + 2 * N * P) * b * L * H


def ssd_compulsory_bytes(b, L, H, N, P=64):
    return 2 * (2 * b * L * H * P + 2 * b * L * N + b * L * H) + 4 * b * H * P * N + 12 * H


def time_ssd(ss, torch, name, device, steps, warmup):
    from ss_inputs import ssd_inputs
    b, L, H, N = SSD_SHAPES[name]
    inp = ssd_inputs(b, L, H, N, seed=3, device=device)
    y = torch.empty_like(inp["x"])
    st = torch.empty((b, H, 64, N), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def one():
        ss.ss_ssd_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], D=inp["D"], dt_bias=inp["dt_bias"],
                      y=y, final_state=st, stream=stream)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize(device)
    ms = e0.elapsed_time(e1) / steps
    del inp, y, st
    torch.cuda.empty_cache()
    return ms


def time_bwd(ss, torch, cfg, device, steps, warmup):
    """The backward (ss_bwd) of a forward workload: `steps` calls timed
    back to back with CUDA events, inputs and upstream gradients resident."""
    from ss_inputs import bwd_upstream, fwd_inputs
    inp = fwd_inputs(cfg.batch, cfg.seqlen, cfg.d_inner, cfg.d_state, cfg.dtype, cfg.seed, device,
                     gate=cfg.gate, D_kind=cfg.D_kind)
    dy, dl = bwd_upstream(cfg.batch, cfg.seqlen, cfg.d_inner, cfg.d_state, cfg.dtype, cfg.seed, device)
    stream = torch.cuda.current_stream(device)
    ws = torch.empty(ss.bwd_workspace_bytes(cfg.batch, cfg.seqlen, cfg.d_inner, cfg.dtype == "bf16"),
                     dtype=torch.uint8, device=device)
    grads = None

    def one():
        return ss.ss_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy, D=inp["D"], z=inp["z"],
                         delta_bias=inp["delta_bias"], dlast_state=dl, grads=grads, workspace=ws,
                         stream=stream)

    grads = one()
    for _ in range(warmup):
        one()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize(device)
    ms = e0.elapsed_time(e1) / steps
    del inp, dy, dl, grads, ws
    torch.cuda.empty_cache()
    return ms


def time_decode(ss, torch, device, steps_total=1000, reps=3):
    """The decode workload: 1000 successive ss_step calls (batch 256, d_inner
    5120, fresh bf16 inputs per step).  The 84 MB state fits in L2, so each
    step is timed alone with CUDA events after an L2 flush (a 256 MB write
    followed by a 256 MB read of another buffer);
    returns (ms per step, bytes per step, ms per step back to back in one CUDA
    graph with no flush, where the state may stay in L2, and (ms, bytes) of a
    bare in-place stream over the same state timed the same way)."""
    from ss_inputs import CONFIGS, step_inputs, step_sequence_inputs
    c = CONFIGS["decode"]
    base = step_inputs(c.batch, c.d_inner, c.d_state, c.dtype, c.seed, device, gate=c.gate)
    seq = step_sequence_inputs(steps_total, c.batch, c.d_inner, c.d_state, c.dtype, c.seed + 1,
                               device, gate=c.gate)
    y = torch.empty((c.batch, c.d_inner), dtype=torch.bfloat16, device=device)
    state = base["state"]
    # L2 flush: write 256 MB, then read another 256 MB so that the dirty lines
    # are written back during the flush, not during the timed step.
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device=device)
    sink = torch.empty((), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def one(t):
        ss.ss_step(state, seq["u"][t], seq["delta"][t], base["A"], seq["B"][t], seq["C"][t],
                   D=base["D"], z=seq["z"][t], delta_bias=base["delta_bias"], y=y, stream=stream)

    for t in range(3):
        one(t)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps_total)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps_total)]
    for t in range(steps_total):
        flush_w.zero_()
        torch.sum(flush_r, dim=None, out=sink)
        starts[t].record(stream)
        one(t)
        ends[t].record(stream)
    torch.cuda.synchronize(device)
    ms_cold = sum(s.elapsed_time(e) for s, e in zip(starts, ends)) / steps_total

    # Calibration: the bare in-place stream over the same state (multiply by
    # one, torch's elementwise kernel), timed the same way -- the ceiling of a
    # read-modify-write stream of this size, below the long-stream copy peak.
    cal = []
    for i in range(30):
        flush_w.zero_()
        torch.sum(flush_r, dim=None, out=sink)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        state.mul_(1.0)
        e1.record(stream)
        torch.cuda.synchronize(device)
        if i >= 5:
            cal.append(e0.elapsed_time(e1))
    ms_inplace = statistics.median(cal)
    inplace_bytes = 2 * state.numel() * state.element_size()

    def run_all():
        # launches on whatever stream is current (the capture stream in graph mode)
        for t in range(steps_total):
            ss.ss_step(state, seq["u"][t], seq["delta"][t], base["A"], seq["B"][t], seq["C"][t],
                       D=base["D"], z=seq["z"][t], delta_bias=base["delta_bias"], y=y)

    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        run_all()
    stream.wait_stream(side)
    torch.cuda.synchronize(device)
    with torch.cuda.graph(g):
        run_all()
    g.replay()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize(device)
    ms_warm = e0.elapsed_time(e1) / (reps * steps_total)
    del g
    return ms_cold, c.compulsory_bytes_per_step(), ms_warm, (ms_inplace, inplace_bytes)


def cpu_baseline(cfg, budget_s=10.0):
    """The oracle (fp32 state, as it stands) on a bounded sample of the
    workload: the first k channels of batch entry 0 over the full sequence."""
    import numpy as np

    import oracle
    from ss_inputs import fwd_inputs, to_f64
    cores = oracle.max_threads()
    L = cfg.seqlen

    def run(k):
        inp = fwd_inputs(1, L, k, cfg.d_state, cfg.dtype, cfg.seed, "cpu", gate=cfg.gate,
                         D_kind=cfg.D_kind)
        args = [to_f64(inp[n]) for n in ("u", "delta", "A", "B", "C")]
        t = time.perf_counter()
        oracle.fwd(*args, D=to_f64(inp["D"]), z=to_f64(inp["z"]),
                   delta_bias=to_f64(inp["delta_bias"]), precision="f32")
        return time.perf_counter() - t

    k0 = max(cores, 8)
    t0 = run(k0)
    k = int(min(cfg.d_inner, max(k0, k0 * budget_s / max(t0, 1e-6))))
    k = max(cores, (k // cores) * cores) if k >= cores else k
    t = run(k)
    chts_per_s = L * k / t
    bytes_per_chts = cfg.compulsory_bytes() / cfg.ch_ts
    return {"value": chts_per_s * bytes_per_chts / 1e9, "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{k} channels x {L} steps of batch entry 0 ({L * k} channel-timesteps, "
                      f"{t:.1f} s), fp32-state oracle; effective bytes scaled per channel-timestep",
            "ch_ts_per_s": chts_per_s}


def run_ours(args):
    import torch

    import selective_state_space_37_b200 as ss
    from ss_inputs import CONFIGS

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=device)
        dist = tdist
    ss.lib()
    cfg = CONFIGS[args.workload]
    hbm, peak_kind = peaks()
    clocks = ClockSampler(local)
    ms, inp, y, st, ws = time_fwd(ss, torch, cfg, device, args.steps, args.warmup,
                                  seed_offset=shard_seed(0, rank), dist=dist, clocks=clocks)
    ms = reduce_max(dist, ms, device)
    step_ms = ms / args.steps
    per_gpu_bytes = cfg.compulsory_bytes()
    value = aggregate_value(world, per_gpu_bytes, args.steps, ms)
    achieved = per_gpu_bytes / (step_ms * 1e-3) / 1e9

    e2e = None
    if args.e2e_steps > 0:
        e_ms, h2d, d2h = time_e2e(ss, torch, cfg, device, inp, args.e2e_steps)
        e_ms = reduce_max(dist, e_ms, device)
        e2e = {"value": world * per_gpu_bytes / (e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
               "path": "ss_fwd_host on pinned host buffers, 1-row batch slices, uploads / scans / "
                       "downloads overlapped"}
    del inp, y, st, ws
    torch.cuda.empty_cache()

    extras = {}
    if not args.no_extras and world == 1:
        for name in ("mamba130m", "million"):
            c = CONFIGS[name]
            steps = 20 if name == "mamba130m" else 3
            m, i2, y2, s2, w2 = time_fwd(ss, torch, c, device, steps, 2)
            sms = m / steps
            gbs = c.compulsory_bytes() / (sms * 1e-3) / 1e9
            extras[name] = {"ms_per_step": sms, "GB_s": gbs, "frac_of_hbm": gbs / hbm,
                            "ch_ts_per_s": c.ch_ts / (sms * 1e-3),
                            "chunk_len": ss.fwd_chunk_len(c.batch, c.seqlen, c.d_inner)}
            del i2, y2, s2, w2
            torch.cuda.empty_cache()
        gms = time_fwd_general(ss, torch, cfg, device, 20, 3)
        ggbs = cfg.compulsory_bytes() / (gms * 1e-3) / 1e9
        extras["general_A_" + cfg.name] = {"ms_per_step": gms, "GB_s": ggbs, "frac_of_hbm": ggbs / hbm,
                                           "ratio_to_structured": gms / step_ms,
                                           "note": "A perturbed off the A[d,n] = a_d (n+1) ladder: one "
                                                   "exponential per state and step"}
        extras["launch_overhead_mamba130m"] = launch_overhead(ss, torch, CONFIGS["mamba130m"], device)
        dms, dbytes, dms_warm, (ims, ibytes) = time_decode(ss, torch, device)
        igbs = ibytes / (ims * 1e-3) / 1e9
        extras["decode"] = {"ms_per_step": dms, "steps_per_s": 1e3 / dms,
                            "GB_s": dbytes / (dms * 1e-3) / 1e9,
                            "frac_of_hbm": dbytes / (dms * 1e-3) / 1e9 / hbm,
                            "note": "1000 ss_step calls, batch 256, d_inner 5120; each step "
                                    "timed alone after an L2 flush (the 84 MB state fits in L2)",
                            "graph_back_to_back_ms_per_step": dms_warm,
                            "graph_back_to_back_steps_per_s": 1e3 / dms_warm,
                            "inplace_stream_same_size": {"ms": ims, "GB_s": igbs,
                                                         "what": "torch in-place multiply of the same "
                                                                 "state, timed the same way"},
                            "frac_of_inplace_stream": dbytes / (dms * 1e-3) / 1e9 / igbs}
        torch.cuda.empty_cache()
        for name in ("mamba2p8b", "mamba130m"):
            c = CONFIGS[name]
            cms = time_fwd_conv(ss, torch, c, device, 20, 3)
            gbs = c.compulsory_bytes(conv=True) / (cms * 1e-3) / 1e9
            fwd_ms = step_ms if name == cfg.name else extras.get(name, {}).get("ms_per_step")
            extras["conv_fwd_" + name] = {"ms_per_step": cms, "GB_s": gbs, "frac_of_hbm": gbs / hbm,
                                          "ratio_to_fwd": (cms / fwd_ms) if fwd_ms else None,
                                          "note": "ss_fwd_conv: causal conv1d (width 4) + SiLU prologue "
                                                  "fused; x read in place of u"}
        _, bf16_peak, _ = tensor_peak()
        for name, (b, L, H, N) in SSD_SHAPES.items():
            sms = time_ssd(ss, torch, name, device, 10, 3)
            tf = ssd_useful_flops(b, L, H, N) / (sms * 1e-3) / 1e12
            gbs = ssd_compulsory_bytes(b, L, H, N) / (sms * 1e-3) / 1e9
            extras[name] = {"ms_per_step": sms, "TFLOP_s": tf, "frac_of_bf16_peak": tf / bf16_peak,
                            "GB_s": gbs, "frac_of_hbm": gbs / hbm,
                            "shape": {"batch": b, "seq_len": L, "nheads": H, "headdim": 64, "d_state": N},
                            "note": "ss_ssd_fwd: chunked matrix form, d_state 128 on tcgen05.mma (TMEM "
                                    "accumulators, TMA SWIZZLE_128B tiles, 128-step chunks); TFLOP_s "
                                    "counts the causal-half products of 64-step chunks, a fixed "
                                    "definition independent of the kernel's chunk"}
        for name in BLOCK_SHAPES:
            kms, toks, flops = time_block(ss, torch, name, device, 10, 3)
            extras[name] = {"ms_per_step": kms, "tokens_per_s": toks / (kms * 1e-3),
                            "projection_TFLOP_s": flops / (kms * 1e-3) / 1e12,
                            "shape": dict(zip(("batch", "seq_len", "d_model"), BLOCK_SHAPES[name])),
                            "note": "ss_block_fwd, random-init bf16 weights: in_proj, x_proj, dt_proj, "
                                    "out_proj on cuBLAS; conv1d + SiLU and the scan in this library"}
        for name in ("mamba2p8b", "mamba130m"):
            c = CONFIGS[name]
            bms = time_bwd(ss, torch, c, device, 5, 2)
            fwd_ms = step_ms if name == cfg.name else extras.get(name, {}).get("ms_per_step")
            gbs = c.bwd_compulsory_bytes() / (bms * 1e-3) / 1e9
            extras["bwd_" + name] = {"ms_per_step": bms, "GB_s": gbs, "frac_of_hbm": gbs / hbm,
                                     "ch_ts_per_s": c.ch_ts / (bms * 1e-3),
                                     "ratio_to_fwd": (bms / fwd_ms) if fwd_ms else None,
                                     "note": "ss_bwd (all input gradients), upstream dy and dlast_state "
                                             "resident; three kernel launches (chunk pass, record fold, gradient pass) "
                                                     "plus the zeroing memsets"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg)

    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": cfg.name, "description": cfg.description,
                       "batch": cfg.batch, "seq_len": cfg.seqlen, "d_inner": cfg.d_inner,
                       "d_state": cfg.d_state, "io_dtype": cfg.dtype, "state_dtype": "fp32",
                       "gate": cfg.gate, "parallelism": f"independent replica per GPU x{world}",
                       "chunk_len": ss.fwd_chunk_len(cfg.batch, cfg.seqlen, cfg.d_inner),
                       "l2": "inputs (%.2f GB) larger than the 126 MB L2; no flush"
                             % (cfg.compulsory_bytes() / 1e9),
                       "compulsory_bytes_per_step": per_gpu_bytes},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                         "frac": achieved / hbm, "traffic": profiled_traffic(cfg.name),
                         "traffic_source": ("carried over from the committed ncu summary "
                                            f"profiles/ss_fwd_kernel_{cfg.name}.md (taken on the same "
                                            "kernel source; not measured in this run)")
                                           if profiled_traffic(cfg.name) else None,
                         "peak_kind": f"{peak_kind} copy bandwidth", "kernel": "ss_fwd_kernel"},
            "roofline_alu": alu_roofline(torch, device, cfg.ch_ts / (step_ms * 1e-3), clocks.summary()),
            "e2e": e2e,
            "gpu_launches": args.steps,
            "clocks": clocks.summary(),
            "cpu_baseline": cpu,
            "ch_ts_per_s": world * cfg.ch_ts / (step_ms * 1e-3),
            "extras": extras or None,
        }
        print(json.dumps(out), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------ reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from ss_inputs import CONFIGS, fwd_inputs, to_f64
    cfg = CONFIGS[args.workload]
    cores = oracle.max_threads()
    L = cfg.seqlen
    # size one step to about one second of oracle work
    probe_k = max(cores, 8)
    inp = fwd_inputs(1, L, probe_k, cfg.d_state, cfg.dtype, cfg.seed, "cpu", gate=cfg.gate,
                     D_kind=cfg.D_kind)
    arrs = {n: to_f64(inp[n]) for n in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}

    def step(a):
        oracle.fwd(a["u"], a["delta"], a["A"], a["B"], a["C"], D=a["D"], z=a["z"],
                   delta_bias=a["delta_bias"], precision="f32")

    t = time.perf_counter()
    step(arrs)
    t_probe = time.perf_counter() - t
    k = int(min(cfg.d_inner, max(probe_k, probe_k * 1.0 / max(t_probe, 1e-6))))
    inp = fwd_inputs(1, L, k, cfg.d_state, cfg.dtype, cfg.seed, "cpu", gate=cfg.gate,
                     D_kind=cfg.D_kind)
    arrs = {n: to_f64(inp[n]) for n in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    for _ in range(args.warmup):
        step(arrs)
    t = time.perf_counter()
    for _ in range(args.steps):
        step(arrs)
    el = time.perf_counter() - t
    bytes_per_chts = cfg.compulsory_bytes() / cfg.ch_ts
    value = L * k * args.steps * bytes_per_chts / el / 1e9
    sample = (f"{k} channels x {L} steps of batch entry 0 per step ({L * k} channel-timesteps), "
              f"fp32-state oracle; effective bytes scaled per channel-timestep")
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
           "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
           "config": {"workload": cfg.name, "description": cfg.description, "batch": cfg.batch,
                      "seq_len": cfg.seqlen, "d_inner": cfg.d_inner, "d_state": cfg.d_state,
                      "io_dtype": cfg.dtype, "state_dtype": "fp32", "gate": cfg.gate},
           "cpu_baseline": {"kind": "oracle", "cores": cores, "sample": sample, "value": value,
                            "unit": "GB/s"},
           "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0},
           "gpu_launches": 0}
    print(json.dumps(out), flush=True)


def run_decode_only(args):
    """Decode workload alone (for profiling and quick checks): --steps single
    token steps of batch 256 x d_inner 5120, each timed after an L2 flush."""
    import torch

    import selective_state_space_37_b200 as ss
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(device)
    ss.lib()
    hbm, peak_kind = peaks()
    ms, nbytes, ms_warm, (ims, ibytes) = time_decode(ss, torch, device, steps_total=max(args.steps, 4), reps=1)
    gbs = nbytes / (ms * 1e-3) / 1e9
    print(json.dumps({"metric": "decode steps/s", "value": 1e3 / ms, "unit": "steps/s",
                      "n_gpus": 1, "steps": args.steps, "ms_per_step": ms,
                      "GB_s": gbs, "frac_of_hbm": gbs / hbm,
                      "peak_kind": peak_kind, "graph_back_to_back_ms_per_step": ms_warm,
                      "frac_of_inplace_stream": gbs / (ibytes / (ims * 1e-3) / 1e9)}), flush=True)


def run_bwd_only(args):
    """Backward workload alone (for profiling and quick checks): --steps ss_bwd
    calls on --workload."""
    import torch

    import selective_state_space_37_b200 as ss
    from ss_inputs import CONFIGS
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(device)
    ss.lib()
    hbm, peak_kind = peaks()
    c = CONFIGS[args.workload]
    ms = time_bwd(ss, torch, c, device, max(args.steps, 1), args.warmup)
    gbs = c.bwd_compulsory_bytes() / (ms * 1e-3) / 1e9
    print(json.dumps({"metric": "selective-scan bwd effective HBM GB/s", "value": gbs, "unit": "GB/s",
                      "n_gpus": 1, "steps": args.steps, "ms_per_step": ms, "workload": c.name,
                      "frac_of_hbm": gbs / hbm, "peak_kind": peak_kind,
                      "bwd_compulsory_bytes": c.bwd_compulsory_bytes(),
                      "ch_ts_per_s": c.ch_ts / (ms * 1e-3)}), flush=True)


def run_block_only(args):
    """Mamba-block inner path alone (for profiling): --steps ss_block_fwd calls
    on the 2.8B-shaped block (or the 130M one with --workload mamba130m)."""
    import torch

    import selective_state_space_37_b200 as ss
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(device)
    ss.lib()
    name = "block_" + args.workload
    ms, toks, flops = time_block(ss, torch, name, device, max(args.steps, 1), args.warmup)
    print(json.dumps({"metric": "Mamba block inner path tokens/s", "value": toks / (ms * 1e-3),
                      "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "ms_per_step": ms,
                      "workload": name, "projection_TFLOP_s": flops / (ms * 1e-3) / 1e12}), flush=True)


def run_ssd_only(args):
    """SSD scan alone (for profiling): --steps ss_ssd_fwd calls on the
    2.7B-shaped Mamba-2 layer (or the 130M one with --workload mamba130m)."""
    import torch

    import selective_state_space_37_b200 as ss
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(device)
    ss.lib()
    name = "ssd_mamba2_130m" if args.workload == "mamba130m" else "ssd_mamba2_2p7b"
    b, L, H, N = SSD_SHAPES[name]
    ms = time_ssd(ss, torch, name, device, max(args.steps, 1), args.warmup)
    _, peak, _ = tensor_peak()
    tf = ssd_useful_flops(b, L, H, N) / (ms * 1e-3) / 1e12
    print(json.dumps({"metric": "SSD scan useful TFLOP/s", "value": tf, "unit": "TFLOP/s", "n_gpus": 1,
                      "steps": args.steps, "ms_per_step": ms, "workload": name, "frac_of_bf16_peak": tf / peak,
                      "GB_s": ssd_compulsory_bytes(b, L, H, N) / (ms * 1e-3) / 1e9}), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.mode == "decode":
        run_decode_only(args)
    elif args.mode == "bwd":
        run_bwd_only(args)
    elif args.mode == "block":
        run_block_only(args)
    elif args.mode == "ssd":
        run_ssd_only(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
