#!/usr/bin/env python
"""Benchmark of the Local-Hessian NVFP4 calibration hot path on B200.

One step = the whole hot path for one layer, every kernel from liblh.so:
    lh_absmax -> lh_accumulate_hessian -> lh_sweep_scales_ws (126 candidates) -> lh_fake_quant
over the seeded synthetic layer (default: the attention projection,
W [4096,4096] bf16, X [2048,4096] bf16; --config picks another).

    python bench.py [--gpus N --steps K --warmup W] [--impl ours|reference] [--config 0..4]

Prints one JSON line (rank 0). `value` is NVFP4 blocks calibrated per second
of the whole step, summed over ranks (each rank calibrates its own layer: the
path shards by layer/expert with no collective, weak scaling). Timing: CUDA
events on the launching stream, L2 flushed before every timed step, max over
ranks. `--impl reference` times the FP64 CPU oracle on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 blocks swept/sec (126 cands) + Hessian tokens/sec; % of roofline, 1 B200"
UNIT = "blocks/s"
SWEEP_FLOP_PER_BLOCK = 126 * 152 * 2   # 16 dw FMA + 136 symmetric-form FMA per candidate
FP32_LANES_PER_SM = 128


def profiled_traffic(kernel_src: str, summary: str):
    """DRAM bytes per launch of a kernel, from the ncu summary committed under
    profiles/, or None when the kernel's source has changed since the counters
    were taken (the summary records the SHA-256 of the source it profiled)."""
    import hashlib
    import re
    src = os.path.join(ROOT, kernel_src)
    prof = os.path.join(ROOT, "profiles", summary)
    if not (os.path.exists(src) and os.path.exists(prof)):
        return None
    text = open(prof).read()
    m_sha = re.search(r"source sha256: ([0-9a-f]{64})", text)
    m_b = re.search(r"dram bytes per launch: (\d+)", text)
    if not (m_sha and m_b):
        return None
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != m_sha.group(1):
        return None
    return int(m_b.group(1))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=float(d["hbm_gbs"]), sm_max_mhz=float(d.get("sm_max_mhz", 1965.0)), source="measured")
    return dict(hbm_gbs=6650.0, sm_max_mhz=1965.0, source="fallback")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.rows = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)

    def stop(self):
        if self.proc is None:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["unsampled"], samples=0)
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.th.join(timeout=2)
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in self.rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return dict(sm_mhz=statistics.median(sm) if sm else None, sm_max_mhz=max(mx) if mx else None,
                    reasons=reasons, samples=len(self.rows))


def dist_setup(backend):
    import torch
    import torch.distributed as dist
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        from datetime import timedelta
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=timedelta(seconds=600))
    return ws, rank, local


def max_over_ranks(x: float, ws: int, device=None) -> float:
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def workload_desc(layer) -> str:
    dt = layer.w_dtype
    if layer.n_mats > 1:
        return (f"{layer.name}: {layer.n_mats} x W[{layer.c_out},{layer.c_in}] {dt}, "
                f"X[{layer.n_tok},{layer.c_in}] bf16 grouped by expert")
    return f"{layer.name}: W[{layer.c_out},{layer.c_in}] {dt}, X[{layer.n_tok},{layer.c_in}] bf16"


# ----------------------------------------------------------------------------- oracle (CPU) timing
def oracle_step(layer, W_f32, n_sweep: int, rng) -> tuple[float, float, float, int]:
    """Times the oracle on one bounded sample of the step: the full Hessian
    (up to 4096 tokens, scaled by token count), `n_sweep` sampled blocks of
    the sweep, and fake-quant of 8 sampled rows. Returns (estimated seconds for
    the whole step, hessian s, sweep s, sampled blocks)."""
    import oracle
    n_tok = layer.n_tok
    t_h = min(n_tok, 4096)
    Xs = layer.X[:t_h]
    off = None
    if layer.offsets is not None:
        off = np.minimum(layer.offsets, t_h)
    t0 = time.perf_counter()
    H = oracle.hessian(Xs, c_in=layer.c_in, offsets=off)
    th = (time.perf_counter() - t0) * (n_tok / t_h)
    J = layer.c_in // 16
    amax = np.array([oracle.absmax(W_f32[m]) for m in range(layer.n_mats)], np.float32) \
        if layer.n_mats <= 4 else np.max(np.abs(W_f32), axis=(1, 2)).astype(np.float32)
    mats = rng.integers(0, layer.n_mats, n_sweep)
    rows = rng.integers(0, layer.c_out, n_sweep)
    cols = rng.integers(0, J, n_sweep)
    Hfull = np.broadcast_to(H, (layer.n_mats,) + H.shape[1:]) if H.shape[0] == 1 else H
    t0 = time.perf_counter()
    codes, _, _ = oracle.sweep_blocks(W_f32, amax, np.ascontiguousarray(Hfull), mats, rows, cols)
    ts = (time.perf_counter() - t0) * (layer.n_blocks / n_sweep)
    nr = 8
    t0 = time.perf_counter()
    for i in range(nr):
        m, r = int(mats[i]), int(rows[i])
        oracle.fake_quant(W_f32[m, r:r + 1], amax[m:m + 1], np.ones((1, J), np.uint8))
    tf = (time.perf_counter() - t0) * (layer.n_mats * layer.c_out / nr)
    return th + ts + tf, th, ts, n_sweep


def run_reference(args):
    ws, rank, _ = dist_setup("gloo")
    if rank != 0:
        return
    import oracle
    import synth
    oracle.build()
    layer = synth.make_config(args.config)
    W_f32 = layer.W_f32()
    rng = np.random.default_rng(0)
    n_sweep = 4000
    for _ in range(args.warmup):
        oracle_step(layer, W_f32, 400, rng)
    est = []
    for _ in range(args.steps):
        est.append(oracle_step(layer, W_f32, n_sweep, rng)[0])
    t = float(sum(est))
    value = layer.n_blocks * args.steps / t
    sample = (f"per step: full Hessian (<=4096 tokens, scaled), {n_sweep} random blocks of the sweep, "
              f"8 rows of fake-quant; times scaled to the whole layer")
    line = dict(metric=METRIC, value=value, unit=UNIT, n_gpus=args.gpus, steps=args.steps, warmup=args.warmup,
                ms_per_step=1e3 * t / args.steps, higher_is_better=True, scaling="weak", vs_baseline=None,
                dtype="f64", data="synthetic", impl="reference",
                config=dict(workload=workload_desc(layer), l2="n/a (CPU)", parallelism="none"),
                cpu_baseline=dict(value=value, unit=UNIT, cores=1, kind="oracle", sample=sample),
                e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0),
                gpu_launches=0)
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- CUDA path
def run_ours(args):
    import torch
    ws, rank, local = dist_setup("nccl")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import scale_calibration_b200 as lh
    import synth

    layer = synth.make_config(args.config)
    n_mats, c_out, c_in, n_tok = layer.n_mats, layer.c_out, layer.c_in, layer.n_tok
    J = c_in // 16
    grouped = layer.offsets is not None
    n_groups = n_mats if grouped else 1

    if layer.w_dtype == "bf16":
        W_host = torch.from_numpy(layer.W.view(np.int16)).view(torch.bfloat16)
    else:
        W_host = torch.from_numpy(np.ascontiguousarray(layer.W))
    X_host = torch.from_numpy(layer.X.view(np.int16)).view(torch.bfloat16)
    W = W_host.to(dev)
    X = X_host.to(dev)
    off = torch.from_numpy(layer.offsets).to(dev) if grouped else None

    amax = torch.empty(n_mats, dtype=torch.float32, device=dev)
    H = torch.zeros(n_groups, J, 16, 16, dtype=torch.float32, device=dev)
    wsb = lh.lh_hessian_workspace_bytes(n_tok, c_in, n_groups)
    wsp = torch.empty(max(wsb, 256), dtype=torch.uint8, device=dev)
    swsb = lh.lh_sweep_workspace_bytes(n_mats, c_in)
    swsp = torch.empty(max(swsb, 16), dtype=torch.uint8, device=dev)
    codes = torch.empty(n_mats, c_out, J, dtype=torch.uint8, device=dev)
    bamax = torch.empty(n_mats, c_out, J, dtype=torch.float32, device=dev)
    Wq = torch.empty(n_mats, c_out, c_in, dtype=W.dtype, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 1 << 28) // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    s = stream.cuda_stream
    ld = W.stride(1)
    launches_per_step = 1 + 2 + (1 if grouped else 0) + 2 + 1  # sweep: bounds kernel + sweep kernel

    def step(ev=None):
        H.zero_()
        if ev: ev[0].record(stream)
        lh.lh_absmax(W, W, n_mats, c_out, c_in, ld, amax, s)
        if ev: ev[1].record(stream)
        lh.lh_accumulate_hessian(X, lh.LH_BF16, n_tok, c_in, X.stride(0), off, n_groups, H, wsp, wsb, s)
        if ev: ev[2].record(stream)
        lh.lh_sweep_scales_ws(W, W, n_mats, c_out, c_in, ld, amax, H, bamax, codes, swsp, swsb, s)
        if ev: ev[3].record(stream)
        lh.lh_fake_quant(W, W, n_mats, c_out, c_in, ld, amax, codes, Wq, Wq, s)
        if ev: ev[4].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    assert lh.lh_workspace_status(wsp, s) == 0

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    sampler = ClockSampler(dev.index)
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    for i in range(args.steps):
        flush.zero_()  # cold L2 for every step
        step(evs[i])
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if ws > 1:
        torch.distributed.barrier()
    per = np.array([[e[k].elapsed_time(e[k + 1]) for k in range(4)] for e in evs])  # ms [steps, 4]
    t_rank = float(per.sum()) / 1e3
    t_all = max_over_ranks(t_rank, ws, dev)
    value = n_mats * c_out * J * ws * args.steps / t_all
    t_abs, t_hess, t_sweep, t_fq = (float(x) for x in per.mean(axis=0))  # ms
    names = ("absmax", "hessian", "sweep", "fake_quant")
    per_median = {n: float(v) for n, v in zip(names, np.median(per, axis=0))}
    per_min = {n: float(v) for n, v in zip(names, per.min(axis=0))}

    # ---- the Hessian call with X left in L2 (no flush between calls): X of the attention,
    # MLP-up and MoE layers (17, 67, 134 MB) fits or nearly fits the 126 MB L2
    warm = []
    for i in range(3 + args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        lh.lh_accumulate_hessian(X, lh.LH_BF16, n_tok, c_in, X.stride(0), off, n_groups, H, wsp, wsb, s)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if i >= 3:
            warm.append(e0.elapsed_time(e1))
    t_hess_warm = float(np.median(warm))
    H.zero_()  # back to one accumulation (deterministic: the same H as the timed steps)
    lh.lh_accumulate_hessian(X, lh.LH_BF16, n_tok, c_in, X.stride(0), off, n_groups, H, wsp, wsb, s)

    # ---- packed NVFP4 export fused with the fake quantisation (one read of W writes the
    # packed nibbles, the scale bytes and W_q), timed like the step, L2 flushed each time
    packed = torch.empty(n_mats, c_out, c_in // 2, dtype=torch.uint8, device=dev)
    scales = torch.empty(n_mats, c_out, J, dtype=torch.uint8, device=dev)
    gscale = torch.empty(n_mats, dtype=torch.float32, device=dev)
    qdt = lh.LH_BF16 if Wq.dtype == torch.bfloat16 else lh.LH_F32
    for _ in range(3):
        lh.lh_quantize_nvfp4(W, W, n_mats, c_out, c_in, ld, amax, codes, packed, scales, gscale, Wq, qdt, s)
    ex_t = []
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        lh.lh_quantize_nvfp4(W, W, n_mats, c_out, c_in, ld, amax, codes, packed, scales, gscale, Wq, qdt, s)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ex_t.append(e0.elapsed_time(e1))
    t_ex = float(np.median(ex_t))  # ms
    ex_bytes = (W.numel() * W.element_size() + 2 * codes.numel() + packed.numel() + Wq.numel() * Wq.element_size()
                + 8 * n_mats)

    # ---- the pages' baseline scalers on the same layer (context beside the Local-Hessian sweep)
    bl_codes = torch.empty_like(codes)
    bl_amax = torch.empty_like(bamax)
    baselines = {}
    for name, meth in (("max", lh.LH_SCALE_MAX), ("four_over_six", lh.LH_SCALE_FOUR_OVER_SIX),
                       ("mse_sweep", lh.LH_SCALE_MSE)):
        for _ in range(3):
            lh.lh_baseline_scales(W, W, n_mats, c_out, c_in, ld, amax, meth, bl_amax, bl_codes, s)
        tb = []
        for _ in range(max(3, min(args.steps, 10))):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            lh.lh_baseline_scales(W, W, n_mats, c_out, c_in, ld, amax, meth, bl_amax, bl_codes, s)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            tb.append(e0.elapsed_time(e1))
        t_b = float(np.median(tb))
        baselines[name] = dict(ms=t_b, blocks_per_s=n_mats * c_out * J / (t_b / 1e3))
    # the amax multiplier search (0.25 + 0.1 k, 38 multipliers) with this layer's H
    for _ in range(3):
        lh.lh_search_amax(W, W, n_mats, c_out, c_in, ld, amax, H, bl_amax, bl_codes, stream=s)
    tb = []
    for _ in range(max(3, min(args.steps, 10))):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        lh.lh_search_amax(W, W, n_mats, c_out, c_in, ld, amax, H, bl_amax, bl_codes, stream=s)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        tb.append(e0.elapsed_time(e1))
    t_b = float(np.median(tb))
    baselines["amax_search_hessian"] = dict(ms=t_b, blocks_per_s=n_mats * c_out * J / (t_b / 1e3))

    # ---- end to end through the public API with host buffers: every step copies its
    # inputs from pinned host memory and its results (codes, best amax, W_q) back.
    # Consecutive steps are pipelined over two device buffer sets on three streams
    # (copy-in, compute, copy-out), ordered by events, so copies overlap compute.
    W_pin = W_host.pin_memory()
    X_pin = X_host.pin_memory()
    off_host = torch.from_numpy(layer.offsets).pin_memory() if grouped else None
    sets = []
    for _ in range(2):
        d = dict(W=torch.empty_like(W), X=torch.empty_like(X), off=torch.empty_like(off) if grouped else None,
                 amax=torch.empty_like(amax), H=torch.empty_like(H), ws=torch.empty_like(wsp),
                 sws=torch.empty_like(swsp),
                 codes=torch.empty_like(codes), bamax=torch.empty_like(bamax), Wq=torch.empty_like(Wq),
                 codes_pin=torch.empty(codes.shape, dtype=codes.dtype).pin_memory(),
                 bam_pin=torch.empty(bamax.shape, dtype=bamax.dtype).pin_memory(),
                 Wq_pin=torch.empty(Wq.shape, dtype=Wq.dtype).pin_memory(),
                 ev_in=torch.cuda.Event(), ev_done=torch.cuda.Event(), ev_out=torch.cuda.Event())
        sets.append(d)
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))

    def e2e_step(i):
        d = sets[i % 2]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(d["ev_done"])  # step i-2 finished reading this set
            d["W"].copy_(W_pin, non_blocking=True)
            d["X"].copy_(X_pin, non_blocking=True)
            if grouped:
                d["off"].copy_(off_host, non_blocking=True)
            d["ev_in"].record(s_in)
        cs = s_cmp.cuda_stream
        s_cmp.wait_event(d["ev_in"])
        if i >= 2:
            s_cmp.wait_event(d["ev_out"])  # results of step i-2 copied out of this set
        with torch.cuda.stream(s_cmp):
            d["H"].zero_()
        lh.lh_absmax(d["W"], d["W"], n_mats, c_out, c_in, ld, d["amax"], cs)
        lh.lh_accumulate_hessian(d["X"], lh.LH_BF16, n_tok, c_in, d["X"].stride(0), d["off"], n_groups, d["H"],
                                 d["ws"], wsb, cs)
        lh.lh_sweep_scales_ws(d["W"], d["W"], n_mats, c_out, c_in, ld, d["amax"], d["H"], d["bamax"], d["codes"],
                              d["sws"], swsb, cs)
        lh.lh_fake_quant(d["W"], d["W"], n_mats, c_out, c_in, ld, d["amax"], d["codes"], d["Wq"], d["Wq"], cs)
        d["ev_done"].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(d["ev_done"])
            d["codes_pin"].copy_(d["codes"], non_blocking=True)
            d["bam_pin"].copy_(d["bamax"], non_blocking=True)
            d["Wq_pin"].copy_(d["Wq"], non_blocking=True)
            d["ev_out"].record(s_out)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    e_start.record(s_in)
    for i in range(args.steps):
        e2e_step(i)
    for st in (s_in, s_cmp):
        s_out.wait_stream(st)
    e_end.record(s_out)
    torch.cuda.synchronize(dev)
    t_e2e = max_over_ranks(e_start.elapsed_time(e_end) / 1e3, ws, dev)
    h2d = W.numel() * W.element_size() + X.numel() * X.element_size() + (off.numel() * 8 if grouped else 0)
    d2h = codes.numel() + bamax.numel() * 4 + Wq.numel() * Wq.element_size()
    e2e = dict(value=n_mats * c_out * J * ws * args.steps / t_e2e, unit=UNIT, h2d_bytes_per_step=int(h2d),
               d2h_bytes_per_step=int(d2h), pipelined="2 buffer sets, copy-in / compute / copy-out streams")
    # the last step's results equal those of the device-resident run
    dl = sets[(args.steps - 1) % 2]
    assert torch.equal(dl["codes_pin"], codes.cpu()), "end-to-end results differ from the device run"

    # ---- rooflines
    peaks = load_peaks()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    fp32_peak = sms * FP32_LANES_PER_SM * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12  # TFLOP/s
    n_blocks = n_mats * c_out * J
    sweep_tflops = SWEEP_FLOP_PER_BLOCK * n_blocks / (t_sweep / 1e3) / 1e12
    hess_bytes = 2 * c_in * n_tok
    hess_gbs = hess_bytes / (t_hess / 1e3) / 1e9
    sweep_traffic = profiled_traffic("scale_calibration_b200/csrc/sweep.cu", "sweep_kernel_attn_proj.md") \
        if args.config == 1 else None
    roofline = dict(bound="alu", kernel="sweep_kernel", achieved=sweep_tflops, peak=fp32_peak, unit="TFLOP/s",
                    frac=sweep_tflops / fp32_peak, traffic=sweep_traffic,
                    traffic_note="DRAM bytes per launch from the committed ncu summary (null if the kernel changed)",
                    peak_note=f"FP32 CUDA-core peak {sms} SMs x 128 lanes x 2 flop x {peaks['sm_max_mhz']:.0f} MHz",
                    flop_per_block=SWEEP_FLOP_PER_BLOCK)
    if clocks.get("sm_mhz"):
        roofline["frac_at_measured_clock"] = sweep_tflops / (fp32_peak * clocks["sm_mhz"] / peaks["sm_max_mhz"])
    hessian = dict(tokens_per_s=n_tok * ws / (t_hess / 1e3) if t_hess > 0 else None, bound="hbm",
                   achieved=hess_gbs, peak=peaks["hbm_gbs"], unit="GB/s", frac=hess_gbs / peaks["hbm_gbs"],
                   bytes_per_launch=hess_bytes, peak_source=peaks["source"],
                   traffic=profiled_traffic("scale_calibration_b200/csrc/hessian.cu", "hessian_tc_kernel_mlp_down.md")
                   if args.config == 3 else None,
                   warm_l2=dict(ms=t_hess_warm, tokens_per_s=n_tok * ws / (t_hess_warm / 1e3),
                                achieved=hess_bytes / (t_hess_warm / 1e3) / 1e9,
                                note="median of back-to-back calls without an L2 flush (X partly or wholly in L2); "
                                     "the HBM fraction above is the cold-L2 one"))

    line = dict(metric=METRIC, value=value, unit=UNIT, n_gpus=ws, steps=args.steps, warmup=args.warmup,
                ms_per_step=1e3 * t_all / args.steps, higher_is_better=True, scaling="weak", vs_baseline=None,
                dtype="f32", data="synthetic",
                config=dict(workload=workload_desc(layer), blocks=n_blocks, tokens=n_tok, l2="flushed",
                            parallelism=f"{ws} independent layers, no collective"),
                kernels_ms=dict(absmax=t_abs, hessian=t_hess, sweep=t_sweep, fake_quant=t_fq),
                kernels_ms_median=per_median, kernels_ms_min=per_min,
                baseline_scalers=baselines,
                nvfp4_export=dict(ms=t_ex, bytes_per_launch=int(ex_bytes), bound="hbm",
                                  achieved=ex_bytes / (t_ex / 1e3) / 1e9, unit="GB/s",
                                  frac=ex_bytes / (t_ex / 1e3) / 1e9 / load_peaks()["hbm_gbs"],
                                  note="lh_quantize_nvfp4: packed E2M1 + scale bytes + W_q in one pass; "
                                       "not part of the timed step"),
                sweep_blocks_per_s=n_blocks * ws / (t_sweep / 1e3), roofline=roofline, hessian=hessian,
                e2e=e2e, gpu_launches=launches_per_step * args.steps, clocks=clocks)

    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        rng = np.random.default_rng(1)
        W_f32 = layer.W_f32()
        t0 = time.perf_counter()
        tot, th, tsw, ns = 0.0, 0.0, 0.0, 0
        reps = 0
        while time.perf_counter() - t0 < args.cpu_seconds and reps < 50:
            e, a, b, n = oracle_step(layer, W_f32, 20000, rng)
            tot += e; th += a; tsw += b; ns += n; reps += 1
        cpu_value = n_blocks * reps / tot
        line["cpu_baseline"] = dict(value=cpu_value, unit=UNIT, cores=1, kind="oracle",
                                    sample=(f"{reps} x (full Hessian of <=4096 tokens, 20000 random sweep blocks, "
                                            f"8 fake-quant rows), scaled to the whole layer"))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.destroy_process_group()


def run_sharded(args):
    """One layer split over the ranks (strong scaling): each rank holds a share of
    the calibration tokens and of the rows; the global amax is a MAX all-reduce,
    the Hessian a SUM all-reduce of the ranks' partial H (NCCL), and each rank
    sweeps and fake-quantises its rows with the full H."""
    import torch
    import torch.distributed as dist
    ws, rank, local = dist_setup("nccl")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import scale_calibration_b200 as lh
    import synth
    from scale_calibration_b200 import distributed as lhd

    layer = synth.make_config(args.config)
    n_mats, c_out, c_in, n_tok = layer.n_mats, layer.c_out, layer.c_in, layer.n_tok
    J = c_in // 16
    grouped = layer.offsets is not None
    n_groups = n_mats if grouped else 1
    t0, t1, loc = lhd.token_shard(n_tok, rank, ws, layer.offsets)
    r0, r1 = lhd.row_shard(c_out, rank, ws)
    rows = r1 - r0
    Wn = layer.W[:, r0:r1]
    W_host = (torch.from_numpy(np.ascontiguousarray(Wn).view(np.int16)).view(torch.bfloat16) if layer.w_dtype == "bf16"
              else torch.from_numpy(np.ascontiguousarray(Wn)))
    X_host = torch.from_numpy(np.ascontiguousarray(layer.X[t0:t1]).view(np.int16)).view(torch.bfloat16)
    W = W_host.to(dev)
    X = X_host.to(dev)
    n_loc = t1 - t0
    off = torch.from_numpy(loc).to(dev) if grouped else None
    amax = torch.empty(n_mats, dtype=torch.float32, device=dev)
    H = torch.zeros(n_groups, J, 16, 16, dtype=torch.float32, device=dev)
    wsb = lh.lh_hessian_workspace_bytes(max(n_loc, 1), c_in, n_groups)
    wsp = torch.empty(max(wsb, 256), dtype=torch.uint8, device=dev)
    swsb = lh.lh_sweep_workspace_bytes(n_mats, c_in)
    swsp = torch.empty(max(swsb, 16), dtype=torch.uint8, device=dev)
    codes = torch.empty(n_mats, rows, J, dtype=torch.uint8, device=dev)
    bamax = torch.empty(n_mats, rows, J, dtype=torch.float32, device=dev)
    Wq = torch.empty(n_mats, rows, c_in, dtype=W.dtype, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 1 << 28) // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    s = stream.cuda_stream
    ld = W.stride(1)

    def step():
        H.zero_()
        lh.lh_absmax(W, W, n_mats, rows, c_in, ld, amax, s)
        if ws > 1:
            dist.all_reduce(amax, op=dist.ReduceOp.MAX)
        if n_loc > 0:
            lhd.accumulate_hessian_sharded(X, n_loc, c_in, off, n_groups, H, wsp, wsb, s, check_status=False)
        else:
            lhd.allreduce_hessian(H)
        lh.lh_sweep_scales_ws(W, W, n_mats, rows, c_in, ld, amax, H, bamax, codes, swsp, swsb, s)
        lh.lh_fake_quant(W, W, n_mats, rows, c_in, ld, amax, codes, Wq, Wq, s)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    assert n_loc == 0 or lh.lh_workspace_status(wsp, s) == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ts = []
    sampler = ClockSampler(dev.index)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    for _ in range(args.steps):
        flush.zero_()
        e0.record(stream)
        step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ts.append(e0.elapsed_time(e1) / 1e3)
    clocks = sampler.stop()
    t_all = max_over_ranks(float(sum(ts)), ws, dev)
    n_blocks = n_mats * c_out * J
    value = n_blocks * args.steps / t_all
    line = dict(metric=METRIC, value=value, unit=UNIT, n_gpus=ws, steps=args.steps, warmup=args.warmup,
                ms_per_step=1e3 * t_all / args.steps, higher_is_better=True, scaling="strong", vs_baseline=None,
                dtype="f32", data="synthetic",
                config=dict(workload=workload_desc(layer), blocks=n_blocks, tokens=n_tok, l2="flushed",
                            parallelism=f"{ws} ranks: tokens and rows sharded, amax MAX and H SUM all-reduce (NCCL)"),
                gpu_launches=(4 + (1 if grouped else 0) + 1) * args.steps, clocks=clocks)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=4, help="0 tiny, 1 attn_proj, 2 mlp_up, 3 mlp_down, 4 moe_experts (default: the largest single-GPU layer)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--mode", choices=["layers", "sharded"], default="layers",
                    help="layers: each rank calibrates its own layer (weak scaling); sharded: one layer split over "
                         "the ranks with an all-reduce of H (strong scaling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.mode == "sharded":
        run_sharded(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
