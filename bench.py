#!/usr/bin/env python
"""Benchmark of the Local-Hessian NVFP4 calibration hot path on B200.

One step = the whole hot path for one layer, every kernel from liblh.so:
    H = 0 -> lh_absmax -> lh_accumulate_hessian -> lh_sweep_scales_ws (126 candidates) -> lh_fake_quant
over a seeded synthetic layer. The default is the largest single-GPU layer, the
MoE expert bank (64 x W [1536,2048] bf16, X [32768,2048] bf16 grouped by expert
with Zipf(1.1) token counts); --config picks another.

    python bench.py [--gpus N --steps K --warmup W] [--impl ours|reference] [--config 0..4]

With N > 1 (torchrun, or `--gpus N` alone, which starts N local ranks) one layer
is split over the ranks: each rank accumulates the Hessian of its share of the
tokens and one SUM all-reduce of H (NCCL) gives every rank the layer's H; each
rank then sweeps and fake-quantises its share of the blocks (whole experts of an
expert bank, else a range of block columns), so the global amax of a matrix
split over ranks is a MAX all-reduce. Total work is fixed (strong scaling).

Prints one JSON line (rank 0). `value` is NVFP4 blocks calibrated per second of
the whole step over all ranks. Timing: CUDA events on the launching stream, L2
flushed before every timed step (a 256 MB write, then a 256 MB read of another
buffer, so that the lines the flush wrote are written back before the step
rather than during it), max over ranks.
`--impl reference` times the FP64 CPU oracle on the host cores on bounded
samples of the same layer, extrapolated to it (labelled so in the line).
"""
from __future__ import annotations

import argparse
import json
import os
import socket
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
# kernels of ours launched per call (counted in the timed region's gpu_launches)
LAUNCHES = dict(absmax=2, hessian_plain=1, hessian_grouped=1, sweep_ws=2, fake_quant=1)


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
        dist.init_process_group(backend, timeout=timedelta(seconds=300))
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


def parallelism_desc(ws: int) -> str:
    if ws == 1:
        return "1 GPU"
    return (f"{ws} ranks: tokens sharded, H SUM all-reduce (NCCL); sweep and fake-quant sharded by expert or "
            f"block column; amax MAX all-reduce where a matrix is split")


def bench_config(layer, ws: int) -> dict:
    """The `config` of the JSON line; the same dict on both arms."""
    return dict(workload=workload_desc(layer), blocks=int(layer.n_blocks), tokens=int(layer.n_tok),
                l2="flushed before every timed step (256 MB write, then 256 MB read of another buffer)",
                parallelism=parallelism_desc(ws))


def spawn_ranks(args) -> int:
    """`--gpus N` (N > 1) without a launcher: run this script as N local ranks
    under torch.distributed.run (rendezvous on 127.0.0.1) and return its exit code."""
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd, cwd=ROOT)


# ----------------------------------------------------------------------------- oracle (CPU) timing
def oracle_step(layer, W_f32, n_sweep: int, rng) -> tuple[float, float, float, int, float]:
    """Times the oracle on one bounded sample of the step: the full Hessian
    (up to 4096 tokens, scaled by token count), `n_sweep` sampled blocks of
    the sweep, and fake-quant of 8 sampled rows. Returns (estimated seconds for
    the whole step, hessian s, sweep s, sampled blocks, measured seconds)."""
    import oracle
    n_tok = layer.n_tok
    t_h = min(n_tok, 4096)
    Xs = layer.X[:t_h]
    off = None
    if layer.offsets is not None:
        off = np.minimum(layer.offsets, t_h)
    t0 = time.perf_counter()
    H = oracle.hessian(Xs, c_in=layer.c_in, offsets=off)
    m_h = time.perf_counter() - t0
    th = m_h * (n_tok / t_h)
    J = layer.c_in // 16
    amax = np.array([oracle.absmax(W_f32[m]) for m in range(layer.n_mats)], np.float32) \
        if layer.n_mats <= 4 else np.max(np.abs(W_f32), axis=(1, 2)).astype(np.float32)
    mats = rng.integers(0, layer.n_mats, n_sweep)
    rows = rng.integers(0, layer.c_out, n_sweep)
    cols = rng.integers(0, J, n_sweep)
    Hfull = np.broadcast_to(H, (layer.n_mats,) + H.shape[1:]) if H.shape[0] == 1 else H
    t0 = time.perf_counter()
    codes, _, _ = oracle.sweep_blocks(W_f32, amax, np.ascontiguousarray(Hfull), mats, rows, cols)
    m_s = time.perf_counter() - t0
    ts = m_s * (layer.n_blocks / n_sweep)
    nr = 8
    t0 = time.perf_counter()
    for i in range(nr):
        m, r = int(mats[i]), int(rows[i])
        oracle.fake_quant(W_f32[m, r:r + 1], amax[m:m + 1], np.ones((1, J), np.uint8))
    m_f = time.perf_counter() - t0
    tf = m_f * (layer.n_mats * layer.c_out / nr)
    return th + ts + tf, th, ts, n_sweep, m_h + m_s + m_f


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
    est, meas = [], []
    for _ in range(args.steps):
        e = oracle_step(layer, W_f32, n_sweep, rng)
        est.append(e[0])
        meas.append(e[4])
    t = float(sum(est))
    value = layer.n_blocks * args.steps / t
    sample = (f"per step: oracle Hessian of the first <= 4096 tokens (scaled by the token count), {n_sweep} random "
              f"blocks of the 126-code sweep (scaled by the block count), fake-quant of 8 rows (scaled by the row "
              f"count); one host core of {os.cpu_count()}")
    line = dict(metric=METRIC, value=value, unit=UNIT, n_gpus=args.gpus, steps=args.steps, warmup=args.warmup,
                ms_per_step=1e3 * t / args.steps, higher_is_better=True, scaling="strong", vs_baseline=None,
                dtype="f64", data="synthetic", impl="reference",
                extrapolated=True, measured_seconds=float(sum(meas)), sampled_blocks_per_step=n_sweep,
                host="CPU oracle (FP64, single-threaded); no GPU, no L2 flush",
                config=bench_config(layer, ws),
                cpu_baseline=dict(value=value, unit=UNIT, cores=1, host_cores=os.cpu_count(), kind="oracle",
                                  sample=sample, extrapolated=True),
                e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0),
                gpu_launches=0)
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- CUDA path
def fma_probe(lh, torch, dev, stream) -> dict:
    """Measured FP32 FMA throughput on every SM, scalar (fma.rn.f32) and packed
    (fma.rn.f32x2), with the library's probe kernel (CUDA events, best of 3)."""
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    out = torch.zeros(1, device=dev)
    blocks, iters = 8 * sms, 4000
    res = dict(blocks=blocks, iters=iters)
    for name, packed in (("scalar_tflops", False), ("packed_tflops", True)):
        for _ in range(2):
            lh.lh_probe_fma(packed, blocks, iters, out, stream.cuda_stream)
        ts = []
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            lh.lh_probe_fma(packed, blocks, iters, out, stream.cuda_stream)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ts.append(e0.elapsed_time(e1) / 1e3)
        res[name] = lh.lh_probe_fma_flop(blocks, iters) / min(ts) / 1e12
    return res


def sweep_work(lh, torch, dev, s, W, n_mats, c_out, c_in, ld, amax, H, codes, t_sweep_ms, fp32_peak):
    """What the sweep executes, from its measurement build (liblh_counters.so, the
    same sources with work counters compiled in): one extra untimed call on the
    same inputs, whose codes must equal the timed library's. The executed FP32 work
    counts 272 flop per full form (136 FMA) and 64 per quantised candidate (16 FMA
    for dw, 16 for the diagonal bound), per block; its rate uses the timed sweep."""
    import ctypes
    path = os.path.join(ROOT, "scale_calibration_b200", "liblh_counters.so")
    if not os.path.exists(path):
        return None
    lib = ctypes.CDLL(path)
    P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    lib.lh_sweep_scales_ws.argtypes = [P, I32, I64, I64, I64, I64, P, P, P, P, P, SZ, P]
    lib.lh_sweep_scales_ws.restype = I32
    lib.lh_sweep_workspace_bytes.argtypes = [I64, I64]
    lib.lh_sweep_workspace_bytes.restype = SZ
    lib.lh_debug_sweep_counts.argtypes = [P, I32]
    lib.lh_debug_sweep_counts.restype = I32
    wsb = lib.lh_sweep_workspace_bytes(n_mats, c_in)
    wsp = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
    c2 = torch.empty_like(codes)
    a2 = torch.empty(codes.shape, dtype=torch.float32, device=dev)
    torch.cuda.synchronize(dev)
    if lib.lh_debug_sweep_counts(None, 1) != 0:
        return None
    dt = lh.LH_BF16 if W.dtype == torch.bfloat16 else lh.LH_F32
    st = lib.lh_sweep_scales_ws(W.data_ptr(), dt, n_mats, c_out, c_in, ld, amax.data_ptr(), H.data_ptr(),
                                a2.data_ptr(), c2.data_ptr(), wsp.data_ptr(), wsb, s)
    torch.cuda.synchronize(dev)
    cnt = (ctypes.c_uint64 * 9)()
    if st != 0 or lib.lh_debug_sweep_counts(cnt, 0) != 0:
        return None
    chunks, blocks, cand, forms, need, below, resweep, classes, pairs = (int(x) for x in cnt)
    if blocks == 0:
        return None
    fpb = 32.0 * forms / blocks
    qpb = 32.0 * cand / blocks
    flop = 272.0 * fpb + 64.0 * qpb
    tf = flop * blocks / (t_sweep_ms / 1e3) / 1e12
    return dict(forms_per_block=fpb, lane_needed_forms_per_block=need / blocks,
                candidates_quantised_per_block=qpb, class_bound_tests_per_block=32.0 * below / blocks,
                fp64_resweeps_per_1000_blocks=1000.0 * resweep / blocks,
                fp64_pairs_per_1000_blocks=1000.0 * pairs / blocks, flop_per_block=flop,
                achieved=tf, unit="TFLOP/s", frac=tf / fp32_peak, same_codes=bool(torch.equal(codes, c2)),
                note="measurement build (liblh_counters.so): forms and candidates are counted per 32-lane warp, "
                     "so every lane pays for a form any lane needs; flop = 272 per form + 64 per quantised "
                     "candidate, over the timed sweep")


def make_share(layer, rank: int, ws: int) -> dict:
    """This rank's inputs: a contiguous token share (with its group offsets) for
    the Hessian and a share of the blocks for the sweep (see sweep_shard)."""
    from scale_calibration_b200 import distributed as lhd
    n_mats, c_out, c_in, n_tok = layer.n_mats, layer.c_out, layer.c_in, layer.n_tok
    J = c_in // 16
    t0, t1, loc = lhd.token_shard(n_tok, rank, ws, layer.offsets)
    kind, lo, hi = lhd.sweep_shard(n_mats, c_out, J, rank, ws)
    if kind == "mats":
        Wn = layer.W[lo:hi]
    elif kind == "cols":
        Wn = layer.W[:, :, 16 * lo:16 * hi]
    else:
        Wn = layer.W[:, lo:hi]
    return dict(t0=t0, t1=t1, offsets=loc, kind=kind, lo=lo, hi=hi, W=np.ascontiguousarray(Wn),
                amax_allreduce=(kind != "mats" and ws > 1))


def run_ours(args):
    import torch
    import torch.distributed as dist
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
    sh = make_share(layer, rank, ws)
    s_mats, s_out, s_cin = sh["W"].shape
    s_J = s_cin // 16
    s_blocks = s_mats * s_out * s_J
    n_loc = sh["t1"] - sh["t0"]

    if layer.w_dtype == "bf16":
        W_host = torch.from_numpy(sh["W"].view(np.int16)).view(torch.bfloat16)
    else:
        W_host = torch.from_numpy(sh["W"])
    X_host = torch.from_numpy(np.ascontiguousarray(layer.X[sh["t0"]:sh["t1"]]).view(np.int16)).view(torch.bfloat16)
    W = W_host.to(dev)
    X = X_host.to(dev)
    off = torch.from_numpy(sh["offsets"]).to(dev) if grouped else None

    amax = torch.zeros(s_mats, dtype=torch.float32, device=dev)
    H = torch.zeros(n_groups, J, 16, 16, dtype=torch.float32, device=dev)

    def sweep_h(Hf):   # the rows of H this rank's sweep reads (contiguous views)
        if sh["kind"] == "mats":
            return Hf[sh["lo"]:sh["hi"]]
        if sh["kind"] == "cols":
            return Hf[:, sh["lo"]:sh["hi"]]
        return Hf

    wsb = lh.lh_hessian_workspace_bytes(max(n_loc, 1), c_in, n_groups)
    wsp = torch.empty(max(wsb, 256), dtype=torch.uint8, device=dev)
    swsb = lh.lh_sweep_workspace_bytes(s_mats, max(s_cin, 16))
    swsp = torch.empty(max(swsb, 16), dtype=torch.uint8, device=dev)
    codes = torch.empty(s_mats, s_out, s_J, dtype=torch.uint8, device=dev)
    bamax = torch.empty(s_mats, s_out, s_J, dtype=torch.float32, device=dev)
    Wq = torch.empty(s_mats, s_out, s_cin, dtype=W.dtype, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 1 << 28) // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.zeros_like(flush)

    def flush_l2():
        """Cold L2: write a buffer twice its size, then read another one as large, so no
        dirty line of the flush is left to be written back inside the timed region."""
        flush.zero_()
        flush_rd.amax()
    stream = torch.cuda.current_stream(dev)
    s = stream.cuda_stream
    ld = W.stride(1)
    hl = LAUNCHES["hessian_grouped" if grouped else "hessian_plain"]
    launches_per_step = (LAUNCHES["absmax"] if s_blocks else 0) + (hl if n_loc else 0) + \
        ((LAUNCHES["sweep_ws"] + LAUNCHES["fake_quant"]) if s_blocks else 0)

    def step_into(d, cs, rec=None):
        """One step on buffer set d (device tensors) on the raw stream cs; rec(k)
        records the k-th event on the current torch stream."""
        r = rec or (lambda k: None)
        r(0)
        d["H"].zero_()
        r(1)
        if s_blocks:
            lh.lh_absmax(d["W"], d["W"], s_mats, s_out, s_cin, ld, d["amax"], cs)
        r(2)
        if sh["amax_allreduce"]:
            dist.all_reduce(d["amax"], op=dist.ReduceOp.MAX)
        r(3)
        if n_loc:
            lh.lh_accumulate_hessian(d["X"], lh.LH_BF16, n_loc, c_in, d["X"].stride(0), d["off"], n_groups, d["H"],
                                     d["ws"], wsb, cs)
        r(4)
        if ws > 1:
            dist.all_reduce(d["H"], op=dist.ReduceOp.SUM)
        r(5)
        if s_blocks:
            lh.lh_sweep_scales_ws(d["W"], d["W"], s_mats, s_out, s_cin, ld, d["amax"], sweep_h(d["H"]),
                                  d["bamax"], d["codes"], d["sws"], swsb, cs)
        r(6)
        if s_blocks:
            lh.lh_fake_quant(d["W"], d["W"], s_mats, s_out, s_cin, ld, d["amax"], d["codes"], d["Wq"], d["Wq"], cs)
        r(7)

    main = dict(W=W, X=X, off=off, amax=amax, H=H, ws=wsp, sws=swsp, codes=codes, bamax=bamax, Wq=Wq)
    for _ in range(args.warmup):
        flush_l2()
        step_into(main, s)
    torch.cuda.synchronize(dev)
    assert n_loc == 0 or lh.lh_workspace_status(wsp, s) == 0

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(args.steps)]
    sampler = ClockSampler(dev.index)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    for i in range(args.steps):
        flush_l2()  # cold L2 for every step
        step_into(main, s, lambda k, e=evs[i]: e[k].record(stream))
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if ws > 1:
        dist.barrier()
    names = ("h_zero", "absmax", "amax_allreduce", "hessian", "h_allreduce", "sweep", "fake_quant")
    per = np.array([[e[k].elapsed_time(e[k + 1]) for k in range(7)] for e in evs])  # ms [steps, 7]
    t_rank = float(per.sum()) / 1e3
    t_all = max_over_ranks(t_rank, ws, dev)
    value = layer.n_blocks * args.steps / t_all
    means = {n: float(v) for n, v in zip(names, per.mean(axis=0))}
    per_median = {n: float(v) for n, v in zip(names, np.median(per, axis=0))}
    per_min = {n: float(v) for n, v in zip(names, per.min(axis=0))}
    if ws == 1:
        for d in (means, per_median, per_min):
            del d["amax_allreduce"], d["h_allreduce"]
    t_hess, t_sweep = means["hessian"], means["sweep"]

    # ---- the Hessian call with X left in L2 (no flush between calls): X of the attention,
    # MLP-up and MoE layers (17, 67, 134 MB) fits or nearly fits the 126 MB L2
    warm = []
    if n_loc:
        H_warm = torch.zeros_like(H)  # the step's H stays as the last timed step left it
        for i in range(3 + args.steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            lh.lh_accumulate_hessian(X, lh.LH_BF16, n_loc, c_in, X.stride(0), off, n_groups, H_warm, wsp, wsb, s)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if i >= 3:
                warm.append(e0.elapsed_time(e1))
    t_hess_warm = float(np.median(warm)) if warm else 0.0

    extras = {}
    if s_blocks:
        # ---- packed NVFP4 export fused with the fake quantisation (one read of W writes the
        # packed nibbles, the scale bytes and W_q), timed like the step, L2 flushed each time
        packed = torch.empty(s_mats, s_out, s_cin // 2, dtype=torch.uint8, device=dev)
        scales = torch.empty(s_mats, s_out, s_J, dtype=torch.uint8, device=dev)
        gscale = torch.empty(s_mats, dtype=torch.float32, device=dev)
        qdt = lh.LH_BF16 if Wq.dtype == torch.bfloat16 else lh.LH_F32

        def timed(fn, reps):
            for _ in range(3):
                fn()
            ts = []
            for _ in range(reps):
                flush_l2()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn()
                e1.record(stream)
                torch.cuda.synchronize(dev)
                ts.append(e0.elapsed_time(e1))
            return float(np.median(ts))

        t_ex = timed(lambda: lh.lh_quantize_nvfp4(W, W, s_mats, s_out, s_cin, ld, amax, codes, packed, scales,
                                                  gscale, Wq, qdt, s), args.steps)
        ex_bytes = (W.numel() * W.element_size() + 2 * codes.numel() + packed.numel() +
                    Wq.numel() * Wq.element_size() + 8 * s_mats)
        fq_bytes = W.numel() * W.element_size() + codes.numel() + Wq.numel() * Wq.element_size()
        abs_bytes = W.numel() * W.element_size()
        hbm = load_peaks()["hbm_gbs"]
        extras["streaming"] = dict(
            unit="GB/s", peak=hbm, note="one pass over W per call; bytes = W read (+ codes read, W_q written)",
            absmax=dict(ms=means["absmax"], bytes=int(abs_bytes), achieved=abs_bytes / means["absmax"] / 1e6,
                        frac=abs_bytes / means["absmax"] / 1e6 / hbm),
            fake_quant=dict(ms=means["fake_quant"], bytes=int(fq_bytes),
                            achieved=fq_bytes / means["fake_quant"] / 1e6,
                            frac=fq_bytes / means["fake_quant"] / 1e6 / hbm),
            nvfp4_export=dict(ms=t_ex, bytes=int(ex_bytes), achieved=ex_bytes / t_ex / 1e6,
                              frac=ex_bytes / t_ex / 1e6 / hbm,
                              note="lh_quantize_nvfp4: packed E2M1 + scale bytes + W_q in one pass; not part of "
                                   "the timed step"))

        # ---- the pages' baseline scalers on the same blocks (context beside the Local-Hessian sweep)
        bl_codes = torch.empty_like(codes)
        bl_amax = torch.empty_like(bamax)
        baselines = {}
        reps = max(3, min(args.steps, 10))
        for name, meth in (("max", lh.LH_SCALE_MAX), ("four_over_six", lh.LH_SCALE_FOUR_OVER_SIX),
                           ("mse_sweep", lh.LH_SCALE_MSE)):
            t_b = timed(lambda: lh.lh_baseline_scales(W, W, s_mats, s_out, s_cin, ld, amax, meth, bl_amax, bl_codes,
                                                      s), reps)
            baselines[name] = dict(ms=t_b, blocks_per_s=s_blocks / (t_b / 1e3))
        # the amax multiplier search (0.25 + 0.1 k, 38 multipliers) with this layer's H
        t_b = timed(lambda: lh.lh_search_amax(W, W, s_mats, s_out, s_cin, ld, amax, sweep_h(H), bl_amax, bl_codes,
                                              stream=s), reps)
        baselines["amax_search_hessian"] = dict(ms=t_b, blocks_per_s=s_blocks / (t_b / 1e3))
        extras["baseline_scalers"] = baselines

    # ---- end to end through the public API with host buffers: every step copies its
    # inputs from pinned host memory and its results (codes, best amax, W_q) back.
    # Consecutive steps are pipelined over two device buffer sets on three streams
    # (copy-in, compute, copy-out), ordered by events, so copies overlap compute.
    W_pin = W_host.pin_memory()
    X_pin = X_host.pin_memory()
    off_host = torch.from_numpy(sh["offsets"]).pin_memory() if grouped else None
    sets = []
    for _ in range(2):
        d = dict(W=torch.empty_like(W), X=torch.empty_like(X), off=torch.empty_like(off) if grouped else None,
                 amax=torch.empty_like(amax), H=torch.empty_like(H), ws=torch.empty_like(wsp),
                 sws=torch.empty_like(swsp), codes=torch.empty_like(codes), bamax=torch.empty_like(bamax),
                 Wq=torch.empty_like(Wq),
                 codes_pin=torch.empty(codes.shape, dtype=codes.dtype).pin_memory(),
                 bam_pin=torch.empty(bamax.shape, dtype=bamax.dtype).pin_memory(),
                 Wq_pin=torch.empty(Wq.shape, dtype=Wq.dtype).pin_memory(),
                 ev_in=torch.cuda.Event(), ev_done=torch.cuda.Event(), ev_out=torch.cuda.Event())
        sets.append(d)
    s_in, s_cmp, s_out_st = (torch.cuda.Stream(dev) for _ in range(3))

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
        s_cmp.wait_event(d["ev_in"])
        if i >= 2:
            s_cmp.wait_event(d["ev_out"])  # results of step i-2 copied out of this set
        with torch.cuda.stream(s_cmp):
            step_into(d, s_cmp.cuda_stream)
        d["ev_done"].record(s_cmp)
        with torch.cuda.stream(s_out_st):
            s_out_st.wait_event(d["ev_done"])
            d["codes_pin"].copy_(d["codes"], non_blocking=True)
            d["bam_pin"].copy_(d["bamax"], non_blocking=True)
            d["Wq_pin"].copy_(d["Wq"], non_blocking=True)
            d["ev_out"].record(s_out_st)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e_start.record(s_in)
    for i in range(args.steps):
        e2e_step(i)
    for st in (s_in, s_cmp):
        s_out_st.wait_stream(st)
    e_end.record(s_out_st)
    torch.cuda.synchronize(dev)
    t_e2e = max_over_ranks(e_start.elapsed_time(e_end) / 1e3, ws, dev)
    h2d = W.numel() * W.element_size() + X.numel() * X.element_size() + (off.numel() * 8 if grouped else 0)
    d2h = codes.numel() + bamax.numel() * 4 + Wq.numel() * Wq.element_size()
    e2e = dict(value=layer.n_blocks * args.steps / t_e2e, unit=UNIT, h2d_bytes_per_step=int(h2d),
               d2h_bytes_per_step=int(d2h), pipelined="2 buffer sets, copy-in / compute / copy-out streams",
               bytes_note="per rank" if ws > 1 else "whole layer")
    # the last step's results equal those of the device-resident run
    dl = sets[(args.steps - 1) % 2]
    assert torch.equal(dl["codes_pin"], codes.cpu()), "end-to-end results differ from the device run"

    # ---- rooflines (this rank's share: the whole layer at one GPU)
    peaks = load_peaks()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    probe = fma_probe(lh, torch, dev, stream)
    # packed two-lane FMAs count twice when the probe shows they retire at twice the scalar rate
    fma_width = 2 if probe["packed_tflops"] > 1.5 * probe["scalar_tflops"] else 1
    fp32_peak = sms * FP32_LANES_PER_SM * 2 * fma_width * peaks["sm_max_mhz"] * 1e6 / 1e12  # TFLOP/s
    sweep_tflops = SWEEP_FLOP_PER_BLOCK * s_blocks / (t_sweep / 1e3) / 1e12 if t_sweep > 0 else 0.0
    hess_bytes = 2 * c_in * n_loc
    hess_gbs = hess_bytes / (t_hess / 1e3) / 1e9 if t_hess > 0 else 0.0
    full = ws == 1
    roofline = dict(bound="alu", kernel="sweep_kernel", achieved=sweep_tflops, peak=fp32_peak, unit="TFLOP/s",
                    frac=sweep_tflops / fp32_peak,
                    traffic=profiled_traffic("scale_calibration_b200/csrc/sweep.cu",
                                             f"sweep_kernel_{layer.name}.md") if full else None,
                    traffic_note="DRAM bytes per launch from the committed ncu summary of this layer (null if the "
                                 "kernel changed since, or none was taken)",
                    peak_note=(f"FP32 CUDA-core peak {sms} SMs x 128 lanes x 2 flop x {fma_width} (FMAs per lane per "
                               f"cycle, from the probe) x {peaks['sm_max_mhz']:.0f} MHz"),
                    fma_probe=probe, flop_per_block=SWEEP_FLOP_PER_BLOCK, blocks_per_launch=int(s_blocks))
    if clocks.get("sm_mhz"):
        roofline["frac_at_measured_clock"] = sweep_tflops / (fp32_peak * clocks["sm_mhz"] / peaks["sm_max_mhz"])
    if s_blocks:
        ex = sweep_work(lh, torch, dev, s, W, s_mats, s_out, s_cin, ld, amax, sweep_h(H), codes, t_sweep, fp32_peak)
        if ex:
            roofline["executed"] = ex
    hessian = dict(tokens_per_s=n_loc / (t_hess / 1e3) if t_hess > 0 else None, bound="hbm",
                   achieved=hess_gbs, peak=peaks["hbm_gbs"], unit="GB/s", frac=hess_gbs / peaks["hbm_gbs"],
                   bytes_per_launch=hess_bytes, peak_source=peaks["source"],
                   traffic=profiled_traffic("scale_calibration_b200/csrc/hessian.cu",
                                            f"hessian_tc_kernel_{layer.name}.md") if full else None,
                   warm_l2=dict(ms=t_hess_warm, tokens_per_s=n_loc / (t_hess_warm / 1e3) if t_hess_warm else None,
                                achieved=hess_bytes / (t_hess_warm / 1e3) / 1e9 if t_hess_warm else None,
                                note="median of back-to-back calls without an L2 flush (X partly or wholly in L2); "
                                     "the HBM fraction above is the cold-L2 one"))

    line = dict(metric=METRIC, value=value, unit=UNIT, n_gpus=ws, steps=args.steps, warmup=args.warmup,
                ms_per_step=1e3 * t_all / args.steps, higher_is_better=True, scaling="strong", vs_baseline=None,
                dtype="f32", data="synthetic", config=bench_config(layer, ws),
                kernels_ms=means, kernels_ms_median=per_median, kernels_ms_min=per_min,
                sweep_blocks_per_s=layer.n_blocks / (t_sweep / 1e3) if t_sweep > 0 else None,
                roofline=roofline, hessian=hessian, e2e=e2e, gpu_launches=launches_per_step * args.steps,
                clocks=clocks, **extras)

    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        rng = np.random.default_rng(1)
        W_f32 = layer.W_f32()
        t0 = time.perf_counter()
        tot, reps = 0.0, 0
        while time.perf_counter() - t0 < args.cpu_seconds and reps < 50:
            tot += oracle_step(layer, W_f32, 20000, rng)[0]
            reps += 1
        cpu_value = layer.n_blocks * reps / tot
        line["cpu_baseline"] = dict(value=cpu_value, unit=UNIT, cores=1, host_cores=os.cpu_count(), kind="oracle",
                                    extrapolated=True,
                                    sample=(f"{reps} x (oracle Hessian of <= 4096 tokens, 20000 random sweep blocks, "
                                            f"8 fake-quant rows), each scaled to the whole layer; "
                                            f"{time.perf_counter() - t0:.1f} s measured"))
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
    ap.add_argument("--config", type=int, default=4,
                    help="0 tiny, 1 attn_proj, 2 mlp_up, 3 mlp_down, 4 moe_experts (default: the largest single-GPU "
                         "layer)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(spawn_ranks(args))
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
