#!/usr/bin/env python
"""Benchmark of the SmoothQuant W8A8 linear hot path on B200.

One step = one pass of the whole path over one batch, for each linear of an 8B-class
transformer layer at prefill size (8192 tokens): QKV 4096 -> 6144 and gate+up
4096 -> 28672 (LayerNorm in front), O 4096 -> 4096 and down 14336 -> 4096 (input from a
previous GEMM).  Per linear:
  calibration absmax of the linear's input (of the LayerNorm output where there is one)
  -> weight row absmax -> smoothing factors (alpha = 0.5) -> fold + per-channel weight
  INT8 -> LayerNorm / smoothing + per-token INT8 -> INT8 tensor-core GEMM with the
  dequant epilogue to bf16.
Synthetic seeded inputs: bf16 activations with 1% fixed outlier channels x100, W ~
N(0, 0.02), gamma ~ U(0.5, 1.5).  Under torchrun every rank runs its own batch (weak
scaling); the calibration statistic is combined across ranks with an all-reduce(MAX).

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "W8A8 smoothed linear TOPS & quantizer GB/s on 1 B200; % of INT8/HBM roofline"
TOKENS = 8192
LAYERS = (("qkv", 4096, 6144, True), ("o", 4096, 4096, False), ("gate_up", 4096, 28672, True),
          ("down", 14336, 4096, False))
ALPHA = 0.5
W_STD = 0.02
WORKLOAD = ("prefill 8B-class linear set: 8192 tokens x {QKV 4096->6144 (LN), O 4096->4096, "
            "gate+up 4096->28672 (LN), down 14336->4096}; calibration on the batch, alpha 0.5")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
INT8_PER_BF16 = 2.0  # dense INT8 tensor rate / dense BF16 rate on B200 (4.5 vs 2.25 PFLOP/s nominal)


def gemm_traffic() -> int | None:
    """DRAM bytes per GEMM launch of this step from the committed ncu summary, or None when the
    GEMM sources changed since the counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "w8a8_gemm_pair_prefill8b_traffic.md")
    if not os.path.exists(path):
        return None
    fields = {}
    for line in open(path):
        if ":" in line and line.split(":")[0].strip().isidentifier():
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    src = os.path.join(ROOT, "w8a8_smoothquant_gemm_b200", "csrc")
    h = hashlib.sha256()
    for f in ("sq_gemm.cu", "sq_ptx.cuh"):
        h.update(open(os.path.join(src, f), "rb").read())
    if fields.get("gemm_source_sha256_16") != h.hexdigest()[:16]:
        return None
    try:
        return int(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def step_ops(M: int = TOKENS) -> float:
    return float(sum(2.0 * M * N * K for _, K, N, _ in LAYERS))


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    return dict(FALLBACK_PEAKS)


# ----------------------------------------------------------------------------- distributed
def init_dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int, device) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def combine_statistic(ax: torch.Tensor, world: int) -> None:
    """Each rank calibrates on its own tokens; the absmax over the whole calibration set is the
    element-wise max over ranks (an all-reduce, in place).  A no-op on one rank."""
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(ax, op=dist.ReduceOp.MAX)


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of one GPU while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "100"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self) -> dict:
        rows = [r.split(",") for r in (self.out or "").strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        clk = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(clk), "sm_max_mhz": float(rows[0][2]), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows)}


# ----------------------------------------------------------------------------- the device path
class Linear:
    """Device buffers of one linear of the step."""

    def __init__(self, name, K, N, ln, M, device, seed):
        import sq_inputs
        import w8a8_smoothquant_gemm_b200 as sq
        self.name, self.K, self.N, self.ln, self.M = name, K, N, ln, M
        self.x, self.W, self.gamma, _ = sq_inputs.torch_case(M, K, N, seed, device, w_std=W_STD)
        f32 = dict(dtype=torch.float32, device=device)
        self.ax, self.aw, self.s = torch.empty(K, **f32), torch.empty(K, **f32), torch.empty(K, **f32)
        self.gf = torch.empty(K, **f32) if ln else None
        self.wq = torch.empty(N, K, dtype=torch.int8, device=device)
        self.sw = torch.empty(N, **f32)
        self.xq = torch.empty(M, K, dtype=torch.int8, device=device)
        self.sx = torch.empty(M, **f32)
        self.y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
        need = sq.sq_w8a8_gemm_workspace_size(M, N, K)
        self.ws = torch.empty(need, dtype=torch.uint8, device=device) if need else None
        # this module's kernels per pass: calibration, weight absmax, factors, fold (one, or
        # three on the streaming route), quantiser, GEMM (+ the split-K reduction when the
        # GEMM splits K)
        self.launches = 5 + sq.sq_fold_kernel_launches(self.W) + (1 if need else 0)

    def run(self, sq, world: int, ev=None):
        if self.ln:
            sq.sq_calib_ln_absmax(self.x, self.gamma, out=self.ax)
        else:
            sq.sq_calib_absmax(self.x, 0, out=self.ax)
        combine_statistic(self.ax, world)
        sq.sq_calib_absmax(self.W, 1, out=self.aw)
        sq.sq_smooth_factors(self.ax, self.aw, ALPHA, out=self.s)
        sq.sq_fold_quant_weights(self.W, self.s, self.gamma if self.ln else None, wq=self.wq, sw=self.sw,
                                 gamma_f=self.gf)
        if self.ln:
            sq.sq_ln_smooth_quant(self.x, gamma_f=self.gf, xq=self.xq, sx=self.sx)
        else:
            sq.sq_ln_smooth_quant(self.x, s=self.s, xq=self.xq, sx=self.sx)
        if ev is not None:
            ev[0].record()
        sq.sq_w8a8_gemm(self.xq, self.sx, self.wq, self.sw, y=self.y, workspace=self.ws)
        if ev is not None:
            ev[1].record()

    # algorithmic bytes of the bandwidth kernels (one read of each input, one write of each output)
    def bytes_calib(self):
        return self.M * self.K * 2 + 4 * self.K + (4 * self.K if self.ln else 0)

    def bytes_wabsmax(self):
        return self.K * self.N * 2 + 4 * self.K

    def bytes_fold(self):
        return self.K * self.N * 2 + self.N * self.K + 4 * self.N + 4 * self.K + (8 * self.K if self.ln else 0)

    def bytes_quant(self):
        return self.M * self.K * 2 + self.M * self.K + 4 * self.M + 4 * self.K


def quantizer_profile(sq, layers, world, reps=5) -> dict:
    """Per-kernel CUDA-event times of the bandwidth kernels (separate from the timed steps).

    Before each timed kernel a 256 MB buffer is zeroed on the same stream: the L2 starts cold,
    and the device is still busy with it when the host has enqueued the kernel and its closing
    event, so an interval holds the kernel's device time, not the host's launch latency."""
    kinds = ("calib", "wabsmax", "fold", "quant")
    tot = {k: 0.0 for k in kinds}
    byt = {k: 0 for k in kinds}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=layers[0].x.device)
    pending = []

    def timed(kind, nbytes, fn):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        pending.append((kind, nbytes, a, b))

    for _ in range(reps):
        for L in layers:
            if L.ln:
                timed("calib", L.bytes_calib(), lambda: sq.sq_calib_ln_absmax(L.x, L.gamma, out=L.ax))
            else:
                timed("calib", L.bytes_calib(), lambda: sq.sq_calib_absmax(L.x, 0, out=L.ax))
            timed("wabsmax", L.bytes_wabsmax(), lambda: sq.sq_calib_absmax(L.W, 1, out=L.aw))
            sq.sq_smooth_factors(L.ax, L.aw, ALPHA, out=L.s)
            timed("fold", L.bytes_fold(),
                  lambda: sq.sq_fold_quant_weights(L.W, L.s, L.gamma if L.ln else None, wq=L.wq, sw=L.sw,
                                                   gamma_f=L.gf))
            if L.ln:
                timed("quant", L.bytes_quant(), lambda: sq.sq_ln_smooth_quant(L.x, gamma_f=L.gf, xq=L.xq, sx=L.sx))
            else:
                timed("quant", L.bytes_quant(), lambda: sq.sq_ln_smooth_quant(L.x, s=L.s, xq=L.xq, sx=L.sx))
    torch.cuda.synchronize()
    for kind, nbytes, a, b in pending:
        tot[kind] += a.elapsed_time(b) / 1e3
        byt[kind] += nbytes
    return {f"{k}_gbs": round(byt[k] / tot[k] / 1e9, 1) for k in kinds}


# ----------------------------------------------------------------------------- CPU oracle sample
def oracle_sample(host_layers, rows: int, cols: int, threads_note: str = "") -> dict:
    """Times the CPU oracle on a bounded sample of the step -- per linear `rows` tokens and
    `cols` output channels -- and extrapolates each part to the full step by its share:
    activation side x M/rows, weight side x N/cols, GEMM x (M N)/(rows cols)."""
    import oracle as O
    t_x = t_w = t_g = 0.0
    full = 0.0
    for (name, K, N, ln), (xh, Wh, gh) in zip(LAYERS, host_layers):
        r = min(rows, xh.shape[0])
        c = min(cols, N)
        xs = xh[:r]
        Ws = np.ascontiguousarray(Wh[:, :c])
        t0 = time.perf_counter()
        ax = O.calib_ln_absmax(xs, gh) if ln else O.calib_absmax(xs, 0)
        t1 = time.perf_counter()
        aw = O.calib_absmax(Ws, 1)
        s = O.smooth_factors(ax, aw, ALPHA)
        wq, sw, gf, _ = O.fold_quant_weights(Ws, s, gh if ln else None)
        t2 = time.perf_counter()
        xq, sx = O.ln_smooth_quant(xs, gamma_f=gf) if ln else O.ln_smooth_quant(xs, s=s)
        t3 = time.perf_counter()
        O.w8a8_gemm(xq, sx, wq, sw, "bf16")
        t4 = time.perf_counter()
        tx = (t1 - t0) + (t3 - t2)
        tw = t2 - t1
        tg = t4 - t3
        t_x, t_w, t_g = t_x + tx, t_w + tw, t_g + tg
        full += tx * TOKENS / r + tw * N / c + tg * (TOKENS * N) / (r * c)
    return {"sample_s": t_x + t_w + t_g, "full_step_s": full}


def host_layers_from_device(layers, rows: int):
    out = []
    for L in layers:
        xh = L.x[:rows].contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
        Wh = L.W.cpu().view(torch.int16).numpy().view(np.uint16)
        out.append((xh, Wh, L.gamma.cpu().numpy()))
    return out


def host_layers_synthetic(rows: int, cols_max: int):
    """CPU-only inputs for the reference arm: the same recipe drawn with numpy."""
    import sq_inputs
    out = []
    for i, (name, K, N, ln) in enumerate(LAYERS):
        c = sq_inputs.make_case(rows, K, min(N, cols_max), 1000 + i, w_std=W_STD)
        out.append((c.x, c.W, c.gamma))
    return out


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle as O
    budget = 150.0  # seconds of oracle work for the whole run
    per_step = budget / max(1, args.steps + args.warmup)
    # sample size scaled to the per-step budget (probe with a tiny sample first)
    rows, cols = 4, 64
    host = host_layers_synthetic(64, 1024)
    probe = oracle_sample(host, rows, cols)
    scale = max(1.0, min(16.0, (per_step / max(probe["sample_s"], 1e-4)) ** 0.5))
    rows, cols = max(1, min(64, int(rows * scale))), max(16, min(1024, int(cols * scale)))
    for _ in range(args.warmup):
        oracle_sample(host, rows, cols)
    fulls, samples = [], []
    for _ in range(args.steps):
        r = oracle_sample(host, rows, cols)
        fulls.append(r["full_step_s"])
        samples.append(r["sample_s"])
    t = statistics.mean(fulls)
    value = step_ops() / t / 1e12
    sample = (f"per linear {rows} tokens x {cols} output channels (all K) per step, times extrapolated to "
              f"8192 tokens x N by the share of each part; {args.steps} steps")
    line = {"metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD, "tokens": TOKENS, "alpha": ALPHA},
            "cpu_baseline": {"value": value, "unit": "TOPS", "cores": O.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- main arm
def run_device(args, rank, world, local):
    import w8a8_smoothquant_gemm_b200 as sq
    device = torch.device("cuda", local)
    sq.lib()
    layers = [Linear(n, K, N, ln, TOKENS, device, 1000 * rank + i) for i, (n, K, N, ln) in enumerate(LAYERS)]
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        for L in layers:
            L.run(sq, world)
    torch.cuda.synchronize()
    if sq.sq_device_error(clear=True) != 0:
        raise RuntimeError("a kernel gave up on a bounded wait during warm-up")

    # ---- timed region: K steps, device time with CUDA events, GEMM launches bracketed too
    gemm_ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in layers]
               for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local) as clk:
        start.record()
        for k in range(args.steps):
            for i, L in enumerate(layers):
                L.run(sq, world, gemm_ev[k][i])
        end.record()
        torch.cuda.synchronize()
    barrier(world)
    elapsed = start.elapsed_time(end) / 1e3
    elapsed = max_over_ranks(elapsed, world, device)
    if sq.sq_device_error(clear=True) != 0:
        raise RuntimeError("a kernel gave up on a bounded wait during the timed steps")
    gemm_s = [sum(gemm_ev[k][i][0].elapsed_time(gemm_ev[k][i][1]) for k in range(args.steps)) / 1e3 / args.steps
              for i in range(len(layers))]

    peaks = load_peaks()
    int8_peak = INT8_PER_BF16 * peaks["bf16_tflops"]
    ops_step = step_ops()
    value = ops_step * world * args.steps / elapsed / 1e12
    gemm_ops = [2.0 * L.M * L.N * L.K for L in layers]
    achieved = sum(gemm_ops) / sum(gemm_s) / 1e12
    roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": int8_peak, "unit": "TOPS",
                "frac": round(achieved / int8_peak, 4), "traffic": gemm_traffic(),
                "traffic_unit": "DRAM bytes per GEMM launch (mean of the 4 launches of a step)",
                "algorithmic_bytes_per_launch": int(sum(L.M * L.K + L.N * L.K + 2 * L.M * L.N for L in layers) / 4),
                "kernel": "w8a8_gemm_kernel (tcgen05 kind::i8), 4 launches per step",
                "peak_note": f"2 x {peaks['source']} burst bf16 {peaks['bf16_tflops']} TFLOP/s"}
    per_gemm = {L.name: {"us": round(t * 1e6, 1), "tops": round(o / t / 1e12, 1),
                         "frac": round(o / t / 1e12 / int8_peak, 3)} for L, t, o in zip(layers, gemm_s, gemm_ops)}

    quant = quantizer_profile(sq, layers, world)
    quant["hbm_peak_gbs"] = peaks["hbm_gbs"]
    quant["quant_frac"] = round(quant["quant_gbs"] / peaks["hbm_gbs"], 3)

    # ---- end to end through the public API: pinned host inputs -> device -> path -> host output.
    # Copies run on their own streams (host->device and device->host in parallel over the
    # full-duplex link), ordered by events so that a linear's copies overlap its neighbours'
    # compute; every byte of every step's inputs and outputs crosses the link inside the
    # timed region.
    h = [{"x": L.x.cpu().pin_memory(), "W": L.W.cpu().pin_memory(), "g": L.gamma.cpu().pin_memory(),
          "y": torch.empty(L.y.shape, dtype=L.y.dtype, pin_memory=True)} for L in layers]
    h2d = sum(b["x"].numel() * 2 + b["W"].numel() * 2 + b["g"].numel() * 4 for b in h)
    d2h = sum(b["y"].numel() * 2 for b in h)
    e2e_steps = max(3, args.steps // 10)
    cs = torch.cuda.current_stream()
    hs, ds = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(nsteps):
        comp = [None] * len(layers)
        back = [None] * len(layers)
        for _ in range(nsteps):
            for i, (L, b) in enumerate(zip(layers, h)):
                with torch.cuda.stream(hs):
                    if comp[i] is not None:
                        hs.wait_event(comp[i])  # the previous step's compute has read these buffers
                    L.x.copy_(b["x"], non_blocking=True)
                    L.W.copy_(b["W"], non_blocking=True)
                    L.gamma.copy_(b["g"], non_blocking=True)
                    loaded = torch.cuda.Event()
                    loaded.record(hs)
                cs.wait_event(loaded)
                if back[i] is not None:
                    cs.wait_event(back[i])  # the previous step's output has left the device
                L.run(sq, world)
                comp[i] = torch.cuda.Event()
                comp[i].record(cs)
                with torch.cuda.stream(ds):
                    ds.wait_event(comp[i])
                    b["y"].copy_(L.y, non_blocking=True)
                    back[i] = torch.cuda.Event()
                    back[i].record(ds)
        cs.wait_stream(hs)
        cs.wait_stream(ds)

    e2e_run(1)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cs)
    hs.wait_event(e0)
    ds.wait_event(e0)
    e2e_run(e2e_steps)
    e1.record(cs)
    torch.cuda.synchronize()
    barrier(world)
    e2e_t = max_over_ranks(e0.elapsed_time(e1) / 1e3, world, device)
    e2e = {"value": ops_step * world * e2e_steps / e2e_t / 1e12, "unit": "TOPS", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "steps": e2e_steps, "ms_per_step": e2e_t / e2e_steps * 1e3,
           "link": "pinned host buffers; host->device and device->host copies on separate streams"}

    # ---- CPU oracle baseline (rank 0, one GPU only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle as O
        rows, cols = 16, 2048
        host = host_layers_from_device(layers, rows)
        r = oracle_sample(host, rows, cols)
        cpu = {"value": ops_step / r["full_step_s"] / 1e12, "unit": "TOPS", "cores": O.num_threads(),
               "kind": "oracle",
               "sample": (f"per linear {rows} tokens x {cols} output channels (all K) of this step's inputs; "
                          f"{r['sample_s']:.1f} s of oracle work, extrapolated to the full step "
                          f"({r['full_step_s']:.1f} s) by each part's share")}

    launches = sum(L.launches for L in layers) * args.steps
    line = {"metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": WORKLOAD, "tokens_per_gpu": TOKENS, "alpha": ALPHA,
                       "shapes_KN": [[K, N] for _, K, N, _ in LAYERS],
                       "l2": "inputs larger than L2: 0.85 GB of activations + bf16 weights read per step (L2 126 MB)",
                       "parallelism": f"dp{world}"},
            "roofline": roofline, "gemm": per_gemm, "quantizer": quant, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "clocks": clk.summary()}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_kernel(args):
    """One kernel of the path on one shape, `--steps` times, CUDA-event timed (profiling aid).

    --shape M,N,K; the activation is [M, K] with a LayerNorm in front, the weight [K, N]."""
    import w8a8_smoothquant_gemm_b200 as sq
    M, N, K = (int(v) for v in args.shape.split(","))
    device = torch.device("cuda", 0)
    L = Linear("k", K, N, True, M, device, 7)
    L.run(sq, 1)
    torch.cuda.synchronize()
    # GEMM operands rotate over enough copies that successive calls miss in L2 (126 MB)
    gemm_bytes = M * K + N * K + 2 * M * N + 4 * (M + N)
    n_copies = max(1, min(32, -(-300 * 2 ** 20 // gemm_bytes)))
    copies = [(L.xq.clone(), L.wq.clone(), torch.empty_like(L.y)) for _ in range(n_copies)]
    rot = [0]

    def gemm_call():
        xq, wq, y = copies[rot[0] % n_copies]
        rot[0] += 1
        sq.sq_w8a8_gemm(xq, L.sx, wq, L.sw, y=y, workspace=L.ws)

    # the bandwidth kernels' inputs rotate the same way (activations and weights as copies
    # whose total exceeds 300 MB), so every call reads its input from HBM
    def rotation(t):
        n = max(1, min(16, -(-300 * 2 ** 20 // (t.numel() * t.element_size()))))
        return [t] + [t.clone() for _ in range(n - 1)]

    xs = rotation(L.x) if args.kernel in ("lnquant", "quant", "calib", "xabsmax") else [L.x]
    ws = rotation(L.W) if args.kernel in ("fold", "wabsmax") else [L.W]
    xq_out = [L.xq] + [torch.empty_like(L.xq) for _ in range(min(len(xs), 4) - 1)]
    wq_out = [L.wq] + [torch.empty_like(L.wq) for _ in range(min(len(ws), 2) - 1)]
    nxt = [0]

    def pick(seq):
        return seq[nxt[0] % len(seq)]

    def rotated(f):
        def call():
            f()
            nxt[0] += 1
        return call

    if args.kernel == "gemm8":
        # the FP8 variant on the same linear: E4M3 codes of the same smoothed operands
        wq8, sw8, gf8, _ = sq.sq_fold_quant_weights_fp8(L.W, L.s, L.gamma)
        xq8, sx8 = sq.sq_ln_smooth_quant_fp8(L.x, gamma_f=gf8)
        copies8 = [(xq8.clone(), wq8.clone(), torch.empty_like(L.y)) for _ in range(n_copies)]

    def gemm8_call():
        xq, wq, y = copies8[rot[0] % n_copies]
        rot[0] += 1
        sq.sq_w8a8_gemm_fp8(xq, sx8, wq, sw8, y=y, workspace=L.ws)

    if args.kernel == "alpha":
        # the whole 20-strength search on this batch (calibration statistics, reference product,
        # 20 x (factors, fold, quantiser, GEMM, error)); the workspace is allocated once
        alpha_ws = torch.empty(sq.lib().sq_alpha_search_workspace_size(M, K, N), dtype=torch.uint8, device=device)

    calls = {
        "alpha": (lambda: sq.sq_alpha_search(L.x, L.W, None, gamma=L.gamma, workspace=alpha_ws), 0, 0.0),
        "gemm": (gemm_call, gemm_bytes, 2.0 * M * N * K),
        "gemm8": (gemm8_call, gemm_bytes, 2.0 * M * N * K),
        "fold": (rotated(lambda: sq.sq_fold_quant_weights(pick(ws), L.s, L.gamma, wq=pick(wq_out), sw=L.sw,
                                                          gamma_f=L.gf)), L.bytes_fold(), 0.0),
        "lnquant": (rotated(lambda: sq.sq_ln_smooth_quant(pick(xs), gamma_f=L.gf, xq=pick(xq_out), sx=L.sx)),
                    L.bytes_quant(), 0.0),
        "quant": (rotated(lambda: sq.sq_ln_smooth_quant(pick(xs), s=L.s, xq=pick(xq_out), sx=L.sx)),
                  L.bytes_quant(), 0.0),
        "calib": (rotated(lambda: sq.sq_calib_ln_absmax(pick(xs), L.gamma, out=L.ax)), L.bytes_calib(), 0.0),
        "xabsmax": (rotated(lambda: sq.sq_calib_absmax(pick(xs), 0, out=L.ax)), M * K * 2 + 4 * K, 0.0),
        "wabsmax": (rotated(lambda: sq.sq_calib_absmax(pick(ws), 1, out=L.aw)), L.bytes_wabsmax(), 0.0),
    }
    fn, nbytes, ops = calls[args.kernel]
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    # device time per call: `steps` calls captured in one CUDA graph (no host launch cost in
    # the timed region), replayed a few times; the median replay / steps
    reps = 5
    if args.kernel in ("gemm", "gemm8"):
        args.steps = max(args.steps, n_copies)
    else:
        args.steps = max(args.steps, len(xs), len(ws))
    g = torch.cuda.CUDAGraph()
    s_cap = torch.cuda.Stream()
    s_cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s_cap):
        with torch.cuda.graph(g, stream=s_cap):
            for _ in range(args.steps):
                fn()
    torch.cuda.current_stream().wait_stream(s_cap)
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in evs:
        a.record()
        g.replay()
        b.record()
    torch.cuda.synchronize()
    t = sorted(a.elapsed_time(b) / 1e3 / args.steps for a, b in evs)
    med = t[len(t) // 2]
    peaks = load_peaks()
    out = {"kernel": args.kernel, "shape": [M, N, K], "steps": args.steps, "median_us": round(med * 1e6, 2),
           "device_error": sq.sq_device_error(clear=True)}
    if nbytes:
        out["gbs"] = round(nbytes / med / 1e9, 1)
        out["hbm_frac"] = round(nbytes / med / 1e9 / peaks["hbm_gbs"], 3)
    if ops:
        out["tops"] = round(ops / med / 1e12, 1)
        out["int8_frac"] = round(ops / med / 1e12 / (INT8_PER_BF16 * peaks["bf16_tflops"]), 3)
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel", choices=("alpha", "gemm", "gemm8", "fold", "lnquant", "quant", "calib", "wabsmax", "xabsmax"),
                    help="run only this kernel on --shape M,N,K (profiling aid; prints no bench line)")
    ap.add_argument("--shape", default="2048,4096,4096")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.kernel:
        run_kernel(args)
        return
    rank, world, local = init_dist()
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_device(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
