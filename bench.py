#!/usr/bin/env python
"""Benchmark of the SmoothQuant W8A8 linear hot path on B200.

One step = one pass of the whole path over one batch, for each linear of a transformer layer:
  calibration absmax of the linear's input (of the LayerNorm output where there is one)
  -> weight row absmax -> smoothing factors (alpha = 0.5) -> fold + per-channel weight INT8
  -> LayerNorm / smoothing + per-token INT8 -> INT8 tensor-core GEMM with the dequant
  epilogue to bf16.
The timed step (the JSON line's `value`) is the 175B-class linear set at 2048 tokens: QKV
12288 -> 36864 and up 12288 -> 49152 (LayerNorm in front), O 12288 -> 12288 and down
49152 -> 12288 (input from a previous GEMM), W ~ N(0, 0.015).  Measured beside it, each with
its own CUDA events: the 8B-class prefill set (8192 tokens; QKV 4096 -> 6144, O 4096 -> 4096,
gate+up 4096 -> 28672, down 14336 -> 4096), decode-sized GEMMs and their quantiser (1, 16, 64
tokens on the 8B shapes; 16 tokens on the 175B shapes), the calibration reduction over 512 x 512
tokens x 4096 channels, and the bandwidth kernels one by one.
Synthetic seeded inputs: bf16 activations with 1% fixed outlier channels x100, gamma ~
U(0.5, 1.5).  Under torchrun every rank runs its own batch (weak scaling); the calibration
statistic is combined across ranks with an all-reduce(MAX).

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
ALPHA = 0.5
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
INT8_PER_BF16 = 2.0        # dense INT8 tensor rate / dense BF16 rate on B200 (4.5 vs 2.25 PFLOP/s nominal)
INT8_NOMINAL_TOPS = 4500.0  # NVIDIA's dense INT8 figure for B200 (context)


class Workload:
    def __init__(self, key, text, tokens, w_std, layers):
        self.key, self.text, self.tokens, self.w_std, self.layers = key, text, tokens, w_std, layers

    def ops(self) -> float:
        return float(sum(2.0 * self.tokens * N * K for _, K, N, _ in self.layers))


HEADLINE = Workload("175b_m2048", "175B-class linear set: 2048 tokens x {QKV 12288->36864 (LN), O 12288->12288, "
                    "up 12288->49152 (LN), down 49152->12288}; W ~ N(0, 0.015); calibration on the batch, alpha 0.5",
                    2048, 0.015, (("qkv", 12288, 36864, True), ("o", 12288, 12288, False),
                                  ("up", 12288, 49152, True), ("down", 49152, 12288, False)))
PREFILL_8B = Workload("8b_m8192", "8B-class prefill linear set: 8192 tokens x {QKV 4096->6144 (LN), O 4096->4096, "
                      "gate+up 4096->28672 (LN), down 14336->4096}; W ~ N(0, 0.02); calibration on the batch, alpha 0.5",
                      8192, 0.02, (("qkv", 4096, 6144, True), ("o", 4096, 4096, False),
                                   ("gate_up", 4096, 28672, True), ("down", 14336, 4096, False)))
DECODE_M_8B = (1, 16, 64)
DECODE_M_175B = (16,)
CALIB_TOKENS, CALIB_K, CALIB_ALPHAS = 512 * 512, 4096, (0.4, 0.5, 0.6, 0.75)
CPU_GEMM_ROWS = 16   # oracle GEMM rows per linear (extrapolated linearly in rows)


def gemm_traffic(workload_key: str) -> int | None:
    """DRAM bytes per GEMM launch of this workload's step from the committed ncu summary, or
    None when the GEMM sources changed since the counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"w8a8_gemm_traffic_{workload_key}.md")
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
                                          "-i", str(self.gpu), "-lms", "50"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.1)
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
    """Device buffers of one linear of a step."""

    def __init__(self, name, K, N, ln, M, device, seed, w_std):
        import sq_inputs
        import w8a8_smoothquant_gemm_b200 as sq
        self.name, self.K, self.N, self.ln, self.M = name, K, N, ln, M
        self.x, self.W, self.gamma, _ = sq_inputs.torch_case(M, K, N, seed, device, w_std=w_std)
        f32 = dict(dtype=torch.float32, device=device)
        self.ax, self.aw, self.s = torch.empty(K, **f32), torch.empty(K, **f32), torch.empty(K, **f32)
        self.gf = torch.empty(K, **f32) if ln else None
        self.wq = torch.empty(N, K, dtype=torch.int8, device=device)
        self.sw = torch.empty(N, **f32)
        self.xq = torch.empty(M, K, dtype=torch.int8, device=device)
        self.sx = torch.empty(M, **f32)
        self.y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
        need = sq.sq_w8a8_gemm_workspace_size(M, N, K)
        self.ws = torch.zeros(need, dtype=torch.uint8, device=device) if need else None

    def run(self, sq, world: int, ev=None):
        """The whole path of this linear; ev = (before quantiser, before GEMM, after GEMM) events."""
        if self.ln:
            sq.sq_calib_ln_absmax(self.x, self.gamma, out=self.ax)
        else:
            sq.sq_calib_absmax(self.x, 0, out=self.ax)
        combine_statistic(self.ax, world)
        sq.sq_calib_absmax(self.W, 1, out=self.aw)
        sq.sq_smooth_factors(self.ax, self.aw, ALPHA, out=self.s)
        sq.sq_fold_quant_weights(self.W, self.s, self.gamma if self.ln else None, wq=self.wq, sw=self.sw,
                                 gamma_f=self.gf)
        if ev is not None:
            ev[0].record()
        self.quantise(sq)
        if ev is not None:
            ev[1].record()
        sq.sq_w8a8_gemm(self.xq, self.sx, self.wq, self.sw, y=self.y, workspace=self.ws)
        if ev is not None:
            ev[2].record()

    def quantise(self, sq, x=None, xq=None, sx=None):
        x = self.x if x is None else x
        xq = self.xq if xq is None else xq
        sx = self.sx if sx is None else sx
        if self.ln:
            sq.sq_ln_smooth_quant(x, gamma_f=self.gf, xq=xq, sx=sx)
        else:
            sq.sq_ln_smooth_quant(x, s=self.s, xq=xq, sx=sx)

    # algorithmic bytes of the bandwidth kernels (one read of each input, one write of each output)
    def bytes_calib(self):
        return self.M * self.K * 2 + 4 * self.K + (4 * self.K if self.ln else 0)

    def bytes_wabsmax(self):
        return self.K * self.N * 2 + 4 * self.K

    def bytes_fold(self):
        return self.K * self.N * 2 + self.N * self.K + 4 * self.N + 4 * self.K + (8 * self.K if self.ln else 0)

    def bytes_quant(self):
        return self.M * self.K * 2 + self.M * self.K + 4 * self.M + 4 * self.K

    def gemm_ops(self):
        return 2.0 * self.M * self.N * self.K


def build_set(wl: Workload, device, rank: int):
    return [Linear(n, K, N, ln, wl.tokens, device, 1000 * rank + 17 * i + wl.tokens, wl.w_std)
            for i, (n, K, N, ln) in enumerate(wl.layers)]


def new_events(n):
    return [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(n)]


def time_steps(sq, layers, steps, world, device):
    """`steps` timed passes of the whole path over the set: device time of the whole region and,
    per linear, of its quantiser + GEMM and of its GEMM alone (CUDA events on the launching
    stream)."""
    evs = [new_events(len(layers)) for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record()
    for k in range(steps):
        for i, L in enumerate(layers):
            L.run(sq, world, evs[k][i])
    end.record()
    torch.cuda.synchronize()
    barrier(world)
    elapsed = max_over_ranks(start.elapsed_time(end) / 1e3, world, device)
    gemm = [statistics.median(evs[k][i][1].elapsed_time(evs[k][i][2]) / 1e3 for k in range(steps))
            for i in range(len(layers))]
    runtime = [statistics.median(evs[k][i][0].elapsed_time(evs[k][i][2]) / 1e3 for k in range(steps))
               for i in range(len(layers))]
    return elapsed, gemm, runtime


def count_launches(sq, layers, world) -> int | None:
    """Kernels of this library (namespace sqk) that one step launches, counted by the profiler on
    an untimed step; None if the profiler is unavailable."""
    try:
        from torch.profiler import ProfilerActivity, profile
        torch.cuda.synchronize()
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            for L in layers:
                L.run(sq, world)
            torch.cuda.synchronize()
        n = sum(1 for e in prof.events() if e.device_type.name == "CUDA" and "sqk::" in e.name)
        return n or None
    except Exception:  # noqa: BLE001 -- the count is reported as unknown
        return None


def time_graph(fn, calls: int, reps: int = 5) -> float:
    """Device seconds per call: `calls` calls captured in one CUDA graph (no host launch cost in
    the timed interval), replayed `reps` times; the median replay / calls."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for _ in range(calls):
                fn()
    torch.cuda.current_stream().wait_stream(s)
    g.replay()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in evs:
        a.record()
        g.replay()
        b.record()
    torch.cuda.synchronize()
    del g
    return statistics.median(a.elapsed_time(b) / 1e3 / calls for a, b in evs)


def copies_past_l2(t: torch.Tensor, total: int = 300 << 20, cap: int = 24):
    """t and clones of it whose total size exceeds `total` bytes (L2 is 126 MB), so that a call
    rotating over them reads its operand from HBM."""
    n = max(1, min(cap, -(-total // (t.numel() * t.element_size()))))
    return [t] + [t.clone() for _ in range(n - 1)]


def decode_sweep(sq, layers, Ms, hbm_gbs) -> dict:
    """Decode-sized GEMMs on the set's folded weights (rotated past L2), and the runtime path of
    each (the per-token quantiser of the linear's first M tokens + the GEMM)."""
    out = {}
    for L in layers:
        wqs = copies_past_l2(L.wq)
        for M in Ms:
            x = L.x[:M]
            xq = torch.empty(M, L.K, dtype=torch.int8, device=L.x.device)
            sx = torch.empty(M, dtype=torch.float32, device=L.x.device)
            y = torch.empty(M, L.N, dtype=torch.bfloat16, device=L.x.device)
            need = sq.sq_w8a8_gemm_workspace_size(M, L.N, L.K)
            ws = torch.zeros(need, dtype=torch.uint8, device=L.x.device) if need else None
            L.quantise(sq, x, xq, sx)
            rot = [0]

            def gemm():
                w = wqs[rot[0] % len(wqs)]
                rot[0] += 1
                sq.sq_w8a8_gemm(xq, sx, w, L.sw, y=y, workspace=ws)

            def path():
                L.quantise(sq, x, xq, sx)
                gemm()

            calls = max(2 * len(wqs), 20)
            t_g = time_graph(gemm, calls)
            t_p = time_graph(path, calls)
            b_g = M * L.K + L.N * L.K + 2 * M * L.N + 4 * (M + L.N)
            b_p = 2 * M * L.K + L.N * L.K + 2 * M * L.N + 4 * (L.N + L.K)
            out[f"{L.name}_m{M}"] = {
                "shape_MNK": [M, L.N, L.K], "gemm_us": round(t_g * 1e6, 2), "gemm_gbs": round(b_g / t_g / 1e9, 1),
                "gemm_hbm_frac": round(b_g / t_g / 1e9 / hbm_gbs, 3), "path_us": round(t_p * 1e6, 2),
                "path_hbm_frac": round(b_p / t_p / 1e9 / hbm_gbs, 3)}
        del wqs
    return out


def quantizer_profile(sq, layers, reps=3) -> dict:
    """Per-kernel CUDA-event times of the bandwidth kernels (separate from the timed steps).

    Before each timed kernel a 256 MB buffer is zeroed on the same stream: the L2 starts cold,
    and the device is still busy with it when the host has enqueued the kernel and its closing
    event, so an interval holds the kernel's device time, not the host's launch latency."""
    kinds = ("calib", "wabsmax", "fold", "quant")
    tot = {k: 0.0 for k in kinds}
    byt = {k: 0 for k in kinds}
    per = {}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=layers[0].x.device)
    pending = []

    def timed(kind, L, nbytes, fn):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        pending.append((kind, L.name, nbytes, a, b))

    for _ in range(reps):
        for L in layers:
            if L.ln:
                timed("calib", L, L.bytes_calib(), lambda: sq.sq_calib_ln_absmax(L.x, L.gamma, out=L.ax))
            else:
                timed("calib", L, L.bytes_calib(), lambda: sq.sq_calib_absmax(L.x, 0, out=L.ax))
            timed("wabsmax", L, L.bytes_wabsmax(), lambda: sq.sq_calib_absmax(L.W, 1, out=L.aw))
            sq.sq_smooth_factors(L.ax, L.aw, ALPHA, out=L.s)
            timed("fold", L, L.bytes_fold(),
                  lambda: sq.sq_fold_quant_weights(L.W, L.s, L.gamma if L.ln else None, wq=L.wq, sw=L.sw,
                                                   gamma_f=L.gf))
            timed("quant", L, L.bytes_quant(), lambda: L.quantise(sq))
    torch.cuda.synchronize()
    for kind, name, nbytes, a, b in pending:
        t = a.elapsed_time(b) / 1e3
        tot[kind] += t
        byt[kind] += nbytes
        per.setdefault(f"{kind}_{name}", []).append(nbytes / t / 1e9)
    del flush
    out = {f"{k}_gbs": round(byt[k] / tot[k] / 1e9, 1) for k in kinds}
    out["per_kernel_gbs"] = {k: round(statistics.median(v), 1) for k, v in per.items()}
    return out


def next_linear_fused(sq, up, down, hbm_gbs) -> dict:
    """The down linear's quantiser fused into the up linear's GEMM: the up GEMM (with the down
    linear's smoothing folded into its output scales) stores the down input and its row maxima,
    and a codes pass quantises it; against the same GEMM followed by the full per-token quantiser
    (statistics pass + codes pass over the stored output)."""
    M, N = up.M, up.N
    sw2 = sq.sq_fold_next_smoothing(up.sw, down.s)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=up.x.device)
    rmax = torch.empty(M, dtype=torch.float32, device=up.x.device)
    xq = torch.empty(M, N, dtype=torch.int8, device=up.x.device)
    sx = torch.empty(M, dtype=torch.float32, device=up.x.device)
    ones = torch.ones(N, dtype=torch.float32, device=up.x.device)
    t_gemm = time_graph(lambda: sq.sq_w8a8_gemm(up.xq, up.sx, up.wq, sw2, y=y, workspace=up.ws), 4)
    t_gemm_rm = time_graph(lambda: sq.sq_w8a8_gemm_rowmax(up.xq, up.sx, up.wq, sw2, y=y, rowmax=rmax,
                                                          workspace=up.ws), 4)
    t_quant = time_graph(lambda: sq.sq_ln_smooth_quant(y, s=ones, xq=xq, sx=sx), 8)
    t_codes = time_graph(lambda: sq.sq_quant_codes(y, rmax, xq=xq, sx=sx), 8)
    b_codes = M * N * 3 + 8 * M
    return {"workload": f"up {M}x{N}x{up.K} GEMM -> down input {M}x{N}",
            "gemm_us": round(t_gemm * 1e6, 1), "gemm_rowmax_us": round(t_gemm_rm * 1e6, 1),
            "quantiser_us": round(t_quant * 1e6, 1), "codes_pass_us": round(t_codes * 1e6, 1),
            "codes_pass_hbm_frac": round(b_codes / t_codes / 1e9 / hbm_gbs, 3),
            "unfused_us": round((t_gemm + t_quant) * 1e6, 1), "fused_us": round((t_gemm_rm + t_codes) * 1e6, 1)}


def calibration_config(sq, device, hbm_gbs) -> dict:
    """The calibration reduction: per-channel absmax over 512 x 512 tokens x 4096 bf16 channels
    (2 GiB, ~1% channels x log-uniform [20, 100]), the weight absmax of W [4096, 4096] and s for
    four alphas.  Inputs far larger than L2; CUDA events around each repetition."""
    import sq_inputs
    x, W, _, _ = sq_inputs.torch_case(CALIB_TOKENS, CALIB_K, CALIB_K, 2, device, outlier_mult=(20.0, 100.0))
    f32 = dict(dtype=torch.float32, device=device)
    ax, aw = torch.empty(CALIB_K, **f32), torch.empty(CALIB_K, **f32)
    ss = [torch.empty(CALIB_K, **f32) for _ in CALIB_ALPHAS]

    def once(evs=None):
        if evs:
            evs[0].record()
        sq.sq_calib_absmax(x, 0, out=ax)
        if evs:
            evs[1].record()
        sq.sq_calib_absmax(W, 1, out=aw)
        for a, o in zip(CALIB_ALPHAS, ss):
            sq.sq_smooth_factors(ax, aw, a, out=o)
        if evs:
            evs[2].record()

    for _ in range(2):
        once()
    evs = new_events(5)
    for e in evs:
        once(e)
    torch.cuda.synchronize()
    t_x = statistics.median(e[0].elapsed_time(e[1]) / 1e3 for e in evs)
    t_all = statistics.median(e[0].elapsed_time(e[2]) / 1e3 for e in evs)
    bx = CALIB_TOKENS * CALIB_K * 2
    b_all = bx + CALIB_K * CALIB_K * 2 + 4 * CALIB_K * (2 + 2 * len(CALIB_ALPHAS))
    del x, W
    torch.cuda.empty_cache()
    return {"workload": "512 x 512 tokens x K 4096 bf16 (2 GiB) activation absmax + W [4096, 4096] absmax + s for "
                        "alpha in {0.4, 0.5, 0.6, 0.75}",
            "us": round(t_all * 1e6, 1), "gbs": round(b_all / t_all / 1e9, 1),
            "hbm_frac": round(b_all / t_all / 1e9 / hbm_gbs, 3), "activation_absmax_us": round(t_x * 1e6, 1),
            "activation_absmax_gbs": round(bx / t_x / 1e9, 1),
            "activation_absmax_hbm_frac": round(bx / t_x / 1e9 / hbm_gbs, 3)}


def int8_probe(device) -> float | None:
    """Dense INT8 GEMM rate of the device's own library path (torch._int_mm, 8192^3): a measured
    ceiling for the INT8 tensor cores, best of 10."""
    try:
        n = 8192
        a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=device)
        b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=device).t()
        for _ in range(3):
            torch._int_mm(a, b)
        torch.cuda.synchronize()
        best = None
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._int_mm(a, b)
            e1.record()
            torch.cuda.synchronize()
            t = e0.elapsed_time(e1) / 1e3
            best = t if best is None else min(best, t)
        return 2.0 * n ** 3 / best / 1e12
    except Exception:  # noqa: BLE001 -- reported as unavailable
        return None


# ----------------------------------------------------------------------------- CPU oracle timing
def host_inputs(layers):
    out = []
    for L in layers:
        xh = L.x.cpu().view(torch.int16).numpy().view(np.uint16)
        Wh = L.W.cpu().view(torch.int16).numpy().view(np.uint16)
        out.append((xh, Wh, L.gamma.cpu().numpy()))
    return out


def oracle_pass(wl: Workload, host, gemm_rows: int) -> dict:
    """The oracle on the workload: calibration, weight absmax, smoothing factors, fold and the
    per-token quantiser at full size (measured), and the GEMM on the first `gemm_rows` rows of
    each linear, all columns (measured; the full GEMM time is that x tokens / gemm_rows, exact
    for a row-parallel product)."""
    import oracle as O
    t_a15 = t_g = 0.0
    for (name, K, N, ln), (xh, Wh, gh) in zip(wl.layers, host):
        t0 = time.perf_counter()
        ax = O.calib_ln_absmax(xh, gh) if ln else O.calib_absmax(xh, 0)
        aw = O.calib_absmax(Wh, 1)
        s = O.smooth_factors(ax, aw, ALPHA)
        wq, sw, gf, _ = O.fold_quant_weights(Wh, s, gh if ln else None)
        xq, sx = O.ln_smooth_quant(xh, gamma_f=gf) if ln else O.ln_smooth_quant(xh, s=s)
        t1 = time.perf_counter()
        O.w8a8_gemm(xq[:gemm_rows], sx[:gemm_rows], wq, sw, "bf16")
        t2 = time.perf_counter()
        t_a15 += t1 - t0
        t_g += t2 - t1
    full = t_a15 + t_g * wl.tokens / gemm_rows
    return {"a1_a5_s": t_a15, "gemm_sample_s": t_g, "full_step_s": full, "spent_s": t_a15 + t_g}


def cpu_baseline(layers, wl: Workload, single_thread_wl_layers=None) -> dict:
    import oracle as O
    host = host_inputs(layers)
    cores = O.num_threads()
    r = oracle_pass(wl, host, CPU_GEMM_ROWS)
    del host
    out = {"value": wl.ops() / r["full_step_s"] / 1e12, "unit": "TOPS", "cores": cores, "kind": "oracle",
           "sample": (f"{wl.key}: calibration, weight absmax, factors, fold and per-token quantiser at full size on "
                      f"{cores} threads ({r['a1_a5_s']:.2f} s measured); GEMM on the first {CPU_GEMM_ROWS} of "
                      f"{wl.tokens} tokens of each linear, all columns ({r['gemm_sample_s']:.2f} s measured), "
                      f"x {wl.tokens // CPU_GEMM_ROWS} for the full step (extrapolated, row-parallel); "
                      f"full step {r['full_step_s']:.1f} s"),
           "a1_a5_s": round(r["a1_a5_s"], 3), "gemm_sample_s": round(r["gemm_sample_s"], 3),
           "full_step_s_extrapolated": round(r["full_step_s"], 2)}
    if single_thread_wl_layers is not None:
        wl1, layers1 = single_thread_wl_layers
        host1 = host_inputs(layers1)
        r_all = oracle_pass(wl1, host1, 4)
        O.set_num_threads(1)
        try:
            r_one = oracle_pass(wl1, host1, 4)
        finally:
            O.set_num_threads(cores)
        out["threads_1_vs_all"] = {"workload": wl1.key, "a1_a5_s_1_thread": round(r_one["a1_a5_s"], 3),
                                   f"a1_a5_s_{cores}_threads": round(r_all["a1_a5_s"], 3),
                                   "gemm_4_rows_s_1_thread": round(r_one["gemm_sample_s"], 3),
                                   f"gemm_4_rows_s_{cores}_threads": round(r_all["gemm_sample_s"], 3)}
    return out


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    """The CPU oracle, as it stands, on this machine's cores, on the headline workload: each step
    runs calibration, weight absmax, factors, fold and quantiser at full size and the GEMM on a
    row sample of every linear; `ms_per_step` is the time actually spent per step, `value` the
    full step's TOPS (GEMM part extrapolated linearly in rows)."""
    if rank != 0:
        return
    import oracle as O
    import sq_inputs
    host = []
    for i, (name, K, N, ln) in enumerate(HEADLINE.layers):
        x, W, g, _ = sq_inputs.torch_case(HEADLINE.tokens, K, N, 1000 + i, "cpu", w_std=HEADLINE.w_std)
        host.append((x.view(torch.int16).numpy().view(np.uint16), W.view(torch.int16).numpy().view(np.uint16),
                     g.numpy()))
    rows = 4
    for _ in range(args.warmup):  # warm-up: one small oracle pass (no timing)
        xh, Wh, gh = host[1]
        O.calib_absmax(xh[:64], 0)
        O.calib_absmax(Wh[:, :64].copy(), 1)
    spent, fulls = [], []
    for _ in range(args.steps):
        r = oracle_pass(HEADLINE, host, rows)
        spent.append(r["spent_s"])
        fulls.append(r["full_step_s"])
    t_spent = statistics.mean(spent)
    t_full = statistics.mean(fulls)
    value = HEADLINE.ops() / t_full / 1e12
    sample = (f"per step: calibration, weight absmax, factors, fold, quantiser at full size; GEMM on {rows} of "
              f"{HEADLINE.tokens} tokens per linear, all columns; value extrapolates the GEMM linearly in rows "
              f"(full step {t_full:.1f} s)")
    line = {"metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_spent * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic", "impl": "reference",
            "config": {"workload": HEADLINE.text, "tokens": HEADLINE.tokens, "alpha": ALPHA},
            "full_step_ms_extrapolated": t_full * 1e3,
            "cpu_baseline": {"value": value, "unit": "TOPS", "cores": O.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- main arm
def e2e_measure(sq, layers, world, device, steps: int, ops: float) -> dict:
    """End to end through the public API: pinned host inputs -> device -> path -> host output.
    Copies run on their own streams (host->device and device->host in parallel over the
    full-duplex link), ordered by events so that a linear's copies overlap its neighbours'
    compute; every byte of every step's inputs and outputs crosses the link inside the timed
    region."""
    h = [{"x": L.x.cpu().pin_memory(), "W": L.W.cpu().pin_memory(), "g": L.gamma.cpu().pin_memory(),
          "y": torch.empty(L.y.shape, dtype=L.y.dtype, pin_memory=True)} for L in layers]
    h2d = sum(b["x"].numel() * 2 + b["W"].numel() * 2 + b["g"].numel() * 4 for b in h)
    d2h = sum(b["y"].numel() * 2 for b in h)
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
    e2e_run(steps)
    e1.record(cs)
    torch.cuda.synchronize()
    barrier(world)
    t = max_over_ranks(e0.elapsed_time(e1) / 1e3, world, device)
    del h
    return {"value": ops * world * steps / t / 1e12, "unit": "TOPS", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": t / steps * 1e3,
            "link": "pinned host buffers; host->device and device->host copies on separate streams"}


def gemm_summary(layers, gemm_s, runtime_s, peak) -> dict:
    return {L.name: {"shape_MNK": [L.M, L.N, L.K], "gemm_us": round(t * 1e6, 1),
                     "tops": round(L.gemm_ops() / t / 1e12, 1), "frac": round(L.gemm_ops() / t / 1e12 / peak, 3),
                     "quant_plus_gemm_us": round(r * 1e6, 1)}
            for L, t, r in zip(layers, gemm_s, runtime_s)}


def run_device(args, rank, world, local):
    import w8a8_smoothquant_gemm_b200 as sq
    device = torch.device("cuda", local)
    sq.lib()
    peaks = load_peaks()
    hbm = peaks["hbm_gbs"]
    probe = int8_probe(device) if not args.quick else None
    int8_peak = max(INT8_PER_BF16 * peaks["bf16_tflops"], probe or 0.0)

    # ---------------------------------------------------------------- headline: 175B-class set
    layers = build_set(HEADLINE, device, rank)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        for L in layers:
            L.run(sq, world)
    torch.cuda.synchronize()
    if sq.sq_device_error(clear=True) != 0:
        raise RuntimeError("a kernel gave up on a bounded wait during warm-up")
    with ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local) as clk:
        elapsed, gemm_s, runtime_s = time_steps(sq, layers, args.steps, world, device)
    if sq.sq_device_error(clear=True) != 0:
        raise RuntimeError("a kernel gave up on a bounded wait during the timed steps")
    ops_step = HEADLINE.ops()
    value = ops_step * world * args.steps / elapsed / 1e12
    achieved = sum(L.gemm_ops() for L in layers) / sum(gemm_s) / 1e12
    roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(int8_peak, 1), "unit": "TOPS",
                "frac": round(achieved / int8_peak, 4), "traffic": gemm_traffic(HEADLINE.key),
                "traffic_unit": "DRAM bytes per GEMM launch (mean of the 4 launches of a step)",
                "algorithmic_bytes_per_launch": int(sum(L.M * L.K + L.N * L.K + 2 * L.M * L.N for L in layers) / 4),
                "kernel": "w8a8_gemm_kernel (tcgen05 kind::i8), 4 launches per step",
                "peak_note": (f"max(2 x {peaks['source']} burst bf16 {peaks['bf16_tflops']} TFLOP/s, "
                              f"torch._int_mm 8192^3 probe {None if probe is None else round(probe, 1)} TOPS)"),
                "int8_probe_tops": None if probe is None else round(probe, 1),
                "frac_of_nominal_4500": round(achieved / INT8_NOMINAL_TOPS, 4)}
    runtime_tops = sum(L.gemm_ops() for L in layers) / sum(runtime_s) / 1e12
    headline = {"gemm": gemm_summary(layers, gemm_s, runtime_s, int8_peak),
                "runtime_only_tops": round(runtime_tops, 1),
                "runtime_only_note": "per-token quantiser + GEMM of each linear (the deployed forward pass), "
                                     "median over the timed steps"}
    launches = count_launches(sq, layers, world)
    decode_175 = {} if args.quick else decode_sweep(sq, layers, DECODE_M_175B, hbm)
    next2 = next_linear_fused(sq, layers[2], layers[3], hbm)
    quant_175 = quantizer_profile(sq, layers)
    e2e = e2e_measure(sq, layers, world, device, max(2, args.steps // 10), ops_step)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_layers = layers
    else:
        cpu_layers = None

    # ---------------------------------------------------------------- 8B-class prefill set
    layers8 = build_set(PREFILL_8B, device, rank)
    for _ in range(args.warmup):
        for L in layers8:
            L.run(sq, world)
    el8, g8, r8 = time_steps(sq, layers8, args.steps, world, device)
    prefill8 = {"workload": PREFILL_8B.text, "tops": round(PREFILL_8B.ops() * world * args.steps / el8 / 1e12, 1),
                "ms_per_step": round(el8 / args.steps * 1e3, 4),
                "gemm": gemm_summary(layers8, g8, r8, int8_peak),
                "runtime_only_tops": round(sum(L.gemm_ops() for L in layers8) / sum(r8) / 1e12, 1),
                "quantizer": quantizer_profile(sq, layers8)}
    decode_8b = {} if args.quick else decode_sweep(sq, layers8, DECODE_M_8B, hbm)
    if cpu_layers is not None:
        cpu = cpu_baseline(cpu_layers, HEADLINE, (PREFILL_8B, layers8))
    del layers8
    torch.cuda.empty_cache()

    # ---------------------------------------------------------------- calibration reduction
    del layers
    torch.cuda.empty_cache()
    calib = None if args.quick else calibration_config(sq, device, hbm)
    if sq.sq_device_error(clear=True) != 0:
        raise RuntimeError("a kernel gave up on a bounded wait")

    quant_175["hbm_peak_gbs"] = hbm
    quant_175["quant_frac"] = round(quant_175["quant_gbs"] / hbm, 3)
    line = {"metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": HEADLINE.text, "tokens_per_gpu": HEADLINE.tokens, "alpha": ALPHA,
                       "shapes_KN": [[K, N] for _, K, N, _ in HEADLINE.layers],
                       "l2": "inputs larger than L2: 3.62 GB of bf16 weights + 0.35 GB of activations read per "
                             "step (L2 126 MB)",
                       "parallelism": f"dp{world}"},
            "roofline": roofline, "headline": headline, "quantizer": quant_175, "decode_175b": decode_175,
            "next_linear_fused": next2,
            "prefill_8b": prefill8, "decode_8b": decode_8b, "calibration": calib,
            "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": None if launches is None else launches * args.steps,
            "gpu_launches_note": "this library's kernels (namespace sqk) in one step, counted by the profiler on an "
                                 "untimed step, x steps",
            "clocks": clk.summary()}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_kernel(args):
    """One kernel of the path on one shape, `--steps` times, CUDA-event timed (profiling aid).

    --shape M,N,K; the activation is [M, K] with a LayerNorm in front, the weight [K, N]."""
    import w8a8_smoothquant_gemm_b200 as sq
    M, N, K = (int(v) for v in args.shape.split(","))
    device = torch.device("cuda", 0)
    L = Linear("k", K, N, True, M, device, 7, 0.02)
    L.run(sq, 1)
    torch.cuda.synchronize()
    gemm_bytes = M * K + N * K + 2 * M * N + 4 * (M + N)
    n_copies = max(1, min(32, -(-300 * 2 ** 20 // gemm_bytes)))
    copies = [(L.xq.clone(), L.wq.clone(), torch.empty_like(L.y)) for _ in range(n_copies)]
    rot = [0]

    def gemm_call():
        xq, wq, y = copies[rot[0] % n_copies]
        rot[0] += 1
        sq.sq_w8a8_gemm(xq, L.sx, wq, L.sw, y=y, workspace=L.ws)

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
        wq8, sw8, gf8, _ = sq.sq_fold_quant_weights_fp8(L.W, L.s, L.gamma)
        xq8, sx8 = sq.sq_ln_smooth_quant_fp8(L.x, gamma_f=gf8)
        copies8 = [(xq8.clone(), wq8.clone(), torch.empty_like(L.y)) for _ in range(n_copies)]

    def gemm8_call():
        xq, wq, y = copies8[rot[0] % n_copies]
        rot[0] += 1
        sq.sq_w8a8_gemm_fp8(xq, sx8, wq, sw8, y=y, workspace=L.ws)

    if args.kernel == "alpha":
        alpha_ws = torch.empty(sq.lib().sq_alpha_search_workspace_size(M, K, N), dtype=torch.uint8, device=device)

    s_plain = L.s
    calls = {
        "alpha": (lambda: sq.sq_alpha_search(L.x, L.W, None, gamma=L.gamma, workspace=alpha_ws), 0, 0.0),
        "gemm": (gemm_call, gemm_bytes, 2.0 * M * N * K),
        "gemm8": (gemm8_call, gemm_bytes, 2.0 * M * N * K),
        "fold": (rotated(lambda: sq.sq_fold_quant_weights(pick(ws), L.s, L.gamma, wq=pick(wq_out), sw=L.sw,
                                                          gamma_f=L.gf)), L.bytes_fold(), 0.0),
        "lnquant": (rotated(lambda: sq.sq_ln_smooth_quant(pick(xs), gamma_f=L.gf, xq=pick(xq_out), sx=L.sx)),
                    L.bytes_quant(), 0.0),
        "quant": (rotated(lambda: sq.sq_ln_smooth_quant(pick(xs), s=s_plain, xq=pick(xq_out), sx=L.sx)),
                  L.bytes_quant(), 0.0),
        "calib": (rotated(lambda: sq.sq_calib_ln_absmax(pick(xs), L.gamma, out=L.ax)), L.bytes_calib(), 0.0),
        "xabsmax": (rotated(lambda: sq.sq_calib_absmax(pick(xs), 0, out=L.ax)), M * K * 2 + 4 * K, 0.0),
        "wabsmax": (rotated(lambda: sq.sq_calib_absmax(pick(ws), 1, out=L.aw)), L.bytes_wabsmax(), 0.0),
    }
    fn, nbytes, ops = calls[args.kernel]
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    if args.kernel in ("gemm", "gemm8"):
        args.steps = max(args.steps, n_copies)
    else:
        args.steps = max(args.steps, len(xs), len(ws))
    med = time_graph(fn, args.steps)
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
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--quick", action="store_true", help="headline and 8B sets only (no decode sweep, probe or "
                                                         "calibration config)")
    ap.add_argument("--kernel", choices=("alpha", "gemm", "gemm8", "fold", "lnquant", "quant", "calib", "wabsmax",
                                         "xabsmax"),
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
