"""Benchmark: fully quantized NVFP4 linear layers at Llama-7B shapes on B200.

One step = forward + backward of the seven linear layers of a Llama-7B block
at 32768 tokens (batch 64 x seq 512): QKVO 4 x (4096 <- 4096), gate/up
2 x (11008 <- 4096), down 1 x (4096 <- 11008).  Per layer: quantize X
(row-wise RTN for fprop, transposed SR for wgrad), quantize W (16x16 tiles,
both orientations), fprop, quantize dY (row-wise and transposed, SR), dgrad,
wgrad -- the calls fqt_linear_fwd / fqt_linear_bwd make, issued one by one
through the public API so that each GEMM and quantizer is bracketed by CUDA
events on the launching stream.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--fmt nvfp4|mxfp4] [--wgrad-rht]

Prints ONE JSON line (rank 0).  value = 6 * sum(M N K) flops of all ranks /
max-over-ranks device time.  Inputs are synthetic (seeded), resident in HBM
and larger than L2 (126 MB) -- no L2 flush is needed between steps.
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
sys.path.insert(0, ROOT)

M_TOKENS = 32768
LAYERS = [("qkvo", 4096, 4096)] * 4 + [("gate_up", 11008, 4096)] * 2 + [("down", 4096, 11008)]
METRIC = "NVFP4 linear fwd+bwd TFLOPS & % FP4 peak; quantizer GB/s & % HBM BW"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_PER_BF16 = 4.0          # nominal dense FP4 / dense BF16 tensor throughput (9 / 2.25 PF)
# DRAM bytes (read + write) per FLOP of fp4_gemm_sfst_kernel as it stands,
# from one ncu capture of one launch per GEMM shape of the step at reduced
# size (the committed launch-list profile gives the command and the
# figures); multiplied by the step's average FLOPs per GEMM launch it is
# `roofline.traffic`.  None whenever the GEMM kernel changes until
# re-measured.
GEMM_DRAM_BYTES_PER_FLOP = 3.006e-4
# Algorithmic bytes per element of one quantize call producing row-wise and
# transposed outputs with an in-kernel amax: amax read 2 B + encode read 2 B
# + two outputs of (0.5 B codes + 1/16 B scales).
Q_BYTES_PER_ELEM = 2 + 2 + 2 * (0.5 + 1 / 16)


def max_over_ranks(x: float, device, world: int) -> float:
    """The largest of every rank's `x` (all ranks take part; any backend)."""
    t = torch.tensor([x], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms_max: float) -> float:
    """Units processed by all ranks per second, timed by the slowest rank."""
    return world * units_per_rank / (ms_max * 1e-3)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------------------
# clocks sampling (nvidia-smi during the timed region)
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.dev = device_index

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self, t_start=None, t_end=None):
        """Median SM clock and active throttle reasons of the samples taken
        between the wall-clock times t_start and t_end (all if not given)."""
        import datetime
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 7:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                if t_start is not None and not (t_start <= ts <= t_end):
                    continue
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
class Layer:
    def __init__(self, F, name, N, K, cfg, src, device):
        self.name, self.N, self.K, self.M = name, N, K, M_TOKENS
        self.x = src["X"].to(device, non_blocking=False)
        self.w = src["W"].to(device)
        self.dy = src["dY"].to(device)
        self.cfg = cfg
        self.sv = F.Saved.empty(self.M, N, K, cfg, device=device, logical_scales=False)
        self.y = torch.empty((self.M, N), dtype=torch.bfloat16, device=device)
        self.dx = torch.empty((self.M, K), dtype=torch.bfloat16, device=device)
        self.dw = torch.empty((N, K), dtype=torch.float32, device=device)


def step_config(fmt: str, wgrad_rht: bool, world: int, dp_allreduce: bool) -> dict:
    """The `config` of the step's JSON line, shared by both arms."""
    nv = fmt == "nvfp4"
    rht = ("wgrad 16-pt" if wgrad_rht else "off") if nv else "all GEMMs 32-pt"
    return {"workload": "Llama-7B linear layers fwd+bwd (QKVO x4 4096x4096, gate/up x2 "
                        "11008x4096, down 11008->4096), tokens 32768 (bs 64 x seq 512)",
            "format": fmt, "rounding": "RTN fwd, SR bwd/update" if nv else "RTN fwd/bwd",
            "weights": "16x16 tiles" if nv else "1x32", "rht": rht,
            "l2": "inputs larger than L2 (no flush)",
            "parallelism": f"dp x{world}, dW all-reduce (NCCL, overlapped)" if dp_allreduce
            else f"replicas x{world}"}


def make_layers(F, cfg, device, seed):
    import fqt_synth as S
    cache = {}
    layers = []
    for name, N, K in LAYERS:
        if (N, K) not in cache:
            cache[(N, K)] = S.llama_linear(N, K, M=M_TOKENS, seed=seed)
        layers.append(Layer(F, name, N, K, cfg, cache[(N, K)], device))
    return layers, cache


def qparams_for(cfg, which):
    """The quantize requests fqt_linear_fwd / fqt_linear_bwd issue."""
    rn, m = cfg.rht_n, cfg.rht_mask
    if which == "x":
        return dict(fmt=cfg.fmt, round=cfg.round_fwd, round_t=cfg.round_x_t,
                    rht_n=rn if m & 1 else 0, rht_n_t=rn if m & 4 else 0, rht_seed=cfg.seed,
                    sr_seed=cfg.seed, sr_stream=0, sr_stream_t=3)
    if which == "w":
        # W^T feeds dgrad: the QuEST-style forward scale does not apply there
        return dict(fmt=cfg.fmt, block=cfg.w_block, round=cfg.round_fwd,
                    round_t=0 if cfg.round_fwd == 2 else cfg.round_fwd,
                    rht_n=rn if m & 1 else 0, rht_n_t=rn if m & 2 else 0, rht_seed=cfg.seed)
    return dict(fmt=cfg.fmt, round=cfg.round_bwd, round_t=cfg.round_bwd,
                rht_n=rn if m & 2 else 0, rht_n_t=rn if m & 4 else 0, rht_seed=cfg.seed,
                sr_seed=cfg.seed, sr_stream=1, sr_stream_t=2)


class DwAllReduce:
    """Data-parallel gradient exchange: each layer's FP32 dW [N, K] summed over
    all ranks.  It is issued right after that layer's wgrad and runs on a
    stream of its own, after the work already queued, so it overlaps the next
    layer's kernels.  `finish` makes the launching stream wait for every
    pending sum; every rank issues the same sums in the same order.

    With `F` and `comm` (an F.NcclComm) the sums go through the library's
    fp4_allreduce_sum_f32 (NCCL on the comm stream); without them, through
    torch.distributed (any backend: the CPU tests run it on gloo)."""

    def __init__(self, world: int, F=None, comm=None):
        self.world, self.works, self.F, self.comm = world, [], F, comm
        self.stream = torch.cuda.Stream() if comm is not None else None

    def issue(self, dw: torch.Tensor):
        """Starts the sum of dw after the work queued on the current stream;
        returns its handle (None on one rank)."""
        if self.world <= 1:
            return None
        if self.comm is None:
            work = torch.distributed.all_reduce(dw, async_op=True)
            self.works.append(work)
            return work
        ready = torch.cuda.Event()
        ready.record()
        self.stream.wait_event(ready)
        self.F.fp4_allreduce_sum_f32(self.comm, dw, stream=self.stream)
        done = torch.cuda.Event()
        done.record(self.stream)
        work = _StreamWork(done)
        self.works.append(work)
        return work

    def finish(self) -> None:
        for w in self.works:
            w.wait()
        self.works.clear()


class _StreamWork:
    """A sum enqueued on the comm stream: wait() orders the current stream
    after it (the torch work handle's meaning for NCCL)."""

    def __init__(self, event):
        self.event = event

    def wait(self):
        torch.cuda.current_stream().wait_event(self.event)


def plan(F, layers, ws, dp=None):
    """The calls of one step: (kind, units, thunk, label) -- the calls
    fqt_linear_fwd / fqt_linear_bwd make for each layer, and with `dp` (a
    DwAllReduce) the dW sum after each wgrad and the wait for all of them at
    the end of the step."""
    calls = []
    for L in layers:
        sv = L.sv
        qx, qw, qd = (qparams_for(L.cfg, k) for k in ("x", "w", "dy"))
        tag = f"{L.name}[{L.N}x{L.K}]"
        calls += [
            ("quant", L.M * L.K, lambda L=L, sv=sv, q=qx: F.fp4_quantize(L.x, sv.xq, sv.xq_t, ws=ws, **q),
             f"quant X {tag}"),
            ("quant", L.N * L.K, lambda L=L, sv=sv, q=qw: F.fp4_quantize(L.w, sv.wq, sv.wq_t, ws=ws, **q),
             f"quant W {tag}"),
            ("gemm", 2 * L.M * L.N * L.K, lambda L=L, sv=sv: F.fp4_gemm(sv.xq, sv.wq, L.y, ws=ws),
             f"fprop {tag}"),
            ("quant", L.M * L.N, lambda L=L, sv=sv, q=qd: F.fp4_quantize(L.dy, sv.dyq, sv.dyq_t, ws=ws, **q),
             f"quant dY {tag}"),
            ("gemm", 2 * L.M * L.N * L.K, lambda L=L, sv=sv: F.fp4_gemm(sv.dyq, sv.wq_t, L.dx, ws=ws),
             f"dgrad {tag}"),
            ("gemm", 2 * L.M * L.N * L.K, lambda L=L, sv=sv: F.fp4_gemm(sv.dyq_t, sv.xq_t, L.dw, ws=ws),
             f"wgrad {tag}"),
        ]
        if dp is not None:
            calls.append(("comm", L.N * L.K * 4, lambda L=L: dp.issue(L.dw), f"dW all-reduce {tag}"))
    if dp is not None:
        calls.append(("comm", 0, dp.finish, "dW all-reduce wait"))
    return calls


def step(calls, events=None):
    """One pass of the hot path; `events` (pre-created pairs) brackets each call."""
    for i, (kind, units, fn, _label) in enumerate(calls):
        if events is not None:
            events[i][0].record()
            fn()
            events[i][1].record()
        else:
            fn()


def e2e_run(F, layers, cache, cfg, ws, steps, device, dp=None):
    """Same workload through fqt_linear_fwd / fqt_linear_bwd with HOST buffers:
    every step copies X, W, dY in from pinned memory and Y, dX, dW out (dW
    after its sum over ranks when `dp` is given).

    Three streams pipeline the layers and the steps: host-to-device copies of
    layer i + 1 and device-to-host copies of layer i - 1 run while layer i
    computes, and the two copy directions overlap each other.  The forward
    starts once X and W have landed (dY still on its way) and Y goes out
    while the backward runs.  Events order each layer's buffers: its inputs
    are overwritten only after the previous step's compute read them, its
    outputs only after the previous step's copy-out.
    Returns (ms per step, H2D bytes, D2H bytes, the pinned host buffers by
    layer shape)."""
    host = {}
    for (N, K), src in cache.items():
        host[(N, K)] = {
            "X": src["X"].pin_memory(), "W": src["W"].pin_memory(), "dY": src["dY"].pin_memory(),
            "Y": torch.empty((M_TOKENS, N), dtype=torch.bfloat16).pin_memory(),
            "dX": torch.empty((M_TOKENS, K), dtype=torch.bfloat16).pin_memory(),
            "dW": torch.empty((N, K), dtype=torch.float32).pin_memory()}
    h2d_s, comp_s, d2h_s = (torch.cuda.Stream(device) for _ in range(3))
    ev = lambda: torch.cuda.Event()
    loaded_xw = [ev() for _ in layers]     # X and W of layer i on the device
    loaded_dy = [ev() for _ in layers]     # dY of layer i on the device
    fwd_done = [ev() for _ in layers]      # layer i's forward done (Y ready)
    computed = [ev() for _ in layers]      # layer i's kernels done (inputs free)
    drained_y = [ev() for _ in layers]     # layer i's Y copied out
    drained = [ev() for _ in layers]       # layer i's dX and dW copied out

    def one():
        for i, L in enumerate(layers):
            h = host[(L.N, L.K)]
            with torch.cuda.stream(h2d_s):
                h2d_s.wait_event(computed[i])
                L.x.copy_(h["X"], non_blocking=True)
                L.w.copy_(h["W"], non_blocking=True)
                loaded_xw[i].record(h2d_s)
                L.dy.copy_(h["dY"], non_blocking=True)
                loaded_dy[i].record(h2d_s)
            with torch.cuda.stream(comp_s):
                comp_s.wait_event(loaded_xw[i])
                comp_s.wait_event(drained_y[i])
                F.fqt_linear_fwd(L.cfg, L.x, L.w, L.y, L.sv, ws)
                fwd_done[i].record(comp_s)
                comp_s.wait_event(loaded_dy[i])
                comp_s.wait_event(drained[i])
                F.fqt_linear_bwd(L.cfg, L.dy, L.sv, L.dx, L.dw, ws)
                work = dp.issue(L.dw) if dp is not None else None
                computed[i].record(comp_s)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(fwd_done[i])
                h["Y"].copy_(L.y, non_blocking=True)
                drained_y[i].record(d2h_s)
                d2h_s.wait_event(computed[i])
                h["dX"].copy_(L.dx, non_blocking=True)
                if work is not None:
                    work.wait()                  # d2h stream waits for the dW sum
                h["dW"].copy_(L.dw, non_blocking=True)
                drained[i].record(d2h_s)
        if dp is not None:
            dp.works.clear()                     # each sum was joined on the d2h stream

    one()
    torch.cuda.synchronize()
    h2d = sum((L.x.numel() + L.w.numel() + L.dy.numel()) * 2 for L in layers)
    d2h = sum(L.y.numel() * 2 + L.dx.numel() * 2 + L.dw.numel() * 4 for L in layers)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(h2d_s)
    for _ in range(steps):
        one()
    # the last step's final copy-out is the last work of the region
    d2h_s.wait_stream(h2d_s)
    d2h_s.wait_stream(comp_s)
    b.record(d2h_s)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    return ms, h2d, d2h, host


def cpu_baseline(rows_sample: int = 1024, cols_sample: int = 2048, seed: int = 0, cache=None,
                 fmt: str = "nvfp4", wgrad_rht: bool = False):
    """The oracle, as it stands, on a bounded sample of the same workload: for
    each of the 7 layers the first `rows_sample` tokens and the first
    `cols_sample` output features (X[:r], W[:c], dY[:r, :c]): the step's
    quantizations of X, W, dY in both orientations (NVFP4: RTN X and 16x16
    W, SR dY and X^T, optionally the 16-point rotation on the wgrad operands;
    MXFP4: RTN with the 32-point rotation everywhere), then the three GEMMs
    in float64.  Throughput in the metric's unit: 6 * r * c * K flops per
    second."""
    import fqt_synth as S
    import oracle as O
    t_total = 0.0
    flops = 0
    seen = {}
    if cache is None:
        cache = {}
    r, c = rows_sample, cols_sample
    nv = fmt == "nvfp4"
    rw = 16 if wgrad_rht else 0
    for name, N, K in LAYERS:
        if (N, K) not in seen:
            if (N, K) not in cache:
                cache[(N, K)] = S.llama_linear(N, K, M=M_TOKENS, seed=seed)
            d = cache[(N, K)]
            seen[(N, K)] = (S.as_f32(d["X"][:r]), S.as_f32(d["W"][:c]), S.as_f32(d["dY"][:r, :c]))
        X, W, dY = seen[(N, K)]
        T = lambda a: np.ascontiguousarray(a.T)
        t0 = time.perf_counter()
        if nv:
            qx = O.nvfp4_quantize_1d(X)
            qxt = O.nvfp4_quantize_1d(T(X), "sr", rht_n=rw, rht_seed=seed, sr_seed=seed,
                                      sr_stream=3)
            qw = O.nvfp4_quantize_2d(W)
            qwt = O.nvfp4_quantize_2d(T(W))
            qd = O.nvfp4_quantize_1d(dY, "sr", sr_seed=seed, sr_stream=1)
            qdt = O.nvfp4_quantize_1d(T(dY), "sr", rht_n=rw, rht_seed=seed, sr_seed=seed,
                                      sr_stream=2)
            deq = lambda q, b=(1, 16): O.dequantize(q["codes"], q["scales"], b)
            wb = (16, 16)
        else:
            mx = lambda a: O.mxfp4_quantize(a, "rtn", rht_n=32, rht_seed=seed)
            qx, qxt, qw, qwt, qd, qdt = mx(X), mx(T(X)), mx(W), mx(T(W)), mx(dY), mx(T(dY))
            deq = lambda q, b=None: O.dequantize(q["codes"], q["scales"], (1, 32), True)
            wb = None
        O.gemm(deq(qx), deq(qw, wb), s_dec_a=qx["s_dec"], s_dec_b=qw["s_dec"])
        O.gemm(deq(qd), deq(qwt, wb), s_dec_a=qd["s_dec"], s_dec_b=qwt["s_dec"])
        O.gemm(deq(qdt), deq(qxt), s_dec_a=qdt["s_dec"], s_dec_b=qxt["s_dec"])
        t_total += time.perf_counter() - t0
        flops += 6 * r * c * K
    return {"value": flops / t_total / 1e12, "unit": "TFLOP/s", "cores": O.num_threads(),
            "kind": "oracle", "seconds": round(t_total, 2),
            "sample": f"first {r} of {M_TOKENS} tokens x first {c} output features of each of "
                      f"the 7 layers: {fmt.upper()} quantize (both orientations) + 3 float64 "
                      "GEMMs"}


def run_ours(args, rank, world, device):
    import fp4_fully_quantized_b200 as F
    F.load()
    fmt = F.MXFP4 if args.fmt == "mxfp4" else F.NVFP4
    cfg = F.linear_cfg(fmt, out_dtype=F.OUT_BF16, seed=args.seed)
    if args.wgrad_rht and fmt == F.NVFP4:
        cfg.rht_mask = F.RHT_WGRAD
    if args.quest and fmt == F.MXFP4:
        cfg.round_fwd = F.QUEST           # Quartet: QuEST-style forward quantizer
    layers, cache = make_layers(F, cfg, device, args.seed + rank)
    ws = F.Workspace(device=device)
    dp = None
    if args.dp_allreduce:
        comm = F.NcclComm(rank, world) if world > 1 else None
        dp = DwAllReduce(world, F, comm)
    calls = plan(F, layers, ws, dp)
    clk = ClockSampler(device.index).__enter__()     # sampling before the timed region
    for _ in range(args.warmup):
        step(calls)
    torch.cuda.synchronize()
    if ws.status() != 0:
        raise RuntimeError(f"device status {ws.status()} after warm-up")
    time.sleep(0.5)

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    mk = lambda: torch.cuda.Event(enable_timing=True)
    evs = [[(mk(), mk()) for _ in calls] for _ in range(args.steps)]
    launches0 = F.kernel_launches()
    t0, t1 = mk(), mk()
    wall0 = time.time()
    t0.record()
    for i in range(args.steps):
        step(calls, evs[i])
    t1.record()
    torch.cuda.synchronize()
    wall1 = time.time()
    clk.__exit__(None, None, None)
    launches = F.kernel_launches() - launches0
    if world > 1:
        torch.distributed.barrier()
    ms = t0.elapsed_time(t1) / args.steps
    ms_max = max_over_ranks(ms, device, world)
    assert ws.status() == 0, f"device status {ws.status()}"

    ev = [(kind, units, a, b) for per in evs for (kind, units, _f, _l), (a, b) in zip(calls, per)]
    breakdown = {}
    for per in evs:
        for (kind, units, _f, label), (a, b) in zip(calls, per):
            if kind == "comm":          # enqueue only; the sum runs on NCCL's stream
                continue
            d = breakdown.setdefault(label, [kind, units, 0.0, 0])
            d[2] += a.elapsed_time(b)
            d[3] += 1
    detail = []
    for label, (kind, units, ms_sum, n) in breakdown.items():
        ms_avg = ms_sum / n
        rate = units / (ms_avg * 1e-3)
        detail.append({"call": label, "ms": round(ms_avg, 4),
                       "rate": round(rate / 1e12, 1) if kind == "gemm" else
                       round(rate * Q_BYTES_PER_ELEM / 1e9, 1),
                       "unit": "TFLOP/s" if kind == "gemm" else "GB/s"})
    flops_step = sum(6 * M_TOKENS * N * K for _, N, K in LAYERS)
    gemm_ms = sum(a.elapsed_time(b) for k, u, a, b in ev if k == "gemm")
    gemm_fl = sum(u for k, u, a, b in ev if k == "gemm")
    gemm_n = sum(1 for k, *_ in ev if k == "gemm")
    q_ms = sum(a.elapsed_time(b) for k, u, a, b in ev if k == "quant")
    q_elems = sum(u for k, u, a, b in ev if k == "quant")
    q_n = sum(1 for k, *_ in ev if k == "quant")
    pk, pk_src = peaks()
    # The GEMMs run in a step far shorter than a second at full clock: the
    # burst BF16 figure (not the seconds-long power-capped one) is their base.
    clk_now = clk.summary(wall0, wall1)
    near_max = (clk_now["sm_mhz"] or 0) >= 0.95 * (clk_now["sm_max_mhz"] or 1e9)
    burst = ms_max * args.steps < 1000.0 and near_max
    bf16_base = pk["bf16_tflops"] if burst else pk["bf16_tflops_sustained"]
    fp4_peak = bf16_base * FP4_PER_BF16
    mma_ceiling = F.mma_rate(0, 20000)      # back-to-back MMAs on resident operands
    gemm_tflops = gemm_fl / (gemm_ms * 1e-3) / 1e12
    q_gbs = q_elems * Q_BYTES_PER_ELEM / (q_ms * 1e-3) / 1e9

    e2e = None
    if not args.no_e2e:
        e_ms, h2d, d2h, _host = e2e_run(F, layers, cache, cfg, ws, args.e2e_steps, device, dp)
        e_max = max_over_ranks(e_ms, device, world)
        e2e = {"value": round(whole_job_rate(flops_step, world, e_max) / 1e12, 2),
               "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(e_max, 3), "steps": args.e2e_steps,
               "api": "fqt_linear_fwd + fqt_linear_bwd, host buffers, copies pipelined "
                      "across layers and steps on two copy streams"}

    out = {
        "metric": METRIC,
        "value": round(whole_job_rate(flops_step, world, ms_max) / 1e12, 2),
        "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_max, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp4(e2m1)+e4m3 scales, fp32 accumulate" if fmt == F.NVFP4 else
                 "fp4(e2m1)+e8m0 scales, fp32 accumulate",
        "data": "synthetic (seeded): X N(0,1) with 1% Student-t(3) channels, W N(0,0.02^2), "
                "dY N(0,1e-6)",
        "config": step_config(args.fmt, bool(args.wgrad_rht and fmt == F.NVFP4), world,
                              dp is not None),
        "roofline": {"kernel": "fp4_gemm_sfst_kernel (tcgen05 block-scaled, scales staged by tcgen05.st)", "bound": "tensor",
                     "achieved": round(gemm_tflops, 1), "peak": round(fp4_peak, 1),
                     "unit": "TFLOP/s", "frac": round(gemm_tflops / fp4_peak, 4),
                     "peak_source": f"{pk_src}: bf16 {'burst' if burst else 'sustained'} "
                                    f"{bf16_base:g} x {FP4_PER_BF16:g} (nominal FP4/BF16)",
                     "mma_ceiling": round(mma_ceiling, 1),
                     "frac_of_mma_ceiling": round(gemm_tflops / mma_ceiling, 4),
                     "mma_ceiling_source": "fp4_mma_rate: 128x256x64 NVFP4 MMAs back to back on "
                                           "operands resident in shared memory, this run",
                     "traffic": (round(GEMM_DRAM_BYTES_PER_FLOP * gemm_fl / gemm_n)
                                 if GEMM_DRAM_BYTES_PER_FLOP else None),
                     "traffic_unit": "DRAM bytes per launch (ncu per-shape captures, scaled by FLOPs)",
                     "launches": gemm_n,
                     "avg_ms": round(gemm_ms / max(gemm_n, 1), 4),
                     "share_of_step": round(gemm_ms / (ms_max * args.steps), 3)},
        "quantizer": {"bound": "hbm", "achieved": round(q_gbs, 1), "peak": pk["hbm_gbs"],
                      "unit": "GB/s", "frac": round(q_gbs / pk["hbm_gbs"], 4),
                      "bytes_per_elem": Q_BYTES_PER_ELEM, "launches": q_n,
                      "share_of_step": round(q_ms / (ms_max * args.steps), 3)},
        "gpu_launches": launches,
        "breakdown": detail,
        "clocks": clk_now,
    }
    if not args.no_sweep:
        out["quantizer_sweep"] = quantizer_sweep_line(F, device, 28, pk["hbm_gbs"])
    if e2e is not None:
        out["e2e"] = e2e
    return out, cache


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, on bounded samples.  The
    token sample of each step shrinks with the number of steps so that the
    whole run stays within about two and a half minutes (1024 tokens take
    about 7.5 s on 16 cores)."""
    f = min(1.0, 20.0 / max(1, args.steps + args.warmup)) ** 0.5   # sample side scale
    rows = args.ref_rows or max(64, int(1024 * f) // 64 * 64)
    cols = args.ref_cols or max(128, int(2048 * f) // 128 * 128)
    steps = []
    cache = {}                    # the synthetic layers are generated once, not per step
    for _ in range(args.warmup):
        cpu_baseline(rows, cols, args.seed, cache, args.fmt, args.wgrad_rht)
    for _ in range(args.steps):
        steps.append(cpu_baseline(rows, cols, args.seed, cache, args.fmt, args.wgrad_rht))
    v = statistics.median(s["value"] for s in steps)
    secs = sum(s["seconds"] for s in steps)
    flops_step = sum(6 * M_TOKENS * N * K for _, N, K in LAYERS)
    ms = flops_step / (v * 1e12) * 1e3
    cb = dict(steps[-1])
    cb["value"] = round(v, 6)
    return {"metric": METRIC, "impl": "reference", "value": round(v, 6), "unit": "TFLOP/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 1), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic (seeded)",
            "config": step_config(args.fmt, bool(args.wgrad_rht and args.fmt == "nvfp4"), 1,
                                  args.dp_allreduce),
            "cpu_baseline": cb, "seconds_total": round(secs, 1),
            "extrapolated": True,
            "extrapolation": f"each step times the oracle on {rows} of {M_TOKENS} tokens x {cols} "
                             "output features of every layer; ms_per_step scales that sample's "
                             "rate to the full step's FLOPs",
            "e2e": {"value": round(v, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# Quantizer sweep: (name, format, block, rounding, Hadamard points, algorithmic
# bytes per element).  One output (row-wise), tensor-core scale layout only,
# amax computed in the call: 2 B amax read + 2 B encode read + 0.5 B codes +
# 1/16 B scales (NVFP4; the 16x16 tile scale is written once per row of its
# tile in that layout); MXFP4 needs no amax pass: 2 + 0.5 + 1/32.
SWEEP_MODES = [
    ("nvfp4_1x16_rtn", "nvfp4", "1d", "rtn", 0, 4.5625),
    ("nvfp4_1x16_sr", "nvfp4", "1d", "sr", 0, 4.5625),
    ("nvfp4_1x16_rtn_rht16", "nvfp4", "1d", "rtn", 16, 4.5625),
    ("nvfp4_1x16_sr_rht16", "nvfp4", "1d", "sr", 16, 4.5625),
    ("nvfp4_16x16_rtn", "nvfp4", "2d", "rtn", 0, 4.5625),
    ("mxfp4_1x32_rtn", "mxfp4", "1d", "rtn", 0, 2.53125),
    ("mxfp4_1x32_rtn_rht32", "mxfp4", "1d", "rtn", 32, 2.53125),
]


def quantizer_sweep_line(F, device, log2n: int, hbm_gbs: float, reps: int = 5) -> dict:
    """The config-3 quantizer modes at 2^log2n elements (one row-wise output,
    amax computed in the call), each timed `reps` times after a 256 MiB write
    that evicts L2; median GB/s of algorithmic bytes and its fraction of the
    measured HBM copy bandwidth."""
    import fqt_synth as S
    ws = F.Workspace(device=device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    rows, cols = (1 << log2n) // 4096, 4096
    x = S.sweep_tensor(log2n, seed=log2n, width=cols).to(device)
    res = {"log2_elems": log2n, "shape": [rows, cols], "reps": reps, "l2": "256 MiB write between calls",
           "unit": "GB/s", "peak": hbm_gbs, "modes": {}}
    for name, fmt_s, blk_s, rnd_s, rht, bpe in SWEEP_MODES:
        fmt = F.MXFP4 if fmt_s == "mxfp4" else F.NVFP4
        blk = F.BLOCK_2D if blk_s == "2d" else F.BLOCK_1D
        q = F.QTensor.empty(rows, cols, fmt, blk, device=device, logical_scales=False)
        fn = lambda: F.fp4_quantize(x, q, fmt=fmt, block=blk, round=F.SR if rnd_s == "sr" else F.RTN,
                                    rht_n=rht, rht_seed=7, sr_seed=11, sr_stream=1, ws=ws)
        fn()
        times = []
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        ms = statistics.median(times)
        gbs = rows * cols * bpe / (ms * 1e-3) / 1e9
        res["modes"][name] = {"ms": round(ms, 4), "rate": round(gbs, 1), "frac": round(gbs / hbm_gbs, 4),
                              "bytes_per_elem": bpe}
        del q
    assert ws.status() == 0, f"device status {ws.status()}"
    return res


def run_sweep(args, device):
    """Quantizer sweep over 2^n elements shaped [2^n / 4096, 4096], N(0,1) with
    0.1 % of the elements x100; each timed call follows a 256 MiB write that
    evicts L2; median of the repetitions."""
    import fp4_fully_quantized_b200 as F
    import fqt_synth as S
    F.load()
    ws = F.Workspace(device=device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    lines = []
    for n in range(args.sweep_min, args.sweep_max + 1):
        rows, cols = (1 << n) // 4096, 4096
        x = S.sweep_tensor(n, seed=n, width=cols).to(device)
        for name, fmt_s, blk_s, rnd_s, rht, bpe in SWEEP_MODES:
            fmt = F.MXFP4 if fmt_s == "mxfp4" else F.NVFP4
            blk = F.BLOCK_2D if blk_s == "2d" else F.BLOCK_1D
            q = F.QTensor.empty(rows, cols, fmt, blk, device=device, logical_scales=False)
            fn = lambda: F.fp4_quantize(x, q, fmt=fmt, block=blk,
                                        round=F.SR if rnd_s == "sr" else F.RTN, rht_n=rht,
                                        rht_seed=7, sr_seed=11, sr_stream=1, ws=ws)
            reps = 20 if n < 28 else 5
            for _ in range(3):
                fn()
            times = []
            for _ in range(reps):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                fn()
                b.record()
                torch.cuda.synchronize()
                times.append(a.elapsed_time(b))
            assert ws.status() == 0, f"device status {ws.status()}"
            ms = statistics.median(times)
            gbs = rows * cols * bpe / (ms * 1e-3) / 1e9
            lines.append({"case": "sweep", "mode": name, "log2_elems": n, "rows": rows,
                          "cols": cols, "ms": round(ms, 5), "bytes_per_elem": bpe,
                          "rate": round(gbs, 1), "unit": "GB/s"})
            del q
        del x
    return lines


def run_swiglu(device, layers=8, hidden=2048, ffn=8192, tokens=16384, seed=0, check_rows=8,
               chained=False):
    """Chained SwiGLU MLP stack through the library's linear layer: NVFP4 fprop
    through all layers (RTN, 16x16 weight tiles), then dgrad / wgrad back with
    stochastically rounded gradients.  Every linear is fqt_linear_fwd /
    fqt_linear_bwd; the SwiGLU glue, silu(g) * u and its derivative, is harness
    code (torch, FP32 math on BF16 tensors).  The same stack in unquantized FP32
    is the comparison.  Returns per-layer relative Frobenius errors of the
    activations, input gradients and both weight gradients, the device time of
    the quantized pass, and the oracle spot check of the first and last layers'
    quantized operands (sampled rows, codes and scales bit-exact)."""
    import fp4_fully_quantized_b200 as F
    import fqt_synth as S
    F.load()
    L, H, Fd, M = layers, hidden, ffn, tokens
    cfg = F.linear_cfg(F.NVFP4, out_dtype=F.OUT_BF16, seed=seed)
    w_gu = [S.normal((2 * Fd, H), 0.02, seed=100 + l).to(device) for l in range(L)]
    w_d = [S.normal((H, Fd), 0.02, seed=200 + l).to(device) for l in range(L)]
    x0 = S.normal((M, H), 1.0, seed=1).to(device)
    dy_top = S.normal((M, H), 1e-3, seed=2).to(device)
    ws = F.Workspace(M, 2 * Fd, max(H, Fd), device=device)
    chk = {0, L - 1}
    sv_gu = [F.Saved.empty(M, 2 * Fd, H, cfg, device, logical_scales=l in chk) for l in range(L)]
    sv_d = [F.Saved.empty(M, H, Fd, cfg, device, logical_scales=l in chk) for l in range(L)]

    def silu(g):
        return g * torch.sigmoid(g)

    def dsilu(g):
        sg = torch.sigmoid(g)
        return sg * (1 + g * (1 - sg))

    # ---- quantized stack
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record()
    h, acts, gus, hin = x0, [], [], []
    for l in range(L):
        hin.append(h)
        y = torch.empty((M, 2 * Fd), dtype=torch.bfloat16, device=device)
        F.fqt_linear_fwd(cfg, h, w_gu[l], y, sv_gu[l], ws)
        gu = y.float()
        gus.append(gu)
        a = (silu(gu[:, :Fd]) * gu[:, Fd:]).to(torch.bfloat16).contiguous()
        hin.append(a)
        h = torch.empty((M, H), dtype=torch.bfloat16, device=device)
        F.fqt_linear_fwd(cfg, a, w_d[l], h, sv_d[l], ws)
        acts.append(h)
    fwd_end = torch.cuda.Event(enable_timing=True)
    fwd_end.record()

    def backward(chain_amax=None):
        """The backward pass.  With chain_amax (one supplied amax per block
        boundary, from an earlier pass: delayed scaling), block l's gate_up
        dgrad encodes block l-1's down-projection dY operand (row-wise, SR) in
        its epilogue and also stores it as BF16; that down layer then only
        quantizes the transposed operand, in one pass with the same supplied
        amax.  Returns the gradients, the dY tensors each linear consumed,
        and each block boundary's measured |dX| max."""
        d, dxs, dwg, dwd, dys, das = dy_top, [None] * L, [None] * L, [None] * L, {}, [None] * L
        cam = [torch.zeros(1, dtype=torch.float32, device=device) for _ in range(L)]
        for l in reversed(range(L)):
            dys[(l, "d")] = d
            da = torch.empty((M, Fd), dtype=torch.bfloat16, device=device)
            das[l] = da
            dwd[l] = torch.empty((H, Fd), dtype=torch.float32, device=device)
            if chain_amax is not None and l < L - 1:
                sv = sv_d[l]          # sv.dyq was encoded by block l + 1's dgrad epilogue
                F.fp4_quantize(d, None, sv.dyq_t, round_t=F.SR, sr_seed=seed, sr_stream_t=2,
                               amax_in_t=chain_amax[l], ws=ws)
                F.fp4_gemm(sv.dyq, sv.wq_t, da, ws=ws)
                F.fp4_gemm(sv.dyq_t, sv.xq_t, dwd[l], ws=ws)
            else:
                F.fqt_linear_bwd(cfg, d, sv_d[l], da, dwd[l], ws)
            g, u = gus[l][:, :Fd], gus[l][:, Fd:]
            daf = da.float()
            dgu = torch.cat([daf * u * dsilu(g), daf * silu(g)], dim=1).to(torch.bfloat16).contiguous()
            dys[(l, "gu")] = dgu
            dx = torch.empty((M, H), dtype=torch.bfloat16, device=device)
            dwg[l] = torch.empty((2 * Fd, H), dtype=torch.float32, device=device)
            if chain_amax is not None and l > 0:
                sv = sv_gu[l]
                F.fp4_quantize(dgu, sv.dyq, sv.dyq_t, round=F.SR, round_t=F.SR, sr_seed=seed,
                               sr_stream=1, sr_stream_t=2, ws=ws)
                F.fp4_gemm_quant_ex(sv.dyq, sv.wq_t, sv_d[l - 1].dyq, chain_amax[l - 1], round=F.SR,
                                    sr_seed=seed, sr_stream=1, c_bf16=dx, c_amax=cam[l - 1], ws=ws)
                F.fp4_gemm(sv.dyq_t, sv.xq_t, dwg[l], ws=ws)
            else:
                F.fqt_linear_bwd(cfg, dgu, sv_gu[l], dx, dwg[l], ws)
                if l > 0:
                    cam[l - 1].copy_(dx.float().abs().max().reshape(1))
            dxs[l] = dx
            d = dx
        return dxs, dwg, dwd, dys, das, cam

    dxs, dwg, dwd, dys, das, cam = backward()
    t1.record()
    torch.cuda.synchronize()
    assert ws.status() == 0, f"device status {ws.status()}"
    ms = t0.elapsed_time(t1)
    ms_bwd = fwd_end.elapsed_time(t1)
    chain = None
    if chained:
        # delayed scaling: this pass encodes with the amax the previous pass measured
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record()
        dxs, dwg, dwd, dys, das, cam2 = backward(chain_amax=cam)
        c1.record()
        torch.cuda.synchronize()
        assert ws.status() == 0, f"device status {ws.status()}"
        n_dx = (L - 1) * M * H            # gradient elements crossing a block boundary
        chain = {"ms_bwd_chained": round(c0.elapsed_time(c1), 3), "ms_bwd_unchained": round(ms_bwd, 3),
                 "boundaries": L - 1,
                 # per element of such a gradient: the unchained path writes BF16 (2 B),
                 # reads it for the amax (2 B) and for the fused row + transposed encode
                 # (2 B); chained, the epilogue writes BF16 and the row-wise codes, and
                 # one transposed-only pass reads the BF16 once
                 "hbm_bytes_removed": n_dx * 2,
                 "bf16_reads_removed": n_dx * 2 * 2 // 2,
                 "amax_supplied_vs_measured": [[float(a.item()), float(b.item())]
                                               for a, b in zip(cam[:L - 1], cam2[:L - 1])]}
    # gradient norm against the SR quantization noise of each layer's dY
    # (the two quantities the "FP4 All the Way" page relates)
    sums = torch.zeros(2, dtype=torch.float64, device=device)
    snr = {}
    for l in range(L):
        for key, sv in (("down", sv_d[l]), ("gate_up", sv_gu[l])):
            g = dys[(l, "d" if key == "down" else "gu")]
            F.fp4_quant_noise(g, sv.dyq, sums, ws)
            sx, sn = sums.tolist()
            snr[(l, key)] = (sx / sn) ** 0.5 if sn > 0 else float("inf")

    # ---- FP32 reference stack (no quantization, no BF16 rounding in between)
    prev_tf32 = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        hr, racts, rgus, rins = x0.float(), [], [], []
        for l in range(L):
            rins.append(hr)
            gu = hr @ w_gu[l].float().t()
            rgus.append(gu)
            a = silu(gu[:, :Fd]) * gu[:, Fd:]
            rins.append(a)
            hr = a @ w_d[l].float().t()
            racts.append(hr)
        dr = dy_top.float()
        rdx, rdwg, rdwd = [None] * L, [None] * L, [None] * L
        for l in reversed(range(L)):
            rdwd[l] = dr.t() @ rins[2 * l + 1]
            da = dr @ w_d[l].float()
            g, u = rgus[l][:, :Fd], rgus[l][:, Fd:]
            dgu = torch.cat([da * u * dsilu(g), da * silu(g)], dim=1)
            rdwg[l] = dgu.t() @ rins[2 * l]
            dr = dgu @ w_gu[l].float()
            rdx[l] = dr
        # the same forward stack with every GEMM input and output rounded to
        # BF16 (no FP4): the stack's own amplification of small rounding errors
        hb, bacts = x0.float(), []
        for l in range(L):
            gu = (hb @ w_gu[l].float().t()).to(torch.bfloat16).float()
            a = (silu(gu[:, :Fd]) * gu[:, Fd:]).to(torch.bfloat16).float()
            hb = (a @ w_d[l].float().t()).to(torch.bfloat16).float()
            bacts.append(hb)
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev_tf32

    def rel(a, b):
        return float((a.float() - b).norm() / b.norm())

    # ---- per-layer local check: each linear's Y, dX and dW against FP32
    # products of THAT linear's own inputs in the quantized stack (its BF16
    # input activation and incoming gradient), so that the comparison does not
    # depend on the errors the layers below or above carried in.  The bound
    # comes from the quantization noise of the operands themselves: with
    # relative noise r_a, r_b (||q(a) - a|| / ||a||, from fp4_quant_noise) a
    # product's relative error is about sqrt(r_a^2 + r_b^2); twice that is
    # allowed.  A wrong or missing gradient has a relative error near 1.
    def nsr(x, q):
        F.fp4_quant_noise(x, q, sums, ws)
        sx, sn = sums.tolist()
        return (sn / sx) ** 0.5 if sx > 0 else 0.0

    local = []
    prev_tf32 = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        for l in range(L):
            for key, sv, xin, w, y, dyin, dx, dw in (
                    ("gate_up", sv_gu[l], hin[2 * l], w_gu[l], gus[l], dys[(l, "gu")], dxs[l],
                     dwg[l]),
                    ("down", sv_d[l], hin[2 * l + 1], w_d[l], acts[l], dys[(l, "d")], das[l],
                     dwd[l])):
                xf, wf, gf = xin.float(), w.float(), dyin.float()
                r_x, r_w, r_g = nsr(xin, sv.xq), nsr(w, sv.wq), nsr(dyin, sv.dyq)
                r_xt = nsr(xin.t().contiguous(), sv.xq_t)
                r_wt = nsr(w.t().contiguous(), sv.wq_t)
                r_gt = nsr(dyin.t().contiguous(), sv.dyq_t)
                e = {"y": rel(y, xf @ wf.t()), "dx": rel(dx, gf @ wf), "dw": rel(dw, gf.t() @ xf)}
                b = {"y": (r_x ** 2 + r_w ** 2) ** 0.5, "dx": (r_g ** 2 + r_wt ** 2) ** 0.5,
                     "dw": (r_gt ** 2 + r_xt ** 2) ** 0.5}
                local.append({"layer": l + 1, "linear": key,
                              **{f"{k}_local": round(v, 5) for k, v in e.items()},
                              **{f"{k}_noise": round(v, 5) for k, v in b.items()}})
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev_tf32

    per_layer = [{"layer": l + 1, "act": round(rel(acts[l], racts[l]), 5),
                  "act_bf16_only": round(rel(bacts[l], racts[l]), 5),
                  "dx": round(rel(dxs[l], rdx[l]), 5),
                  "dw_gate_up": round(rel(dwg[l], rdwg[l]), 5),
                  "dw_down": round(rel(dwd[l], rdwd[l]), 5),
                  "grad_snr_dy_down": round(snr[(l, "down")], 3),
                  "grad_snr_dy_gate_up": round(snr[(l, "gate_up")], 3)} for l in range(L)]

    # ---- oracle spot check: sampled rows of the first and last layers'
    # quantized X (RTN) and dY (SR), codes and logical scales bit-exact
    import oracle as O
    rng = np.random.default_rng(seed + 7)
    mism = 0
    checked = 0
    for l in sorted(chk):
        for sv, xin, dyin in ((sv_gu[l], hin[2 * l], dys[(l, "gu")]), (sv_d[l], hin[2 * l + 1], dys[(l, "d")])):
            for q, src, rnd, stream in ((sv.xq, xin, "rtn", 0), (sv.dyq, dyin, "sr", 1)):
                if chained and q is sv.dyq and sv is sv_d[l] and l < L - 1:
                    continue      # encoded from the FP32 product in the epilogue, not from dyin
                rows_ = np.sort(rng.choice(M, check_rows, replace=False))
                amax = float(q.amax.item())
                C_ = src.shape[1]
                codes = q.codes.view(M, C_ // 2)
                scales = q.scales.view(M, C_ // 16)
                for r in rows_:
                    xr = src[int(r):int(r) + 1].float().cpu().numpy()
                    ref = O.nvfp4_quantize_1d(xr, round_mode=rnd, sr_seed=seed, sr_stream=stream,
                                              amax_in=amax, row_offset=int(r))
                    mism += int((codes[int(r)].cpu().numpy() != ref["codes"][0]).sum())
                    mism += int((scales[int(r)].cpu().numpy() != ref["scales"][0]).sum())
                    checked += 1
    return {"case": "swiglu", "layers": L, "hidden": H, "ffn": Fd, "tokens": M,
            "ms_quantized_fwd_bwd": round(ms, 3),
            "tflops_gemm_equiv": round(L * 6 * M * (2 * Fd * H + H * Fd) / (ms * 1e-3) / 1e12, 1),
            "rel_err_vs_fp32": per_layer, "local": local, "chained": chain,
            "oracle_rows_checked": checked,
            "oracle_mismatches": mism}


def run_formats(device, seed=0, rows_checked=128, M=M_TOKENS):
    """Config 4: MXFP4 against NVFP4 on the same seeded Llama-7B tensors.

    Per distinct layer shape and operand (X, W, dY), the relative
    quantization noise ||deq(q(x)) - x|| / ||x|| of the row-wise operand,
    rounded to nearest without rotation in both formats (NVFP4 weights in
    16x16 tiles, as its layer stores them; the layer's stochastically rounded
    NVFP4 dY is listed beside as dY_sr), from fp4_quant_noise; and the relative
    Frobenius error of the layer's three products, each format in its own
    layer configuration (NVFP4 without Hadamard, MXFP4 with the 32-point
    transform on every operand), on `rows_checked` sampled output rows
    against the unquantized float64 product of the BF16 inputs.  The "FP4"
    page (Components, NVFP4) says NVFP4 has the lower quantization error."""
    import fp4_fully_quantized_b200 as F
    import fqt_synth as S
    F.load()
    ws = F.Workspace(device=device)
    sums = torch.zeros(2, dtype=torch.float64, device=device)
    rng = np.random.default_rng(seed + 11)
    out = {"case": "formats", "tokens": M, "rows_checked": rows_checked, "shapes": []}
    for name, N, K in [("qkvo", 4096, 4096), ("gate_up", 11008, 4096), ("down", 4096, 11008)]:
        d = S.llama_linear(N, K, M=M, seed=seed)
        X, W, dY = d["X"].to(device), d["W"].to(device), d["dY"].to(device)
        row = {"layer": name, "N": N, "K": K, "noise": {}, "gemm_err": {}}
        for fmt_name, fmt in (("nvfp4", F.NVFP4), ("mxfp4", F.MXFP4)):
            nz = {}
            ops = [("X", X, F.BLOCK_1D, F.RTN), ("W", W, F.BLOCK_2D, F.RTN),
                   ("dY", dY, F.BLOCK_1D, F.RTN)]
            if fmt == F.NVFP4:
                ops.append(("dY_sr", dY, F.BLOCK_1D, F.SR))
            for opn, t, blk, rnd in ops:
                if fmt == F.MXFP4:
                    blk = F.BLOCK_1D
                q = F.QTensor.empty(t.shape[0], t.shape[1], fmt, blk, device=device, logical_scales=False)
                F.fp4_quantize(t, q, fmt=fmt, block=blk, round=rnd, sr_seed=seed, sr_stream=1, ws=ws)
                F.fp4_quant_noise(t, q, sums, ws)
                sx, sn = sums.tolist()
                nz[opn] = round((sn / sx) ** 0.5, 5)
                del q
            row["noise"][fmt_name] = nz
            cfg = F.linear_cfg(fmt, out_dtype=F.OUT_F32, seed=seed)
            sv = F.Saved.empty(M, N, K, cfg, device=device, logical_scales=False)
            y = torch.empty((M, N), dtype=torch.float32, device=device)
            dx = torch.empty((M, K), dtype=torch.float32, device=device)
            dw = torch.empty((N, K), dtype=torch.float32, device=device)
            F.fqt_linear_fwd(cfg, X, W, y, sv, ws)
            F.fqt_linear_bwd(cfg, dY, sv, dx, dw, ws)
            torch.cuda.synchronize()
            assert ws.status() == 0
            r = torch.from_numpy(np.sort(rng.choice(M, rows_checked, replace=False))).to(device)
            c = torch.from_numpy(np.sort(rng.choice(N, rows_checked, replace=False))).to(device)
            Xd, Wd, dYd = X.double(), W.double(), dY.double()
            refs = {"Y": (Xd[r] @ Wd.t(), y[r]), "dX": (dYd[r] @ Wd, dx[r]),
                    "dW": (dYd[:, c].t() @ Xd, dw[c])}
            row["gemm_err"][fmt_name] = {k: round(float((g.double() - ref).norm() / ref.norm()), 5)
                                         for k, (ref, g) in refs.items()}
            del sv, y, dx, dw
        out["shapes"].append(row)
        del X, W, dY
    return out


def _time(fn, steps, warmup):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps


def run_gemm_vendor(F, qa, qb, y, ws, args):
    """Comparison only, never the library's path: the vendor's block-scaled
    FP4 GEMM (cuBLASLt through torch.nn.functional.scaled_mm) on the very
    operand bytes fp4_gemm reads (E2M1 codes; E4M3 block scales and FP32
    tensor scales for NVFP4, E8M0 block scales for MXFP4; scales in the
    128-row x 4-block atom layout), BF16 out, both timed the same way; the two
    products are compared element by element."""
    import torch.nn.functional as Fn
    M, N, K = qa.rows, qb.rows, qa.cols
    fp4 = torch.float4_e2m1fn_x2
    a = qa.codes.view(M, K // 2).view(fp4)
    b = qb.codes.view(N, K // 2).view(fp4).t()
    ST, SW = Fn.ScalingType, Fn.SwizzleType
    if qa.fmt == F.MXFP4:             # E8M0 1x32 block scales, tensor scale 1
        sa = qa.scales_mma.view(torch.float8_e8m0fnu)
        sb = qb.scales_mma.view(torch.float8_e8m0fnu)
        vend = lambda: Fn.scaled_mm(a, b, sa, ST.BlockWise1x32, sb, ST.BlockWise1x32,
                                    swizzle_a=SW.SWIZZLE_32_4_4, swizzle_b=SW.SWIZZLE_32_4_4,
                                    output_dtype=torch.bfloat16)
        recipe = "MXFP4"
    else:
        sa = qa.scales_mma.view(torch.float8_e4m3fn)
        sb = qb.scales_mma.view(torch.float8_e4m3fn)
        vend = lambda: Fn.scaled_mm(a, b, [sa, qa.s_dec], [ST.BlockWise1x16, ST.TensorWise],
                                    [sb, qb.s_dec], [ST.BlockWise1x16, ST.TensorWise],
                                    swizzle_a=[SW.SWIZZLE_32_4_4, SW.NO_SWIZZLE],
                                    swizzle_b=[SW.SWIZZLE_32_4_4, SW.NO_SWIZZLE],
                                    output_dtype=torch.bfloat16)
        recipe = "NVFP4 two-level"
    ours = lambda: F.fp4_gemm(qa, qb, y, ws=ws)
    ms_v = _time(vend, args.steps, args.warmup)
    ms_o = _time(ours, args.steps, args.warmup)
    yv = vend()
    ours()
    torch.cuda.synchronize()
    assert ws.status() == 0
    d = (yv.float() - y.float()).abs()
    fl = 2.0 * M * N * K / 1e12
    return {"case": "gemm_vendor", "m": M, "n": N, "k": K, "unit": "TFLOP/s",
            "vendor": {"ms": round(ms_v, 4), "rate": round(fl / (ms_v * 1e-3), 1),
                       "kernel": "torch.nn.functional.scaled_mm (cuBLASLt), " + recipe},
            "ours": {"ms": round(ms_o, 4), "rate": round(fl / (ms_o * 1e-3), 1)},
            "ratio_ours_to_vendor": round(ms_v / ms_o, 3),
            "bf16_equal_frac": round(float((yv == y).float().mean().item()), 4),
            "max_abs_diff_over_max": float(d.max().item() / max(float(y.float().abs().max().item()), 1e-30))}


def run_case(args, device):
    """A single kernel family on one small problem (for profiler captures):
    --case gemm: NVFP4 fprop-style GEMM [m, k] x [n, k]^T, BF16 out;
    --case gemm_vendor: the same operands through the vendor's NVFP4 GEMM,
    timed beside fp4_gemm (comparison only);
    --case quant: NVFP4 row-wise RTN + transposed SR of a [m, k] tensor;
    --case quant_sr: both outputs stochastically rounded (the dY quantization);
    --case gemm_quant / gemm_then_quant: the GEMM with its result encoded to
    NVFP4 in the epilogue, against the GEMM's BF16 output quantized afterwards
    (both with a supplied output amax)."""
    import fp4_fully_quantized_b200 as F
    import fqt_synth as S
    F.load()
    M, N, K = args.m, args.n, args.k
    ws = F.Workspace(device=device)
    x = S.student_t_channels(M, K, seed=1)[0].to(device)
    qa = F.QTensor.empty(M, K, device=device, logical_scales=False)
    qat = F.QTensor.empty(K, M, device=device, logical_scales=False)
    if args.case in ("quant", "quant_sr"):
        rr, rc = (args.rounds or ("sr,sr" if args.case == "quant_sr" else "rtn,sr")).split(",")
        r, rt = (F.SR if rr == "sr" else F.RTN), (F.SR if rc == "sr" else F.RTN)
        amax_in = None
        if args.amax_supplied:        # time the fused encode alone: amax computed once, then supplied
            F.fp4_quantize(x, qa, qat, round=r, round_t=rt, sr_seed=1, sr_stream=1, sr_stream_t=3, ws=ws)
            amax_in = qa.amax.clone()
        fn = lambda: F.fp4_quantize(x, qa, qat, round=r, round_t=rt, sr_seed=1, sr_stream=1,
                                    sr_stream_t=3, amax_in=amax_in, amax_in_t=amax_in, ws=ws)
        bpe = Q_BYTES_PER_ELEM - (2 if args.amax_supplied else 0)
        units, unit = M * K * bpe / 1e9, "GB/s"
    else:
        w = S.normal((N, K), 0.02, seed=2).to(device)
        if args.case == "gemm_vendor" and args.fmt == "mxfp4":
            qa = F.QTensor.empty(M, K, F.MXFP4, device=device, logical_scales=False)
            qb = F.QTensor.empty(N, K, F.MXFP4, device=device, logical_scales=False)
            F.fp4_quantize(x, qa, fmt=F.MXFP4, ws=ws)
            F.fp4_quantize(w, qb, fmt=F.MXFP4, ws=ws)
            y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
            return run_gemm_vendor(F, qa, qb, y, ws, args)
        qb = F.QTensor.empty(N, K, F.NVFP4, F.BLOCK_2D, device=device, logical_scales=False)
        qbt = F.QTensor.empty(K, N, F.NVFP4, F.BLOCK_2D, device=device, logical_scales=False)
        F.fp4_quantize(x, qa, ws=ws)
        F.fp4_quantize(w, qb, qbt, block=F.BLOCK_2D, ws=ws)
        y = torch.empty((M, N), dtype=torch.float32 if args.out == "f32" else torch.bfloat16,
                        device=device)
        qy = F.QTensor.empty(M, N, device=device, logical_scales=False)
        y_amax = torch.ones(1, dtype=torch.float32, device=device)   # supplied (delayed) amax
        if args.case == "gemm_vendor":
            return run_gemm_vendor(F, qa, qb, y, ws, args)
        if args.case == "gemm_quant":          # result encoded to NVFP4 in the epilogue
            fn = lambda: F.fp4_gemm_quant(qa, qb, qy, y_amax, ws=ws)
        elif args.case == "gemm_then_quant":   # BF16 result, then the quantizer
            fn = lambda: (F.fp4_gemm(qa, qb, y, ws=ws), F.fp4_quantize(y, qy, amax_in=y_amax, ws=ws))
        else:
            fn = lambda: F.fp4_gemm(qa, qb, y, ws=ws)
        units, unit = 2 * M * N * K / 1e12, "TFLOP/s"
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        fn()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.steps
    assert ws.status() == 0
    return {"case": args.case, "m": M, "n": N, "k": K, "ms": round(ms, 4),
            "rate": round(units / (ms * 1e-3), 1), "unit": unit}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", choices=["gemm", "gemm_vendor", "gemm_quant", "gemm_then_quant", "quant",
                                       "quant_sr", "sweep", "swiglu", "formats"], default=None,
                    help="time one kernel family on one problem (profiling), or the "
                         "quantizer sweep over 2^n elements")
    ap.add_argument("--rounds", default=None,
                    help="--case quant: rounding of the row and transposed outputs, e.g. rtn,sr")
    ap.add_argument("--amax-supplied", action="store_true",
                    help="--case quant: supply the tensor amax (times the fused encode alone)")
    ap.add_argument("--sweep-min", type=int, default=20)
    ap.add_argument("--sweep-max", type=int, default=30)
    ap.add_argument("--out", choices=["bf16", "f32"], default="bf16",
                    help="--case gemm: output type (the weight gradient is FP32)")
    ap.add_argument("--m", type=int, default=8192)
    ap.add_argument("--n", type=int, default=4096)
    ap.add_argument("--k", type=int, default=4096)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--fmt", choices=["nvfp4", "mxfp4"], default="nvfp4")
    ap.add_argument("--wgrad-rht", action="store_true")
    ap.add_argument("--quest", action="store_true",
                    help="--fmt mxfp4: QuEST-style forward quantizer (RMS-based clipping scale)")
    ap.add_argument("--dp-allreduce", action="store_true",
                    help="data parallel: sum each layer's dW over the ranks (NCCL) inside the step")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--chained", action="store_true",
                    help="--case swiglu: also run the backward with each block's dgrad epilogue "
                         "encoding the next block's dY operand (delayed amax)")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the compact quantizer sweep (config 3 at 2^28) after the step")
    ap.add_argument("--e2e-steps", type=int, default=5,
                    help="timed steps of the host-buffer leg (the copy pipeline fills once "
                         "per timed region)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-rows", type=int, default=None,
                    help="tokens per layer in each oracle sample (default: 1024 for the "
                         "cpu_baseline leg; scaled to the step count for --impl reference)")
    ap.add_argument("--ref-cols", type=int, default=None)
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.case is not None:
        dev = torch.device("cuda", local)
        torch.cuda.set_device(dev)
        if args.case == "sweep":
            for line in run_sweep(args, dev):
                print(json.dumps(line), flush=True)
        elif args.case == "formats":
            print(json.dumps(run_formats(dev, seed=args.seed)), flush=True)
        elif args.case == "swiglu":
            print(json.dumps(run_swiglu(dev, seed=args.seed, chained=args.chained)), flush=True)
        else:
            print(json.dumps(run_case(args, dev)), flush=True)
        return

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    out, cache = run_ours(args, rank, world, device)
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.ref_rows or 1024, args.ref_cols or 2048, args.seed,
                                           cache, args.fmt, args.wgrad_rht)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
