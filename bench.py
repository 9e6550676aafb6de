#!/usr/bin/env python3
"""Benchmark of the SmoothQuant W8A8 linear hot path on B200.

One step = one pass of the whole path over one batch of synthetic inputs:
  a1 calibrate the activation ranges (LayerNorm output absmax over the
     calibration tokens)          sq_calibrate_absmax(calib, gamma, beta)
  a2 weight ranges                sq_calibrate_absmax(W)
  a3/a4 smoothing factor + fold   sq_smooth_fold(..., gamma, beta -> gamma', beta')
  a4/a5 fold + quantize W         sq_quantize_weight(W, s)
  a6 LayerNorm + per-token quant  sq_ln_quant_act(h, gamma', beta')
  a7/a8 INT8 GEMM + dequant       sq_w8a8_linear(xq, sx, wq, sw, bias)
With N > 1 GPUs every rank runs its own batch (data parallel, weak scaling);
the activation ranges are max-all-reduced over the ranks (NCCL) between a1
and a3 so every rank derives the same smoothing.

Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle on a
bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import sq_inputs  # noqa: E402

METRIC = "W8A8 linear TOPS and % of INT8 peak (large M); GB/s % HBM (decode M≤32)"
DECODE_M = 32  # the metric's decode range: up to this many tokens the step is reported in GB/s
DESCR = {
    "tiny": "tiny: K=N=256, M=16, calib 128, outliers x60 on channels 3/77",
    "attn": "OPT-6.7B attention projection: K=N=4096, M=2048 tokens, calib 512, 6 outlier channels x40-100, LN folded, alpha 0.5",
    "ffn_up": "OPT-6.7B FFN up: K=4096, N=16384, M=4096 tokens, calib 512, 4 outlier channels x50, bias, LN folded, alpha 0.5",
    "decode": "OPT-175B FFN up decode: K=12288, N=49152, M tokens, calib 512, 12 outlier channels x80, LN folded, alpha 0.5",
    "ffn_down": "OPT-175B FFN down: K=49152, N=12288, M=8192 tokens, calib 1024, 25 outlier channels x100 on X, alpha 0.5",
}
STEP = ("calibrate(LN absmax) + weight absmax + smoothing/fold + fold-and-quantize weight + "
        "LN/per-token quantize + INT8 GEMM with dequant epilogue")
LEVEL_DESCR = {
    "channel": "activations per token (dynamic), weights per output channel",
    "O1": "activations per token (dynamic), weights per tensor",
    "O2": "activations per tensor (dynamic, two passes), weights per tensor",
    "O3": "activations per tensor (static range from calibration, one clamped pass), weights per tensor",
}
I8_PER_BF16 = 2.0  # nominal dense INT8 : BF16 tensor throughput on B200 (4.5 : 2.25 POPS)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ helpers --
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# scale granularities of each level: (activations, weights); "channel" is the
# default (per-token activations, per-output-channel weights), O1-O3 the
# explainer's efficiency levels (section "inference")
LEVELS = {"channel": ("token", "channel"), "O1": ("token", "tensor"), "O2": ("tensor", "tensor"),
          "O3": ("static", "tensor")}


def stage_bytes_ops(wl, M, level="channel"):
    """Algorithmic bytes of every stage of the step (a per-tensor pass reads its
    input twice) and the GEMM's 2MNK ops."""
    K, N, C = wl.K, wl.N, wl.calib
    act, wgt = LEVELS[level]
    b = {
        "calib_reset": 3 * 4 * K,
        "calibrate_x": 2 * C * K + 4 * K,
        "calibrate_w": 2 * N * K + 4 * K,
        "smooth_fold": 4 * K * 6,
    }
    if act == "static":
        if wl.ln:
            b["static_calib"] = 2 * C * K + 4 * K
        b["static_range"] = 8 * K + 4
    b["quantize_weight"] = (2 if wgt == "tensor" else 1) * 2 * N * K + N * K + 4 * N + 4 * K
    b["ln_quant_act"] = (2 if act == "tensor" else 1) * 2 * M * K + M * K + 4 * M + 8 * K
    b["w8a8_linear"] = M * K + N * K + 4 * M + 4 * N + 2 * M * N + (2 * N if wl.bias else 0)
    return b, 2 * M * N * K


def traffic_from_profile(kernel_src: str, profile_md: str):
    """DRAM bytes per launch from a committed ncu summary, or None if the kernel
    source changed since the counters were taken."""
    if not os.path.exists(profile_md):
        return None
    sha = hashlib.sha256(open(kernel_src, "rb").read()).hexdigest()[:16]
    got = {}
    for line in open(profile_md):
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            got[k.strip()] = v.strip().strip("`")
    m = re.search(r"\b[0-9a-f]{16}\b", got.get("source_sha256_16", ""))
    if m is None or m.group(0) != sha:
        return None
    n = re.match(r"[0-9.]+", got.get("dram_bytes_per_launch", ""))
    return int(float(n.group(0))) if n else None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons of one GPU, sampled every 100 ms."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, uuid: str):
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None
        self.uuid = uuid

    def start(self):
        try:
            self.proc = subprocess.Popen(  # noqa: S603
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, TypeError, ValueError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        rows = [[c.strip() for c in r.split(",")] for r in self.out.read().strip().splitlines() if r.strip()]
        os.unlink(self.out.name)
        mine = [r for r in rows if self.uuid and r[0].lower().endswith(self.uuid.lower())]
        if not mine:  # uuid unknown: keep the first GPU's rows
            first = rows[0][0] if rows else None
            mine = [r for r in rows if r[0] == first]
        sm, mx, reasons = [], [], set()
        for r in mine:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(self.REASONS, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        load = [x for x in sm if x > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def workload_of(args):
    wl = sq_inputs.WORKLOADS[args.workload]
    if args.alpha is not None:
        wl = sq_inputs.with_(wl, alpha=float(args.alpha))
    return wl


def common_config(args, wl, M, world):
    """The workload keys, identical in the GPU arm and the reference arm."""
    return {"workload": DESCR[args.workload] + ("" if M == wl.M else f" (M={M})") +
                        ("" if args.alpha is None else f" (alpha={wl.alpha})"),
            "M": M, "N": wl.N, "K": wl.K, "calib_tokens": wl.calib, "alpha": wl.alpha,
            "level": args.level, "granularity": LEVEL_DESCR[args.level], "step": STEP,
            "parallelism": f"dp{world}"}


# ------------------------------------------------------------ GPU arm -------
class Plan:
    """Device buffers and prepared C-ABI calls of one step (argument
    marshalling done once, so the per-step host cost is a few C calls)."""

    def __init__(self, wl, M, rank, device, sq, torch, two_streams=False, level="channel"):
        self.torch, self.sq, self.wl, self.M = torch, sq, wl, M
        self.level = level
        self.two_streams = two_streams
        dev = device
        data_wl = sq_inputs.with_(wl, seed=wl.seed + 1000 * rank)  # this rank's tokens
        w = sq_inputs.weight(wl)
        calib = sq_inputs.calib_rows(data_wl)
        h = sq_inputs.run_rows(data_wl, 0, M)
        g, b, bias = sq_inputs.gamma(wl), sq_inputs.beta(wl), sq_inputs.bias(wl)
        self.host = {"w": w, "calib": calib, "h": h, "gamma": g, "beta": b, "bias": bias}
        T = lambda a, dt=None: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dev)
        self.w, self.calib, self.h = T(w), T(calib), T(h)
        self.gamma, self.beta, self.bias = T(g), T(b), T(bias)
        K, N = wl.K, wl.N
        f32 = dict(dtype=torch.float32, device=dev)
        # activation ranges, weight ranges and (level O3) the folded transform's
        # ranges, zeroed together at the start of every step
        self.amax = torch.zeros(3 * K, **f32)
        self.amax_x, self.amax_w, self.amax_hat = self.amax[:K], self.amax[K:2 * K], self.amax[2 * K:]
        self.w_range = torch.zeros(4, **f32)  # per-tensor ranges (16-byte aligned slots)
        self.a_range = torch.zeros(4, **f32)
        self.s, self.inv_s = torch.empty(K, **f32), torch.empty(K, **f32)
        self.gamma_f = torch.empty(K, **f32) if g is not None else None
        self.beta_f = torch.empty(K, **f32) if b is not None else None
        self.wq = torch.empty((N, K), dtype=torch.int8, device=dev)
        self.sw = torch.empty(N, **f32)
        self.xq = torch.empty((M, K), dtype=torch.int8, device=dev)
        self.sx = torch.empty(M, **f32)
        self.y = torch.empty((M, N), dtype=torch.float16, device=dev)
        self.ws = sq.new_workspace(M, N, K, device=dev)
        self.main = torch.cuda.current_stream()
        self.side = torch.cuda.Stream()
        self.runtime_inv_s = None if g is not None else self.inv_s
        self.ws_bytes = 0 if self.ws is None else self.ws.numel()
        self.calib_rows = calib.shape[0]
        self.bind(self.main)
        # libsq kernels per step (a per-tensor quantization is two kernels)
        self.launches_per_step = sum(self.kernels.values())

    def bind(self, main_stream, single=False):
        """(Re)build the prepared C calls for the given main stream (all of them
        on it when `single`, else the weight stages on the side stream when the
        plan uses two streams)."""
        torch, wl, M = self.torch, self.wl, self.M
        K, N = wl.K, wl.N
        L = self.sq._L
        p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
        self.cur = main_stream
        stream = ctypes.c_void_p(main_stream.cuda_stream)
        side = ctypes.c_void_p(self.side.cuda_stream) if self.two_streams and not single else stream
        eps = ctypes.c_float(1e-5)
        runtime_inv_s, ws_bytes = self.runtime_inv_s, self.ws_bytes
        act, wgt = LEVELS[self.level]
        calls = [
            ("calib_reset", L.sq_calibrate_reset, (p(self.amax), 3 * K, stream)),
            ("calibrate_x", L.sq_calibrate_absmax, (p(self.calib), self.calib_rows, K, K, p(self.gamma),
                                                    p(self.beta), eps, p(self.amax_x), stream)),
            ("calibrate_w", L.sq_calibrate_absmax, (p(self.w), N, K, K, None, None, eps, p(self.amax_w),
                                                    side)),
            ("smooth_fold", L.sq_smooth_fold, (p(self.amax_x), p(self.amax_w), K, ctypes.c_float(wl.alpha),
                                               p(self.s), p(self.inv_s), p(self.gamma), p(self.beta),
                                               p(self.gamma_f), p(self.beta_f), None, None, 0, stream)),
        ]
        if act == "static":  # level O3: the static range of the runtime transform
            if self.gamma is not None:
                calls.append(("static_calib", L.sq_calibrate_absmax,
                              (p(self.calib), self.calib_rows, K, K, p(self.gamma_f), p(self.beta_f), eps,
                               p(self.amax_hat), stream)))
                calls.append(("static_range", L.sq_tensor_range, (p(self.amax_hat), None, K, p(self.a_range),
                                                                  stream)))
            else:
                calls.append(("static_range", L.sq_tensor_range, (p(self.amax_x), p(self.inv_s), K,
                                                                  p(self.a_range), stream)))
        if wgt == "tensor":
            calls.append(("quantize_weight", L.sq_quantize_weight_tensor,
                          (p(self.w), N, K, p(self.s), p(self.wq), p(self.sw), p(self.w_range), side)))
        else:
            calls.append(("quantize_weight", L.sq_quantize_weight,
                          (p(self.w), N, K, p(self.s), p(self.wq), p(self.sw), side)))
        act_common = (p(self.h), M, K, K, p(self.gamma_f), p(self.beta_f), p(runtime_inv_s), eps)
        if act == "tensor":
            calls.append(("ln_quant_act", L.sq_ln_quant_act_tensor,
                          act_common + (p(self.xq), p(self.sx), p(self.a_range), stream)))
        elif act == "static":
            calls.append(("ln_quant_act", L.sq_ln_quant_act_static,
                          act_common + (p(self.a_range), p(self.xq), p(self.sx), stream)))
        else:
            calls.append(("ln_quant_act", L.sq_ln_quant_act, act_common + (p(self.xq), p(self.sx), stream)))
        calls.append(("w8a8_linear", L.sq_w8a8_linear, (p(self.xq), p(self.sx), p(self.wq), p(self.sw),
                                                        p(self.bias), p(self.y), M, N, K, p(self.ws),
                                                        ws_bytes, stream)))
        self.calls = calls
        self.kernels = {name: (2 if (name == "quantize_weight" and wgt == "tensor") or
                               (name == "ln_quant_act" and act == "tensor") else 1)
                        for name, _, _ in calls}

    def step(self, events=None, allreduce=None, part=None):
        """Run one step.  With two streams the independent stages overlap:
            main: calib_reset | calibrate_x | smooth_fold | ln_quant_act    | w8a8_linear
            side:             | calibrate_w |             | quantize_weight |
        with events joining them where a stage needs the other stream's output.
        With `events` (one per call + 1), the stages instead run one after the
        other on the main stream timing order (for the per-stage breakdown)."""
        torch = self.torch
        if events is not None:  # serialized, one event before each call
            for i, (name, fn, args) in enumerate(self.calls):
                events[i].record(self.main)
                if name in ("calibrate_w", "quantize_weight"):
                    self.side.wait_stream(self.main)
                if name == "smooth_fold" and allreduce is not None:
                    allreduce(self.amax_x)
                self._call(name, fn, args)
                if name in ("calibrate_w", "quantize_weight"):
                    self.main.wait_stream(self.side)
            events[-1].record(self.main)
            return
        if not self.two_streams:  # one stream: consecutive kernels overlap their launches (PDL)
            for name, fn, args in self.calls:
                if name == "smooth_fold" and allreduce is not None:
                    allreduce(self.amax_x)
                self._call(name, fn, args)
            return
        main = self.cur
        calls = self.calls
        if part == "rest":  # smooth_fold onwards (the ranges are complete and all-reduced)
            calls = calls[[c[0] for c in calls].index("smooth_fold"):]
        for name, fn, args in calls:
            if name == "smooth_fold" and part != "rest":  # needs both ranges
                if allreduce is not None:              # on main after calibrate_x: overlaps calibrate_w
                    allreduce(self.amax_x)
                main.wait_stream(self.side)
            if name == "quantize_weight":              # needs s
                self.side.wait_stream(main)
            if name == "w8a8_linear":                  # needs wq and xq
                main.wait_stream(self.side)
            self._call(name, fn, args)                 # calibrate_w / quantize_weight run on side
            if name == "calib_reset":                  # ranges zeroed (and the previous step done)
                self.side.wait_stream(main)

    def capture(self, world):
        """Capture the step into CUDA graphs: one graph for N = 1; for N > 1 two
        graphs around the NCCL all-reduce, which runs eagerly between them (with
        two streams, three: see capture_split)."""
        torch = self.torch
        if self.two_streams and world > 1:
            return self.capture_split()
        cap = torch.cuda.Stream()
        cap.wait_stream(self.main)
        names = [c[0] for c in self.calls]
        cut = names.index("smooth_fold") if world > 1 else len(names)
        segs = [names[:cut], names[cut:]] if world > 1 else [names]
        self.graphs = []
        with torch.cuda.stream(cap):
            self.bind(cap)
            for i, seg in enumerate(segs):
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr, stream=cap):
                    if self.two_streams:  # the side stream forks from and joins the capture
                        self.step()
                    else:
                        for name, fn, args in self.calls:
                            if name in seg:
                                self._call(name, fn, args)
                self.graphs.append(gr)
        self.bind(self.main)
        self.main.wait_stream(cap)

    def capture_staged(self):
        """Capture the step once more with an event-record node before every
        call and after the last (N = 1): replaying it gives each kernel's
        device time without host launch gaps; the event nodes serialize the
        kernels, so no stage overlaps its neighbour here."""
        torch = self.torch
        self.sev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(self.calls) + 1)]
        cap = torch.cuda.Stream()
        cap.wait_stream(self.main)
        with torch.cuda.stream(cap):
            self.bind(cap, single=True)
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=cap):
                for i, (name, fn, args) in enumerate(self.calls):
                    self.sev[i].record(cap)
                    self._call(name, fn, args)
                self.sev[-1].record(cap)
        self.bind(self.main)
        self.main.wait_stream(cap)
        self.staged = gr

    def capture_gemm_burst(self, reps):
        """Capture `reps` back-to-back launches of the step's W8A8 linear (same
        buffers, main-stream order, launch overlap between them) into one
        graph: its replay time / reps is the kernel's average launch duration
        with no host gap and no per-launch event."""
        torch = self.torch
        cap = torch.cuda.Stream()
        cap.wait_stream(self.main)
        with torch.cuda.stream(cap):
            self.bind(cap, single=True)
            name, fn, args = self.calls[-1]
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=cap):
                for _ in range(reps):
                    self._call(name, fn, args)
        self.bind(self.main)
        self.main.wait_stream(cap)
        self.burst, self.burst_reps = gr, reps

    def capture_burst_of(self, calls, reps):
        """One graph of `reps` rounds of the given (fn, args-builder) calls on a
        capture stream; args-builder(stream) returns the C arguments."""
        torch = self.torch
        cap = torch.cuda.Stream()
        cap.wait_stream(self.main)
        with torch.cuda.stream(cap):
            st = ctypes.c_void_p(cap.cuda_stream)
            bound = [(fn, mk(st)) for fn, mk in calls]
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=cap):
                for _ in range(reps):
                    for fn, a in bound:
                        self._call("producer", fn, a)
        self.main.wait_stream(cap)
        return gr

    def capture_split(self):
        """N > 1 with two streams: [zero the ranges, calibrate_x] and
        [smooth_fold .. w8a8_linear] (which forks the side stream for the weight
        quantization) captured for the main stream, [calibrate_w] for the side
        stream; replay_split runs the range all-reduce eagerly on the main stream
        between the first and the last while the side graph runs."""
        torch = self.torch
        calls = lambda: {c[0]: c for c in self.calls}
        cap = torch.cuda.Stream()
        cap.wait_stream(self.main)
        with torch.cuda.stream(cap):
            self.bind(cap)
            g_x = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_x, stream=cap):
                self._call(*calls()["calib_reset"])
                self._call(*calls()["calibrate_x"])
            g_rest = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_rest, stream=cap):
                self.step(part="rest")
            self.bind(cap, single=True)  # calibrate_w on the capturing stream
            g_w = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_w, stream=cap):
                self._call(*calls()["calibrate_w"])
        self.bind(self.main)
        self.main.wait_stream(cap)
        self.graphs = [g_x, g_w, g_rest]
        self.split = True

    def replay_split(self, allreduce):
        torch, main = self.torch, self.main
        self.graphs[0].replay()                # zero the ranges, calibrate_x
        self.side.wait_stream(main)
        with torch.cuda.stream(self.side):
            self.graphs[1].replay()            # calibrate_w
        allreduce(self.amax_x)                 # main stream: overlaps calibrate_w
        main.wait_stream(self.side)
        self.graphs[2].replay()                # smooth_fold .. w8a8_linear

    def replay(self, allreduce=None):
        if getattr(self, "split", False):
            return self.replay_split(allreduce)
        self.graphs[0].replay()
        if len(self.graphs) > 1:
            allreduce(self.amax_x)
            self.graphs[1].replay()

    @staticmethod
    def _call(name, fn, args):
        st = fn(*args)
        if st != 0:
            raise RuntimeError(f"{name}: status {st}")


def run_gpu(args):
    import torch
    import torch.distributed as dist

    import w8a8_int8_linear_channel_b200 as sq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device (the product path has no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)

    wl = workload_of(args)
    M = args.m if args.m else wl.M
    plan = Plan(wl, M, rank, device, sq, torch, two_streams=args.streams == 2, level=args.level)
    allreduce = None
    if world > 1:
        allreduce = lambda t: dist.all_reduce(t, op=dist.ReduceOp.MAX)
    # L2 flush between steps: write a 256 MiB buffer (> the 126 MB L2), then
    # read another one so the flush's dirty lines are written back before the
    # step starts (outside the timed events); the step then starts cold.
    flush_w = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
    flush_r = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=device)

    def flush():
        flush_w.zero_()
        flush_r.sum()

    ncalls = len(plan.calls)

    for _ in range(args.warmup):
        flush()
        plan.step(allreduce=allreduce)
    torch.cuda.synchronize()
    if sq.sq_poll_status() != 0:
        raise RuntimeError("device wait timed out during warm-up")
    use_graph = not args.no_graph
    graph_note = None
    if use_graph:
        try:
            plan.capture(world)
            for _ in range(3):
                flush()
                plan.replay(allreduce)
            torch.cuda.synchronize()
        except RuntimeError as e:  # capture refused: time the eager launches instead
            use_graph, graph_note = False, f"capture failed: {str(e)[:200]}"
            torch.cuda.synchronize()
    run_step = (lambda: plan.replay(allreduce)) if use_graph else (lambda: plan.step(None, allreduce))

    # timed region: events only at step boundaries, so consecutive kernels of a
    # step overlap their launches (programmatic dependent launch)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    try:
        uuid = str(torch.cuda.get_device_properties(local).uuid)
    except Exception:  # no uuid attribute: the sampler falls back to the first GPU
        uuid = ""
    sampler = ClockSampler(uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    for i in range(args.steps):
        flush()
        events[i][0].record()
        run_step()
        events[i][1].record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    if sq.sq_poll_status() != 0:
        raise RuntimeError("device wait timed out in the timed region")
    total = sum(ev[0].elapsed_time(ev[1]) for ev in events)
    t_local = torch.tensor([total], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t_local, op=dist.ReduceOp.MAX)
    total_ms = float(t_local.item())
    ms_per_step = total_ms / args.steps

    # the same steps with a warm L2 (no flush between them), reported beside
    # the cold-L2 value the headline uses
    n_warm = min(args.steps, 300)
    wev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    wev[0].record()
    for _ in range(n_warm):
        run_step()
    wev[1].record()
    torch.cuda.synchronize()
    t_warm = torch.tensor([wev[0].elapsed_time(wev[1])], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t_warm, op=dist.ReduceOp.MAX)
    warm_ms_per_step = float(t_warm.item()) / n_warm

    # stage breakdown: a second loop with an event around every call.  With a
    # graph (N = 1) the events are graph nodes, so each stage is its kernel's
    # device time; otherwise eager launches, and each stage also carries its
    # own launch latency.  The GEMM's time here is the roofline's launch
    # duration.
    n_stage = min(args.steps, args.stage_steps)
    per_stage = np.zeros(ncalls)
    stage_mode = "eager"
    if use_graph and world == 1:
        try:
            plan.capture_staged()
            for _ in range(3):
                flush()
                plan.staged.replay()
            torch.cuda.synchronize()
            for i in range(n_stage):
                flush()
                plan.staged.replay()
                torch.cuda.synchronize()
                for j in range(ncalls):
                    per_stage[j] += plan.sev[j].elapsed_time(plan.sev[j + 1])
            stage_mode = "graph"
        except RuntimeError:
            torch.cuda.synchronize()
            per_stage[:] = 0.0
    if stage_mode == "eager":
        sev = [[torch.cuda.Event(enable_timing=True) for _ in range(ncalls + 1)] for _ in range(n_stage)]
        for i in range(n_stage):
            flush()
            plan.step(sev[i], allreduce)
        torch.cuda.synchronize()
        for ev in sev:
            for j in range(ncalls):
                per_stage[j] += ev[j].elapsed_time(ev[j + 1])
    if sq.sq_poll_status() != 0:
        raise RuntimeError("device wait timed out in the stage loop")
    stage_us = {c[0]: 1e3 * per_stage[j] / n_stage for j, c in enumerate(plan.calls)}
    stage_cold = run_stage_cold(plan, torch, flush, args.burst_iters) if use_graph and world == 1 else None
    if sq.sq_poll_status() != 0:
        raise RuntimeError("device wait timed out in the cold stage loop")

    # the roofline's launch duration: back-to-back launches of the linear in
    # one graph (inputs as the step leaves them: L2-warm for the large-M
    # shapes, far larger than L2 for decode), L2 flushed before each burst
    gemm_us, gemm_mode = stage_us["w8a8_linear"], "stage loop (one event pair per launch)"
    # about 2 ms of launches per burst: enough to amortize the event pair on a
    # short kernel, short enough that a long kernel is still timed as a burst
    # (not under the sustained power cap of a seconds-long loop)
    reps = int(max(1, min(args.burst, round(2000.0 / max(stage_us["w8a8_linear"], 1.0)))))
    if use_graph:
        try:
            plan.capture_gemm_burst(reps)
            for _ in range(2):
                flush()
                plan.burst.replay()
            torch.cuda.synchronize()
            bev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.burst_iters)]
            for i in range(args.burst_iters):
                flush()
                bev[i][0].record()
                plan.burst.replay()
                bev[i][1].record()
            torch.cuda.synchronize()
            tb = sum(e[0].elapsed_time(e[1]) for e in bev) / args.burst_iters
            gemm_us = 1e3 * tb / reps
            gemm_mode = (f"{reps} back-to-back launches in one CUDA graph, events around the replay, "
                         f"mean of {args.burst_iters} replays")
        except RuntimeError:
            torch.cuda.synchronize()
    if sq.sq_poll_status() != 0:
        raise RuntimeError("device wait timed out in the GEMM burst")

    producer = run_producer(plan, sq, torch, flush, reps, args) if args.producer and use_graph else None
    bmm = run_bmm(sq, torch, device, flush, args) if args.bmm and use_graph else None
    # one-GPU extras: the forward alone, the decode half of the metric, reconstruction quality
    forward = decode_rec = quality = quality_sweep = None
    if world == 1 and use_graph and not args.no_extras:
        forward = run_forward(plan, sq, torch, flush, args.burst_iters)
        quality = run_quality(plan, sq, torch)
    peaks_early, _ = load_peaks()
    if world == 1 and use_graph and not args.no_extras and not args.no_decode:
        decode_rec = run_decode_sweep(sq, torch, device, flush, args.burst_iters, peaks_early)
    if world == 1 and not args.no_extras and not args.no_quality_sweep:
        quality_sweep = run_quality_sweep(sq, torch, device, sq_inputs.FFN_DOWN_ALPHAS)
    gemm_shapes = None
    if world == 1 and use_graph and not args.no_extras:
        gemm_shapes = run_gemm_shapes(sq, torch, device, flush, args)

    nbytes, ops = stage_bytes_ops(wl, M, args.level)
    step_bytes = sum(nbytes.values())
    decode = M <= DECODE_M
    if decode:
        value = world * step_bytes * args.steps / (total_ms * 1e-3) / 1e9
        value_warm = world * step_bytes / (warm_ms_per_step * 1e-3) / 1e9
        unit = "GB/s"
    else:
        value = world * ops * args.steps / (total_ms * 1e-3) / 1e12
        value_warm = world * ops / (warm_ms_per_step * 1e-3) / 1e12
        unit = "TOPS"

    peaks, peak_kind = load_peaks()
    gemm_s = gemm_us * 1e-6
    prof = os.path.join(ROOT, "profiles", f"w8a8_linear_{args.workload}{'_m%d' % M if M != wl.M else ''}.md")
    pair = M > 128  # the library's automatic choice (sq_w8a8_linear): CTA pairs above 128 tokens
    gemm_src = "k_gemm_splitk.cu" if decode else "k_gemm_pair.cu" if pair else "k_gemm_tiled.cu"
    gemm_name = ("k_gemm_splitk (swap-AB stream-K)" if decode else
                 "k_gemm_pair (tcgen05 cta_group::2 kind::i8, 256x256 tiles)" if pair else
                 "k_gemm_tiled (tcgen05 kind::i8, 128x256 tiles)")
    src = os.path.join(ROOT, "w8a8_int8_linear_channel_b200", "csrc", gemm_src)
    traffic = traffic_from_profile(src, prof)
    if decode:
        ach = nbytes["w8a8_linear"] / gemm_s / 1e9
        peak = float(peaks["hbm_gbs"])
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
                "frac": round(ach / peak, 4), "traffic": traffic,
                "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"}
    else:
        ach = ops / gemm_s / 1e12
        peak = float(peaks["bf16_tflops"]) * I8_PER_BF16
        roof = {"bound": "tensor", "achieved": round(ach, 1), "peak": round(peak, 1), "unit": "TOPS",
                "frac": round(ach / peak, 4), "traffic": traffic,
                "peak_source": f"{peak_kind} cuBLAS bf16 burst {peaks['bf16_tflops']} TFLOP/s x 2 "
                               "(nominal dense INT8:BF16 ratio 4.5:2.25)"}
    roof["kernel"] = gemm_name
    roof["per_launch_us"] = round(gemm_us, 2)
    roof["launch_timing"] = gemm_mode
    if forward is not None:  # the same kernel with its operands coming from HBM (L2 flushed first)
        cold_us = forward["linear"]["cold_us"]
        cold_ach = (nbytes["w8a8_linear"] / (cold_us * 1e-6) / 1e9) if decode else (ops / (cold_us * 1e-6) / 1e12)
        roof["per_launch_us_cold"] = cold_us
        roof["achieved_cold"] = round(cold_ach, 1)
        roof["frac_cold"] = round(cold_ach / roof["peak"], 4)

    e2e = e2e_fwd = None
    if not args.no_e2e:
        e2e = run_e2e(plan, sq, torch, world, allreduce, min(args.steps, args.e2e_steps), dist)
        e2e_fwd = run_e2e_forward(plan, sq, torch, world, min(args.steps, 10 * args.e2e_steps), dist)

    result = None
    if rank == 0:
        result = {
            "metric": METRIC, "value": round(value, 2), "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8",
            "data": "synthetic (seeded PCG64, OPT-shaped with persistent outlier channels)",
            "config": common_config(args, wl, M, world),
            "run": {"streams": args.streams, "cuda_graph": use_graph,
                    **({"cuda_graph_note": graph_note} if graph_note else {}),
                    "l2": "flushed before every step (256 MiB write, then 256 MiB read so no dirty "
                          "lines remain), outside the timed events",
                    "timing": "CUDA events at the boundaries of every step, summed over steps, max over "
                              "ranks; stage_us and the roofline's launch time from a second loop with "
                              "events around every call (" + ("event nodes in a CUDA graph of the step"
                              if stage_mode == "graph" else "eager launches") + "); stage_us_cold: each "
                              "stage alone, a graph of 10 x [L2 flush, stage] minus a graph of the flushes, "
                              "per stage"},
            "roofline": roof,
            "warm_l2": {"value": round(value_warm, 2), "unit": unit, "ms_per_step": round(warm_ms_per_step, 5),
                        "steps": n_warm, "note": "back-to-back steps with no flush between them"},
            "stage_us": {k: round(v, 2) for k, v in stage_us.items()},
            # each stage alone with its operands in HBM (flush-difference method,
            # no event pair in the figure); the bandwidth figures use these when
            # they exist, else the event-pair stage times (which read low)
            "stage_us_cold": ({k: round(v, 2) for k, v in stage_cold.items()} if stage_cold else None),
            # side kernels are HBM-bound: algorithmic bytes / stage time, and its
            # share of the measured copy bandwidth
            "stage_gbs": {k: round(nbytes[k] / (v * 1e-6) / 1e9, 1) for k, v in (stage_cold or stage_us).items()
                          if v > 0},
            "stage_hbm_frac": {k: round(nbytes[k] / (v * 1e-6) / 1e9 / float(peaks["hbm_gbs"]), 3)
                               for k, v in (stage_cold or stage_us).items()
                               if v > 0 and (k != "w8a8_linear" or decode)},
            "gpu_launches": plan.launches_per_step * args.steps,
            "launch": (("the step captured once into a CUDA graph and replayed (the C-ABI calls are "
                        "capture-safe); every libsq kernel uses programmatic dependent launch")
                       if use_graph and world == 1 else
                       ("the step captured into CUDA graphs replayed around the NCCL all-reduce of the "
                        "activation ranges, which runs eagerly" +
                        (" on the main stream while the weight-range graph runs on the side stream"
                         if plan.two_streams else "") +
                        "; every libsq kernel uses programmatic dependent launch")
                       if use_graph else "eager C-ABI calls; every libsq kernel uses programmatic "
                       "dependent launch"),
            "clocks": clocks,
            "e2e": e2e,
            "e2e_forward": e2e_fwd,
        }
        for key, rec in (("forward", forward), ("decode", decode_rec), ("quality", quality),
                         ("quality_alpha_sweep", quality_sweep), ("gemm_shapes", gemm_shapes)):
            if rec is not None:
                result[key] = rec
        if producer is not None:
            result["producer_quant"] = producer
        if bmm is not None:
            result["bmm"] = bmm
        if world == 1 and not args.no_cpu_baseline:
            result["cpu_baseline"] = oracle_baseline(wl, M, budget_s=args.cpu_budget, level=args.level)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


def run_producer(plan, sq, torch, flush, reps, args):
    """Producer-side quantization on the step's linear: the fused linear that
    emits the next linear's INT8 input at a static scale (times 1/s of the
    next layer), against the unfused pair (linear to fp16, then the static
    quantization pass), each as back-to-back launches in one graph."""
    L = sq._L
    wl, M = plan.wl, plan.M
    N, K = wl.N, wl.K
    dev = plan.y.device
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    g = torch.Generator(device="cpu").manual_seed(5)
    inv_next = (torch.rand(N, generator=g) * 1.5 + 0.5).to(dev)
    rng_next = torch.full((4,), 4.0, dtype=torch.float32, device=dev)
    q_next = torch.empty((M, N), dtype=torch.int8, device=dev)
    s_next = torch.empty(M, dtype=torch.float32, device=dev)
    y = plan.y
    fused = [(L.sq_w8a8_linear_quant, lambda st: (p(plan.xq), p(plan.sx), p(plan.wq), p(plan.sw), p(plan.bias), 0,
                                                  p(inv_next), p(rng_next), p(q_next), p(s_next), M, N, K,
                                                  p(plan.ws), plan.ws_bytes, st))]
    unfused = [(L.sq_w8a8_linear, lambda st: (p(plan.xq), p(plan.sx), p(plan.wq), p(plan.sw), p(plan.bias), p(y),
                                              M, N, K, p(plan.ws), plan.ws_bytes, st)),
               (L.sq_ln_quant_act_static, lambda st: (p(y), M, N, N, None, None, p(inv_next), ctypes.c_float(1e-5),
                                                      p(rng_next), p(q_next), p(s_next), st))]
    # the next linear's per-token dynamic scale: the GEMM with a row-maximum epilogue plus the
    # codes pass, against the linear to fp16 then the per-token quantization (sq_ln_quant_act)
    ws_dyn = sq.new_quant_dyn_workspace(M, N, K, device=dev)
    fused_dyn = [(L.sq_w8a8_linear_quant_dyn, lambda st: (p(plan.xq), p(plan.sx), p(plan.wq), p(plan.sw),
                                                          p(plan.bias), 0, p(inv_next), p(q_next), p(s_next),
                                                          M, N, K, p(ws_dyn), ws_dyn.numel(), st))]
    unfused_dyn = [unfused[0],
                   (L.sq_ln_quant_act, lambda st: (p(y), M, N, N, None, None, p(inv_next), ctypes.c_float(1e-5),
                                                   p(q_next), p(s_next), st))]
    out = {}
    for name, calls in (("fused", fused), ("unfused", unfused), ("dynamic_fused", fused_dyn),
                        ("dynamic_unfused", unfused_dyn)):
        gr = plan.capture_burst_of(calls, reps)
        flush()
        gr.replay()
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.burst_iters)]
        for e in ev:
            flush()
            e[0].record()
            gr.replay()
            e[1].record()
        torch.cuda.synchronize()
        out[name + "_us"] = round(1e3 * sum(a.elapsed_time(b) for a, b in ev) / len(ev) / reps, 2)
    if sq.sq_poll_status() != 0:
        raise RuntimeError("device wait timed out in the producer-quantization loop")
    # algorithmic bytes: the linear's operands and scales, then its output
    base = M * K + N * K + 4 * M + 4 * N + (2 * N if plan.bias is not None else 0)
    out["fused_bytes"] = base + M * N + 4 * N + 4 * M
    out["unfused_bytes"] = base + 2 * M * N + (2 * M * N + M * N + 4 * M + 4 * N)
    out["ops"] = 2 * M * N * K
    out["what"] = ("linear + the next linear's static (level O3) input quantization with its 1/s: fused into "
                   "the GEMM epilogue (sq_w8a8_linear_quant) vs sq_w8a8_linear then sq_ln_quant_act_static; "
                   "and at the next linear's per-token dynamic scale: sq_w8a8_linear_quant_dyn (GEMM with a "
                   "row-maximum epilogue writing fp16, then a codes pass) vs sq_w8a8_linear then "
                   f"sq_ln_quant_act; {reps} back-to-back launches per graph, L2 flushed before each replay")
    return out


def run_bmm(sq, torch, device, flush, args):
    """INT8 BMM on the OPT-6.7B attention shapes (32 heads, 2048 tokens, head
    dim 128): Q K^T and P V (V stored transposed), per-head scales, random
    codes; back-to-back launches in one graph, L2 flushed before each replay.
    Both are HBM-bound (fp16 scores out, or the [2048 x 2048] probabilities
    in): the roofline is the algorithmic bytes against the measured copy
    bandwidth, with the tensor-core time beside it."""
    L = sq._L
    peaks, kind = load_peaks()
    out = {}
    g = torch.Generator(device="cpu").manual_seed(9)
    for name, (B, M, N, K) in (("qk", (32, 2048, 2048, 128)), ("pv", (32, 2048, 128, 2048))):
        a = torch.randint(-127, 128, (B, M, K), dtype=torch.int8, generator=g).to(device)
        b = torch.randint(-127, 128, (B, N, K), dtype=torch.int8, generator=g).to(device)
        sa = (torch.rand(B, 1, generator=g) * 1e-2).expand(B, M).contiguous().to(device)
        sb = (torch.rand(B, 1, generator=g) * 1e-2).expand(B, N).contiguous().to(device)
        y = torch.empty((B, M, N), dtype=torch.float16, device=device)
        p = lambda t: ctypes.c_void_p(t.data_ptr())
        reps = 10
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cap):
            st = ctypes.c_void_p(cap.cuda_stream)
            for _ in range(2):
                Plan._call("bmm", L.sq_w8a8_bmm, (p(a), p(sa), p(b), p(sb), p(y), B, M, N, K, st))
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=cap):
                for _ in range(reps):
                    Plan._call("bmm", L.sq_w8a8_bmm, (p(a), p(sa), p(b), p(sb), p(y), B, M, N, K, st))
        torch.cuda.current_stream().wait_stream(cap)
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.burst_iters)]
        for e in ev:
            flush()
            e[0].record()
            gr.replay()
            e[1].record()
        torch.cuda.synchronize()
        us = 1e3 * sum(x.elapsed_time(z) for x, z in ev) / len(ev) / reps
        nbytes = B * (M * K + N * K + 4 * M + 4 * N + 2 * M * N)
        ops = 2 * B * M * N * K
        gbs = nbytes / (us * 1e-6) / 1e9
        out[name] = {"shape": f"{B} x [{M} x {K}] x [{N} x {K}]^T", "us": round(us, 2),
                     "tops": round(ops / (us * 1e-6) / 1e12, 1), "gbs": round(gbs, 1), "bound": "hbm",
                     "frac": round(gbs / float(peaks["hbm_gbs"]), 4),
                     "tensor_time_us_at_peak": round(ops / (float(peaks["bf16_tflops"]) * I8_PER_BF16 * 1e12) * 1e6, 2)}
        del a, b, y
    if sq.sq_poll_status() != 0:
        raise RuntimeError("device wait timed out in the BMM loop")
    return out


def run_gemm_shapes(sq, torch, device, flush, args):
    """The INT8 linear alone on the other large-M configurations (FFN-up of
    OPT-6.7B and FFN-down of OPT-175B): random codes of the workload's shape,
    per-token / per-channel scales and a bias; back-to-back launches in one
    graph with the L2 flushed before each replay (the operands of FFN-down,
    1 GB, do not fit in L2 anyway).  Tensor-bound: 2MNK against the measured
    bf16 burst x the nominal INT8:BF16 ratio."""
    L = sq._L
    peaks, _ = load_peaks()
    peak = float(peaks["bf16_tflops"]) * I8_PER_BF16
    out = {}
    g = torch.Generator(device="cpu").manual_seed(11)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    for name, reps in (("ffn_up", 10), ("ffn_down", 3)):
        wl = sq_inputs.WORKLOADS[name]
        M, N, K = wl.M, wl.N, wl.K
        xq = torch.randint(-127, 128, (M, K), dtype=torch.int8, device=device)
        wq = torch.randint(-127, 128, (N, K), dtype=torch.int8, device=device)
        sx = (torch.rand(M, generator=g) * 1e-3).to(device)
        sw = (torch.rand(N, generator=g) * 1e-3).to(device)
        bias = (torch.randn(N, generator=g) * 0.1).half().to(device)
        y = torch.empty((M, N), dtype=torch.float16, device=device)
        ws_n = int(sq.sq_w8a8_workspace_bytes(M, N, K))
        ws = torch.zeros(max(ws_n, 16), dtype=torch.uint8, device=device)
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cap):
            st = ctypes.c_void_p(cap.cuda_stream)
            cargs = (p(xq), p(sx), p(wq), p(sw), p(bias), p(y), M, N, K, p(ws), ws_n, st)
            for _ in range(2):
                Plan._call("linear", L.sq_w8a8_linear, cargs)
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=cap):
                for _ in range(reps):
                    Plan._call("linear", L.sq_w8a8_linear, cargs)
        torch.cuda.current_stream().wait_stream(cap)
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(max(3, args.burst_iters // 4))]
        for e in ev:
            flush()
            e[0].record()
            gr.replay()
            e[1].record()
        torch.cuda.synchronize()
        us = 1e3 * sum(x.elapsed_time(z) for x, z in ev) / len(ev) / reps
        tops = 2.0 * M * N * K / (us * 1e-6) / 1e12
        out[name] = {"shape": f"M={M} N={N} K={K}", "us": round(us, 2), "tops": round(tops, 1),
                     "frac": round(tops / peak, 4), "bound": "tensor", "launches_per_replay": reps}
        del xq, wq, y, ws, gr
        torch.cuda.empty_cache()
    if sq.sq_poll_status() != 0:
        raise RuntimeError("device wait timed out in the GEMM-shape loop")
    out["peak_tops"] = round(peak, 1)
    out["timing"] = "back-to-back launches in one CUDA graph, L2 flushed before each replay"
    return out


def graph_of(torch, calls, reps, pre=None):
    """One CUDA graph of `reps` rounds of the given (fn, args-builder(stream)) C calls,
    captured on a side stream (consecutive launches overlap through PDL); `pre` (torch work,
    e.g. an L2 flush) is captured before every round."""
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        st = ctypes.c_void_p(cap.cuda_stream)
        bound = [(fn, mk(st)) for fn, mk in calls]
        for fn, a in bound:  # once eagerly (lazy set-up outside the capture)
            Plan._call("call", fn, a)
        if pre is not None:
            pre()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=cap):
            for _ in range(reps):
                if pre is not None:
                    pre()
                for fn, a in bound:
                    Plan._call("call", fn, a)
    torch.cuda.current_stream().wait_stream(cap)
    torch.cuda.synchronize()
    return gr


def time_graph(torch, gr, iters, flush, reps=1):
    """Mean device time (us) of one round of a graph of `reps` rounds: events around each
    replay on the current stream, the L2 flushed before each replay (outside the events)."""
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(iters)]
    flush()
    gr.replay()
    for e in ev:
        flush()
        e[0].record()
        gr.replay()
        e[1].record()
    torch.cuda.synchronize()
    return 1e3 * sum(a.elapsed_time(b) for a, b in ev) / iters / reps


COLD_REPS = 10


def cold_warm(torch, calls, flush, iters, warm_reps, flush_graph=None):
    """(cold, warm) microseconds per round of `calls`.  Cold: a graph of COLD_REPS x [L2 flush,
    round] minus a graph of COLD_REPS x [L2 flush] (so neither the flush nor an event pair around
    a single short launch enters the figure), divided by COLD_REPS; every round starts with its
    operands in HBM.  Warm: `warm_reps` back-to-back rounds per replay (operands stay in L2 when
    they fit)."""
    with_flush = graph_of(torch, calls, COLD_REPS, pre=flush)
    if flush_graph is None:
        flush_graph = graph_of(torch, [], COLD_REPS, pre=flush)
    nrep = max(3, iters // 4)
    cold = (time_graph(torch, with_flush, nrep, flush, COLD_REPS)
            - time_graph(torch, flush_graph, nrep, flush, COLD_REPS))
    warm = time_graph(torch, graph_of(torch, calls, warm_reps), nrep, flush, warm_reps)
    return cold, warm


def run_stage_cold(plan, torch, flush, iters):
    """Each stage of the step alone, cold: a graph of COLD_REPS x [L2 flush, stage] minus a
    graph of the flushes, per stage (the stages are idempotent on the step's own buffers:
    ranges max-merged into themselves, the same factors, codes and output rewritten)."""
    flush_graph = graph_of(torch, [], COLD_REPS, pre=flush)
    out = {}
    for name, fn, args in plan.calls:
        call = (fn, lambda st, a=args: a[:-1] + (st,))
        out[name] = cold_warm(torch, [call], flush, iters, 2, flush_graph)[0]
    return out


def run_forward(plan, sq, torch, flush, iters):
    """The per-forward part of the step (a6 + a7 + a8: LayerNorm / per-token quantization, the
    INT8 GEMM and its epilogue) with the weight already quantized, as a model runs it; and
    the linear (a7 + a8) alone.  Cold: L2 flushed before every forward; warm: back to back."""
    calls = {name: (fn, args) for name, fn, args in plan.calls}
    rebind = lambda name: (calls[name][0], lambda st, a=calls[name][1]: a[:-1] + (st,))
    wl, M = plan.wl, plan.M
    nbytes, ops = stage_bytes_ops(wl, M, plan.level)
    fwd_bytes = nbytes["ln_quant_act"] + nbytes["w8a8_linear"]
    out = {}
    for key, names in (("forward", ("ln_quant_act", "w8a8_linear")), ("linear", ("w8a8_linear",)),
                       ("ln_quant_act", ("ln_quant_act",))):
        cold, warm = cold_warm(torch, [rebind(n) for n in names], flush, iters, 20)
        rec = {"cold_us": round(cold, 2), "warm_us": round(warm, 2)}
        b = fwd_bytes if key == "forward" else nbytes[names[0]]
        rec["gbs_cold"] = round(b / (cold * 1e-6) / 1e9, 1)
        if key != "ln_quant_act":
            rec["tops_cold"] = round(ops / (cold * 1e-6) / 1e12, 1)
            rec["tops_warm"] = round(ops / (warm * 1e-6) / 1e12, 1)
        else:
            rec["gbs_warm"] = round(b / (warm * 1e-6) / 1e9, 1)
        out[key] = rec
    out["what"] = ("forward = sq_ln_quant_act + sq_w8a8_linear with the weight already quantized; cold: a "
                   f"graph of {COLD_REPS} x [256 MiB L2 flush, forward] minus a graph of the flushes alone, per "
                   "forward; warm: 20 back-to-back forwards per replay")
    if sq.sq_poll_status() != 0:
        raise RuntimeError("device wait timed out in the forward loop")
    return out


def run_decode_sweep(sq, torch, device, flush, iters, peaks):
    """The metric's decode half: the OPT-175B FFN-up linear (K = 12288, N = 49152) at
    M in {1, 4, 8, 16, 32}: per-launch time of the stream-K kernel (cold: one launch after an
    L2 flush; warm: back-to-back launches; the 604 MB weight never fits the 126 MB L2), its
    algorithmic GB/s and the fraction of the measured copy bandwidth; and the forward
    (per-token quantization + linear)."""
    wl = sq_inputs.WORKLOADS["decode"]
    Mmax = max(sq_inputs.DECODE_M)
    plan = Plan(wl, Mmax, 0, device, sq, torch)
    plan.step()
    torch.cuda.synchronize()
    L = sq._L
    K, N = wl.K, wl.N
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    hbm = float(peaks["hbm_gbs"])
    uuid = ""
    try:
        uuid = str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    if sampler:
        sampler.start()
    rows = []
    for M in sq_inputs.DECODE_M:
        y = plan.y[:M]
        lin = (L.sq_w8a8_linear, lambda st, M=M, y=y: (p(plan.xq), p(plan.sx), p(plan.wq), p(plan.sw), None,
                                                      p(y), M, N, K, p(plan.ws), plan.ws_bytes, st))
        act = (L.sq_ln_quant_act, lambda st, M=M: (p(plan.h), M, K, K, p(plan.gamma_f), p(plan.beta_f), None,
                                                  ctypes.c_float(1e-5), p(plan.xq), p(plan.sx), st))
        cold, warm = cold_warm(torch, [lin], flush, iters, 10)
        fcold, fwarm = cold_warm(torch, [act, lin], flush, iters, 10)
        b = M * K + N * K + 4 * M + 4 * N + 2 * M * N
        fb = b + 3 * M * K + 4 * M + 8 * K
        rows.append({"M": M, "linear_cold_us": round(cold, 2), "linear_warm_us": round(warm, 2),
                     "gbs_cold": round(b / (cold * 1e-6) / 1e9, 1), "gbs_warm": round(b / (warm * 1e-6) / 1e9, 1),
                     "hbm_frac_cold": round(b / (cold * 1e-6) / 1e9 / hbm, 4),
                     "hbm_frac_warm": round(b / (warm * 1e-6) / 1e9 / hbm, 4),
                     "forward_cold_us": round(fcold, 2), "forward_warm_us": round(fwarm, 2),
                     "forward_gbs_cold": round(fb / (fcold * 1e-6) / 1e9, 1),
                     "algorithmic_bytes": b})
    clocks = sampler.stop() if sampler else None
    if sq.sq_poll_status() != 0:
        raise RuntimeError("device wait timed out in the decode sweep")
    del plan
    torch.cuda.empty_cache()
    return {"workload": DESCR["decode"], "kernel": "k_gemm_splitk (swap-AB stream-K, tcgen05 kind::i8)",
            "peak_gbs": hbm, "peak_source": "measured copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
            "bytes": "M*K + N*K + 4M + 4N + 2MN per linear launch; the forward adds 3MK + 4M + 8K",
            "timing": f"cold: a graph of {COLD_REPS} x [256 MiB L2 flush, launch] minus a graph of the flushes "
                      "alone, per launch; warm: 10 back-to-back launches per replay",
            "sweep": rows, "clocks": clocks}


# ------------------------------------------------------------ quality -------
def layernorm_fp64(torch, h, gamma, beta, eps):
    """The LayerNorm the linear's input comes from, in fp64 (biased variance)."""
    x = h.double()
    mu = x.mean(1, keepdim=True)
    var = ((x - mu) ** 2).mean(1, keepdim=True)
    x = (x - mu) / torch.sqrt(var + eps)
    if gamma is not None:
        x = x * gamma.double()
    if beta is not None:
        x = x + beta.double()
    return x


def product_fp64(torch, X64, w, bias):
    """Y = X W^T + b in fp64 (W converted in blocks of rows to bound the memory)."""
    N = w.shape[0]
    Y = torch.empty((X64.shape[0], N), dtype=torch.float64, device=X64.device)
    step = 4096
    for n0 in range(0, N, step):
        Y[:, n0:n0 + step] = X64 @ w[n0:n0 + step].double().t()
    if bias is not None:
        Y += bias.double()
    return Y


def unsmoothed_w8a8(sq, torch, h_s, w, gamma, beta, bias, per_tensor):
    """W8A8 without smoothing through the library's own entry points: per token and per output
    channel (sq_ln_quant_act + sq_quantize_weight), or naive, one scale for all of X and one for
    all of W (level O2 for X, sq_quantize_weight_tensor)."""
    m, K = h_s.shape
    N = w.shape[0]
    dev = h_s.device
    xq = torch.empty((m, K), dtype=torch.int8, device=dev)
    sx = torch.empty(m, dtype=torch.float32, device=dev)
    wq = torch.empty((N, K), dtype=torch.int8, device=dev)
    sw = torch.empty(N, dtype=torch.float32, device=dev)
    if per_tensor:
        rx = torch.zeros(4, dtype=torch.float32, device=dev)
        rw = torch.zeros(4, dtype=torch.float32, device=dev)
        sq.sq_ln_quant_act_tensor(h_s, xq, sx, rx[:1], gamma, beta)
        sq.sq_quantize_weight_tensor(w, wq, sw, rw[:1])
    else:
        sq.sq_ln_quant_act(h_s, xq, sx, gamma, beta)
        sq.sq_quantize_weight(w, wq, sw)
    y = torch.empty((m, N), dtype=torch.float16, device=dev)
    sq.sq_w8a8_linear(xq, sx, wq, sw, y, bias, workspace=sq.new_workspace(m, N, K, device=dev))
    return y


def rel_err(torch, y, Y64):
    return float(torch.linalg.norm(y.double() - Y64) / torch.linalg.norm(Y64))


def quality_of(sq, torch, y_sq, h_s, w, gamma, beta, bias, eps=1e-5):
    """Relative Frobenius error against the unquantized fp64 X W^T (+ b) of the SmoothQuant
    output y_sq and of the two unsmoothed W8A8 baselines, on the same sampled token rows."""
    X64 = layernorm_fp64(torch, h_s, gamma, beta, float(np.float32(eps))) if gamma is not None else h_s.double()
    Y64 = product_fp64(torch, X64, w, bias)
    out = {"e_sq": rel_err(torch, y_sq, Y64),
           "e_naive_per_tensor": rel_err(torch, unsmoothed_w8a8(sq, torch, h_s, w, gamma, beta, bias, True), Y64),
           "e_per_token_per_channel": rel_err(torch, unsmoothed_w8a8(sq, torch, h_s, w, gamma, beta, bias, False),
                                              Y64)}
    return {k: round(v, 6) for k, v in out.items()}


def sample_rows(M, m):
    return np.unique(np.linspace(0, M - 1, min(m, M)).astype(np.int64))


def run_quality(plan, sq, torch, m=128):
    """Quality of the step's own output on the step's workload (sampled token rows x all N)."""
    idx = sample_rows(plan.M, m)
    it = torch.from_numpy(idx).to(plan.h.device)
    q = quality_of(sq, torch, plan.y.index_select(0, it), plan.h.index_select(0, it).contiguous(), plan.w,
                   plan.gamma, plan.beta, plan.bias)
    q.update({"rows": f"{idx.size} of {plan.M} tokens (evenly spaced) x all {plan.wl.N} outputs",
              "alpha": plan.wl.alpha, "reference": "fp64 X W^T (+ b), X the fp64 LayerNorm of h where the "
              "workload has one", "metric": "||y - Y64||_F / ||Y64||_F",
              "naive_per_tensor": "no smoothing; one scale for all of X (dynamic) and one for all of W",
              "per_token_per_channel": "no smoothing; one scale per token and per output channel"})
    return q


def run_quality_sweep(sq, torch, device, alphas, m=64, name="ffn_down"):
    """The alpha sweep on an outlier workload: for each alpha a SmoothQuantLinear built from the
    full weight and calibration set, run on sampled token rows; the unsmoothed baselines once."""
    wl = sq_inputs.WORKLOADS[name]
    T = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(device)
    w, calib = T(sq_inputs.weight(wl)), T(sq_inputs.calib_rows(wl))
    h_s = T(sq_inputs.run_rows(wl, 0, m))
    g, b, bias = T(sq_inputs.gamma(wl)), T(sq_inputs.beta(wl)), T(sq_inputs.bias(wl))
    X64 = layernorm_fp64(torch, h_s, g, b, float(np.float32(1e-5))) if g is not None else h_s.double()
    Y64 = product_fp64(torch, X64, w, bias)
    base = {"e_naive_per_tensor": round(rel_err(torch, unsmoothed_w8a8(sq, torch, h_s, w, g, b, bias, True), Y64), 6),
            "e_per_token_per_channel": round(rel_err(torch, unsmoothed_w8a8(sq, torch, h_s, w, g, b, bias, False),
                                                     Y64), 6)}
    sweep = []
    for a in alphas:
        layer = sq.SmoothQuantLinear.from_float(w, calib, float(a), g, b, bias)
        sweep.append({"alpha": a, "e_sq": round(rel_err(torch, layer(h_s), Y64), 6)})
        del layer
    torch.cuda.synchronize()
    if sq.sq_poll_status() != 0:
        raise RuntimeError("device wait timed out in the quality sweep")
    del w, calib
    torch.cuda.empty_cache()
    return {"workload": DESCR[name], "rows": f"the first {m} of {wl.M} tokens x all {wl.N} outputs", **base,
            "sweep": sweep}


def run_e2e_forward(plan, sq, torch, world, steps, dist):
    """The forward through the public API with the layer resident: every step copies that
    step's tokens h from pinned host memory, runs SmoothQuantLinear.forward (LayerNorm /
    per-token quantization + INT8 GEMM) and copies y back to pinned host memory, all inside
    the timed events; consecutive steps alternate between two streams."""
    dev = plan.w.device
    layer = sq.SmoothQuantLinear.from_float(plan.w, plan.calib, plan.wl.alpha, plan.gamma, plan.beta, plan.bias,
                                            level=plan.level)
    h_host = torch.from_numpy(np.ascontiguousarray(plan.host["h"])).pin_memory()
    y_host = [torch.empty(tuple(plan.y.shape), dtype=torch.float16).pin_memory() for _ in range(2)]
    streams = [torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)]
    h_dev = [torch.empty_like(h_host, device=dev) for _ in range(2)]
    y_dev = [torch.empty(tuple(plan.y.shape), dtype=torch.float16, device=dev) for _ in range(2)]

    def one(i):
        j = i % 2
        with torch.cuda.stream(streams[j]):
            h_dev[j].copy_(h_host, non_blocking=True)
            layer(h_dev[j], y_dev[j])
            y_host[j].copy_(y_dev[j], non_blocking=True)

    for i in range(4):
        one(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    main = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    for st in streams:
        st.wait_stream(main)
    for i in range(steps):
        one(i)
    for st in streams:
        main.wait_stream(st)
    e1.record(main)
    e1.synchronize()
    t = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item())
    M, N, K = plan.M, plan.wl.N, plan.wl.K
    ops = 2 * M * N * K
    fb = M * K * 2 + M * N * 2
    if M <= DECODE_M:
        v, u = world * (M * K * 3 + N * K + 2 * M * N) * steps / (ms * 1e-3) / 1e9, "GB/s"
    else:
        v, u = world * ops * steps / (ms * 1e-3) / 1e12, "TOPS"
    return {"value": round(v, 3), "unit": u, "h2d_bytes_per_step": int(M * K * 2),
            "d2h_bytes_per_step": int(M * N * 2), "steps": steps, "ms_per_step": round(ms / steps, 4),
            "api": "SmoothQuantLinear.forward with the quantized layer resident on the device; h in and y out "
                   "over pinned host memory inside the timed region; consecutive steps on two streams",
            "pcie_bytes_per_step": fb}


def run_e2e(plan, sq, torch, world, allreduce, steps, dist):
    """The same step through the public Python API (SmoothQuantLinear) with the
    inputs in pinned host memory: H2D copies, the whole path, D2H of y, all
    inside the timed events.  Steps are independent batches, so consecutive
    steps alternate between two streams (each with its own pinned output):
    the H2D copy of one step overlaps the compute and the D2H copy of the
    previous one, as a serving loop would run them."""
    dev = plan.w.device
    hp = {k: (None if v is None else torch.from_numpy(np.ascontiguousarray(v)).pin_memory())
          for k, v in plan.host.items()}
    y_host = [torch.empty(tuple(plan.y.shape), dtype=torch.float16).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in hp.values() if v is not None)
    d2h = y_host[0].numel() * 2
    pg = dist.group.WORLD if world > 1 else None
    streams = [torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)]

    def one(i):
        with torch.cuda.stream(streams[i % 2]):
            d = {k: (None if v is None else v.to(dev, non_blocking=True)) for k, v in hp.items()}
            layer = sq.SmoothQuantLinear.from_float(d["w"], d["calib"], plan.wl.alpha, d["gamma"], d["beta"],
                                                    d["bias"], process_group=pg, level=plan.level)
            y = layer(d["h"])
            y_host[i % 2].copy_(y, non_blocking=True)

    for i in range(4):
        one(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    main = torch.cuda.current_stream(dev)
    e0.record(main)
    for st in streams:
        st.wait_stream(main)
    for i in range(steps):
        one(i)
    for st in streams:
        main.wait_stream(st)
    e1.record(main)
    e1.synchronize()
    t = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item())
    M, N, K = plan.M, plan.wl.N, plan.wl.K
    nbytes, ops = stage_bytes_ops(plan.wl, M, plan.level)
    if M <= DECODE_M:
        v, u = world * sum(nbytes.values()) * steps / (ms * 1e-3) / 1e9, "GB/s"
    else:
        v, u = world * ops * steps / (ms * 1e-3) / 1e12, "TOPS"
    return {"value": round(v, 3), "unit": u, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "steps": steps, "ms_per_step": round(ms / steps, 4),
            "api": "SmoothQuantLinear.from_float + forward, pinned host buffers, consecutive steps on two "
                   "streams (copies of one step overlap the previous step)"}


# ------------------------------------------------------ oracle (CPU) arm -----
def oracle_sample_inputs(wl, M, c_s, n_s, m_s):
    bias = sq_inputs.bias(wl)
    return {"calib": sq_inputs.calib_rows(wl, 0, c_s), "w": sq_inputs.weight(wl, 0, n_s),
            "h": sq_inputs.run_rows(wl, 0, m_s), "g": sq_inputs.gamma(wl), "b": sq_inputs.beta(wl),
            "bias": None if bias is None else bias[:n_s]}


def oracle_stage_times(wl, inp, level="channel"):
    """Time each oracle stage (as it stands) on one sample; seconds per stage."""
    import oracle
    act, wgt = LEVELS[level]
    g, b = inp["g"], inp["b"]
    st = {}
    t = time.perf_counter()

    def lap(name):
        nonlocal t
        now = time.perf_counter()
        st[name] = now - t
        t = now

    ax = oracle.calibrate_absmax(inp["calib"], gamma=g, beta=b)
    lap("calibrate_x")
    aw = oracle.calibrate_absmax(inp["w"])
    lap("calibrate_w")
    s, inv_s = oracle.smooth(ax, aw, wl.alpha)
    gf, bf = oracle.fold_ln(g, b, inv_s) if g is not None else (None, None)
    lap("smooth_fold")
    rt_inv = None if g is not None else inv_s
    if act == "static":
        if g is not None:
            ahat = oracle.calibrate_absmax(inp["calib"], gamma=gf, beta=bf)
            lap("static_calib")
            rng_ = oracle.tensor_range(ahat)
        else:
            rng_ = oracle.tensor_range(ax, inv_s)
        lap("static_range")
    w_f = oracle.fold_weight(inp["w"], s)
    wq, sw = oracle.quantize_weight_tensor(w_f)[:2] if wgt == "tensor" else oracle.quantize_weight(w_f)
    lap("quantize_weight")
    if act == "tensor":
        xq, sx, _ = oracle.ln_quant_act_tensor(inp["h"], gf, bf, rt_inv)
    elif act == "static":
        xq, sx = oracle.ln_quant_act_static(inp["h"], rng_, gf, bf, rt_inv)
    else:
        xq, sx = oracle.ln_quant_act(inp["h"], gf, bf, rt_inv)
    lap("ln_quant_act")
    oracle.w8a8_linear(xq, sx, wq, sw, inp["bias"])
    lap("w8a8_linear")
    return st


def oracle_full_time(wl, M, st, c_s, n_s, m_s):
    """Extrapolate sampled stage times linearly to the full workload."""
    return (st["calibrate_x"] * wl.calib / c_s + st["calibrate_w"] * wl.N / n_s
            + st["smooth_fold"] + st.get("static_calib", 0.0) * wl.calib / c_s + st.get("static_range", 0.0)
            + st["quantize_weight"] * wl.N / n_s
            + st["ln_quant_act"] * M / m_s + st["w8a8_linear"] * (M * wl.N) / (m_s * n_s))


def pick_sample(wl, M, budget_s, level="channel"):
    """Sample sizes whose oracle step takes about budget_s seconds."""
    import oracle
    c_s, n_s, m_s = min(wl.calib, 16), min(wl.N, 128), min(M, 4)
    for _ in range(3):  # a small sample's time is mostly fixed costs: refine twice
        st = oracle_stage_times(wl, oracle_sample_inputs(wl, M, c_s, n_s, m_s), level)
        if oracle_full_time(wl, M, st, c_s, n_s, m_s) <= budget_s:  # the whole workload fits the budget
            return wl.calib, wl.N, M
        dt = sum(st.values())
        if dt >= 0.5 * budget_s:
            break
        # grow the token and weight samples together (the GEMM is ~ m_s * n_s)
        f = (budget_s / max(dt, 1e-6)) ** 0.5
        n_s = int(min(wl.N, max(n_s, n_s * f)))
        m_s = int(min(M, max(m_s, m_s * f)))
        c_s = int(min(wl.calib, max(c_s, c_s * f)))
    return c_s, n_s, m_s


def host_cpu_model():
    """The host CPU's model name from /proc/cpuinfo, or None where it cannot be read."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                key, sep, val = line.partition(":")
                if sep and key.strip() == "model name":
                    return val.strip()
    except OSError:
        pass
    return None


def oracle_baseline(wl, M, budget_s, level="channel"):
    import oracle
    c_s, n_s, m_s = pick_sample(wl, M, budget_s, level)
    st = oracle_stage_times(wl, oracle_sample_inputs(wl, M, c_s, n_s, m_s), level)
    full = oracle_full_time(wl, M, st, c_s, n_s, m_s)
    nbytes, ops = stage_bytes_ops(wl, M, level)
    rate = lambda t: (sum(nbytes.values()) / t / 1e9) if M <= DECODE_M else (ops / t / 1e12)
    u = "GB/s" if M <= DECODE_M else "TOPS"
    v = rate(full)
    # the same oracle on one thread, on a sample a tenth the size
    cores = oracle.num_threads()
    c1, n1, m1 = max(1, c_s // 10), max(1, n_s // 10), max(1, m_s // 10)
    oracle.set_num_threads(1)
    try:
        st1 = oracle_stage_times(wl, oracle_sample_inputs(wl, M, c1, n1, m1), level)
    finally:
        oracle.set_num_threads(cores)
    full1 = oracle_full_time(wl, M, st1, c1, n1, m1)
    return {"value": round(v, 6), "unit": u, "cores": cores, "kind": "oracle", "cpu_model": host_cpu_model(),
            "sample": (f"{c_s}/{wl.calib} calibration rows, {n_s}/{wl.N} weight rows, {m_s}/{M} tokens; " +
                       (f"the whole workload, timed directly ({sum(st.values()):.2f} s of CPU work)"
                        if (c_s, n_s, m_s) == (wl.calib, wl.N, M) else
                        f"each stage timed on its sample and scaled linearly to the full workload "
                        f"({sum(st.values()):.2f} s of CPU work; full step estimated {full:.1f} s)")),
            "single_thread": {"value": round(rate(full1), 6), "unit": u, "cores": 1,
                              "sample": f"{c1} calibration rows, {n1} weight rows, {m1} tokens, scaled linearly"}}


def run_reference(args):
    """The oracle as the reference arm: each step one bounded sample of the
    workload, sized so the whole run ends within a few minutes."""
    import oracle
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    wl = workload_of(args)
    M = args.m if args.m else wl.M
    per_step = max(0.02, min(10.0, args.ref_budget / max(1, args.steps + args.warmup)))
    c_s, n_s, m_s = pick_sample(wl, M, per_step, args.level)
    inp = oracle_sample_inputs(wl, M, c_s, n_s, m_s)
    for _ in range(args.warmup):
        oracle_stage_times(wl, inp, args.level)
    fulls = []
    work = 0.0
    for _ in range(args.steps):
        st = oracle_stage_times(wl, inp, args.level)
        work += sum(st.values())
        fulls.append(oracle_full_time(wl, M, st, c_s, n_s, m_s))
    full = sum(fulls) / len(fulls)
    nbytes, ops = stage_bytes_ops(wl, M, args.level)
    if M <= DECODE_M:
        v, u = sum(nbytes.values()) / full / 1e9, "GB/s"
    else:
        v, u = ops / full / 1e12, "TOPS"
    sample = (f"per step {c_s}/{wl.calib} calibration rows, {n_s}/{wl.N} weight rows, {m_s}/{M} tokens; "
              f"stage times scaled linearly to the full workload")
    return {"metric": METRIC, "value": round(v, 6), "unit": u, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(full * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
            "impl": "reference",
            "config": common_config(args, wl, M, world),
            "run": {"where": "CPU oracle on the host cores, rank 0 only"},
            "cpu_baseline": {"value": round(v, 6), "unit": u, "cores": oracle.num_threads(),
                             "kind": "oracle", "cpu_model": host_cpu_model(), "sample": sample},
            "e2e": {"value": round(v, 6), "unit": u, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "cpu_seconds": round(work, 2)}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["sq", "reference"], default="sq")
    ap.add_argument("--workload", choices=sorted(DESCR), default="attn")
    ap.add_argument("--m", type=int, default=0, help="token count override (decode sweep)")
    ap.add_argument("--level", choices=["channel", "O1", "O2", "O3"], default="channel",
                    help="scale granularities (default: per-token activations, per-channel weights)")
    ap.add_argument("--alpha", type=float, default=None, help="override the workload's smoothing alpha")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the forward, decode-sweep and quality records (N = 1 only anyway)")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode sweep record")
    ap.add_argument("--no-quality-sweep", action="store_true", help="skip the FFN-down alpha sweep")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--stage-steps", type=int, default=300, help="steps of the per-stage timing loop")
    ap.add_argument("--burst", type=int, default=20,
                    help="most back-to-back GEMM launches per timed burst (fewer for long kernels)")
    ap.add_argument("--burst-iters", type=int, default=20, help="timed bursts (roofline launch duration)")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the step's kernels eagerly instead of replaying a captured CUDA graph")
    ap.add_argument("--streams", type=int, choices=[1, 2], default=2,
                    help="2: run the independent stages of a step on two streams")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--bmm", action="store_true", help="also time the INT8 BMMs of attention")
    ap.add_argument("--producer", action="store_true",
                    help="also time the fused producer-side quantization of the linear's output")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle CPU work")
    ap.add_argument("--ref-budget", type=float, default=150.0, help="seconds for the reference arm")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    res = run_reference(args) if args.impl == "reference" else run_gpu(args)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
