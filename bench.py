"""Benchmark of the static FP8 W8A8 hot path on B200.

Workload (one step): the two-tower decoder-MLP pass -- 36 layers, each with
an understanding-tower gated MLP over 1024 tokens and a generation-tower gated
MLP over 4096 tokens, d=3072, I=12288, every layer and tower with its own FP8
weights and static scales.  One gated MLP = quantize X once, gate and up FP8
GEMMs, two-input SwiGLU quantized to FP8, FP8 down GEMM.  Metric: tokens/s of
the whole pass, (1024 + 4096) tokens per step per GPU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun with N>1 every rank runs an independent replica of the pass on
its own GPU (no data-path collective; weak scaling).  Rank 0 prints one JSON
line.  The timed region replays the pass (one grouped composite C-ABI call per
layer) as a CUDA graph, with CUDA events around the region only.  Afterwards
each kind of launch of the step is replayed back to back on its own, which
gives each kernel's average launch duration (for the roofline of the
dominant kernel).  The end-to-end number goes through the composite call with
host buffers: every layer's input is copied from pinned host memory and its
output copied back inside the timed region.  At N=1 the line also carries the
per-workload kernel figures ("configs": the Linear sweep, the SwiGLU sweep, the
shared-quant Q/K/V block, the tiny MLP, the per-token path, the
cross-attention projections and the SwiGLU variant) with their roofline
fractions.

`--impl reference` times the CPU oracle (the only other implementation there
is) on a bounded sample of rows of the same pass on the host cores.
"""

from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "gated-MLP tokens/s + FP8 GEMM TFLOP/s & SwiGLU-quant GB/s vs roofline"
UNIT = "tokens/s"
LAYERS = synth.C4["layers"]
D, I = synth.C4["d"], synth.C4["I"]
TOWERS = (("und", synth.C4["M_und"]), ("gen", synth.C4["M_gen"]))
TOKENS_PER_STEP = sum(m for _, m in TOWERS)
# order of the towers inside a grouped launch: the generation tower's tiles
# first, the understanding tower's fill the ragged last wave
GROUP_ORDER = (TOWERS[1], TOWERS[0])
CALIB_BATCHES = 16
CALIB_ROWS = 256


# DRAM bytes (read + write) per launch of the dominant kernel: the sum of
# dram__bytes_read.sum (166.76 MB) and dram__bytes_write.sum (55.50 MB) from
# an ncu capture of this kernel build on this shape, with L2 flushed before
# the launch.  Remove an entry when its kernel changes.
TRAFFIC = {"gate_up_swiglu@group": 222_259_968}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p["bf16_tflops_sustained"]), source="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        rows = [ln.split(",") for ln in self.out.read().splitlines() if ln.strip()]
        os.unlink(self.out.name)
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
                for name, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(name)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


class NvmlClockSampler:
    """SM clock, power and clock-event reasons read through NVML every 20 ms
    on a host thread while the timed region runs (a 200 ms nvidia-smi loop
    sees only a couple of samples in a sub-second region).  Reads only."""

    INTERVAL_S = 0.02

    def __init__(self, device_index: int):
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(device_index)
        uuid = getattr(props, "uuid", None)
        self.h = None
        if uuid is not None:
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(uuid))
            except Exception:
                self.h = None
        if self.h is None:
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        self.names = (("hw_slowdown", pynvml.nvmlClocksEventReasonHwSlowdown),
                      ("hw_thermal_slowdown", pynvml.nvmlClocksEventReasonHwThermalSlowdown),
                      ("sw_thermal_slowdown", pynvml.nvmlClocksEventReasonSwThermalSlowdown),
                      ("hw_power_brake_slowdown", pynvml.nvmlClocksEventReasonHwPowerBrakeSlowdown),
                      ("sw_power_cap", pynvml.nvmlClocksEventReasonSwPowerCap))
        self.samples = []
        self.stop_flag = threading.Event()
        self.thread = None

    def _run(self):
        nv = self.nv
        while not self.stop_flag.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((float(sm), int(rs), pw))
            except Exception:
                pass
            self.stop_flag.wait(self.INTERVAL_S)

    def start(self):
        self.samples = []
        self.stop_flag.clear()
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def stop(self):
        self.stop_flag.set()
        if self.thread is not None:
            self.thread.join(timeout=5)
        if not self.samples:
            return None
        reasons = sorted({n for _, rs, _ in self.samples for n, bit in self.names if rs & bit})
        return {"sm_mhz": statistics.median(s[0] for s in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples),
                "power_w_max": max(s[2] for s in self.samples),
                "source": f"NVML every {int(self.INTERVAL_S * 1000)} ms during the timed region"}


def clock_sampler(device_index: int):
    try:
        return NvmlClockSampler(device_index)
    except Exception:
        return ClockSampler(device_index)


# ---------------------------------------------------------------- set-up


class Layer:
    pass


def prepare(fw, device, n_layers, log):
    """Synthetic checkpoint of the two-tower pass, made on the GPU with the
    library's own load-time calls: RTN FP8 weights (s_w = max|W|/448) and
    static input scales from the moving-average observer over 16 calibration
    batches (s_in over the batches' inputs; s_down over SiLU(G)*U of the same
    batches, with G and U taken from the FP8 gate/up GEMMs)."""
    layers = []
    t0 = time.time()
    for l in range(n_layers):
        for tower, M in TOWERS:
            src = synth.c4_layer(l, tower, device=device, n_calib=CALIB_BATCHES,
                                 calib_rows=CALIB_ROWS)
            L = Layer()
            L.tower, L.M, L.index = tower, M, l
            L.x = src["x"]
            L.wg, L.s_wg = fw.fp8_rtn_quantize_weight(src["wg"])
            L.wu, L.s_wu = fw.fp8_rtn_quantize_weight(src["wu"])
            L.wd, L.s_wd = fw.fp8_rtn_quantize_weight(src["wd"])
            amax_in = torch.cat([fw.fp8_absmax_bf16(b) for b in src["calib"]])
            L.s_in = fw.fp8_observer_scale(amax_in)
            amax_h = []
            for b in src["calib"]:
                bq = fw.fp8_quant_static(b, L.s_in)
                g = fw.fp8_linear_static(bq, L.wg, L.s_in, L.s_wg)
                u = fw.fp8_linear_static(bq, L.wu, L.s_in, L.s_wu)
                amax_h.append(fw.fp8_silu_mul_absmax(g, u))
            L.s_down = fw.fp8_observer_scale(torch.cat(amax_h))
            del src
            layers.append(L)
    torch.cuda.synchronize()
    # gate and up share one quantized activation: the load-time invariant
    for L in layers:
        st = fw.fp8_check_shared_input_scale([L.s_in, L.s_in])
        if st != 0:
            raise RuntimeError(f"shared input scale check failed: {st}")
    log(f"prepared {len(layers)} layer-towers in {time.time() - t0:.1f}s")
    return layers


def make_buffers(fw, layers, device, fused, grouped=False):
    ws = {}
    bufs = {}
    if grouped:
        Ms = [M for _, M in GROUP_ORDER]
        nbytes = fw.gated_mlp_static_fp8_group_workspace(Ms, D, I)
        ws["group"] = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        for (tower, _), v in zip(GROUP_ORDER, fw.group_workspace_views(ws["group"], Ms, D, I)):
            bufs[tower] = v
        for L in layers:
            L.y = torch.empty((L.M, D), dtype=torch.bfloat16, device=device)
        return ws, bufs
    for tower, M in TOWERS:
        if fused:
            nbytes = fw.gated_mlp_static_fp8_fused_workspace(M, D, I)
            ws[tower] = torch.zeros(nbytes, dtype=torch.uint8, device=device)
            bufs[tower] = fw.fused_workspace_views(ws[tower], M, D, I)
        else:
            nbytes = fw.gated_mlp_static_fp8_workspace(M, D, I)
            ws[tower] = torch.empty(nbytes, dtype=torch.uint8, device=device)
            bufs[tower] = fw.gated_mlp_workspace_views(ws[tower], M, D, I)
    for L in layers:
        L.y = torch.empty((L.M, D), dtype=torch.bfloat16, device=device)
    return ws, bufs


# ---------------------------------------------------------- timed region


def build_value_plan(fw, layers, ws, stream_handle, fused):
    """The pass as one composite C-ABI call per MLP (the call a user makes):
    gated_mlp_static_fp8_fused (or gated_mlp_static_fp8 when unfused)."""
    lib = fw.load()
    fn = lib.gated_mlp_static_fp8_fused if fused else lib.gated_mlp_static_fp8
    plan = []
    for L in layers:
        M = L.M
        head = (L.x.data_ptr(), M, D, I, L.s_in.data_ptr(), L.wg.data_ptr(), L.s_wg.data_ptr(),
                L.wu.data_ptr(), L.s_wu.data_ptr(), L.s_down.data_ptr())
        tail = (L.wd.data_ptr(), L.s_wd.data_ptr(), ws[L.tower].data_ptr(), L.y.data_ptr(),
                stream_handle)
        args = head + ((None,) if fused else ()) + tail
        plan.append(("mlp@" + L.tower, fn, args, 0, 0))
    return plan


def layer_pairs(layers):
    """The layer-towers of the pass as (generation, understanding) pairs, one per layer."""
    by = {}
    for L in layers:
        by.setdefault(L.index, {})[L.tower] = L
    return [tuple(by[l][t] for t, _ in GROUP_ORDER) for l in sorted(by)]


def _tower_struct(fw, L, x=None, y=None):
    x = L.x if x is None else x
    y = L.y if y is None else y
    return fw.MlpTower(x.data_ptr(), L.M, L.s_in.data_ptr(), L.wg.data_ptr(), L.s_wg.data_ptr(),
                       L.wu.data_ptr(), L.s_wu.data_ptr(), L.s_down.data_ptr(), L.wd.data_ptr(),
                       L.s_wd.data_ptr(), y.data_ptr())


def build_group_value_plan(fw, layers, ws, stream_handle):
    """The pass as one grouped composite call per layer (both towers):
    gated_mlp_static_fp8_group -- three launches per layer."""
    lib = fw.load()
    w = ws["group"]
    plan, keep = [], []
    for pair in layer_pairs(layers):
        arr = (fw.MlpTower * len(pair))(*[_tower_struct(fw, L) for L in pair])
        keep.append(arr)  # the call reads the array: keep it alive with the plan
        args = (ctypes.byref(arr), len(pair), D, I, None, w.data_ptr(), w.numel(), stream_handle)
        plan.append(("mlp@group", lib.gated_mlp_static_fp8_group, args, 0, 0))
    return plan, keep


def build_group_plan(fw, layers, bufs, ws, stream_handle):
    """The grouped pass as a flat list of the three grouped C-ABI calls per
    layer, as gated_mlp_static_fp8_group issues them: quantize both towers'
    X, the fused gate/up GEMM + SwiGLU-quant of both, the down GEMM of both
    with the same split-K scratch (the tail of the group workspace), so that
    the outputs are the composite call's, bit for bit."""
    lib = fw.load()
    w = ws["group"]
    off = sum(fw.gated_mlp_static_fp8_fused_workspace(M, D, I) for _, M in GROUP_ORDER)
    splitk, splitk_bytes = w.data_ptr() + off, w.numel() - off
    plan, keep = [], []
    for pair in layer_pairs(layers):
        Msum = sum(L.M for L in pair)
        q = (fw.QuantProblem * len(pair))(*[
            fw.QuantProblem(L.x.data_ptr(), L.M * D, L.s_in.data_ptr(), bufs[L.tower]["xq"].data_ptr())
            for L in pair])
        g = (fw.GateUpProblem * len(pair))(*[
            fw.GateUpProblem(bufs[L.tower]["xq"].data_ptr(), L.wg.data_ptr(), L.wu.data_ptr(), L.M,
                             L.s_in.data_ptr(), L.s_wg.data_ptr(), L.s_wu.data_ptr(),
                             L.s_down.data_ptr(), bufs[L.tower]["h"].data_ptr()) for L in pair])
        dn = (fw.LinearProblem * len(pair))(*[
            fw.LinearProblem(bufs[L.tower]["h"].data_ptr(), L.wd.data_ptr(), L.M,
                             L.s_down.data_ptr(), L.s_wd.data_ptr(), L.y.data_ptr()) for L in pair])
        keep += [q, g, dn]
        plan.append(("quant@group", lib.fp8_quant_static_group,
                     (ctypes.byref(q), len(pair), stream_handle), 3 * Msum * D, 0))
        plan.append(("gate_up_swiglu@group", lib.fp8_gate_up_swiglu_static_group,
                     (ctypes.byref(g), len(pair), I, D, None, stream_handle),
                     Msum * D + 2 * len(pair) * I * D + Msum * I, 4 * Msum * I * D))
        plan.append(("gemm_down@group", lib.fp8_linear_static_group,
                     (ctypes.byref(dn), len(pair), D, I, splitk, splitk_bytes, stream_handle),
                     Msum * I + len(pair) * D * I + 2 * Msum * D, 2 * Msum * D * I))
    return plan, keep


def build_plan(fw, layers, bufs, stream_handle, fused, ws=None):
    """The pass as a flat list of direct C-ABI calls (kind, fn, args,
    algorithmic bytes, flops), in the order the composite gated-MLP call
    issues them.  Fused: quantize X, fused gate/up GEMM + SwiGLU-quant, down
    GEMM.  Unfused: quantize X, gate GEMM, up GEMM, SwiGLU-quant, down GEMM."""
    lib = fw.load()
    plan = []
    for L in layers:
        b = bufs[L.tower]
        M = L.M
        xq, h = b["xq"].data_ptr(), b["h"].data_ptr()
        s_in, s_down = L.s_in.data_ptr(), L.s_down.data_ptr()
        tw = "@" + L.tower
        plan.append(("quant" + tw, lib.fp8_quant_static,
                     (L.x.data_ptr(), M * D, s_in, xq, stream_handle), 3 * M * D, 0))
        if fused:
            plan.append(("gate_up_swiglu" + tw, lib.fp8_gate_up_swiglu_static,
                         (xq, L.wg.data_ptr(), L.wu.data_ptr(), M, I, D, s_in, L.s_wg.data_ptr(),
                          L.s_wu.data_ptr(), s_down, None, h, stream_handle),
                         M * D + 2 * I * D + M * I, 4 * M * I * D))
        else:
            g, u = b["g"].data_ptr(), b["u"].data_ptr()
            plan.append(("gemm_gate" + tw, lib.fp8_linear_static,
                         (xq, L.wg.data_ptr(), M, I, D, s_in, L.s_wg.data_ptr(), g, stream_handle),
                         M * D + I * D + 2 * M * I, 2 * M * I * D))
            plan.append(("gemm_up" + tw, lib.fp8_linear_static,
                         (xq, L.wu.data_ptr(), M, I, D, s_in, L.s_wu.data_ptr(), u, stream_handle),
                         M * D + I * D + 2 * M * I, 2 * M * I * D))
            plan.append(("swiglu" + tw, lib.silu_mul_2in_fp8, (g, u, M * I, s_down, h, stream_handle),
                         5 * M * I, 0))
        plan.append(("gemm_down" + tw, lib.fp8_linear_static,
                     (h, L.wd.data_ptr(), M, D, I, s_down, L.s_wd.data_ptr(), L.y.data_ptr(),
                      stream_handle),
                     M * I + D * I + 2 * M * D, 2 * M * D * I))
    return plan


def run_plan(plan, events=None):
    if events is None:
        for _, fn, args, _, _ in plan:
            if fn(*args) != 0:
                raise RuntimeError("launch failed")
        return
    for i, (_, fn, args, _, _) in enumerate(plan):
        events[i].record()
        if fn(*args) != 0:
            raise RuntimeError("launch failed")
    events[len(plan)].record()


def make_stream_runner(plan, device):
    """The pass with the two towers of each layer on two streams.  Within a
    layer the understanding-tower and generation-tower MLPs are independent,
    so they run concurrently (each stream keeps its own kernel order); at
    every layer boundary the streams join, as the next layer's inputs would
    depend on both towers."""
    main = torch.cuda.current_stream(device)
    side = torch.cuda.Stream(device)
    # group plan entries by layer: each layer is und entries then gen entries
    n_layers = sum(1 for e in plan if e[0] == plan[0][0])  # first entry of every layer
    step = len(plan) // n_layers
    groups = [plan[i:i + step] for i in range(0, len(plan), step)]
    side_handle = side.cuda_stream
    main_handle = main.cuda_stream
    # rebind the stream argument (the last one) of every call
    bound = []
    for g in groups:
        und = [(fn, args[:-1] + (side_handle,)) for k, fn, args, _, _ in g if k.endswith("@und")]
        gen = [(fn, args[:-1] + (main_handle,)) for k, fn, args, _, _ in g if k.endswith("@gen")]
        bound.append((und, gen))
    ev_main = [torch.cuda.Event() for _ in bound]
    ev_side = [torch.cuda.Event() for _ in bound]

    def run():
        side.wait_stream(main)
        for li, (und, gen) in enumerate(bound):
            for fn, args in und:
                if fn(*args) != 0:
                    raise RuntimeError("launch failed")
            for fn, args in gen:
                if fn(*args) != 0:
                    raise RuntimeError("launch failed")
            ev_side[li].record(side)
            ev_main[li].record(main)
            main.wait_event(ev_side[li])
            side.wait_event(ev_main[li])
        main.wait_stream(side)
    return run


def capture_graph(run):
    """One step captured into a CUDA graph (after one eager step outside the
    capture, which does the library's per-device set-up); returns the graph's
    replay."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    torch.cuda.synchronize()
    return g


def time_device(plan, steps, warmup, dist_ctx, sampler=None, runner=None):
    """W untimed steps, then K timed steps between a barrier + synchronize on
    both sides, with CUDA events on the launching stream around the region
    only (an event between two kernels would stop the next kernel from being
    scheduled early)."""
    run = runner if runner is not None else (lambda: run_plan(plan))
    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_ctx.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    start.record()
    for k in range(steps):
        run()
    stop.record()
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    dist_ctx.barrier()
    return start.elapsed_time(stop), clocks


def time_kinds(plan, steps):
    """Average launch duration of each kind of launch in the step.  The
    step's launches of one kind (36 of each in the grouped pass, every one on
    its own layer's buffers) are captured into a CUDA graph that issues them
    back to back on one stream, as the step does; the graph is replayed
    `steps` times, each replay timed by its own event pair, and the median
    replay time is divided by its launch count.  No event sits between two
    launches, so programmatic launch overlap is kept, as in the step.
    Returns {kind: (ms per launch, launches per step, bytes, flops per launch)}."""
    kinds = []
    for e in plan:
        if e[0] not in kinds:
            kinds.append(e[0])
    out = {}
    for kind in kinds:
        entries = [e for e in plan if e[0] == kind]

        def run_current(entries=entries):
            h = torch.cuda.current_stream().cuda_stream
            for _, fn, a, _, _ in entries:
                if fn(*(a[:-1] + (h,))) != 0:
                    raise RuntimeError("launch failed")
        run_current()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run_current()
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        times = []
        for _ in range(steps):
            a.record()
            g.replay()
            b.record()
            b.synchronize()
            times.append(a.elapsed_time(b))
        del g
        n = len(entries)
        out[kind] = (statistics.median(times) / n, n, entries[0][3], entries[0][4])
    return out


def time_e2e(fw, layers, steps, warmup, device, dist_ctx, fused):
    """The pass through the composite C-ABI call with host buffers: each
    layer's X is copied from pinned host memory on a copy stream, the gated
    MLP runs on the compute stream, Y is copied back to pinned host memory on
    a third stream; two device buffer sets per tower let copies overlap the
    previous layer's compute."""
    h_x = [L.x.cpu().pin_memory() for L in layers]
    h_y = [torch.empty((L.M, D), dtype=torch.bfloat16).pin_memory() for L in layers]
    dx = {t: [torch.empty((M, D), dtype=torch.bfloat16, device=device) for _ in range(2)]
          for t, M in TOWERS}
    dy = {t: [torch.empty((M, D), dtype=torch.bfloat16, device=device) for _ in range(2)]
          for t, M in TOWERS}
    wsize = fw.gated_mlp_static_fp8_fused_workspace if fused else fw.gated_mlp_static_fp8_workspace
    mlp = fw.gated_mlp_static_fp8_fused if fused else fw.gated_mlp_static_fp8
    ws = {t: torch.empty(wsize(M, D, I), dtype=torch.uint8, device=device) for t, M in TOWERS}
    comp = torch.cuda.Stream(device)
    h2d = torch.cuda.Stream(device)
    d2h = torch.cuda.Stream(device)
    n = len(layers)

    def one_pass():
        # a pass starts once the previous one is complete (slots are reused)
        h2d.wait_stream(comp)
        d2h.wait_stream(comp)
        ready = [torch.cuda.Event() for _ in range(n)]
        done = [torch.cuda.Event() for _ in range(n)]
        copied_out = [torch.cuda.Event() for _ in range(n)]
        for i, L in enumerate(layers):
            slot = (i // 2) % 2  # layers alternate towers; two slots per tower
            with torch.cuda.stream(h2d):
                if i >= 4:
                    h2d.wait_event(done[i - 4])  # slot's previous user finished compute
                dx[L.tower][slot].copy_(h_x[i], non_blocking=True)
                ready[i].record(h2d)
            with torch.cuda.stream(comp):
                comp.wait_event(ready[i])
                if i >= 4:
                    comp.wait_event(copied_out[i - 4])  # slot's previous output copied out
                mlp(dx[L.tower][slot], L.s_in, L.wg, L.s_wg, L.wu, L.s_wu,
                                        L.s_down, L.wd, L.s_wd, workspace=ws[L.tower],
                                        out=dy[L.tower][slot], stream=comp)
                done[i].record(comp)
            with torch.cuda.stream(d2h):
                d2h.wait_event(done[i])
                h_y[i].copy_(dy[L.tower][slot], non_blocking=True)
                copied_out[i].record(d2h)
        # the step ends when its last result is in host memory
        comp.wait_stream(d2h)
        comp.wait_stream(h2d)

    for _ in range(warmup):
        one_pass()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_ctx.barrier()
    torch.cuda.synchronize()
    comp.wait_stream(torch.cuda.current_stream())
    start.record(comp)
    for _ in range(steps):
        one_pass()
    stop.record(comp)
    torch.cuda.synchronize()
    dist_ctx.barrier()
    ms = start.elapsed_time(stop)
    h2d_bytes = sum(t.numel() * t.element_size() for t in h_x)
    d2h_bytes = sum(t.numel() * t.element_size() for t in h_y)
    # check one output against the device-path result of the same layer
    return ms, h2d_bytes, d2h_bytes, h_y


def time_e2e_group(fw, layers, steps, warmup, device, dist_ctx, slots=4, copy_streams=2):
    """time_e2e for the grouped pass, as a stream of steps: per layer, both
    towers' X are copied in from pinned host memory on a copy stream, one
    gated_mlp_static_fp8_group call runs both towers on the compute stream,
    and both Y are copied back on a third stream.  `slots` device buffer sets
    per tower rotate over the layers of consecutive steps, and each copy or
    call waits only for the earlier users of its slot, so the copies of one
    layer overlap the compute of others across step boundaries too (a later
    step's inputs stream in while the earlier step's last results stream out).
    copy_streams=2 gives each tower its own pair of copy streams.  Four slots
    and per-tower copy streams measured 24.4-24.9 ms per step against 27.0 ms
    for two slots, one copy stream per direction and a full join between
    steps (same box); the copies alone take about 24 ms.  The timed region
    ends when the last step's last result is in host memory."""
    pairs = layer_pairs(layers)
    h_x = [[L.x.cpu().pin_memory() for L in pair] for pair in pairs]
    h_y = [[torch.empty((L.M, D), dtype=torch.bfloat16).pin_memory() for L in pair]
           for pair in pairs]
    dx = {t: [torch.empty((M, D), dtype=torch.bfloat16, device=device) for _ in range(slots)]
          for t, M in TOWERS}
    dy = {t: [torch.empty((M, D), dtype=torch.bfloat16, device=device) for _ in range(slots)]
          for t, M in TOWERS}
    ws = torch.empty(fw.gated_mlp_static_fp8_group_workspace([M for _, M in GROUP_ORDER], D, I),
                     dtype=torch.uint8, device=device)
    comp = torch.cuda.Stream(device)
    h2d_s = [torch.cuda.Stream(device) for _ in range(copy_streams)]
    d2h_s = [torch.cuda.Stream(device) for _ in range(copy_streams)]
    done, copied_out = {}, {}  # per layer-pair issue index k: compute done, results copied out
    counter = [0]

    def one_pass():
        for i, pair in enumerate(pairs):
            k = counter[0]
            counter[0] += 1
            slot = k % slots
            prev = k - slots  # the previous user of this slot
            prev_done = done.pop(prev, None)
            ready = []
            for t, (L, hx) in enumerate(zip(pair, h_x[i])):
                st = h2d_s[t % copy_streams]
                with torch.cuda.stream(st):
                    if prev_done is not None:
                        st.wait_event(prev_done)  # its compute has read the slot's X
                    dx[L.tower][slot].copy_(hx, non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(st)
                    ready.append(ev)
            with torch.cuda.stream(comp):
                for ev in ready:
                    comp.wait_event(ev)
                for ev in copied_out.pop(prev, ()):
                    comp.wait_event(ev)  # its Y has left the slot
                towers = [dict(x=dx[L.tower][slot], s_in=L.s_in, wg=L.wg, s_wg=L.s_wg, wu=L.wu,
                               s_wu=L.s_wu, s_down=L.s_down, wd=L.wd, s_wd=L.s_wd) for L in pair]
                fw.gated_mlp_static_fp8_group(towers, workspace=ws,
                                              outs=[dy[L.tower][slot] for L in pair], stream=comp)
                done[k] = torch.cuda.Event()
                done[k].record(comp)
            copied_out[k] = []
            for t, (L, hy) in enumerate(zip(pair, h_y[i])):
                st = d2h_s[t % copy_streams]
                with torch.cuda.stream(st):
                    st.wait_event(done[k])
                    hy.copy_(dy[L.tower][slot], non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(st)
                    copied_out[k].append(ev)

    cur = torch.cuda.current_stream()
    streams = [comp] + h2d_s + d2h_s

    def join():
        for st in streams:
            cur.wait_stream(st)

    for _ in range(warmup):
        one_pass()
    join()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_ctx.barrier()
    torch.cuda.synchronize()
    start.record(cur)
    for st in streams:
        st.wait_stream(cur)
    for _ in range(steps):
        one_pass()
    join()
    stop.record(cur)
    torch.cuda.synchronize()
    dist_ctx.barrier()
    ms = start.elapsed_time(stop)
    h2d_bytes = sum(t.numel() * t.element_size() for row in h_x for t in row)
    d2h_bytes = sum(t.numel() * t.element_size() for row in h_y for t in row)
    return ms, h2d_bytes, d2h_bytes, [t for row in h_y for t in row], \
        [L for pair in pairs for L in pair]


# ------------------------------------------------------------- CPU oracle


class OracleSample:
    """The oracle on a bounded sample of the same pass: rows of one layer of
    each tower, on all host cores.  Rows are independent under static scales,
    so the time per row extrapolates to the whole pass.  The weights are
    quantized once up front (load time, not timed); the scale values do not
    change the oracle's cost."""

    def __init__(self, layer: int = 0):
        import oracle  # the CPU-baseline leg is the one place the benchmark runs it

        self.oracle = oracle
        self.cores = len(os.sched_getaffinity(0))
        oracle.set_num_threads(self.cores)
        self.layer = layer
        self.towers = []
        for tower, M in TOWERS:
            src = synth.c4_layer(layer, tower, device="cpu", n_calib=0)
            b = {k: src[k].view(torch.int16).numpy().view(np.uint16) for k in ("x", "wg", "wu", "wd")}
            wgq, swg = oracle.rtn_weight(b["wg"])
            wuq, swu = oracle.rtn_weight(b["wu"])
            wdq, swd = oracle.rtn_weight(b["wd"])
            s_in = oracle.scale_from_amax(oracle.absmax(b["x"]))
            self.towers.append((tower, b["x"], (s_in, wgq, swg, wuq, swu, oracle.f32(4 * s_in),
                                                wdq, swd)))

    def run(self, rows_per_tower: int):
        """Seconds per token-layer, averaged over both towers."""
        per_row = []
        for _, x, args in self.towers:
            rows = np.ascontiguousarray(x[:rows_per_tower])
            t0 = time.perf_counter()
            self.oracle.gated_mlp(rows, *args)
            per_row.append((time.perf_counter() - t0) / rows_per_tower)
        return statistics.mean(per_row)

    def tokens_per_s(self, sec_per_token_layer: float) -> float:
        return 1.0 / (sec_per_token_layer * LAYERS)

    def describe(self, rows_per_tower: int, wall: float) -> str:
        return (f"oracle gated MLP (d=3072, I=12288) on {rows_per_tower} rows of layer {self.layer} "
                f"of each tower, {wall:.1f}s wall on {self.cores} threads; rows are independent, "
                f"time per row extrapolated to the 36-layer pass")


def cpu_baseline(rows_per_tower: int = 1024, single_rows: int = 64):
    """The oracle on all host cores, and separately on one thread (a smaller
    sample: about the same wall time)."""
    o = OracleSample()
    t0 = time.perf_counter()
    spt = o.run(rows_per_tower)
    wall = time.perf_counter() - t0
    o.oracle.set_num_threads(1)
    t0 = time.perf_counter()
    spt1 = o.run(single_rows)
    wall1 = time.perf_counter() - t0
    o.oracle.set_num_threads(o.cores)
    single = {"value": o.tokens_per_s(spt1), "threads": 1,
              "sample": f"{single_rows} rows of layer {o.layer} of each tower, {wall1:.1f}s wall"}
    return o.tokens_per_s(spt), o.cores, o.describe(rows_per_tower, wall), single


# ------------------------------------------------------- single kernels


L2_FLUSH_BYTES = 256 * 1024 * 1024  # twice the 126 MB L2
ROTATE_BYTES = 256 * 1024 * 1024    # buffer sets are rotated until they span twice the L2
MAX_SETS = 64
MIN_PER_REPLAY = 20                 # launches per replay of a back-to-back graph


def _scalar(v, device):
    return torch.tensor([v], dtype=torch.float32, device=device)


def _static_linear_inputs(fw, M, N, K, cfg, seed, device):
    x = synth.student_t((M, K), 4, synth.seed(cfg, seed, 0), device)
    w = synth.normal((N, K), synth.W_STD, synth.seed(cfg, seed, 10), device)
    s_in = fw.fp8_observer_scale(fw.fp8_absmax_bf16(x))
    xq = fw.fp8_quant_static(x, s_in)
    wq, s_w = fw.fp8_rtn_quantize_weight(w)
    return xq, wq, s_in, s_w


# The SwiGLU variant timed by the "variants" workload: alpha 1.702 inside the
# sigmoid, beta 1 on up, clamp at 7 (the shape the pages' notes name).
SWIGLU_VARIANT = lambda fw: fw.swiglu(1.702, 1.0, 7.0)  # noqa: E731


def make_kernel(fw, kind, shape, device):
    """One call of a kernel kind on one shape, with synthetic inputs shaped
    like the pages' workloads.  Returns (t, call, work, nbytes): t holds every
    device buffer the call reads or writes (cloning t gives an independent
    set), call(t) issues the call on the current stream, work is its
    algorithmic flops (None for the streaming kernels), nbytes its algorithmic
    bytes (every operand read once, every output written once).  Kind
    "scaled_mm" is torch._scaled_mm (cuBLASLt FP8 with per-tensor scales, BF16
    out): the library ceiling our GEMM is compared with, not part of the path."""
    bf, f8 = torch.bfloat16, fw.FP8
    emp = lambda shp, dt: torch.empty(shp, dtype=dt, device=device)  # noqa: E731
    if kind in ("gemm", "gemm_ws", "scaled_mm"):
        M, N, K = shape
        xq, wq, s_in, s_w = _static_linear_inputs(fw, M, N, K, 1, 90 if kind != "scaled_mm" else 92,
                                                  device)
        t = dict(xq=xq, wq=wq, s_in=s_in, s_w=s_w, y=emp((M, N), bf))
        if kind == "gemm_ws":
            t["ws"] = torch.zeros(fw.load().fp8_linear_static_ws_bytes(), dtype=torch.uint8,
                                  device=device)
            call = lambda t: fw.fp8_linear_static_ws(t["xq"], t["wq"], t["s_in"], t["s_w"],  # noqa: E731
                                                     workspace=t["ws"], out=t["y"])
        elif kind == "gemm":
            call = lambda t: fw.fp8_linear_static(t["xq"], t["wq"], t["s_in"], t["s_w"],  # noqa: E731
                                                  out=t["y"])
        else:
            del t["y"]
            call = lambda t: torch._scaled_mm(t["xq"], t["wq"].t(), scale_a=t["s_in"],  # noqa: E731
                                              scale_b=t["s_w"], out_dtype=bf)
        return t, call, 2.0 * M * N * K, M * K + N * K + 2 * M * N
    if kind == "gemm_scaled":  # per-token activation and per-channel weight scales
        M, N, K = shape
        x = synth.activation_with_outliers(M, K, 9, 6, 0, device)
        xq, sx = fw.fp8_quant_per_token(x)
        wq, sw = fw.fp8_quant_per_token(synth.normal((N, K), synth.W_STD, synth.seed(6, 90, 1),
                                                     device))
        t = dict(xq=xq, wq=wq, sx=sx, sw=sw, y=emp((M, N), bf))
        call = lambda t: fw.fp8_linear_scaled(t["xq"], t["wq"], t["sx"], t["sw"], out=t["y"])  # noqa: E731
        return t, call, 2.0 * M * N * K, M * K + N * K + 2 * M * N + 4 * (M + N)
    if kind in ("dual", "dual_var"):
        M, N, K = shape
        x = synth.activation_with_outliers(M, K, 9, 1, 0, device)
        s_in = fw.fp8_observer_scale(fw.fp8_absmax_bf16(x))
        xq = fw.fp8_quant_static(x, s_in)
        wg, s_wg = fw.fp8_rtn_quantize_weight(synth.normal((N, K), synth.W_STD, synth.seed(4, 90, 1), device))
        wu, s_wu = fw.fp8_rtn_quantize_weight(synth.normal((N, K), synth.W_STD, synth.seed(4, 90, 2), device))
        t = dict(xq=xq, wg=wg, wu=wu, s_in=s_in, s_wg=s_wg, s_wu=s_wu, s_down=_scalar(0.003, device),
                 h=emp((M, N), f8))
        act = SWIGLU_VARIANT(fw) if kind == "dual_var" else None
        call = lambda t: fw.fp8_gate_up_swiglu_static(t["xq"], t["wg"], t["wu"], t["s_in"],  # noqa: E731
                                                      t["s_wg"], t["s_wu"], t["s_down"], act=act,
                                                      out=t["h"])
        return t, call, 4.0 * M * N * K, M * K + 2 * N * K + M * N
    if kind in ("mlp", "mlp_tok"):
        M, dm, Ii = shape
        x = synth.activation_with_outliers(M, dm, 0, 0, 0, device)
        ws_ = [synth.normal(shp, synth.W_STD, synth.seed(0, 90, k), device)
               for k, shp in enumerate(((Ii, dm), (Ii, dm), (dm, Ii)))]
        if kind == "mlp":
            t = dict(x=x, s_in=fw.fp8_observer_scale(fw.fp8_absmax_bf16(x)),
                     s_down=_scalar(0.003, device), y=emp((M, dm), bf),
                     ws=emp(fw.gated_mlp_static_fp8_fused_workspace(M, dm, Ii), torch.uint8))
            for name, w in zip(("g", "u", "d"), ws_):
                t["w" + name], t["s_w" + name] = fw.fp8_rtn_quantize_weight(w)
            call = lambda t: fw.gated_mlp_static_fp8_fused(  # noqa: E731
                t["x"], t["s_in"], t["wg"], t["s_wg"], t["wu"], t["s_wu"], t["s_down"], t["wd"],
                t["s_wd"], workspace=t["ws"], out=t["y"])
        else:  # per-channel weight scales, per-token activation scales computed at run time
            t = dict(x=x, y=emp((M, dm), bf),
                     ws=emp(fw.load().gated_mlp_per_token_fp8_workspace(M, dm, Ii), torch.uint8))
            for name, w in zip(("g", "u", "d"), ws_):
                t["w" + name], t["s_w" + name] = fw.fp8_quant_per_token(w)
            call = lambda t: fw.gated_mlp_per_token_fp8(  # noqa: E731
                t["x"], t["wg"], t["s_wg"], t["wu"], t["s_wu"], t["wd"], t["s_wd"],
                workspace=t["ws"], out=t["y"])
        return t, call, 6.0 * M * dm * Ii, 2 * M * dm + 3 * dm * Ii + 2 * M * dm
    if kind in ("qkv", "qkv_gemm"):
        M, dm, Nq, Nkv = shape
        x = synth.activation_with_outliers(M, dm, 3, 90, 0, device, heavy_tailed_outliers=True)
        s_in = fw.fp8_observer_scale(fw.fp8_absmax_bf16(x))
        t = dict(s_in=s_in)
        for k, (name, n) in enumerate((("q", Nq), ("k", Nkv), ("v", Nkv))):
            t["w" + name], t["s_w" + name] = fw.fp8_rtn_quantize_weight(
                synth.normal((n, dm), synth.W_STD, synth.seed(3, 90, k), device))
            t["y" + name] = emp((M, n), bf)
        proj = lambda t: [(t["wq"], t["s_wq"]), (t["wk"], t["s_wk"]), (t["wv"], t["s_wv"])]  # noqa: E731
        outs = lambda t: [t["yq"], t["yk"], t["yv"]]  # noqa: E731
        nsum = Nq + 2 * Nkv
        if kind == "qkv":
            t["x"] = x
            t["ws"] = emp(fw.qkv_shared_quant_workspace(M, dm), torch.uint8)
            call = lambda t: fw.fp8_shared_quant_linears(t["x"], t["s_in"], proj(t),  # noqa: E731
                                                         workspace=t["ws"], out=outs(t))
            return t, call, 2.0 * M * dm * nsum, 2 * M * dm + dm * nsum + 2 * M * nsum
        t["xq"] = fw.fp8_quant_static(x, s_in)
        call = lambda t: fw.fp8_linears_static(t["xq"], t["s_in"], proj(t), out=outs(t))  # noqa: E731
        return t, call, 2.0 * M * dm * nsum, M * dm + dm * nsum + 2 * M * nsum
    if kind == "xattn":  # cross-attention: Q from x, K and V from a context tensor
        Mq, Mkv, dm, Nq, Nkv = shape
        x = synth.activation_with_outliers(Mq, dm, 5, 5, 0, device)
        ctx = synth.activation_with_outliers(Mkv, dm, 5, 6, 0, device)
        t = dict(x=x, ctx=ctx, s_q=fw.fp8_observer_scale(fw.fp8_absmax_bf16(x)),
                 s_kv=fw.fp8_observer_scale(fw.fp8_absmax_bf16(ctx)),
                 ws=emp(fw.load().cross_attention_qkv_static_fp8_workspace(Mq, Mkv, dm),
                        torch.uint8),
                 yq=emp((Mq, Nq), bf), yk=emp((Mkv, Nkv), bf), yv=emp((Mkv, Nkv), bf))
        for k, (name, n) in enumerate((("q", Nq), ("k", Nkv), ("v", Nkv))):
            t["w" + name], t["s_w" + name] = fw.fp8_rtn_quantize_weight(
                synth.normal((n, dm), synth.W_STD, synth.seed(5, 90, k), device))
        call = lambda t: fw.cross_attention_qkv_static_fp8(  # noqa: E731
            t["x"], t["ctx"], t["s_q"], t["wq"], t["s_wq"], t["s_kv"], t["wk"], t["s_wk"],
            t["wv"], t["s_wv"], workspace=t["ws"], out=(t["yq"], t["yk"], t["yv"]))
        work = 2.0 * dm * (Mq * Nq + 2 * Mkv * Nkv)
        return t, call, work, 2 * (Mq + Mkv) * dm + dm * (Nq + 2 * Nkv) + 2 * (Mq * Nq + 2 * Mkv * Nkv)
    if kind in ("gemm_group", "gemm_group_ws", "dual_group", "quant_group"):
        if kind == "quant_group":
            M0, M1, K = shape
            t = {}
            for p, M in enumerate((M0, M1)):
                t[f"x{p}"] = synth.activation_with_outliers(M, K, 9, p, 0, device)
                t[f"s{p}"] = fw.fp8_observer_scale(fw.fp8_absmax_bf16(t[f"x{p}"]))
                t[f"q{p}"] = emp((M, K), f8)
            call = lambda t: fw.fp8_quant_static_group([t["x0"], t["x1"]], [t["s0"], t["s1"]],  # noqa: E731
                                                       outs=[t["q0"], t["q1"]])
            return t, call, None, 3 * (M0 + M1) * K
        M0, M1, N, K = shape
        t = {}
        for p, M in enumerate((M0, M1)):
            if kind == "dual_group":
                x = synth.activation_with_outliers(M, K, 9, 2 + p, 0, device)
                t[f"s_in{p}"] = fw.fp8_observer_scale(fw.fp8_absmax_bf16(x))
                t[f"xq{p}"] = fw.fp8_quant_static(x, t[f"s_in{p}"])
                for j, nm in enumerate(("wg", "wu")):
                    t[f"{nm}{p}"], t[f"s_{nm}{p}"] = fw.fp8_rtn_quantize_weight(
                        synth.normal((N, K), synth.W_STD, synth.seed(4, 91, 1 + j + 2 * p), device))
                t[f"s_down{p}"] = _scalar(0.003, device)
                t[f"h{p}"] = emp((M, N), f8)
            else:
                t[f"xq{p}"], t[f"wq{p}"], t[f"s_in{p}"], t[f"s_w{p}"] = _static_linear_inputs(
                    fw, M, N, K, 1, 91 + 2 * p, device)
                t[f"y{p}"] = emp((M, N), bf)
        if kind == "dual_group":
            probs = lambda t: [tuple(t[f"{k}{p}"] for k in ("xq", "wg", "wu", "s_in", "s_wg",  # noqa: E731
                                                           "s_wu", "s_down")) for p in range(2)]
            call = lambda t: fw.fp8_gate_up_swiglu_static_group(probs(t), outs=[t["h0"], t["h1"]])  # noqa: E731
            return t, call, 4.0 * (M0 + M1) * N * K, (M0 + M1) * K + 4 * N * K + (M0 + M1) * N
        t["ws"] = torch.zeros(fw.load().fp8_linear_static_ws_bytes(), dtype=torch.uint8, device=device)
        split = kind == "gemm_group_ws"
        probs = lambda t: [tuple(t[f"{k}{p}"] for k in ("xq", "wq", "s_in", "s_w")) for p in range(2)]  # noqa: E731
        call = lambda t: fw.fp8_linear_static_group(probs(t), outs=[t["y0"], t["y1"]],  # noqa: E731
                                                    split_k=split, workspace=t["ws"])
        return t, call, 2.0 * (M0 + M1) * N * K, (M0 + M1) * K + 2 * N * K + 2 * (M0 + M1) * N
    if kind in ("swiglu", "swiglu_tok", "swiglu_var"):
        M, Ii = shape
        t = dict(g=synth.normal((M, Ii), 2.0, synth.seed(2, 90, 7), device),
                 u=synth.normal((M, Ii), 1.0, synth.seed(2, 90, 8), device), h=emp((M, Ii), f8))
        if kind == "swiglu":
            t["s"] = fw.fp8_observer_scale(fw.fp8_silu_mul_absmax(t["g"], t["u"]))
            call = lambda t: fw.silu_mul_2in_fp8(t["g"], t["u"], t["s"], out=t["h"])  # noqa: E731
            return t, call, None, 5 * M * Ii
        if kind == "swiglu_var":
            t["s"] = _scalar(0.01, device)
            act = SWIGLU_VARIANT(fw)
            call = lambda t: fw.swiglu_2in_fp8(t["g"], t["u"], t["s"], act, out=t["h"])  # noqa: E731
            return t, call, None, 5 * M * Ii
        t["s"] = emp((M,), torch.float32)
        call = lambda t: fw.silu_mul_2in_fp8_per_token(t["g"], t["u"], out=t["h"], scales=t["s"])  # noqa: E731
        return t, call, None, 5 * M * Ii + 4 * M
    if kind in ("quant", "quant_tok"):
        M, K = shape
        t = dict(x=synth.activation_with_outliers(M, K, 9, 0, 0, device), q=emp((M, K), f8))
        if kind == "quant":
            t["s"] = fw.fp8_observer_scale(fw.fp8_absmax_bf16(t["x"]))
            call = lambda t: fw.fp8_quant_static(t["x"], t["s"], out=t["q"])  # noqa: E731
            return t, call, None, 3 * M * K
        t["s"] = emp((M,), torch.float32)
        call = lambda t: fw.fp8_quant_per_token(t["x"], out=t["q"], scales=t["s"])  # noqa: E731
        return t, call, None, 3 * M * K + 4 * M
    raise ValueError(kind)


def _set_bytes(t):
    return sum(v.numel() * v.element_size() for v in t.values())


def time_back_to_back(calls, steps, warmup):
    """Per-launch time of calls issued back to back, as a layer stack issues
    them: the calls (one per buffer set, repeated to at least MIN_PER_REPLAY)
    are captured once into a CUDA graph, so that host issue cannot starve the
    GPU, and the graph is replayed; each replay is timed by its own event pair
    and the median replay time is divided by its launch count.  Returns (ms
    per call, calls per replay)."""
    seq = calls * max(1, -(-MIN_PER_REPLAY // len(calls)))
    for c in calls:  # eager once: the library's per-device set-up stays out of the capture
        c()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for c in seq:
            c()
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    times = []
    for _ in range(steps):
        a.record()
        g.replay()
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b) / len(seq))
    del g
    return statistics.median(times), len(seq)


def time_isolated(call, steps, warmup, flush):
    """One launch at a time with L2 flushed before it (a 256 MB read, which
    leaves no dirty lines), timed by an event pair around the launch.  The
    figure includes the launch latency between the event and the kernel."""
    for _ in range(warmup):
        call()
    times = []
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(steps):
        flush.sum()
        a.record()
        call()
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b))
    return statistics.median(times)


def kernel_bench(fw, kind, shape, steps, warmup, device, sustain_s=0.0, isolated=True,
                 clocks=True):
    """One kernel kind on one shape.  The headline "us" is the back-to-back
    per-launch time over buffer sets rotated until they span twice the L2
    (so every launch reads its operands from DRAM, as a layer stack does);
    "us_isolated" is the same launch alone after an L2 flush.  Fractions use
    the burst peaks (these kernels are timed in short runs).  With sustain_s >
    0 the back-to-back graph also replays for that many seconds, the
    power-capped rate.  Returns a dict for one JSON line."""
    pk = peaks()
    t0, call, work, nbytes = make_kernel(fw, kind, shape, device)
    # at least two sets, so that consecutive launches never share buffers
    nsets = int(min(MAX_SETS, max(2, -(-ROTATE_BYTES // max(_set_bytes(t0), 1)))))
    sets = [t0] + [{k: v.clone() for k, v in t0.items()} for _ in range(nsets - 1)]
    calls = [(lambda t=t: call(t)) for t in sets]
    sampler = clock_sampler(device.index if device.index is not None else 0) if clocks else None
    if sampler:
        sampler.start()
    ms, per_replay = time_back_to_back(calls, steps, max(warmup // 5, 2))
    clk = sampler.stop() if sampler else None
    out = {"kernel": kind, "shape": list(shape), "us": ms * 1e3,
           "gbs": nbytes / (ms / 1e3) / 1e9, "hbm_frac": nbytes / (ms / 1e3) / 1e9 / pk["hbm"],
           "timing": f"back to back, {nsets} buffer set(s) of {_set_bytes(t0) / 1e6:.1f} MB rotated, "
                     f"median of {steps} graph replays of {per_replay} launches"}
    if clk:
        out["sm_mhz"] = clk["sm_mhz"]
        out["clock_reasons"] = clk["reasons"]
    if isolated:
        flush = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
        ms_iso = time_isolated(calls[0], steps, warmup, flush)
        out["us_isolated"] = ms_iso * 1e3
        del flush
    if work:
        out["tflops"] = work / (ms / 1e3) / 1e12
        out["fp8_peak_frac"] = out["tflops"] / (2.0 * pk["bf16"])
    if sustain_s > 0:
        seq = calls * max(1, -(-MIN_PER_REPLAY // len(calls)))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for c in seq:
                c()
        g.replay()
        torch.cuda.synchronize()
        n, t_start = 0, time.perf_counter()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        while time.perf_counter() - t_start < sustain_s:
            g.replay()
            n += len(seq)
            torch.cuda.synchronize()
        b.record()
        b.synchronize()
        sus_ms = a.elapsed_time(b) / n
        out["sustained_us"] = sus_ms * 1e3
        if work:
            out["sustained_tflops"] = work / (sus_ms / 1e3) / 1e12
        del g
    st, where = fw.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} at wait site {where}")
    del sets, calls, t0
    torch.cuda.empty_cache()
    return out


SWEEPS = {
    "c1": [("gemm", (m, n, synth.C1_K)) for m in synth.C1_M for n in synth.C1_N],
    "c2": [("swiglu", (m, i)) for m in synth.C2_M for i in synth.C2_I],
    "c3": [("qkv", (synth.C3["M"], synth.C3["d"], synth.C3["Nq"], synth.C3["Nk"])),
           ("qkv_gemm", (synth.C3["M"], synth.C3["d"], synth.C3["Nq"], synth.C3["Nk"])),
           ("quant", (synth.C3["M"], synth.C3["d"]))] +
          [("gemm", (synth.C3["M"], n, synth.C3["d"])) for n in (synth.C3["Nq"], synth.C3["Nk"])],
    "c4": [("dual", (m, synth.C4["I"], synth.C4["d"])) for m in (1024, 4096)] +
          [("gemm", (m, synth.C4["I"], synth.C4["d"])) for m in (1024, 4096)] +
          [("gemm", (m, synth.C4["d"], synth.C4["I"])) for m in (1024, 4096)] +
          [("swiglu", (m, synth.C4["I"])) for m in (1024, 4096)] +
          [("quant", (m, synth.C4["d"])) for m in (1024, 4096)],
    "c0": [("mlp", (synth.C0["M"], synth.C0["d"], synth.C0["I"]))],
    # our FP8 GEMM against cuBLASLt FP8 (torch._scaled_mm) at the same shapes
    "fp8ceil": [(k, shp) for shp in ((8192, 8192, 8192), (4096, 12288, 3072), (4096, 3072, 12288))
                for k in ("gemm", "scaled_mm")],
    # the grouped launches of the same layer (generation tower first)
    "c4g": [("dual_group", (4096, 1024, synth.C4["I"], synth.C4["d"])),
            ("gemm_group", (4096, 1024, synth.C4["d"], synth.C4["I"])),
            ("gemm_group_ws", (4096, 1024, synth.C4["d"], synth.C4["I"])),
            ("quant_group", (4096, 1024, synth.C4["d"]))],
    # per-token activation / per-channel weight scales at the generation tower's size
    "per_token": [("mlp_tok", (4096, synth.C4["d"], synth.C4["I"])),
                  ("quant_tok", (4096, synth.C4["d"])),
                  ("swiglu_tok", (4096, synth.C4["I"])),
                  ("gemm_scaled", (4096, synth.C4["I"], synth.C4["d"]))],
    # cross-attention projections: generation-tower queries over understanding-tower context
    "xattn": [("xattn", (4096, 1024, synth.C3["d"], synth.C3["Nq"], synth.C3["Nk"]))],
    # the swiglu_alpha/beta/limit variant: element-wise and in the gate/up epilogue
    "variants": [("swiglu_var", (4096, synth.C4["I"])),
                 ("dual_var", (4096, synth.C4["I"], synth.C4["d"])),
                 ("dual", (4096, synth.C4["I"], synth.C4["d"]))],
}

# the workloads whose figures go into the default run's line (key "configs")
CONFIG_REPLAYS = 50
# fp8ceil: the measured FP8 ceiling, cuBLASLt (torch._scaled_mm) beside our GEMM at the same shapes
LINE_CONFIGS = ("c0", "c1", "c2", "c3", "per_token", "xattn", "variants", "fp8ceil")


def config_figures(fw, device, steps, warmup, log):
    """The default run's per-workload kernel figures: every shape of the
    Linear sweep (c1), the SwiGLU sweep (c2), the shared-quant Q/K/V block
    (c3, whole call and its grouped GEMM alone), the tiny MLP (c0), the
    per-token path, the cross-attention projections, the SwiGLU variant
    (element-wise, and in the gate/up epilogue beside the plain one) and the
    measured FP8 ceiling (cuBLASLt's FP8 GEMM beside ours at 8192^3 and the
    two-tower shapes), each timed back to back with rotating buffers and alone
    after an L2 flush."""
    pk = peaks()
    out = {"timing": f"back to back over buffer sets spanning >= {ROTATE_BYTES >> 20} MB (twice "
                     f"the L2), median of {steps} CUDA-graph replays of >= {MIN_PER_REPLAY} "
                     f"launches; us_isolated: one launch after a 256 MB L2 flush (includes the "
                     f"launch latency); fractions of the measured burst peaks",
           "peaks": {"fp8_tflops": 2.0 * pk["bf16"], "hbm_gbs": pk["hbm"],
                     "source": f"{pk['source']}: bf16 burst x 2 for FP8; copy bandwidth"}}
    for name in LINE_CONFIGS:
        rows = []
        for kind, shape in SWEEPS[name]:
            r = kernel_bench(fw, kind, shape, steps, warmup, device)
            keep = {k: (round(v, 4) if isinstance(v, float) else v) for k, v in r.items()
                    if k not in ("timing",)}
            if kind in ("swiglu", "swiglu_tok", "swiglu_var", "quant", "quant_tok"):
                keep["hbm_nominal_frac"] = round(r["gbs"] / 8000.0, 4)
            rows.append(keep)
            log(f"{name} {kind} {shape}: {r['us']:.1f} us"
                + (f", {r['tflops']:.0f} TFLOP/s" if "tflops" in r else f", {r['gbs']:.0f} GB/s"))
        out[name] = rows
    return out


# -------------------------------------------------------------- dist glue


class DistCtx:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend="nccl"):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            if backend == "nccl":
                torch.cuda.set_device(self.local_rank)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            if self.pg.get_backend() == "nccl":
                self.pg.barrier(device_ids=[self.local_rank])
            else:
                self.pg.barrier()

    def max(self, v: float) -> float:
        if self.pg is None:
            return v
        dev = torch.device("cuda", self.local_rank) if self.pg.get_backend() == "nccl" else "cpu"
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


def aggregate_value(tokens_per_rank: int, world: int, max_seconds: float) -> float:
    """Whole-job throughput: tokens of every rank over the slowest rank's time."""
    return tokens_per_rank * world / max_seconds


# ------------------------------------------------------------------ main


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 120 for the pass, about 2 s; 50 graph replays "
                         "for --kernel/--sweep)")
    ap.add_argument("--warmup", type=int, default=None,
                    help="untimed warm-up steps (default 3 for the pass; 10 launches for "
                         "--kernel/--sweep)")
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--layers", type=int, default=LAYERS)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload kernel figures (c0-c3, per-token, cross-attention)")
    ap.add_argument("--streams", type=int, choices=(1, 2), default=2,
                    help="towers mode: 2 runs the two towers of each layer on two streams, "
                         "joined per layer")
    ap.add_argument("--eager", action="store_true",
                    help="issue the grouped pass's calls eagerly instead of replaying one step "
                         "captured as a CUDA graph")
    ap.add_argument("--unfused", action="store_true",
                    help="time the five-kernel composition (separate gate/up GEMMs and SwiGLU-quant)")
    ap.add_argument("--kernel", choices=("gemm", "gemm_ws", "dual", "swiglu", "quant", "gemm_group",
                                         "gemm_group_ws", "dual_group", "quant_group", "scaled_mm",
                                         "mlp", "qkv", "qkv_gemm", "mlp_tok", "quant_tok",
                                         "swiglu_tok", "gemm_scaled", "xattn", "swiglu_var",
                                         "dual_var"),
                    help="time one kernel on one shape instead of the pass")
    ap.add_argument("--shape", help="M,N,K for gemm; M,I,K for dual; M,I for swiglu; M,K for quant; "
                                    "M0,M1,N,K / M0,M1,I,K / M0,M1,K for the group kinds; "
                                    "M,d,I for mlp (the fused gated MLP, three launches); "
                                    "M,d,Nq,Nkv for qkv (shared quantize + grouped Q/K/V GEMM) "
                                    "and qkv_gemm (the grouped GEMM alone); M,d,I for mlp_tok; "
                                    "M,N,K for gemm_scaled; Mq,Mkv,d,Nq,Nkv for xattn")
    ap.add_argument("--mode", choices=("group", "towers"), default="group",
                    help="group: one grouped launch per step covers both towers of a layer; "
                         "towers: one launch per tower (see --streams)")
    ap.add_argument("--sweep", choices=tuple(SWEEPS), help="time every kernel shape of a workload")
    ap.add_argument("--sustain", type=float, default=0.0,
                    help="with --kernel/--sweep: also run each kernel back to back for this many "
                         "seconds and report the power-capped rate")
    args = ap.parse_args()
    single = bool(args.kernel or args.sweep)
    if args.steps is None:
        args.steps = 50 if single else 120
    if args.warmup is None:
        args.warmup = 10 if single else 3
    log = lambda m: print(m, file=sys.stderr, flush=True)  # noqa: E731

    if args.kernel or args.sweep:
        import fp8_w8a8_static_b200 as fw
        device = torch.device("cuda", 0)
        torch.cuda.set_device(device)
        fw.load()
        jobs = ([(args.kernel, tuple(int(v) for v in args.shape.split(",")))] if args.kernel
                else SWEEPS[args.sweep])
        for kind, shape in jobs:
            print(json.dumps(kernel_bench(fw, kind, shape, args.steps, max(args.warmup, 3), device,
                                          args.sustain)), flush=True)
            torch.cuda.empty_cache()
        return 0

    ctx = DistCtx()
    if args.impl == "reference":
        if ctx.rank != 0:
            return 0
        o = OracleSample()
        rows = 64
        for _ in range(args.warmup):
            o.run(2)
        step_rates = []
        t0 = time.perf_counter()
        for _ in range(args.steps):
            step_rates.append(o.tokens_per_s(o.run(rows)))
        wall = time.perf_counter() - t0
        cores, sample = o.cores, o.describe(rows, wall / max(args.steps, 1)) + " (per step)"
        # value: the pass's tokens/s implied by the sample's time per row;
        # ms_per_step: the wall time a timed step (the sample) actually took
        value = statistics.median(step_rates)
        line = {
            "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": wall / max(args.steps, 1) * 1e3,
            "extrapolated_ms_per_pass": TOKENS_PER_STEP / value * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": "two-tower MoT decoder-MLP pass, 36 layers x {und M=1024, gen M=4096}, d=3072, I=12288",
                       "global_batch": TOKENS_PER_STEP, "parallelism": "host cores",
                       "step": f"the oracle on {rows} rows of layer 0 of each tower (a bounded "
                               f"sample of the pass; rows are independent under static scales)",
                       "sample_rows_per_tower": rows, "cores": cores},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return 0

    import fp8_w8a8_static_b200 as fw

    ctx.init("nccl")
    device = torch.device("cuda", ctx.local_rank)
    torch.cuda.set_device(device)
    fw.load()
    if fw.device_check() != 0:
        raise RuntimeError("not an sm_100 device")
    pk = peaks()
    layers = prepare(fw, device, args.layers, log)
    fused = not args.unfused
    grouped = fused and args.mode == "group"
    ws, bufs = make_buffers(fw, layers, device, fused, grouped)
    stream = torch.cuda.current_stream(device)
    if grouped:
        plan, keep_plan = build_group_plan(fw, layers, bufs, ws, stream.cuda_stream)
        value_plan, keep_value = build_group_value_plan(fw, layers, ws, stream.cuda_stream)
    else:
        plan = build_plan(fw, layers, bufs, stream.cuda_stream, fused)
        value_plan = build_value_plan(fw, layers, ws, stream.cuda_stream, fused)

    launches_before = fw.launch_count()
    launches_per_step = sum(3 if fused else 5 for _ in value_plan)
    sampler = clock_sampler(device.index if device.index is not None else 0)
    runner = make_stream_runner(value_plan, device) if (args.streams == 2 and not grouped) else None
    graph = None
    if grouped and not args.eager:
        # the plan's calls name the stream they launch on: rebind them to the
        # capture stream, which torch makes current inside the capture
        def run_current():
            h = torch.cuda.current_stream().cuda_stream
            for _, fn, a, _, _ in value_plan:
                if fn(*(a[:-1] + (h,))) != 0:
                    raise RuntimeError("launch failed")
        graph = capture_graph(run_current)
        runner = graph.replay
    total_ms, clocks = time_device(value_plan, args.steps, max(args.warmup, 3), ctx, sampler,
                                   runner)
    # each kind's launches of the step replayed back to back (after the timed region)
    per_kind = time_kinds(plan, args.steps)
    launches = launches_per_step * args.steps
    counted = fw.launch_count() - launches_before
    # launches are counted when issued: eager calls and captures, not graph replays
    kinds_issued = 2 * len(plan)  # time_kinds: one eager pass and one capture of each kind
    if graph is not None:  # the eager step before the capture, and the capture
        expect = 2 * launches_per_step + kinds_issued
    else:
        expect = launches_per_step * (args.steps + max(args.warmup, 3)) + kinds_issued
    if counted != expect:
        raise RuntimeError(f"launch count {counted} != expected {expect}")
    st, where = fw.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} at wait site {where}")

    max_ms = ctx.max(total_ms)
    tokens = TOKENS_PER_STEP * args.steps * args.layers / LAYERS
    value = aggregate_value(tokens, ctx.world, max_ms / 1e3)

    # per-kernel achieved rates: each kind's launches of one step replayed back to back
    step_ms = {k: ms * n for k, (ms, n, _, _) in per_kind.items()}
    comp = {"note": "per-kernel figures: each kind's launches of one step (one per layer, on "
                    "that layer's buffers) captured as a CUDA graph and replayed back to back, "
                    f"median of {args.steps} replays; no event between launches. The kinds' sum "
                    f"is {sum(step_ms.values()):.3f} ms per step against the pass's "
                    f"{max_ms / args.steps:.3f} ms"}
    for kind, (ms, n, nbytes, flops) in per_kind.items():
        d = {"launches_per_step": n, "us_per_launch": ms * 1e3, "ms_per_step": step_ms[kind],
             "share": step_ms[kind] / sum(step_ms.values())}
        if flops:
            d["tflops"] = flops / (ms / 1e3) / 1e12
        d["gbs"] = nbytes / (ms / 1e3) / 1e9
        comp[kind] = d
    # the dominant kernel: the launch shape with the largest share of the pass
    tensor_kinds = [k for k in per_kind if per_kind[k][3]]
    dom = max(tensor_kinds, key=lambda k: step_ms[k])
    fp8_peak = 2.0 * pk["bf16_sustained"]
    ms, n, nbytes, flops = per_kind[dom]
    achieved = flops / (ms / 1e3) / 1e12
    kind, tower = dom.split("@")
    if tower == "group":
        mrows = "+".join(f"{M} ({t})" for t, M in GROUP_ORDER)
        tower_desc = "both towers in one launch"
    else:
        mrows = dict(TOWERS)[tower]
        tower_desc = f"{tower} tower"
    names = {"gemm_down": f"fp8_gemm_pair_kernel, down projection M={mrows} N={D} K={I}",
             "gemm_gate": f"fp8_gemm_pair_kernel, gate projection M={mrows} N={I} K={D}",
             "gemm_up": f"fp8_gemm_pair_kernel, up projection M={mrows} N={I} K={D}",
             "gate_up_swiglu": f"fp8_dual_swiglu_pair_kernel (gate/up GEMMs + SwiGLU-quant), "
                               f"M={mrows} I={I} K={D}"}
    roofline = {"bound": "tensor", "achieved": achieved, "peak": fp8_peak, "unit": "TFLOP/s",
                "frac": achieved / fp8_peak, "traffic": TRAFFIC.get(dom),
                "traffic_unit": "DRAM bytes per launch (ncu)",
                "kernel": f"{names[kind]}, {tower_desc}, {n} launches per step, "
                          f"{flops / 1e9:.1f} GFLOP and {nbytes / 1e6:.1f} MB algorithmic per launch",
                "launch_us": ms * 1e3,
                "peak_source": f"{pk['source']}: bf16 sustained {pk['bf16_sustained']} TFLOP/s x 2 (nominal fp8/bf16 ratio)"}
    for k in list(comp):
        if k.startswith(("swiglu", "quant")) and isinstance(comp[k], dict):
            comp[k]["hbm_frac"] = comp[k]["gbs"] / pk["hbm"]
    all_flops = sum(v[3] * v[1] for v in per_kind.values())
    all_tensor_ms = sum(step_ms[k] for k in tensor_kinds)
    comp["all_tensor_kernels_tflops"] = all_flops / (all_tensor_ms / 1e3) / 1e12

    e2e = None
    if not args.no_e2e:
        if grouped:
            ms, hb, db, h_y, order = time_e2e_group(fw, layers, max(1, args.steps // 2), 1,
                                                    device, ctx)
        else:
            ms, hb, db, h_y = time_e2e(fw, layers, max(1, args.steps // 2), 1, device, ctx, fused)
            order = layers
        ms = ctx.max(ms)
        torch.cuda.synchronize()
        same = torch.equal(h_y[-1], order[-1].y.cpu())
        e2e = {"value": aggregate_value(TOKENS_PER_STEP * max(1, args.steps // 2) * args.layers / LAYERS,
                                        ctx.world, ms / 1e3),
               "unit": UNIT, "h2d_bytes_per_step": hb, "d2h_bytes_per_step": db,
               "matches_device_path": bool(same)}

    cpu = None
    if ctx.rank == 0 and ctx.world == 1 and not args.no_cpu_baseline:
        tps, cores, sample, single = cpu_baseline()
        cpu = {"value": tps, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
               "nproc": os.cpu_count(), "single_thread": single}

    configs = None
    if ctx.world == 1 and not args.no_configs:
        del graph
        graph = None
        torch.cuda.empty_cache()
        configs = config_figures(fw, device, CONFIG_REPLAYS, 10, log)

    if ctx.rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ctx.world,
            "steps": args.steps, "warmup": max(args.warmup, 3),
            "ms_per_step": max_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp8-e4m3 MMA, fp32 accumulate, bf16 out",
            "data": "synthetic",
            "config": {"workload": "two-tower MoT decoder-MLP pass, 36 layers x {und M=1024, gen M=4096}, d=3072, I=12288",
                       "path": ("fused: quantize X -> gate/up GEMM with SwiGLU-quant epilogue -> down GEMM"
                                if fused else "unfused: quantize X -> gate GEMM -> up GEMM -> SwiGLU-quant -> down GEMM"),
                       "launch": ("grouped: one launch per step covers both towers of a layer"
                                  if grouped else f"per tower, {args.streams} stream(s)")
                                 + ("; the step replayed as one CUDA graph" if graph else ""),
                       "layers": args.layers, "global_batch": TOKENS_PER_STEP * ctx.world,
                       "parallelism": f"replicas x{ctx.world}",
                       "l2": "inputs larger than L2 (8.15 GB of FP8 weights per pass)"},
            "roofline": roofline, "components": comp, "e2e": e2e, "cpu_baseline": cpu,
            "gpu_launches": launches, "clocks": clocks, "configs": configs,
        }
        print(json.dumps(line), flush=True)
    del graph
    ctx.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
