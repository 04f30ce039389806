"""Benchmark of the W4A16 weight-only linear layer on B200.

Default workload: the hidden-5120 decode layer set at M = 1 (qkv 5120x7680,
o_proj 5120x5120, gate+up 5120x51200, down 25600x5120; W ~ N(0, 0.02) packed
to INT4 group 128, X ~ N(0, 1) BF16 with 1% salient channels x20).  One step
runs the four layers once.  The headline value is effective packed-weight
bandwidth (GB/s of INT4 code bytes, N*K/2 per layer) for the whole job.

Also measured in the same run: the prefill layer set at M = 4096 on the
hidden-8192 shapes (TFLOP/s), per-kernel rooflines, an end-to-end number
through the public API with host buffers, and the FP64 oracle timed on the
host cores as a CPU baseline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
  (N > 1: launched by torch.distributed.run; every rank runs its own replica,
  weak scaling, no collective on the data path.)
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from synth import workloads  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
METRIC = "W4A16 effective weight GB/s (% HBM peak) at M=1; TFLOP/s (% BF16 peak) at M=4096"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM bytes (read + write) per launch of the dominant kernels, from one ncu capture each
# (summaries under profiles/).  A figure holds only for the kernel source it was taken on,
# so each carries the sha256 of that source file; after any change it reads as null.
NCU_TRAFFIC = {
    # python bench.py --profile decode:gate_up; dram__bytes_read.sum 143392512 + dram__bytes_write.sum 4034048
    ("decode_cc_kernel", "gate_up"): {"source": "weight_only_int4_linear_b200/csrc/gemv.cu",
                                      "sha256": "ab8e6f501913c473315e69ad4e443a993bcb8cd4dd825179dd595b891d690b0e",
                                      "bytes": 147426560},
    # python bench.py --profile prefill:gate_up_m4096; dram__bytes_read.sum 1108846080 + write 454347264
    ("prefill_kernel", "gate_up_m4096"): {"source": "weight_only_int4_linear_b200/csrc/gemm.cu",
                                          "sha256": "6e2f2daa7ddb04a9b7ae69d75359c9f4f41576d570171e6775945c9328b4e6e0",
                                          "bytes": 1563193344},
}


def ncu_traffic(kernel: str, layer: str):
    import hashlib
    rec = NCU_TRAFFIC.get((kernel, layer))
    if not rec or rec["bytes"] is None:
        return None
    with open(os.path.join(ROOT, rec["source"]), "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != rec["sha256"]:
            return None
    return rec["bytes"]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def max_over_ranks(x: float, device: str) -> float:
    """Max of a per-rank float over the process group (device time of the slowest rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(bytes_per_step_per_rank: float, steps: int, ms: float, world: int) -> float:
    """GB/s of the whole job: every rank's bytes over the slowest rank's time."""
    return world * bytes_per_step_per_rank * steps / (ms * 1e-3) / 1e9


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.gpu_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------------------------
# our implementation
# ----------------------------------------------------------------------------------------------

def setup_layers(cases, torch, w4, stream):
    layers = []
    for c in cases:
        W = torch.empty((c.N, c.K), dtype=torch.float32, device="cuda")
        synth.fill_weights_device(c.w_seed, c.w_tag, W.data_ptr(), c.N * c.K, stream=stream.cuda_stream)
        pw = w4.PackedWeight.from_float(W, stream=stream)
        torch.cuda.synchronize()
        del W
        if int(pw.status.item()) != 0:
            raise RuntimeError(f"packing failed for {c.name}: status {int(pw.status.item())}")
        xb = synth.activations_bf16(c.x_seed, c.M, c.K)
        X = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
        Y = torch.empty((c.M, c.N), dtype=torch.bfloat16, device="cuda")
        nb = w4.workspace_bytes(c.M, c.N, c.K)
        ws = torch.zeros(max(nb, 256), dtype=torch.uint8, device="cuda")
        layers.append({"case": c, "pw": pw, "X": X, "Y": Y, "ws": ws if nb else None, "x_host": xb})
    torch.cuda.synchronize()
    return layers


PREFILL_MIN_M = 64  # the library's automatic path choice: M >= 64 takes the tensor-core GEMM


def launches_per_call(c) -> int:
    """Our kernels per linear call: X preparation + GEMM (M >= 64); with K/128
    a multiple of 8, the one-token integer GEMV + its split-K reduction
    (M = 1, X prepared inside the GEMV), or X preparation + integer GEMV +
    reduction (2 <= M <= 16); otherwise X preparation + tensor-core GEMV per
    32-token chunk."""
    if c.M >= PREFILL_MIN_M:
        return 2
    if (c.K // 128) % 8 == 0 and c.M <= 16:
        return 2 if c.M == 1 else 3
    return 2 * ((c.M + 31) // 32)


def _linear_call(w4, L, path):
    w4.linear(L["X"], L["pw"].qweight, L["pw"].scales, L["pw"].zeros, L["Y"], L["ws"], path=path)


def capture(torch, stream, body):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        body()
    return g


def _step_body(sets, path, w4, n):
    """n steps; step i runs every layer once on weight copy i % len(sets)."""
    def f():
        for i in range(n):
            for L in sets[i % len(sets)]:
                _linear_call(w4, L, path)
    return f


def time_steps(sets, steps, warmup, torch, w4, stream, path, block=50):
    """Device time of exactly `steps` steps (step i on weight copy i % len(sets)), replayed from CUDA
    graphs of `block` steps (launch overhead off the timed path), after `warmup` untimed steps."""
    with torch.cuda.stream(stream):
        _step_body(sets, path, w4, max(warmup, 1))()
    torch.cuda.synchronize()
    block = max(1, min(block, steps))
    if block > len(sets):
        block -= block % len(sets)  # every graph starts on copy 0, so blocks keep the rotation
    full, rest = divmod(steps, block)
    g_full = capture(torch, stream, _step_body(sets, path, w4, block))
    g_rest = capture(torch, stream, _step_body(sets, path, w4, rest)) if rest else None
    with torch.cuda.stream(stream):
        g_full.replay()  # graph warm-up
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(full):
            g_full.replay()
        if g_rest is not None:
            g_rest.replay()
    end.record(stream)
    torch.cuda.synchronize()
    total_ms = start.elapsed_time(end)
    del g_full, g_rest
    return total_ms


def protocol_blocks(sets, torch, w4, stream, path, seconds, min_blocks=50, block=20):
    """Repeated timing of the same step outside the headline region: a CUDA graph of `block` steps
    replayed back to back, each replay bracketed by events on the launching stream, until at least
    `min_blocks` replays and `seconds` of device time.  Returns the per-step microseconds of every
    replay."""
    g = capture(torch, stream, _step_body(sets, path, w4, block))
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    per_step, total_ms = [], 0.0
    while len(per_step) < min_blocks or total_ms < seconds * 1e3:
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(51)]
        ev[0].record(stream)
        with torch.cuda.stream(stream):
            for j in range(50):
                g.replay()
                ev[j + 1].record(stream)
        torch.cuda.synchronize()
        for j in range(50):
            ms = ev[j].elapsed_time(ev[j + 1])
            per_step.append(ms * 1e3 / block)
            total_ms += ms
    del g
    return per_step


def _quantiles(xs):
    q = np.quantile(np.asarray(xs), [0.1, 0.5, 0.9])
    return {"p10": float(q[0]), "median": float(q[1]), "p90": float(q[2]), "n": len(xs)}


def packed_copies(c, torch, w4, stream, max_copies=48):
    """Copies of layer c's packed weights, enough that their codes exceed 3x L2 (at most max_copies)."""
    W = torch.empty((c.N, c.K), dtype=torch.float32, device="cuda")
    synth.fill_weights_device(c.w_seed, c.w_tag, W.data_ptr(), c.N * c.K, stream=stream.cuda_stream)
    copies = max(1, min(max_copies, -(-3 * L2_BYTES // c.code_bytes)))
    pws = [w4.PackedWeight.from_float(W, stream=stream) for _ in range(copies)]
    torch.cuda.synchronize()
    del W
    if any(int(pw.status.item()) != 0 for pw in pws):
        raise RuntimeError(f"packing failed for {c.name}")
    return pws


def time_layer_alone(c, torch, w4, stream, min_calls=200, pws=None):
    """Device time of one call of layer `c` (CUDA events on the launching
    stream): back-to-back calls replayed from a CUDA graph, each call reading a
    different copy of the packed weights, rotating through enough copies that
    their codes exceed 3x L2; the median over seven replays of the graph.
    Returns (us per call, copies)."""
    own = pws is None
    if own:
        pws = packed_copies(c, torch, w4, stream)
    copies = len(pws)
    xb = synth.activations_bf16(c.x_seed, c.M, c.K)
    X = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    Y = torch.empty((c.M, c.N), dtype=torch.bfloat16, device="cuda")
    nb = w4.workspace_bytes(c.M, c.N, c.K)
    ws = torch.zeros(max(nb, 256), dtype=torch.uint8, device="cuda")
    passes = max(1, -(-min_calls // copies)) if c.M < 512 else 1

    def body():
        for _ in range(passes):
            for pw in pws:
                w4.linear(X, pw.qweight, pw.scales, pw.zeros, Y, ws)
    with torch.cuda.stream(stream):
        for _ in range(3):
            body()
    torch.cuda.synchronize()
    g = capture(torch, stream, body)
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    # median over replays, each bracketed by events on the launching stream
    reps = 7
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    ev[0].record(stream)
    with torch.cuda.stream(stream):
        for r in range(reps):
            g.replay()
            ev[r + 1].record(stream)
    torch.cuda.synchronize()
    us = statistics.median(ev[r].elapsed_time(ev[r + 1]) for r in range(reps)) * 1e3 / (passes * copies)
    del g, X, Y, ws
    if own:
        del pws
    torch.cuda.empty_cache()
    return us, copies


def layer_roofline(c, us, peaks, peak_src, kernel):
    """One layer's measured rate against the copy bandwidth (HBM-bound GEMV) or the dense BF16 peak (GEMM)."""
    if c.M >= PREFILL_MIN_M:
        achieved = c.flops / us / 1e6
        return {"bound": "tensor", "kernel": kernel, "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"], "per_call_us": us,
                "peak_source": peak_src}
    achieved = c.code_bytes / us / 1e3
    return {"bound": "hbm", "kernel": kernel, "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "per_call_us": us, "algorithmic_bytes_per_launch": c.code_bytes,
            "peak_source": peak_src}


def decode_kernel_name(c) -> str:
    if c.M >= PREFILL_MIN_M:
        return "prefill_kernel"
    if (c.K // 128) % 8 == 0 and c.M <= 16:
        return "decode_cc_kernel" if c.M == 1 else f"decode_mt_kernel<{4 if c.M <= 4 else 8 if c.M <= 8 else 16}>"
    return "decode_tc_kernel<16>" if min(c.M, 32) <= 16 else "decode_tc_kernel<32>"


def run_layer_tables(torch, w4, stream, peaks, peak_src, prefill_ms=(512, 2048)):
    """The other workloads, each layer alone with its weights rotated past 3x L2: the single 4096 x 4096
    GEMV, the small-batch sweep M in {2, 4, 8, 16, 32} and the prefill GEMM at M in prefill_ms, on the
    hidden-8192 shapes (one set of packed copies per shape serves every M)."""
    out = {}
    c1 = workloads.single_gemv()[0]
    us, copies = time_layer_alone(c1, torch, w4, stream)
    out["single_gemv_4096"] = {"workload": c1.workload, "M": 1, "K": c1.K, "N": c1.N, "weight_copies": copies,
                               "roofline": layer_roofline(c1, us, peaks, peak_src, decode_kernel_name(c1))}
    small = workloads.small_batch_8192()
    pre = workloads.prefill_8192(ms=list(prefill_ms))
    rows_small, rows_pre = [], []
    def base(c):
        return c.name.rsplit("_m", 1)[0]
    for shape in [name for name, _, _ in workloads.HIDDEN_8192]:
        cs = [c for c in small if base(c) == shape]
        pws = packed_copies(cs[0], torch, w4, stream, max_copies=12)
        for c in cs:
            us, copies = time_layer_alone(c, torch, w4, stream, pws=pws)
            rows_small.append({"layer": c.name, "M": c.M, "K": c.K, "N": c.N, "weight_copies": copies,
                               "roofline": layer_roofline(c, us, peaks, peak_src, decode_kernel_name(c))})
        for c in [c for c in pre if base(c) == shape]:
            us, copies = time_layer_alone(c, torch, w4, stream, pws=pws[:1])
            rows_pre.append({"layer": c.name, "M": c.M, "K": c.K, "N": c.N,
                             "roofline": layer_roofline(c, us, peaks, peak_src, decode_kernel_name(c))})
        del pws
        torch.cuda.empty_cache()
    out["small_batch_8192"] = rows_small
    out["prefill_8192_other_m"] = rows_pre
    return out


def time_e2e(layers, steps, warmup, torch, w4, stream, path):
    """The C-ABI call with host buffers, once per layer and step: w4a16_linear_host enqueues the
    pinned H2D copy of X, the layer and the D2H copy of Y on the stream (the automatic path choice,
    as `path` is for the timed kernels)."""
    lib = w4.load()
    xs = [torch.from_numpy(L["x_host"].view(np.int16)).pin_memory() for L in layers]
    ys = [torch.empty((L["case"].M, L["case"].N), dtype=torch.int16).pin_memory() for L in layers]
    calls = []
    for L, xh, yh in zip(layers, xs, ys):
        c, pw, ws = L["case"], L["pw"], L["ws"]
        calls.append((xh.data_ptr(), L["X"].data_ptr(), c.M, c.K, pw.qweight.data_ptr(), pw.scales.data_ptr(),
                      pw.zeros.data_ptr(), c.N, L["Y"].data_ptr(), yh.data_ptr(),
                      ws.data_ptr() if ws is not None else None, ws.numel() if ws is not None else 0,
                      stream.cuda_stream))
    fn = lib.w4a16_linear_host

    def one_step():
        for args in calls:
            st = fn(*args)
            if st != 0:
                raise w4.W4A16Error("w4a16_linear_host", st)

    for _ in range(warmup):
        one_step()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        one_step()
    end.record(stream)
    torch.cuda.synchronize()
    h2d = sum(L["X"].numel() * 2 for L in layers)
    d2h = sum(L["Y"].numel() * 2 for L in layers)
    return start.elapsed_time(end), h2d, d2h


def time_e2e_graph(layers, steps, warmup, torch, w4, stream, per_graph=10):
    """The same host-buffer calls, each enqueued by w4a16_linear_host, captured once into a CUDA graph of
    `per_graph` steps and replayed: every replay performs every layer's transfer of X from pinned host memory
    and of Y back to it, without the host's per-call enqueue cost (the way a serving loop replays a captured
    decode step).  Returns ms per step."""
    lib = w4.load()
    xs = [torch.from_numpy(L["x_host"].view(np.int16)).pin_memory() for L in layers]
    ys = [torch.empty((L["case"].M, L["case"].N), dtype=torch.int16).pin_memory() for L in layers]
    calls = []
    for L, xh, yh in zip(layers, xs, ys):
        c, pw, ws = L["case"], L["pw"], L["ws"]
        calls.append((xh.data_ptr(), L["X"].data_ptr(), c.M, c.K, pw.qweight.data_ptr(), pw.scales.data_ptr(),
                      pw.zeros.data_ptr(), c.N, L["Y"].data_ptr(), yh.data_ptr(),
                      ws.data_ptr() if ws is not None else None, ws.numel() if ws is not None else 0,
                      stream.cuda_stream))
    fn = lib.w4a16_linear_host

    def body():
        for _ in range(per_graph):
            for args in calls:
                st = fn(*args)
                if st != 0:
                    raise w4.W4A16Error("w4a16_linear_host", st)
    with torch.cuda.stream(stream):
        body()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    # relaxed: the host entry asks the runtime for the mapped device addresses of the pinned buffers while
    # the capture is open, which is not a stream operation
    with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
        body()
    reps = max(1, (steps + per_graph - 1) // per_graph)
    with torch.cuda.stream(stream):
        for _ in range(max(1, warmup)):
            g.replay()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(reps):
            g.replay()
    end.record(stream)
    torch.cuda.synchronize()
    del g
    return start.elapsed_time(end) / (reps * per_graph)


# ----------------------------------------------------------------------------------------------
# the 80-layer decode stack (hidden 8192, M = 1), all packed weights resident
# ----------------------------------------------------------------------------------------------

STACK_LAYERS = 80
STACK_DOWN_IN = 28672  # down reads the first half of gate+up's output, renormalised


def build_stack(torch, w4, stream, n_layers=STACK_LAYERS):
    """Packed weights of layers 0 .. n_layers-1 (seed = layer index), generated and packed on the device."""
    cases0 = workloads.stack_layer(0)
    Wtmp = torch.empty(max(c.N * c.K for c in cases0), dtype=torch.float32, device="cuda")
    layers = []
    for layer in range(n_layers):
        mats = []
        for c in workloads.stack_layer(layer):
            synth.fill_weights_device(c.w_seed, c.w_tag, Wtmp.data_ptr(), c.N * c.K, stream=stream.cuda_stream)
            mats.append(w4.PackedWeight.from_float(Wtmp[: c.N * c.K].view(c.N, c.K), stream=stream))
        layers.append(mats)
    torch.cuda.synchronize()
    del Wtmp
    for layer, mats in enumerate(layers):
        for pw in mats:
            if int(pw.status.item()) != 0:
                raise RuntimeError(f"packing failed in stack layer {layer}")
    return layers


class StackBuffers:
    def __init__(self, torch, w4, layers):
        qkv, o, gu, down = layers[0]
        bf = dict(dtype=torch.bfloat16, device="cuda")
        self.h = [torch.empty((1, qkv.K), **bf), torch.empty((1, qkv.K), **bf)]
        self.y_qkv = torch.empty((1, qkv.N), **bf)
        self.y_o = torch.empty((1, o.N), **bf)
        self.y_gu = torch.empty((1, gu.N), **bf)
        self.u = torch.empty((1, STACK_DOWN_IN), **bf)
        self.y_down = torch.empty((1, down.N), **bf)
        nb = max(w4.workspace_bytes(1, pw.N, pw.K) for pw in layers[0])
        self.ws = torch.zeros(max(nb, 256), dtype=torch.uint8, device="cuda")


def stack_step(w4, layers, buf, record=()):
    """One decode step through the stack from buf.h[0]: per layer qkv, o and
    gate+up read the hidden state h; down reads u = renorm(gate+up[:, :28672]);
    the next hidden state is renorm(down).  Returns (final h, {layer: copies of
    that layer's inputs and outputs} for the layers in `record`)."""
    h = buf.h[0]
    rec = {}
    for layer, (p_qkv, p_o, p_gu, p_down) in enumerate(layers):
        w4.linear(h, p_qkv.qweight, p_qkv.scales, p_qkv.zeros, buf.y_qkv, buf.ws)
        w4.linear(h, p_o.qweight, p_o.scales, p_o.zeros, buf.y_o, buf.ws)
        w4.linear(h, p_gu.qweight, p_gu.scales, p_gu.zeros, buf.y_gu, buf.ws)
        w4.renorm_rows(buf.y_gu[:, :STACK_DOWN_IN], buf.u)
        w4.linear(buf.u, p_down.qweight, p_down.scales, p_down.zeros, buf.y_down, buf.ws)
        h_next = buf.h[(layer + 1) % 2]
        w4.renorm_rows(buf.y_down, h_next)
        if layer in record:
            rec[layer] = {"h": h.clone(), "qkv": buf.y_qkv.clone(), "o_proj": buf.y_o.clone(),
                          "gate_up": buf.y_gu.clone(), "u": buf.u.clone(), "down": buf.y_down.clone()}
        h = h_next
    return h, rec


def run_stack(torch, w4, stream, steps):
    """Aggregate weight GB/s of the 80-layer stack: one step = 320 linear calls + 160 renorms, replayed
    from a CUDA graph; the step starts from the same X each time."""
    layers = build_stack(torch, w4, stream)
    buf = StackBuffers(torch, w4, layers)
    c0 = workloads.stack_layer(0)
    x0 = torch.from_numpy(synth.activations_bf16(c0[0].x_seed, 1, c0[0].K).view(np.int16)).cuda().view(torch.bfloat16)
    code_bytes = sum(pw.N * pw.K // 2 for mats in layers for pw in mats)

    def body():
        buf.h[0].copy_(x0)
        stack_step(w4, layers, buf)
    with torch.cuda.stream(stream):
        for _ in range(2):
            body()
    torch.cuda.synchronize()
    g = capture(torch, stream, body)
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(steps):
            g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    fault = w4.device_fault()
    del g, layers, buf
    torch.cuda.empty_cache()
    if fault:
        raise RuntimeError(f"a kernel gave up a bounded wait (site {fault}) in the stack")
    return {"value": code_bytes / (ms * 1e-3) / 1e9, "unit": "GB/s", "workload": "decode_stack_80x8192",
            "ms_per_step": ms, "steps": steps, "packed_code_bytes": code_bytes,
            "launches_per_step": STACK_LAYERS * (sum(launches_per_call(c) for c in workloads.stack_layer(0)) + 2),
            "note": "aggregate packed-code GB/s over 80 layers x {qkv, o, gate+up, down} chained on one "
                    "stream with the renorm kernels between them (their time included)"}


def cpu_baseline(cases, budget_s=12.0):
    """The FP64 oracle (as it stands) on a bounded sample of the same workload:
    the first rows of each layer, packed by the oracle, multiplied on all host cores."""
    import oracle
    rows_per_layer = 1024
    samples = []
    for c in cases:
        rows = np.arange(min(rows_per_layer, c.N), dtype=np.int64)
        W = synth.weight_rows_f32(c.w_seed, c.w_tag, c.K, rows)
        st, qw, sc, z = oracle.quantize_pack(W)
        X = synth.activations_bf16(c.x_seed, c.M, c.K)
        samples.append((X, qw, sc, z, rows.size * c.K // 2))
    t0 = time.perf_counter()
    done_bytes, reps = 0, 0
    while True:
        for X, qw, sc, z, nbytes in samples:
            oracle.linear(X, qw, sc, z)
            done_bytes += nbytes
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": done_bytes / dt / 1e9, "unit": "GB/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": f"first {rows_per_layer} output rows of each of the {len(cases)} layers "
                      f"({', '.join(c.name for c in cases)}), M={cases[0].M}, {reps} passes in {dt:.1f} s; "
                      f"GB/s of packed code bytes"}, dt


def run_ours(args):
    import torch
    import weight_only_int4_linear_b200 as w4

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    w4.load()
    stream = torch.cuda.Stream()
    peaks, peak_src = load_peaks()

    # the hidden-5120 layer set at M = 1, two copies of its packed weights: step i runs copy i % 2, so
    # 2 x 251 MB of weights pass between reuses (4x the 126 MB L2)
    cases = workloads.decode_5120()
    sets = [setup_layers(cases, torch, w4, stream) for _ in range(2)]
    code_bytes = sum(c.code_bytes for c in cases)
    all_bytes = sum(c.code_bytes + c.meta_bytes + 2 * c.M * (c.K + c.N) for c in cases)

    # Clock samples cover a window of the same steps around the timed region: repeated blocks of the
    # step (the timing protocol's spread) before and after it, so the sampler (one sample per 200 ms)
    # sees the clocks the timed steps ran at.
    with ClockSampler(local) as clk:
        proto = protocol_blocks(sets, torch, w4, stream, w4.PATH_AUTO, seconds=args.protocol_seconds / 2)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        total_ms = time_steps(sets, args.steps, args.warmup, torch, w4, stream, w4.PATH_AUTO)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        proto += protocol_blocks(sets, torch, w4, stream, w4.PATH_AUTO, seconds=args.protocol_seconds / 2)
    total_ms = max_over_ranks(total_ms, "cuda")
    value = whole_job_rate(code_bytes, args.steps, total_ms, world)
    pq = _quantiles(proto)

    # end to end through the public API with host buffers
    e2e_ms, h2d, d2h = time_e2e(sets[0], args.steps, args.warmup, torch, w4, stream, w4.PATH_AUTO)
    e2e_ms = max_over_ranks(e2e_ms, "cuda")
    e2e_value = whole_job_rate(code_bytes, args.steps, e2e_ms, world)
    e2e_graph_ms = max_over_ranks(time_e2e_graph(sets[0], args.steps, args.warmup, torch, w4, stream), "cuda")
    e2e_graph_value = whole_job_rate(code_bytes, 1, e2e_graph_ms, world)
    del sets
    torch.cuda.empty_cache()

    # each layer's kernel alone (an M = 1 call is one launch); dominant kernel: gate+up
    per_layer = [time_layer_alone(c, torch, w4, stream)[0] for c in cases]
    dom = max(range(len(cases)), key=lambda i: cases[i].code_bytes)
    dom_us = per_layer[dom]
    dom_gbs = cases[dom].code_bytes / dom_us / 1e3
    dom_all = (cases[dom].code_bytes + cases[dom].meta_bytes) / dom_us / 1e3
    fault = w4.device_fault()
    if fault != 0:
        raise RuntimeError(f"a kernel gave up a bounded wait (site {fault}); results invalid")

    # prefill layer set at M = 4096 (hidden-8192 shapes)
    prefill = None
    if not args.no_prefill:
        pcases = workloads.prefill_8192(ms=[4096])
        players = setup_layers(pcases, torch, w4, stream)
        p_ms = time_steps([players], args.prefill_steps, 1, torch, w4, stream, w4.PATH_AUTO, block=1)
        del players
        torch.cuda.empty_cache()
        flops = sum(c.flops for c in pcases)
        tflops = flops * args.prefill_steps / (p_ms * 1e-3) / 1e12
        pdom = max(range(len(pcases)), key=lambda i: pcases[i].flops)
        pdom_us = time_layer_alone(pcases[pdom], torch, w4, stream)[0]  # X preparation + GEMM
        pdom_tf = pcases[pdom].flops / pdom_us / 1e6
        prefill = {"value": tflops, "unit": "TFLOP/s", "workload": "prefill_hidden8192_m4096",
                   "ms_per_step": p_ms / args.prefill_steps, "steps": args.prefill_steps,
                   "frac_of_bf16_peak": tflops / peaks["bf16_tflops"],
                   "roofline": {"bound": "tensor", "kernel": f"prefill_kernel on {pcases[pdom].name} "
                                                             f"({pcases[pdom].K}x{pcases[pdom].N}, M={pcases[pdom].M})",
                                "achieved": pdom_tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                "frac": pdom_tf / peaks["bf16_tflops"],
                                "traffic": ncu_traffic("prefill_kernel", pcases[pdom].name),
                                "per_call_us": pdom_us, "timed": "whole call: X preparation (about 2% of it) + GEMM",
                                "peak_source": peak_src}}

    tables = None if args.no_tables else run_layer_tables(torch, w4, stream, peaks, peak_src)

    stack = None
    if not args.no_stack:
        stack = run_stack(torch, w4, stream, args.stack_steps)

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        cpu, _ = cpu_baseline(cases, args.cpu_budget)

    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    launches = args.steps * sum(launches_per_call(c) for c in cases)
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int4 weights x bf16 activations, fp32 accumulate",
        "data": "synthetic (seeded W ~ N(0,0.02) packed INT4 g128; X ~ N(0,1) bf16, 1% channels x20)",
        "config": {"workload": "decode_hidden5120_m1", "M": 1,
                   "shapes_KxN": [[c.K, c.N] for c in cases], "group": 128,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"inputs larger than L2: two copies of the layer set's weights alternate by step, "
                         f"{2 * all_bytes / 1e6:.0f} MB read between reuses vs {L2_BYTES / 1e6:.0f} MB L2"},
        "frac_of_hbm_peak": value / world / peaks["hbm_gbs"],
        "all_bytes_gbs": world * all_bytes * args.steps / (total_ms * 1e-3) / 1e9,
        "protocol": {"us_per_step": pq, "gbs_median": code_bytes / pq["median"] / 1e3,
                     "frac_median": code_bytes / pq["median"] / 1e3 / peaks["hbm_gbs"],
                     "how": "CUDA graphs of 20 steps replayed back to back around the timed region, "
                            "each replay bracketed by events; weights rotated as above"},
        "roofline": {"bound": "hbm", "kernel": f"{decode_kernel_name(cases[dom])} on {cases[dom].name} "
                                                f"({cases[dom].K}x{cases[dom].N})",
                     "achieved": dom_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": dom_gbs / peaks["hbm_gbs"],
                     "traffic": args.traffic if args.traffic is not None else ncu_traffic("decode_cc_kernel",
                                                                                         cases[dom].name),
                     "achieved_all_bytes": dom_all, "per_launch_us": dom_us,
                     "algorithmic_bytes_per_launch": cases[dom].code_bytes, "peak_source": peak_src},
        "per_layer_us": {c.name: us for c, us in zip(cases, per_layer)},
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms / args.steps},
        "e2e_graph": {"value": e2e_graph_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h, "ms_per_step": e2e_graph_ms,
                      "note": "the same host-buffer calls captured into a CUDA graph and replayed"},
        "prefill": prefill,
        "stack": stack,
        "configs": tables,
        "gpu_launches": launches,
        "cpu_baseline": cpu,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------------------------
# reference arm: the FP64 oracle on the host cores, same workload, metric and unit
# ----------------------------------------------------------------------------------------------

def run_reference(args):
    """The reference arm: the FP64 oracle, as it stands, on the host cores.  A
    step is one pass over a bounded sample of the decode step (the first rows
    of each of the four layers), sized so that warm-up + timed steps take about
    --ref-seconds in all.  Under torch.distributed.run only rank 0 runs."""
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    cases = workloads.decode_5120()

    def sample(rows_per_layer):
        out = []
        for c in cases:
            rows = np.arange(min(rows_per_layer, c.N), dtype=np.int64)
            W = synth.weight_rows_f32(c.w_seed, c.w_tag, c.K, rows)
            st, qw, sc, z = oracle.quantize_pack(W)
            out.append((synth.activations_bf16(c.x_seed, c.M, c.K), qw, sc, z, rows.size * c.K // 2))
        return out

    def step(smp):
        for X, qw, sc, z, _ in smp:
            oracle.linear(X, qw, sc, z)

    probe_rows = 256
    smp = sample(probe_rows)
    t0 = time.perf_counter()
    step(smp)
    t_probe = time.perf_counter() - t0
    per_step = args.ref_seconds / max(1, args.steps + args.warmup)
    rows = int(max(8, min(4096, probe_rows * per_step / max(t_probe, 1e-6))))
    smp = sample(rows)
    for _ in range(args.warmup):
        step(smp)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step(smp)
    dt = time.perf_counter() - t0
    nbytes = sum(x[4] for x in smp)
    value = nbytes * args.steps / dt / 1e9
    sample_desc = (f"first {rows} output rows of each of the {len(cases)} layers ({', '.join(c.name for c in cases)}), "
                   f"M=1, packed by the oracle; {args.steps} timed steps of one pass each in {dt:.2f} s; "
                   f"GB/s of packed code bytes")
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (same seeded workload)",
        "config": {"workload": "decode_hidden5120_m1", "M": 1, "shapes_KxN": [[c.K, c.N] for c in cases],
                   "group": 128, "sample_rows_per_layer": rows},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.threads(), "kind": "oracle",
                         "sample": sample_desc},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_profile(spec: str, repeats: int = 4):
    """Run one layer of a workload a few times, or (layer "all") the whole layer set, for an ncu
    capture; no timing."""
    import torch
    import weight_only_int4_linear_b200 as w4
    w4.load()
    wl, name = spec.split(":")
    if wl == "w8":  # the W8A16 layer on a decode shape (hidden 5120, M = 1)
        stream = torch.cuda.Stream()
        for c in [c for c in workloads.decode_5120() if name in (c.name, "all")]:
            W = torch.empty((c.N, c.K), dtype=torch.float32, device="cuda")
            synth.fill_weights_device(c.w_seed, c.w_tag, W.data_ptr(), c.N * c.K, stream=stream.cuda_stream)
            p8 = w4.PackedW8.from_float(W, stream)
            xb = synth.activations_bf16(c.x_seed, c.M, c.K)
            X = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
            Y = torch.empty((c.M, c.N), dtype=torch.bfloat16, device="cuda")
            ws = torch.zeros(w4.w8_workspace_bytes(c.M, c.N, c.K), dtype=torch.uint8, device="cuda")
            torch.cuda.synchronize()
            del W
            with torch.cuda.stream(stream):
                for _ in range(repeats):
                    w4.w8_linear(X, p8.qweight, p8.scales, Y, ws)
            torch.cuda.synchronize()
        fault = w4.device_fault()
        print(json.dumps({"profiled": spec, "repeats": repeats, "fault": fault}))
        if fault:
            raise SystemExit(1)
        return
    cases = {"decode": workloads.decode_5120(), "small": workloads.small_batch_8192(),
             "prefill": workloads.prefill_8192(ms=[4096])}[wl]
    chosen = cases if name == "all" else [c for c in cases if c.name == name]
    stream = torch.cuda.Stream()
    layers = setup_layers(chosen, torch, w4, stream)
    with torch.cuda.stream(stream):
        for _ in range(repeats):
            for L in layers:
                _linear_call(w4, L, w4.PATH_AUTO)
    torch.cuda.synchronize()
    fault = w4.device_fault()
    print(json.dumps({"profiled": spec, "repeats": repeats, "fault": fault}))
    if fault:
        raise SystemExit(1)


def _time_graph(torch, stream, body, calls):
    """Device time per call of `body` (which makes `calls` calls), replayed from a CUDA graph."""
    with torch.cuda.stream(stream):
        for _ in range(2):
            body()
    torch.cuda.synchronize()
    g = capture(torch, stream, body)
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 3
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(reps):
            g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / (reps * calls)


def run_comparators(which: str):
    """The unfused pipelines the fused kernel replaces ("Quantization I", Concept; "Weight-Only
    Quantization and Mixed Precision", sections 1 and 7), timed per call beside the fused path, one
    JSON line per layer:
      offline_dequant_gemm: W_hat = (q - z) s materialised once in BF16 (not timed), then a cuBLAS
        BF16 GEMM per call (torch.matmul);
      naive_three_kernel: per call, unpack to byte codes (w4a16_unpack), dequantise to BF16
        (w4a16_dequant_codes), cuBLAS BF16 GEMM: every intermediate through HBM.
    Every call of every variant reads weights past L2 (enough copies rotated)."""
    import torch
    import weight_only_int4_linear_b200 as w4
    w4.load()
    stream = torch.cuda.Stream()
    sets = {"decode": workloads.decode_5120(), "prefill": workloads.prefill_8192(ms=[4096])}
    names = list(sets) if which == "all" else which.split(",")
    for wl in names:
        for c in sets[wl]:
            fused_us, _ = time_layer_alone(c, torch, w4, stream)
            W = torch.empty((c.N, c.K), dtype=torch.float32, device="cuda")
            synth.fill_weights_device(c.w_seed, c.w_tag, W.data_ptr(), c.N * c.K, stream=stream.cuda_stream)
            pw = w4.PackedWeight.from_float(W, stream=stream)
            torch.cuda.synchronize()
            del W
            xb = synth.activations_bf16(c.x_seed, c.M, c.K)
            X = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
            Y = torch.empty((c.M, c.N), dtype=torch.bfloat16, device="cuda")
            # offline dequantisation: BF16 weights, copies past 3x L2
            wbytes = c.N * c.K * 2
            ncopy = max(1, min(16, -(-3 * L2_BYTES // wbytes)))
            W_hats = [torch.empty((c.N, c.K), dtype=torch.bfloat16, device="cuda") for _ in range(ncopy)]
            for Wh in W_hats:
                w4.dequant(pw.qweight, pw.scales, pw.zeros, c.K, Wh)
            torch.cuda.synchronize()

            def body_gemm():
                for Wh in W_hats:
                    torch.matmul(X, Wh.t(), out=Y)
            gemm_us = _time_graph(torch, stream, body_gemm, ncopy)
            Y_gemm = Y.clone()
            del W_hats
            torch.cuda.empty_cache()
            # naive three kernels: packed copies past 3x L2, one codes and one W_hat buffer
            pcopy = max(1, min(16, -(-3 * L2_BYTES // c.code_bytes)))
            pws = [(pw.qweight, pw.scales, pw.zeros)] + [(pw.qweight.clone(), pw.scales.clone(), pw.zeros.clone())
                                                         for _ in range(pcopy - 1)]
            codes = torch.empty((c.N, c.K), dtype=torch.uint8, device="cuda")
            Wh = torch.empty((c.N, c.K), dtype=torch.bfloat16, device="cuda")

            def body_naive():
                for qw_, sc_, z_ in pws:
                    w4.unpack(qw_, c.K, codes)
                    w4.dequant_codes(codes, sc_, z_, Wh)
                    torch.matmul(X, Wh.t(), out=Y)
            naive_us = _time_graph(torch, stream, body_naive, pcopy)
            torch.cuda.synchronize()
            agree = bool(torch.equal(Y.view(torch.int16), Y_gemm.view(torch.int16)))
            line = {"comparators": c.workload, "layer": c.name, "M": c.M, "K": c.K, "N": c.N,
                    "fused_us": fused_us, "offline_dequant_gemm_us": gemm_us, "naive_three_kernel_us": naive_us,
                    "fused_speedup_vs_dequant_gemm": gemm_us / fused_us,
                    "fused_speedup_vs_naive": naive_us / fused_us,
                    "fused_code_gbs": c.code_bytes / fused_us / 1e3,
                    "unfused_paths_agree_bitwise": agree, "fault": w4.device_fault()}
            if c.M >= PREFILL_MIN_M:
                line.update({"fused_tflops": c.flops / fused_us / 1e6, "dequant_gemm_tflops": c.flops / gemm_us / 1e6,
                             "naive_tflops": c.flops / naive_us / 1e6})
            print(json.dumps(line), flush=True)
            del pws, codes, Wh, pw
            torch.cuda.empty_cache()


def awq_channel_scales(K: int, seed: int = 42):
    """Synthetic AWQ scales: s_k = mean|x_k|^(1/2) over a seeded 64-token calibration batch
    (salient channels included), normalised to geometric mean 1; r = fp32(1 / s)."""
    xb = synth.activations_bf16(seed, 64, K)
    xf = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    s = np.sqrt(np.abs(xf).mean(axis=0))
    s /= np.exp(np.log(s).mean())
    s = s.astype(np.float32)
    return s, (1.0 / s.astype(np.float64)).astype(np.float32)


def run_variants(which: str):
    """Weight formats and the AWQ fold on the fused kernels, one JSON line per layer: the
    affine layer, the same kernels on symmetric-packed weights (zero point 8), and
    w4a16_linear_awq (activation scaling formed in the kernels' X preparation, weights from
    w4a16_quantize_pack_awq); device time per call (median of three rounds in rotated order),
    each call reading a different copy of the weights past L2, replayed from a CUDA graph."""
    import torch
    import weight_only_int4_linear_b200 as w4
    w4.load()
    stream = torch.cuda.Stream()
    sets = {"decode": workloads.decode_5120(), "small_batch": workloads.small_batch_8192(),
            "prefill": workloads.prefill_8192(ms=[4096])}
    names = list(sets) if which == "all" else which.split(",")
    for wl in names:
        for c in sets[wl]:
            s, r = awq_channel_scales(c.K)
            s_dev, r_dev = torch.from_numpy(s).cuda(), torch.from_numpy(r).cuda()
            copies = max(1, min(16, -(-3 * L2_BYTES // c.code_bytes)))
            W = torch.empty((c.N, c.K), dtype=torch.float32, device="cuda")
            synth.fill_weights_device(c.w_seed, c.w_tag, W.data_ptr(), c.N * c.K, stream=stream.cuda_stream)
            packed = {}
            with torch.cuda.stream(stream):
                packed["affine"] = [w4.PackedWeight.from_float(W, stream=stream) for _ in range(copies)]
                packed["symmetric"] = [w4.PackedWeight.from_float(W, stream=stream, symmetric=True)
                                       for _ in range(copies)]
                awq = []
                for _ in range(copies):
                    pw = w4.PackedWeight(c.N, c.K)
                    pw.status = torch.zeros(1, dtype=torch.int32, device="cuda")
                    w4.quantize_pack_awq(W, s_dev, pw.qweight, pw.scales, pw.zeros, pw.status, stream)
                    awq.append(pw)
                packed["awq"] = awq
            torch.cuda.synchronize()
            del W
            if any(int(pw.status.item()) != 0 for v in packed.values() for pw in v):
                raise RuntimeError(f"packing failed for {c.name}")
            xb = synth.activations_bf16(c.x_seed, c.M, c.K)
            X = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
            Y = torch.empty((c.M, c.N), dtype=torch.bfloat16, device="cuda")
            ws = torch.zeros(max(w4.workspace_bytes(c.M, c.N, c.K), 256), dtype=torch.uint8, device="cuda")
            passes = max(1, -(-200 // copies)) if c.M < 512 else 1
            # three rounds in rotated order, median per variant: under a sustained load the clock
            # drifts down, which would otherwise favour whichever variant is timed first
            samples = {kind: [] for kind in packed}
            kinds = list(packed)
            for rnd in range(3):
                for kind in kinds[rnd:] + kinds[:rnd]:
                    pws = packed[kind]

                    def body(pws=pws, kind=kind):
                        for _ in range(passes):
                            for pw in pws:
                                if kind == "awq":
                                    w4.linear_awq(X, r_dev, pw.qweight, pw.scales, pw.zeros, Y, ws)
                                else:
                                    w4.linear(X, pw.qweight, pw.scales, pw.zeros, Y, ws)
                    samples[kind].append(_time_graph(torch, stream, body, passes * copies))
            us = {kind: statistics.median(v) for kind, v in samples.items()}
            line = {"variants": c.workload, "layer": c.name, "M": c.M, "K": c.K, "N": c.N,
                    "affine_us": us["affine"], "symmetric_us": us["symmetric"], "awq_us": us["awq"],
                    "awq_over_affine": us["awq"] / us["affine"], "fault": w4.device_fault()}
            if c.M >= PREFILL_MIN_M:
                line.update({k + "_tflops": c.flops / v / 1e6 for k, v in us.items()})
            else:
                line.update({k + "_code_gbs": c.code_bytes / v / 1e3 for k, v in us.items()})
            print(json.dumps(line), flush=True)
            del packed, awq, X, Y, ws
            torch.cuda.empty_cache()


def run_w8(which: str):
    """W8A16 ("Weight-Only Quantization and Mixed Precision", sections 5 and 8: INT8 weights,
    16-bit activations, no grouping) beside the W4A16 layer and a cuBLAS BF16 GEMM on the same
    shapes, one JSON line per layer and token count: device time per call, each call reading a
    different copy of the weights past L2, replayed from a CUDA graph.  The W8 roofline bytes are
    N K code bytes + 2 N scale bytes (+ X and Y)."""
    import torch
    import weight_only_int4_linear_b200 as w4
    w4.load()
    stream = torch.cuda.Stream()
    ms = [int(m) for m in which.split(",")] if which not in ("decode", "all") else [1, 2]
    for c in workloads.decode_5120():
        w8_bytes = c.N * c.K + 2 * c.N
        copies8 = max(1, min(16, -(-3 * L2_BYTES // w8_bytes)))
        copies16 = max(1, min(16, -(-3 * L2_BYTES // (2 * c.N * c.K))))
        W = torch.empty((c.N, c.K), dtype=torch.float32, device="cuda")
        synth.fill_weights_device(c.w_seed, c.w_tag, W.data_ptr(), c.N * c.K, stream=stream.cuda_stream)
        with torch.cuda.stream(stream):
            p8 = [w4.PackedW8.from_float(W, stream) for _ in range(copies8)]
            W16 = [W.to(torch.bfloat16) for _ in range(copies16)]
        torch.cuda.synchronize()
        del W
        if any(int(p.status.item()) != 0 for p in p8):
            raise RuntimeError(f"W8 quantisation failed for {c.name}")
        for M in ms:
            cm = dataclasses.replace(c, M=M)
            xb = synth.activations_bf16(c.x_seed, M, c.K)
            X = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
            Y = torch.empty((M, c.N), dtype=torch.bfloat16, device="cuda")
            ws = torch.zeros(max(w4.w8_workspace_bytes(M, c.N, c.K), 256), dtype=torch.uint8, device="cuda")
            passes8 = max(1, -(-200 // copies8))

            def body8():
                for _ in range(passes8):
                    for p in p8:
                        w4.w8_linear(X, p.qweight, p.scales, Y, ws)
            us8 = _time_graph(torch, stream, body8, passes8 * copies8)
            passes16 = max(1, -(-100 // copies16))

            def body16():
                for _ in range(passes16):
                    for Wb in W16:
                        torch.matmul(X, Wb.t(), out=Y)
            us16 = _time_graph(torch, stream, body16, passes16 * copies16)
            us4, _ = time_layer_alone(cm, torch, w4, stream)
            line = {"w8a16": c.workload, "layer": c.name, "M": M, "K": c.K, "N": c.N,
                    "w8_us": us8, "w8_gbs": (w8_bytes + 2 * M * (c.K + c.N)) / us8 / 1e3,
                    "w8_frac_of_hbm": (w8_bytes + 2 * M * (c.K + c.N)) / us8 / 1e3 / load_peaks()[0]["hbm_gbs"],
                    "bf16_cublas_us": us16, "w8_speedup_vs_bf16": us16 / us8,
                    "w4_us": us4, "w4_speedup_vs_bf16": us16 / us4,
                    "fault": w4.device_fault()}
            print(json.dumps(line), flush=True)
            del X, Y, ws
        del p8, W16
        torch.cuda.empty_cache()


def run_groups(which: str):
    """Quantisation groups of 32, 64 and 128 weights, one JSON line per layer and token count: device
    time per call (w4a16_linear_g), each call reading a different copy of the packed weights past L2,
    replayed from a CUDA graph.  "decode": the hidden-5120 shapes at M = 1 (GB/s of code bytes and of
    all weight bytes, codes + 6 B of metadata per group); "batched": the hidden-8192 shapes at M in
    {4, 16, 40, 512} (GB/s of code bytes, and TFLOP/s at M = 512); "all": both."""
    import torch
    import weight_only_int4_linear_b200 as w4
    w4.load()
    stream = torch.cuda.Stream()
    runs = []
    if which in ("decode", "all"):
        runs += [(c, [1]) for c in workloads.decode_5120()]
    if which in ("batched", "all"):
        runs += [(c, [4, 16, 40, 512]) for c in workloads.small_batch_8192(ms=[2])]
    for c0, ms in runs:
        W = torch.empty((c0.N, c0.K), dtype=torch.float32, device="cuda")
        synth.fill_weights_device(c0.w_seed, c0.w_tag, W.data_ptr(), c0.N * c0.K, stream=stream.cuda_stream)
        packs = {}
        for group in (128, 64, 32):
            wbytes = c0.code_bytes + c0.N * (c0.K // group) * 6
            copies = max(1, min(16, -(-3 * L2_BYTES // wbytes)))
            pws = []
            with torch.cuda.stream(stream):
                for _ in range(copies):
                    pw = w4.PackedWeight(c0.N, c0.K, group=group)
                    pw.status = torch.zeros(1, dtype=torch.int32, device="cuda")
                    w4.quantize_pack_g(W, group, pw.qweight, pw.scales, pw.zeros, pw.status, stream=stream)
                    pws.append(pw)
            torch.cuda.synchronize()
            if any(int(p.status.item()) != 0 for p in pws):
                raise RuntimeError(f"packing failed for {c0.name}, group {group}")
            packs[group] = (pws, wbytes)
        del W
        torch.cuda.empty_cache()
        for M in ms:
            name = c0.name.rsplit("_m", 1)[0]
            xb = synth.activations_bf16(c0.x_seed + M, M, c0.K)
            X = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
            Y = torch.empty((M, c0.N), dtype=torch.bfloat16, device="cuda")
            line = {"groups": c0.workload, "layer": name, "M": M, "K": c0.K, "N": c0.N}
            for group in (128, 64, 32):
                pws, wbytes = packs[group]
                ws = torch.zeros(max(w4.workspace_bytes_g(M, c0.N, c0.K, group), 256), dtype=torch.uint8,
                                 device="cuda")
                passes = max(1, -(-200 // len(pws))) if M < 512 else 1

                def body(pws=pws, group=group, ws=ws):
                    for _ in range(passes):
                        for p in pws:
                            w4.linear_g(X, group, p.qweight, p.scales, p.zeros, Y, ws)
                us = _time_graph(torch, stream, body, passes * len(pws))
                line.update({f"g{group}_us": us, f"g{group}_code_gbs": c0.code_bytes / us / 1e3,
                             f"g{group}_all_gbs": wbytes / us / 1e3})
                if M >= 64:
                    line[f"g{group}_tflops"] = 2 * M * c0.N * c0.K / us / 1e6
                del ws
            line["fault"] = w4.device_fault()
            print(json.dumps(line), flush=True)
            del X, Y
        del packs
        torch.cuda.empty_cache()


def run_sweep(which: str):
    """Per-layer device time of every workload shape (one JSON line each): each
    call reads a different copy of the packed weights, rotating through enough
    copies that their codes exceed 3x L2, replayed from a CUDA graph."""
    import torch
    import weight_only_int4_linear_b200 as w4
    w4.load()
    stream = torch.cuda.Stream()
    peaks, peak_src = load_peaks()
    sets = {"single_gemv": workloads.single_gemv(), "decode": workloads.decode_5120(),
            "small": workloads.small_batch_8192(), "prefill": workloads.prefill_8192()}
    names = list(sets) if which == "all" else which.split(",")
    for wl in names:
        for c in sets[wl]:
            us, copies = time_layer_alone(c, torch, w4, stream)
            fault = w4.device_fault()
            line = {"sweep": c.workload, "layer": c.name, "M": c.M, "K": c.K, "N": c.N, "us_per_call": us,
                    "code_gbs": c.code_bytes / us / 1e3, "all_bytes_gbs": (c.code_bytes + c.meta_bytes) / us / 1e3,
                    "tflops": c.flops / us / 1e6, "frac_hbm": c.code_bytes / us / 1e3 / peaks["hbm_gbs"],
                    "frac_bf16": c.flops / us / 1e6 / peaks["bf16_tflops"], "weight_copies": copies,
                    "fault": fault}
            print(json.dumps(line), flush=True)
            if fault:
                raise SystemExit(1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--prefill-steps", type=int, default=3)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--stack-steps", type=int, default=20)
    ap.add_argument("--no-stack", action="store_true")
    ap.add_argument("--no-tables", action="store_true", help="skip the single-GEMV, small-batch and other-M tables")
    ap.add_argument("--protocol-seconds", type=float, default=1.0,
                    help="device seconds of repeated step blocks around the timed region (spread and clocks)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--ref-seconds", type=float, default=90.0,
                    help="reference arm: approximate host seconds for warm-up + timed steps")
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per launch of the dominant kernel, from an ncu capture of the current sources")
    ap.add_argument("--profile", default=None,
                    help="workload:layer (e.g. decode:gate_up, prefill:o_proj_m4096, decode:all, w8:gate_up): run it a few "
                         "times, untimed")
    ap.add_argument("--comparators", default=None,
                    help="decode|prefill|all: the unfused pipelines (offline dequant + GEMM, naive three kernels) "
                         "timed beside the fused path, one JSON line per layer")
    ap.add_argument("--w8", default=None,
                    help="decode, or a comma list of token counts: W8A16 layers timed beside W4A16 and a cuBLAS "
                         "BF16 GEMM on the decode shapes, one JSON line each")
    ap.add_argument("--groups", default=None,
                    help="decode|batched|all: quantisation groups of 32, 64 and 128 timed on the decode shapes "
                         "(M = 1) and the hidden-8192 shapes (M = 4, 16, 40, 512), one line each")
    ap.add_argument("--variants", default=None,
                    help="decode|small_batch|prefill|all: affine, symmetric-packed and AWQ-folded layers timed "
                         "on the same kernels, one JSON line per layer")
    ap.add_argument("--sweep", default=None,
                    help="all, or a comma list of single_gemv, decode, small, prefill: per-layer times, one line each")
    args = ap.parse_args()
    if args.comparators:
        run_comparators(args.comparators)
        return
    if args.variants:
        run_variants(args.variants)
        return
    if args.groups:
        run_groups(args.groups)
        return
    if args.w8:
        run_w8(args.w8)
        return
    if args.sweep:
        run_sweep(args.sweep)
        return
    if args.profile:
        run_profile(args.profile)
        return
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
