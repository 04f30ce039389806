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


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


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
    """Our kernels per linear call: X preparation + GEMM (M >= 64), else
    X preparation + GEMV per 32-token chunk."""
    if c.M >= PREFILL_MIN_M:
        return 2
    return 2 * ((c.M + 31) // 32)


class ExternalEvents:
    """CUDA events recorded as external event nodes inside a captured graph, so
    each replay times the kernels between them (cudaEventRecordExternal)."""

    def __init__(self, n):
        from cuda.bindings import runtime as rt
        self.rt = rt
        self.ev = []
        for _ in range(n):
            err, e = rt.cudaEventCreate()
            assert int(err) == 0, err
            self.ev.append(e)

    def record(self, i, stream_handle):
        err, = self.rt.cudaEventRecordWithFlags(self.ev[i], self.rt.cudaStream_t(stream_handle),
                                                 self.rt.cudaEventRecordExternal)
        assert int(err) == 0, err

    def elapsed(self, i, j):
        err, ms = self.rt.cudaEventElapsedTime(self.ev[i], self.ev[j])
        assert int(err) == 0, err
        return ms

    def close(self):
        for e in self.ev:
            self.rt.cudaEventDestroy(e)


def _linear_call(w4, L, path):
    w4.linear(L["X"], L["pw"].qweight, L["pw"].scales, L["pw"].zeros, L["Y"], L["ws"], path=path)


def capture(torch, stream, body):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        body()
    return g


def time_steps(layers, steps, warmup, torch, w4, stream, path, block=50):
    """Device time of exactly `steps` passes over the layer set, replayed from CUDA
    graphs of `block` steps (launch overhead off the timed path)."""
    with torch.cuda.stream(stream):
        for _ in range(max(warmup, 1)):
            for L in layers:
                _linear_call(w4, L, path)
    torch.cuda.synchronize()
    block = max(1, min(block, steps))
    full, rest = divmod(steps, block)

    def body(n):
        def f():
            for _ in range(n):
                for L in layers:
                    _linear_call(w4, L, path)
        return f

    g_full = capture(torch, stream, body(block))
    g_rest = capture(torch, stream, body(rest)) if rest else None
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


def time_per_layer(layers, torch, w4, stream, path, steps=20, replays=5):
    """Mean device time of each layer's call inside the real step sequence
    (external event nodes around every call of a captured multi-step graph)."""
    n = len(layers)
    ev = ExternalEvents(2 * n * steps)

    def body():
        h = torch.cuda.current_stream().cuda_stream
        for s in range(steps):
            for i, L in enumerate(layers):
                ev.record(2 * (s * n + i), h)
                _linear_call(w4, L, path)
                ev.record(2 * (s * n + i) + 1, h)

    g = capture(torch, stream, body)
    times = [[] for _ in range(n)]
    for _ in range(replays):
        with torch.cuda.stream(stream):
            g.replay()
        torch.cuda.synchronize()
        for s in range(1, steps):  # first step of a replay follows the idle host gap
            for i in range(n):
                times[i].append(ev.elapsed(2 * (s * n + i), 2 * (s * n + i) + 1))
    del g
    ev.close()
    return [statistics.mean(t) for t in times]


def time_e2e(layers, steps, warmup, torch, w4, stream, path):
    """Public-API calls with host buffers: pinned H2D of X and D2H of Y every step."""
    xs = [torch.from_numpy(L["x_host"].view(np.int16)).pin_memory() for L in layers]
    ys = [torch.empty((L["case"].M, L["case"].N), dtype=torch.int16).pin_memory() for L in layers]

    def one_step():
        for L, xh, yh in zip(layers, xs, ys):
            L["X"].view(torch.int16).copy_(xh, non_blocking=True)
            _linear_call(w4, L, path)
            yh.copy_(L["Y"].view(torch.int16), non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            one_step()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(steps):
            one_step()
        end.record(stream)
    torch.cuda.synchronize()
    h2d = sum(L["X"].numel() * 2 for L in layers)
    d2h = sum(L["Y"].numel() * 2 for L in layers)
    return start.elapsed_time(end), h2d, d2h


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

    cases = workloads.decode_5120()
    layers = setup_layers(cases, torch, w4, stream)
    code_bytes = sum(c.code_bytes for c in cases)
    all_bytes = sum(c.code_bytes + c.meta_bytes + 2 * c.M * (c.K + c.N) for c in cases)

    # warm-up + timed region (device time, CUDA events on the launching stream)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        total_ms = time_steps(layers, args.steps, args.warmup, torch, w4, stream, w4.PATH_AUTO)
    if world > 1:
        t = torch.tensor([total_ms], device="cuda")
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        total_ms = float(t.item())
    value = world * code_bytes * args.steps / (total_ms * 1e-3) / 1e9
    per_layer = time_per_layer(layers, torch, w4, stream, w4.PATH_AUTO)
    fault = w4.device_fault()
    if fault != 0:
        raise RuntimeError(f"a kernel gave up a bounded wait (site {fault}); results invalid")

    # dominant kernel: the largest layer (gate+up)
    dom = max(range(len(cases)), key=lambda i: cases[i].code_bytes)
    dom_ms = per_layer[dom]
    dom_gbs = cases[dom].code_bytes / (dom_ms * 1e-3) / 1e9
    dom_all = (cases[dom].code_bytes + cases[dom].meta_bytes) / (dom_ms * 1e-3) / 1e9

    # end to end through the public API with host buffers
    e2e_ms, h2d, d2h = time_e2e(layers, args.steps, args.warmup, torch, w4, stream, w4.PATH_AUTO)
    e2e_value = world * code_bytes * args.steps / (e2e_ms * 1e-3) / 1e9
    del layers
    torch.cuda.empty_cache()

    # prefill layer set at M = 4096 (hidden-8192 shapes)
    prefill = None
    if not args.no_prefill:
        pcases = workloads.prefill_8192(ms=[4096])
        players = setup_layers(pcases, torch, w4, stream)
        p_ms = time_steps(players, args.prefill_steps, 1, torch, w4, stream, w4.PATH_AUTO, block=1)
        p_layer = time_per_layer(players, torch, w4, stream, w4.PATH_AUTO, steps=2, replays=2)
        flops = sum(c.flops for c in pcases)
        tflops = flops * args.prefill_steps / (p_ms * 1e-3) / 1e12
        pdom = max(range(len(pcases)), key=lambda i: pcases[i].flops)
        pdom_tf = pcases[pdom].flops / (p_layer[pdom] * 1e-3) / 1e12
        prefill = {"value": tflops, "unit": "TFLOP/s", "workload": "prefill_hidden8192_m4096",
                   "ms_per_step": p_ms / args.prefill_steps, "steps": args.prefill_steps,
                   "frac_of_bf16_peak": tflops / peaks["bf16_tflops"],
                   "roofline": {"bound": "tensor", "kernel": f"linear {pcases[pdom].name}",
                                "achieved": pdom_tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                "frac": pdom_tf / peaks["bf16_tflops"], "peak_source": peak_src}}
        del players
        torch.cuda.empty_cache()

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
                   "l2": f"inputs larger than L2: {all_bytes / 1e6:.0f} MB read per step vs "
                         f"{L2_BYTES / 1e6:.0f} MB L2, layers run in sequence"},
        "frac_of_hbm_peak": value / world / peaks["hbm_gbs"],
        "all_bytes_gbs": world * all_bytes * args.steps / (total_ms * 1e-3) / 1e9,
        "roofline": {"bound": "hbm", "kernel": f"decode GEMV on {cases[dom].name} "
                                                f"({cases[dom].K}x{cases[dom].N})",
                     "achieved": dom_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": dom_gbs / peaks["hbm_gbs"], "traffic": args.traffic,
                     "achieved_all_bytes": dom_all, "per_launch_ms": dom_ms,
                     "algorithmic_bytes_per_launch": cases[dom].code_bytes, "peak_source": peak_src},
        "per_layer_ms": {c.name: ms for c, ms in zip(cases, per_layer)},
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms / args.steps},
        "prefill": prefill,
        "gpu_launches": launches,
        "cpu_baseline": cpu,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------------------------
# reference arm: the FP64 oracle on the host cores, same workload, metric and unit
# ----------------------------------------------------------------------------------------------

def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    cases = workloads.decode_5120()
    cpu, dt = cpu_baseline(cases, budget_s=max(5.0, min(60.0, args.cpu_budget)))
    steps_equiv = cpu["value"]
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": steps_equiv,
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": sum(c.code_bytes for c in cases) / (cpu["value"] * 1e9) * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (same seeded workload)",
        "config": {"workload": "decode_hidden5120_m1", "M": 1, "shapes_KxN": [[c.K, c.N] for c in cases],
                   "group": 128},
        "cpu_baseline": cpu,
        "e2e": {"value": cpu["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_profile(spec: str, repeats: int = 4):
    """Run one layer of a workload a few times (for an ncu capture; no timing)."""
    import torch
    import weight_only_int4_linear_b200 as w4
    w4.load()
    wl, name = spec.split(":")
    cases = {"decode": workloads.decode_5120(), "small": workloads.small_batch_8192(),
             "prefill": workloads.prefill_8192()}[wl]
    case = [c for c in cases if c.name == name][0]
    stream = torch.cuda.Stream()
    L = setup_layers([case], torch, w4, stream)[0]
    with torch.cuda.stream(stream):
        for _ in range(repeats):
            _linear_call(w4, L, w4.PATH_AUTO)
    torch.cuda.synchronize()
    fault = w4.device_fault()
    print(json.dumps({"profiled": spec, "repeats": repeats, "fault": fault}))
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
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per launch of the dominant kernel from an ncu capture of this build")
    ap.add_argument("--profile", default=None,
                    help="workload:layer (e.g. decode:gate_up, prefill:o_proj_m4096): run it a few times, untimed")
    args = ap.parse_args()
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
