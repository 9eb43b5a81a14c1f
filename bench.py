#!/usr/bin/env python
"""Benchmark of the ConvRot W4A4 linear layer on B200.

One step = the whole online hot path over one batch of the DiT MLP in edit
mode (two images): for the up projection X [8192, 3072] -> W [12288, 3072]
and then the down projection X [8192, 12288] (post-GELU values) -> W
[3072, 12288], each layer rotates X and quantises it dynamically to INT4
(one activation kernel, or two for tensors that do not fit on chip) and runs
the INT4 GEMM with the scale, bias and bf16 epilogue (one kernel).  The
offline weight packing is timed separately and reported, not counted in the
step.  Inputs are seeded synthetic draws of the model cards' shapes (the real
weights are not available); the timed loop rotates over input sets whose total
size is more than three times the L2 size.

``rows`` time every other configuration the same way, each for at least
200 ms: the DiT attention projection, each DiT MLP layer alone, the four
text-encoder projections (21 and 130 tokens, weight-bandwidth bound, with an
HBM roofline), the tiny parity case, shared activation quantisation for
split Q/K/V projections, the W4A8 asymmetric group-16 format, INT8
tensorwise + ConvRot and the INT8 branch of the W4A4 weights.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: the layer does not shard across GPUs (one GPU per layer), so N>1
runs N independent replicas, one process per GPU under torchrun; the time is
the max over ranks and the value counts the work of all ranks.

`--impl reference` times the CPU oracle (a plain float64/integer numpy
implementation) on a bounded sample of the same workload on this machine's
host cores; it is a deliberately slow baseline, not a target.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import platform
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A4 ConvRot linear TOPS and % of INT8 tensor/HBM roofline on 1 B200"
WORKLOAD = "dit_mlp"
# A step of the headline workload: the DiT MLP's two projections, up then down.
STEP_LAYERS = {"dit_mlp": ("dit_mlp_up", "dit_mlp_down")}
UNIT = "TOP/s"
# Recipe's nominal dense ratio int8 : bf16 on B200 (4.5 : 2.25 POPS/PFLOPS).
INT8_PER_BF16 = 2.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
MIN_TIMED_MS = 200.0   # every row (and the sustained headline run) times at least this long
MIN_PART_LAUNCHES = 50  # per-kernel split: at least this many launches of each kernel

CSRC = os.path.join(ROOT, "w4a8_rotated_quantized_b200", "csrc")
PAIR_SOURCES = [os.path.join(CSRC, f) for f in ("gemm_w4a4_pair.cu", "cr_device.cuh")]
SMALL_SOURCES = [os.path.join(CSRC, f) for f in ("gemm_w4a4_small.cu", "cr_device.cuh")]
GEMM_PROFILE = os.path.join(ROOT, "profiles", "gemm_w4a4_dit_mlp.json")
GEMM_SOURCES = PAIR_SOURCES
# ncu summaries (DRAM bytes per launch) of the dominant kernel of each row, keyed to the sources they
# were taken on: a row reports `traffic` only while its kernel's sources are unchanged.
ROW_PROFILES = {
    "dit_attn": (os.path.join(ROOT, "profiles", "gemm_w4a4_dit_attn.json"), PAIR_SOURCES),
    "int8_convrot": (os.path.join(ROOT, "profiles", "gemm_i8_dit_attn.json"),
                     [os.path.join(CSRC, f) for f in ("gemm_i8.cu", "cr_device.cuh")]),
    "w4a8_asym_g16": (os.path.join(ROOT, "profiles", "gemm_w4a8_w4a8_up.json"),
                      [os.path.join(CSRC, f) for f in ("gemm_w4a8.cu", "cr_device.cuh")]),
    "int8_branch_w4": (os.path.join(ROOT, "profiles", "gemm_a8w4_dit_attn.json"),
                       [os.path.join(CSRC, f) for f in ("gemm_a8w4.cu", "cr_device.cuh")]),
}
# The few-token rows' GEMMs: one summary per kernel, DRAM bytes per launch for each workload it serves.
FEW_TOKEN_PROFILES = {
    "small": (os.path.join(ROOT, "profiles", "gemm_w4a4_small_text_enc.json"), SMALL_SOURCES),
    "pair": (os.path.join(ROOT, "profiles", "gemm_w4a4_pair_text_enc_up_130.json"), PAIR_SOURCES),
}


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=400)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=WORKLOAD, help=argparse.SUPPRESS)
    p.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timings (profiling runs)")
    p.add_argument("--e2e-steps", type=int, default=20)
    p.add_argument("--no-rows", action="store_true", help="skip the other configurations (profiling runs)")
    p.add_argument("--rows", default="", help="comma-separated subset of rows to run")
    return p.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def sources_sha256(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profile_traffic(profile, sources, workload=None):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current source (for a
    summary of several workloads, the entry of `workload`)."""
    if not os.path.exists(profile):
        return None
    with open(profile) as f:
        prof = json.load(f)
    if prof.get("source_sha256") != sources_sha256(sources):
        return None
    if workload is not None:
        return prof.get("per_workload", {}).get(workload, {}).get("dram_bytes_per_launch")
    return prof.get("dram_bytes_per_launch")


def few_token_gemm(M, N, num_sms):
    """The GEMM kernel cr_w4a4_gemm runs for M tokens x N outputs (the library's dispatch rule): the
    few-token kernel up to 128 tokens, and up to 256 when its 128-row weight tiles leave room for a K
    split of two or more on the SMs; else the CTA-pair kernel."""
    small = M <= 128 or (M <= 256 and 2 * ((N + 127) // 128) <= num_sms)
    return "small" if small else "pair"


def gemm_traffic_per_launch():
    return profile_traffic(GEMM_PROFILE, GEMM_SOURCES)


def step_layers(workload):
    return STEP_LAYERS.get(workload, (workload,))


# ---------------------------------------------------------------------------
# distributed plumbing (replicas only; no data-path collective)
# ---------------------------------------------------------------------------

def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


def max_over_ranks(value: float, device) -> float:
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        if device is not None and getattr(device, "type", "cpu") == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            import tempfile

            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", self.gpu_id], stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.out.close()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as f:
            for ln in f:
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        sm = [r[0] for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[2]) if v.lower().startswith("active")})
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ---------------------------------------------------------------------------

def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("internal_api") in ("openblas", "mkl", "blis")]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.lower().startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def host_info():
    return {"cores": blas_threads(), "nproc": os.cpu_count(), "cpu_model": cpu_model()}


def oracle_layer_fn(kind, d, K):
    """(step(rows) -> None) running the oracle's whole layer of one format on the given X rows.

    The weights are prepared once by the oracle's own offline path (not timed)."""
    import oracle

    if kind == "w4a4":
        wq, s_w, _, _ = oracle.pack_weight(d["W"])
        return lambda xs: oracle.w4a4_linear(xs, wq, s_w, d["bias"])
    if kind == "int8":
        qw, s_w, _ = oracle.pack_weight8(d["W"])
        return lambda xs: oracle.int8_linear(xs, qw, s_w, d["bias"])
    if kind == "a8w4":
        wq, s_w, _, _ = oracle.pack_weight(d["W"])
        return lambda xs: oracle.a8w4_linear(xs, wq, s_w, d["bias"])
    if kind == "w4a8":
        p = oracle.pack_weight_w4a8(d["W"])
        return lambda xs: oracle.w4a8_linear(xs, p["q"], p["s"], p["z"], d["bias"])
    raise ValueError(kind)


def time_oracle(layers, rows_per_step, budget_s, max_steps=64):
    """Run the oracle on `rows_per_step` token rows of every layer per step, for about budget_s seconds.

    `layers` is a list of (step_fn, X bits, N, K, ops multiplier).  Returns (ops/s, steps, seconds)."""
    for fn, X, N, K, mult in layers:  # warm-up (BLAS thread pool, page faults)
        fn(X[:min(rows_per_step, X.shape[0])])
    t0 = time.perf_counter()
    ops, steps = 0.0, 0
    while True:
        for fn, X, N, K, mult in layers:
            M = X.shape[0]
            r0 = (steps * rows_per_step) % M
            xs = X[r0:r0 + rows_per_step]
            fn(xs)
            ops += mult * 2.0 * xs.shape[0] * N * K
        steps += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s or steps >= max_steps:
            return ops / dt, steps, dt


def cpu_baseline(layer_specs, budget_s, rows_per_step, unit=UNIT, scale=1e12):
    """The oracle as it stands on this host's cores, on a bounded sample of a workload.

    layer_specs: [(kind, workload name or dict of inputs, ops multiplier)]."""
    from w4a8_rotated_quantized_b200 import workloads

    layers, names = [], []
    for kind, w, mult in layer_specs:
        if isinstance(w, str):
            names.append(w)
            d = workloads.make_inputs(w)
        else:
            names.append(w["name"])
            d = w
        X = d["X"]
        N, K = d["W"].shape
        layers.append((oracle_layer_fn(kind, d, K), X, N, K, mult))
    rate, steps, dt = time_oracle(layers, rows_per_step, budget_s)
    out = {"value": rate / scale, "unit": unit, "kind": "oracle",
           "sample": f"{steps} oracle steps, each the whole layer on {rows_per_step} token rows of "
                     f"{' + '.join(names)} (full K and N), {dt:.1f} s"}
    out.update(host_info())
    return out


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from w4a8_rotated_quantized_b200 import workloads

    names = step_layers(args.workload)
    # rows per step sized so that warm-up + timed steps stay within about a minute of CPU work
    rows = int(max(4, min(128, 4096 // max(1, args.steps + args.warmup))))
    layers = []
    for n in names:
        d = workloads.make_inputs(n)
        N, K = d["W"].shape
        layers.append((oracle_layer_fn("w4a4", d, K), d["X"], N, K))

    def step(i):
        ops = 0.0
        for fn, X, N, K in layers:
            r0 = (i * rows) % X.shape[0]
            xs = X[r0:r0 + rows]
            fn(xs)
            ops += 2.0 * xs.shape[0] * N * K
        return ops

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    ops = 0.0
    for i in range(args.steps):
        ops += step(args.warmup + i)
    dt = time.perf_counter() - t0
    value = ops / dt / 1e12
    ws = [workloads.CONFIGS[n] for n in names]
    cpu = {"value": value, "unit": UNIT, "kind": "oracle",
           "sample": f"each step: the whole layer on {rows} token rows of {' + '.join(names)} (full K and N)"}
    cpu.update(host_info())
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / max(1, args.steps) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.workload}: " + "; ".join(w.description for w in ws),
                   "layers": [{"name": w.name, "M": w.M, "N": w.N, "K": w.K} for w in ws],
                   "sample_rows_per_step": rows},
        "cpu_baseline": cpu,
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU timing helpers
# ---------------------------------------------------------------------------

def graph_kernel_nodes(g):
    """Kernel nodes of a captured CUDA graph (our launches: the step issues no library kernel)."""
    try:
        from cuda.bindings import runtime as rt

        graph = g.raw_cuda_graph()
        err, _, n = rt.cudaGraphGetNodes(graph, 0)
        if int(err) != 0:
            return None
        err, nodes, n = rt.cudaGraphGetNodes(graph, n)
        if int(err) != 0:
            return None
        kinds = [rt.cudaGraphNodeGetType(nd)[1] for nd in nodes]
        return sum(1 for k in kinds if k == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel)
    except Exception:
        return None


def capture_graph(torch, stream, body):
    try:
        g = torch.cuda.CUDAGraph(keep_graph=True)
    except TypeError:
        g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        body()
    return g


class Timed:
    """A sequence of launches over R rotating input sets: `parts` = [(name, fn(r))], one step = every
    part once on set r.  Captures one graph per step, one graph of all R steps, and one graph per
    part over all R sets."""

    def __init__(self, torch, stream, parts, R, warmup=3):
        self.torch, self.stream, self.parts, self.R = torch, stream, parts, R
        with torch.cuda.stream(stream):
            for i in range(max(1, warmup)):  # eager warm-up: per-device setup happens outside any capture
                for _, f in parts:
                    f(i % R)
        stream.synchronize()
        self.g_steps = [capture_graph(torch, stream, lambda r=r: [f(r) for _, f in parts]) for r in range(R)]
        self.g_cycle = capture_graph(torch, stream, lambda: [f(r) for r in range(R) for _, f in parts])
        self.g_parts = [capture_graph(torch, stream, lambda f=f: [f(r) for r in range(R)]) for _, f in parts]
        n = graph_kernel_nodes(self.g_steps[0])
        self.launches_per_step = n
        # a graph's first replay also uploads it to the device: replay every graph once before any timing
        with torch.cuda.stream(stream):
            for g in self.g_steps + [self.g_cycle] + self.g_parts:
                g.replay()
        stream.synchronize()

    def events(self):
        return self.torch.cuda.Event(enable_timing=True), self.torch.cuda.Event(enable_timing=True)

    def time_steps(self, k):
        """Exactly k steps (per-step graphs in order), device time in ms."""
        e0, e1 = self.events()
        with self.torch.cuda.stream(self.stream):
            e0.record(self.stream)
            for i in range(k):
                self.g_steps[i % self.R].replay()
            e1.record(self.stream)
        self.stream.synchronize()
        return e0.elapsed_time(e1)

    def time_sustained(self, min_ms=MIN_TIMED_MS):
        """Whole-cycle replays for at least min_ms and at least MIN_PART_LAUNCHES steps: (steps, ms)."""
        one = self.time_cycles(1)
        reps = max(math.ceil(min_ms / max(one, 1e-3)), math.ceil(MIN_PART_LAUNCHES / self.R), 1)
        return reps * self.R, self.time_cycles(reps)

    def time_cycles(self, reps):
        e0, e1 = self.events()
        with self.torch.cuda.stream(self.stream):
            self.g_cycle.replay()
            e0.record(self.stream)
            for _ in range(reps):
                self.g_cycle.replay()
            e1.record(self.stream)
        self.stream.synchronize()
        return e0.elapsed_time(e1)

    def time_parts(self):
        """Average device time of one launch of each part (us), from replays of per-part graphs with
        events between them: at least MIN_PART_LAUNCHES launches of each part."""
        torch = self.torch
        n = max(1, math.ceil(MIN_PART_LAUNCHES / self.R))
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(self.g_parts) + 1)] for _ in range(n)]
        with torch.cuda.stream(self.stream):
            for j in range(n):
                ev[j][0].record(self.stream)
                for i, g in enumerate(self.g_parts):
                    g.replay()
                    ev[j][i + 1].record(self.stream)
        self.stream.synchronize()
        return {name: sum(e[i].elapsed_time(e[i + 1]) for e in ev) / (n * self.R) * 1e3
                for i, (name, _) in enumerate(self.parts)}, n * self.R

    def release(self):
        del self.g_steps, self.g_cycle, self.g_parts


def rotations(l2, set_bytes):
    """Rotating input sets: enough that they hold more than three times the L2 size."""
    return max(2, math.ceil(3 * l2 / set_bytes))


def dev_bf16(torch, device, bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


class Env:
    """Library handle, shared workspace and a private stream for the pre-marshalled C-ABI calls."""

    def __init__(self, torch, device):
        from w4a8_rotated_quantized_b200 import binding

        self.torch, self.device, self.b = torch, device, binding
        self.lib, self.P = binding._lib, binding._ptr
        self.l2 = torch.cuda.get_device_properties(device).L2_cache_size
        # zeroed workspace of the bench's own calls: the one-call layers keep the activation codes in
        # it (at most 4096 x 3072 / 2 bytes in these rows)
        self.ws = torch.zeros(32 << 20, dtype=torch.uint8, device=device)
        self.wsp, self.wsn = self.P(self.ws), self.ws.numel()
        self.stream = torch.cuda.Stream(device)
        self.sp = binding.ctypes.c_void_p(self.stream.cuda_stream)

    def call(self, fn, args):
        st = fn(*args)
        if st:
            raise self.b.ConvRotError(fn.__name__, st)

    def status(self):
        """The device status word of this workspace (synchronises the stream)."""
        st = self.b.ctypes.c_int(0)
        self.call(self.lib.cr_read_device_status, (self.wsp, self.b.ctypes.byref(st), self.sp))
        return st.value


def w4a4_layer(env, wname, R=None, seed_base=1000, extra_bytes=0):
    """R rotating input sets of one W4A4 layer (own X draw and rolled weight rows per set) and the
    pre-marshalled calls: act(r) = cr_rotate_quant_act, gemm(r) = cr_w4a4_gemm."""
    import w4a8_rotated_quantized_b200 as cr
    from w4a8_rotated_quantized_b200 import workloads

    torch, device = env.torch, env.device
    w = workloads.CONFIGS[wname]
    M, N, K = w.M, w.N, w.K
    d = workloads.make_inputs(w)
    X0, W0, B0 = dev_bf16(torch, device, d["X"]), dev_bf16(torch, device, d["W"]), dev_bf16(torch, device, d["bias"])
    set_bytes = M * K * 2 + M * K // 2 + M * N * 2 + N * K // 2
    if R is None:
        R = rotations(env.l2, set_bytes + extra_bytes)
    sets = []
    for r in range(R):
        X = X0 if r == 0 else dev_bf16(torch, device, workloads.make_inputs(w, with_weight=False, seed=seed_base + r)["X"])
        Wq, s_w = cr.cr_pack_weight(W0 if r == 0 else W0.roll(r, dims=0))
        Xq = torch.empty((M, K // 2), dtype=torch.uint8, device=device)
        s_a = torch.empty((1,), dtype=torch.float32, device=device)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        sets.append((X, Wq, s_w, Xq, s_a, Y))
    torch.cuda.synchronize()
    P = env.P
    acts = [(P(X), M, K, K, 256, P(Xq), P(s_a), env.wsp, env.wsn, env.sp) for (X, Wq, s_w, Xq, s_a, Y) in sets]
    gemms = [(P(Xq), P(s_a), P(Wq), P(s_w), P(B0), P(Y), N, M, N, K, env.wsp, env.wsn, env.sp)
             for (X, Wq, s_w, Xq, s_a, Y) in sets]
    lins = [(P(X), K, P(Wq), P(s_w), P(B0), P(Y), N, M, N, K, 256, env.wsp, env.wsn, env.sp)
            for (X, Wq, s_w, Xq, s_a, Y) in sets]
    lins_one = [(P(X), K, P(Wq), P(s_w), P(B0), P(Y), N, M, N, K, 256, 1, env.wsp, env.wsn, env.sp)
                for (X, Wq, s_w, Xq, s_a, Y) in sets]  # cr_w4a4_linear_ex, mode CR_LINEAR_ONE_LAUNCH
    lins_two = [(P(X), K, P(Wq), P(s_w), P(B0), P(Y), N, M, N, K, 256, 2, env.wsp, env.wsn, env.sp)
                for (X, Wq, s_w, Xq, s_a, Y) in sets]  # cr_w4a4_linear_ex, mode CR_LINEAR_TWO_LAUNCHES
    lib = env.lib
    if lib.cr_w4a4_linear_workspace_size(M, N, K, 256) > env.wsn:
        lins = None  # the one-call layer keeps the codes in the workspace: only for inputs that fit it
    return {
        "w": w, "d": d, "R": R, "sets": sets, "W0": W0, "B0": B0, "set_bytes": set_bytes,
        "act": lambda r: env.call(lib.cr_rotate_quant_act, acts[r]),
        "gemm": lambda r: env.call(lib.cr_w4a4_gemm, gemms[r]),
        "linear": None if lins is None else (lambda r: env.call(lib.cr_w4a4_linear, lins[r])),
        "linear_one": None if lins is None else (lambda r: env.call(lib.cr_w4a4_linear_ex, lins_one[r])),
        "linear_two": None if lins is None else (lambda r: env.call(lib.cr_w4a4_linear_ex, lins_two[r])),
    }


def tensor_roofline(kernel, ops, us, peaks, peaks_kind, int8_meas, traffic=None):
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]) * INT8_PER_BF16
    achieved = ops / (us * 1e-6) / 1e12
    out = {"bound": "tensor", "kernel": kernel, "achieved": achieved, "peak": burst, "unit": UNIT,
           "frac": achieved / burst, "traffic": traffic,
           "peak_source": f"{peaks_kind} bf16 dense burst {peaks.get('bf16_tflops')} TFLOP/s x {INT8_PER_BF16} "
                          f"(nominal int8:bf16 ratio)",
           "algorithmic": "2*M*N*K integer ops per launch"}
    if int8_meas:
        out["frac_of_measured_int8_mm"] = achieved / int8_meas
    return out


def hbm_roofline(kernel, nbytes, us, peaks, peaks_kind, what, traffic=None):
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    achieved = nbytes / (us * 1e-6) / 1e9
    return {"bound": "hbm", "kernel": kernel, "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm, "traffic": traffic, "peak_source": f"{peaks_kind} HBM copy bandwidth",
            "algorithmic": what, "algorithmic_bytes_per_launch": nbytes}


def measure_int8_peak(torch, device):
    """Dense INT8 throughput of the library GEMM (torch._int_mm, cuBLASLt) on 8192^3: the measured
    INT8 tensor peak that the INT4/INT8 GEMMs are also reported against."""
    n = 8192
    g = torch.Generator(device=device).manual_seed(0)
    a = torch.randint(-128, 127, (n, n), dtype=torch.int8, device=device, generator=g)
    b = torch.randint(-128, 127, (n, n), dtype=torch.int8, device=device, generator=g)
    for _ in range(5):
        torch._int_mm(a, b.t())
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 20
    e0.record()
    for _ in range(reps):
        torch._int_mm(a, b.t())
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    del a, b
    return {"value": 2.0 * n ** 3 / (ms / 1e3) / 1e12, "unit": UNIT, "how": f"torch._int_mm int8 {n}^3, "
            f"{reps} launches after 5 warm-ups, CUDA events"}


# ---------------------------------------------------------------------------
# rows: every other configuration, timed like the headline
# ---------------------------------------------------------------------------

W4A4_ROWS = ("dit_attn", "dit_mlp_up", "dit_mlp_down", "text_enc_up_21", "text_enc_up_130", "text_enc_down_21",
             "text_enc_down_130", "tiny")
ALL_ROWS = W4A4_ROWS + ("qkv_shared_dit_attn", "w4a8_asym_g16", "int8_convrot", "int8_branch_w4")


def row_w4a4(env, name, peaks, peaks_kind, int8_meas, cpu):
    """One W4A4 layer.  More than 256 tokens: the activation pass and the CTA-pair GEMM (two launches,
    what cr_w4a4_linear runs), tensor roofline of the GEMM.  At most 256 tokens: the one-call layer as the
    library arranges it (cr_w4a4_linear: one launch with the activation phases fused into the few-token
    GEMM, or the activation pass and the few-token GEMM), HBM roofline of its dominant kernel; both
    arrangements are reported beside it (one launch forced through cr_w4a4_linear_ex; the two-launch
    split cr_rotate_quant_act + cr_w4a4_gemm)."""
    torch = env.torch
    L = w4a4_layer(env, name, seed_base=3000)
    w, R = L["w"], L["R"]
    M, N, K = w.M, w.N, w.K
    ops = 2.0 * M * N * K
    gemm_bytes = M * K / 2 + N * K / 2 + 4 * N + 2 * N + 2 * M * N + 4
    act_bytes = 2.0 * M * K + M * K / 2
    t = Timed(torch, env.stream, [("act", L["act"]), ("gemm", L["gemm"])], R)
    steps, ms = t.time_sustained()
    parts, n_part = t.time_parts()
    two = {
        "value": ops * steps / (ms / 1e3) / 1e12, "ms_per_step": ms / steps, "steps": steps, "timed_ms": ms,
        "kernels_us": {"act_rotate_quant": parts["act"], "w4a4_gemm": parts["gemm"]},
        "kernel_launches_timed": n_part,
        "act_path_GBps": act_bytes / (parts["act"] * 1e-6) / 1e9,
        "gpu_launches_per_step": t.launches_per_step,
    }
    t.release()
    small = M <= 256  # the one-call layer can run as one launch for at most 256 tokens
    out = {"workload": f"{w.name}: {w.description}", "M": M, "N": N, "K": K, "dtype": "s4",
           "l2": f"{R} rotating input sets of {L['set_bytes'] / 1e6:.1f} MB"}
    if small and L["linear"] is not None:
        fused_bytes = 2.0 * M * K + N * K / 2 + 4 * N + 2 * N + 2 * M * N
        kern = ("w4a4_gemm_small fused layer (rotation, scale and INT4 codes of X, then weights on the MMA M "
                "side with K split over a cluster; one launch)")
        to = Timed(torch, env.stream, [("layer", L["linear_one"])], R)
        osteps, oms = to.time_sustained()
        oparts, on = to.time_parts()
        one = {
            "api": "cr_w4a4_linear_ex, mode CR_LINEAR_ONE_LAUNCH", "value": ops * osteps / (oms / 1e3) / 1e12,
            "ms_per_step": oms / osteps, "steps": osteps, "timed_ms": oms,
            "kernels_us": {"w4a4_linear_fused": oparts["layer"]}, "kernel_launches_timed": on,
            "gpu_launches_per_step": to.launches_per_step,
            "roofline": hbm_roofline(kern, fused_bytes, oparts["layer"], peaks, peaks_kind,
                                     "X 2MK + Wq N*K/2 + w_scale 4N + bias 2N + Y 2MN bytes per launch"),
        }
        to.release()
        gk = few_token_gemm(M, N, torch.cuda.get_device_properties(env.device).multi_processor_count)
        two["gemm_roofline"] = hbm_roofline(
            "w4a4_gemm_small" if gk == "small" else "w4a4_gemm_pair (tcgen05 cta_group::2 kind::i8)", gemm_bytes,
            parts["gemm"], peaks, peaks_kind, "Xq M*K/2 + Wq N*K/2 + w_scale 4N + bias 2N + Y 2MN bytes per launch",
            profile_traffic(*FEW_TOKEN_PROFILES[gk], workload=name))
        # the one-call layer forced to two launches: the GEMM starts as a programmatic dependent of the pass
        tt = Timed(torch, env.stream, [("layer", L["linear_two"])], R)
        tsteps, tms = tt.time_sustained()
        two["one_call"] = {"api": "cr_w4a4_linear_ex, mode CR_LINEAR_TWO_LAUNCHES (the GEMM as a programmatic "
                                  "dependent of the activation pass)", "value": ops * tsteps / (tms / 1e3) / 1e12,
                           "ms_per_step": tms / tsteps, "steps": tsteps, "timed_ms": tms,
                           "gpu_launches_per_step": tt.launches_per_step}
        two["api"] = "cr_rotate_quant_act + cr_w4a4_gemm (two calls: no programmatic dependence)"
        tt.release()
        tf = Timed(torch, env.stream, [("layer", L["linear"])], R)
        fsteps, fms = tf.time_sustained()
        fparts, fn = tf.time_parts()
        arrangement = "one launch" if tf.launches_per_step == 1 else "two launches"
        out.update({
            "api": f"cr_w4a4_linear (the library's arrangement for this shape: {arrangement})",
            "arrangement": arrangement, "value": ops * fsteps / (fms / 1e3) / 1e12, "unit": UNIT,
            "ms_per_step": fms / fsteps, "steps": fsteps, "timed_ms": fms,
            "kernels_us": {"w4a4_linear": fparts["layer"]}, "kernel_launches_timed": fn,
            "gpu_launches_per_step": tf.launches_per_step,
            # the dominant kernel: the fused layer, or the few-token GEMM of the two-launch arrangement
            "roofline": one["roofline"] if tf.launches_per_step == 1 else two["gemm_roofline"],
            "one_launch": one,
            "two_launches": two,
        })
        tf.release()
    else:
        out.update(two)
        out.update({"api": "cr_rotate_quant_act + cr_w4a4_gemm (the kernels cr_w4a4_linear runs)", "unit": UNIT})
        if M <= 256:  # still bound by the weight stream: HBM roofline of the GEMM and of the whole layer
            out["roofline"] = hbm_roofline("w4a4_gemm_pair (tcgen05 cta_group::2 kind::i8)", gemm_bytes,
                                           parts["gemm"], peaks, peaks_kind,
                                           "Xq M*K/2 + Wq N*K/2 + w_scale 4N + bias 2N + Y 2MN bytes per launch")
            step_bytes = act_bytes + gemm_bytes
            hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
            out["layer_hbm"] = {"bytes_per_step": step_bytes, "achieved_GBps": step_bytes / (ms / steps * 1e-3) / 1e9,
                                "frac": step_bytes / (ms / steps * 1e-3) / 1e9 / hbm}
        else:
            prof = ROW_PROFILES.get(name)
            out["roofline"] = tensor_roofline("w4a4_gemm_pair (tcgen05 cta_group::2 kind::i8)", ops, parts["gemm"],
                                              peaks, peaks_kind, int8_meas, profile_traffic(*prof) if prof else None)
    if cpu:
        out["cpu_baseline"] = cpu_baseline([("w4a4", L["d"] | {"name": name}, 1)], 1.5, min(M, 64))
    del L
    torch.cuda.empty_cache()
    return out


def row_qkv(env, peaks, peaks_kind, int8_meas, cpu):
    """Shared activation quantisation for split projections: X [4096, 3072] of the DiT attention
    feeds three [3072, 3072] projections (query, key, value) through one rotation + quantisation
    and one GEMM launch over all their tiles; compared with three separate layers."""
    import w4a8_rotated_quantized_b200 as cr
    from w4a8_rotated_quantized_b200 import workloads

    torch, device, P, lib = env.torch, env.device, env.P, env.lib
    w = workloads.CONFIGS["dit_attn"]
    M, N, K = w.M, w.N, w.K
    d = workloads.make_inputs(w)
    rng = np.random.default_rng(77)
    Ws = [dev_bf16(torch, device, d["W"])] + [
        dev_bf16(torch, device, workloads.bf16_bits_from_f32((rng.standard_normal((N, K)) * 0.02).astype(np.float32)))
        for _ in range(2)]
    B0 = dev_bf16(torch, device, d["bias"])
    set_bytes = M * K * 2 + M * K // 2 + 3 * (M * N * 2 + N * K // 2)
    R = rotations(env.l2, set_bytes)
    sets = []
    for r in range(R):
        X = dev_bf16(torch, device, workloads.make_inputs(w, with_weight=False, seed=4000 + r)["X"])
        packed = [cr.cr_pack_weight(Wj.roll(r, dims=0)) for Wj in Ws]
        Xq = torch.empty((M, K // 2), dtype=torch.uint8, device=device)
        s_a = torch.empty((1,), dtype=torch.float32, device=device)
        Ys = [torch.empty((M, N), dtype=torch.bfloat16, device=device) for _ in range(3)]
        sets.append((X, packed, Xq, s_a, Ys))
    torch.cuda.synchronize()
    arr = lambda ts: (env.b.ctypes.c_void_p * 3)(*[t.data_ptr() for t in ts])
    i64 = (env.b.ctypes.c_int64 * 3)(N, N, N)
    i32 = (env.b.ctypes.c_int * 3)(N, N, N)
    acts, multis, seps = [], [], []
    for (X, packed, Xq, s_a, Ys) in sets:
        acts.append((P(X), M, K, K, 256, P(Xq), P(s_a), env.wsp, env.wsn, env.sp))
        multis.append((P(Xq), P(s_a), M, K, 3, arr([p[0] for p in packed]), arr([p[1] for p in packed]),
                       arr([B0, B0, B0]), arr(Ys), i64, i32, env.wsp, env.wsn, env.sp))
        seps.append([(P(X), K, P(p[0]), P(p[1]), P(B0), P(Y), N, M, N, K, 256, env.wsp, env.wsn, env.sp)
                     for p, Y in zip(packed, Ys)])
    t = Timed(torch, env.stream, [("act", lambda r: env.call(lib.cr_rotate_quant_act, acts[r])),
                                  ("gemm_multi", lambda r: env.call(lib.cr_w4a4_gemm_multi, multis[r]))], R)
    steps, ms = t.time_sustained()
    parts, n_part = t.time_parts()
    ops = 3 * 2.0 * M * N * K
    t2 = Timed(torch, env.stream, [("three_layers", lambda r: [env.call(lib.cr_w4a4_linear, a) for a in seps[r]])], R)
    steps2, ms2 = t2.time_sustained()
    out = {
        "workload": "DiT attention input X [4096,3072] (1% channels x50) -> query, key, value weights 3 x "
                    "[3072,3072]: one rotation + INT4 quantisation of X, one GEMM launch over all three",
        "M": M, "N": [N, N, N], "K": K, "dtype": "s4",
        "value": ops * steps / (ms / 1e3) / 1e12, "unit": UNIT, "ms_per_step": ms / steps, "steps": steps,
        "timed_ms": ms, "kernels_us": {"act_rotate_quant": parts["act"], "w4a4_gemm_multi": parts["gemm_multi"]},
        "kernel_launches_timed": n_part,
        "separate_layers_ms_per_step": ms2 / steps2,
        "separate_layers_value": ops * steps2 / (ms2 / 1e3) / 1e12,
        "roofline": tensor_roofline("w4a4_gemm_pair over three projections (one launch)", ops, parts["gemm_multi"],
                                    peaks, peaks_kind, int8_meas),
        "gpu_launches_per_step": t.launches_per_step,
        "l2": f"{R} rotating input sets of {set_bytes / 1e6:.1f} MB",
    }
    if cpu:
        # the oracle as it stands: the whole layer once per projection
        out["cpu_baseline"] = cpu_baseline([("w4a4", "dit_attn", 1)] * 3, 1.5, 32)
    t.release()
    t2.release()
    del sets
    torch.cuda.empty_cache()
    return out


def row_format(env, row, peaks, peaks_kind, int8_meas, cpu):
    """The further formats of the model cards, each timed like the headline step:
    * int8_convrot: INT8 tensorwise + ConvRot on the DiT attention projection;
    * w4a8_asym_g16: W4A8 (asymmetric 4-bit weights, group 16) on X [4096, 3072] Student-t ->
      W [12288, 3072], fp16 tensor-core GEMM with in-kernel dequantisation;
    * int8_branch_w4: INT8 activations against the packed INT4 weights of the W4A4 format."""
    import w4a8_rotated_quantized_b200 as cr
    from w4a8_rotated_quantized_b200 import workloads

    torch, device, P, lib = env.torch, env.device, env.P, env.lib
    wname = {"int8_convrot": "dit_attn", "w4a8_asym_g16": "w4a8_up", "int8_branch_w4": "dit_attn"}[row]
    w = workloads.CONFIGS[wname]
    M, N, K = w.M, w.N, w.K
    ops = 2.0 * M * N * K
    d = workloads.make_inputs(w)
    X0, W0, B0 = dev_bf16(torch, device, d["X"]), dev_bf16(torch, device, d["W"]), dev_bf16(torch, device, d["bias"])
    wbytes = {"int8_convrot": N * K, "w4a8_asym_g16": N * K // 2 + N * K // 16 * 2 + N * K // 32,
              "int8_branch_w4": N * K // 2}[row]
    set_bytes = M * K * 2 + M * K + M * N * 2 + wbytes
    R = rotations(env.l2, set_bytes)
    act_calls, gemm_calls, keep = [], [], []
    for r in range(R):
        X = X0 if r == 0 else dev_bf16(torch, device, workloads.make_inputs(w, with_weight=False, seed=2000 + r)["X"])
        Wr = W0 if r == 0 else W0.roll(r, dims=0)
        Xq = torch.empty((M, K), dtype=torch.int8, device=device)
        s_a = torch.empty((1,), dtype=torch.float32, device=device)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        act_calls.append((P(X), M, K, K, 256, 8, 1, P(Xq), P(s_a), env.wsp, env.wsn, env.sp))
        if row in ("int8_convrot", "int8_branch_w4"):
            Wq, s_w = cr.cr_pack_weight_ex(Wr, bits=8, rotate=True) if row == "int8_convrot" else cr.cr_pack_weight(Wr)
            gemm_calls.append((P(Xq), P(s_a), P(Wq), P(s_w), P(B0), P(Y), N, M, N, K, env.wsp, env.wsn, env.sp))
            keep.append((X, Wq, s_w, Xq, s_a, Y))
        else:
            Wq, gs, gz = cr.cr_pack_weight_w4a8(Wr)
            gemm_calls.append((P(Xq), P(s_a), P(Wq), P(gs), P(gz), P(B0), P(Y), N, M, N, K, env.wsp, env.wsn, env.sp))
            keep.append((X, Wq, gs, gz, Xq, s_a, Y))
    torch.cuda.synchronize()
    gemm_fn = {"int8_convrot": lib.cr_int8_gemm, "w4a8_asym_g16": lib.cr_w4a8_gemm,
               "int8_branch_w4": lib.cr_a8w4_gemm}[row]
    t = Timed(torch, env.stream, [("act", lambda r: env.call(lib.cr_rotate_quant_act_ex, act_calls[r])),
                                  ("gemm", lambda r: env.call(gemm_fn, gemm_calls[r]))], R)
    steps, ms = t.time_sustained()
    parts, n_part = t.time_parts()
    prof = ROW_PROFILES.get(row)
    if row == "w4a8_asym_g16":
        peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        achieved = ops / (parts["gemm"] * 1e-6) / 1e12
        roof = {"bound": "tensor", "kernel": "w4a8_gemm (tcgen05 kind::f16, CTA pair, in-kernel dequantisation)",
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": profile_traffic(*prof), "peak_source": f"{peaks_kind} bf16 dense burst (fp16 has the "
                                                                  f"same nominal rate)",
                "algorithmic": "2*M*N*K ops per launch"}
        # the dense layer it replaces: fp16 tensor-core GEMM (cuBLAS) on unquantised operands, same shapes
        a16 = X0.to(torch.float16)
        w16 = W0.to(torch.float16)
        for _ in range(3):
            torch.matmul(a16, w16.t())
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(20):
            torch.matmul(a16, w16.t())
        e1.record()
        torch.cuda.synchronize()
        roof["fp16_library_gemm_us"] = e0.elapsed_time(e1) / 20 * 1e3
        del a16, w16
        dt, unit = "f16", "TFLOP/s"
    else:
        kern = "int8_gemm (tcgen05 kind::i8, CTA pair)" if row == "int8_convrot" else \
            "a8w4_gemm (tcgen05 kind::i8, CTA pair, INT4 weights widened in the kernel)"
        roof = tensor_roofline(kern, ops, parts["gemm"], peaks, peaks_kind, int8_meas, profile_traffic(*prof))
        dt, unit = ("s8" if row == "int8_convrot" else "s8xs4"), UNIT
    out = {
        "workload": f"{w.name}: {w.description}", "M": M, "N": N, "K": K, "dtype": dt,
        "value": ops * steps / (ms / 1e3) / 1e12, "unit": unit, "ms_per_step": ms / steps, "steps": steps,
        "timed_ms": ms, "kernels_us": {"act_rotate_quant8": parts["act"], "gemm": parts["gemm"]},
        "kernel_launches_timed": n_part, "roofline": roof, "gpu_launches_per_step": t.launches_per_step,
        "l2": f"{R} rotating input sets of {set_bytes / 1e6:.1f} MB",
    }
    if cpu:
        kind = {"int8_convrot": "int8", "w4a8_asym_g16": "w4a8", "int8_branch_w4": "a8w4"}[row]
        out["cpu_baseline"] = cpu_baseline([(kind, d | {"name": wname}, 1)], 1.5, 32,
                                           unit=unit)
    t.release()
    del keep
    torch.cuda.empty_cache()
    return out


def bench_rows(env, peaks, peaks_kind, int8_meas, cpu, only=None):
    out = {}
    for name in ALL_ROWS:
        if only and name not in only:
            continue
        if name in W4A4_ROWS:
            out[name] = row_w4a4(env, name, peaks, peaks_kind, int8_meas, cpu)
        elif name == "qkv_shared_dit_attn":
            out[name] = row_qkv(env, peaks, peaks_kind, int8_meas, cpu)
        else:
            out[name] = row_format(env, name, peaks, peaks_kind, int8_meas, cpu)
        env.torch.cuda.synchronize()
        st = env.status()
        if st != 0:
            raise SystemExit(f"device status {st} after row {name}: {env.b.cr_status_string(st)}")
    return out


# ---------------------------------------------------------------------------
# end to end through the public one-call API, host buffers, copies overlapped with compute
# ---------------------------------------------------------------------------

def e2e_pipelined(env, layers, steps):
    """Every step: for each layer, pinned host X -> device, cr_w4a4_linear, device Y -> pinned host.
    Three streams (copy in, compute, copy out) and double-buffered device X/Y, so that the input copy
    of step i+1 and the output copy of step i-1 overlap the compute of step i."""
    import w4a8_rotated_quantized_b200 as cr

    torch, device = env.torch, env.device
    h2d, comp, d2h = (torch.cuda.Stream(device) for _ in range(3))
    hosts, bufs = [], []
    for L in layers:
        w = L["w"]
        hosts.append([L["sets"][r][0].cpu().pin_memory() for r in range(min(2, L["R"]))])
        bufs.append({"X": [torch.empty((w.M, w.K), dtype=torch.bfloat16, device=device) for _ in range(2)],
                     "Y": [torch.empty((w.M, w.N), dtype=torch.bfloat16, device=device) for _ in range(2)],
                     "Yh": [torch.empty((w.M, w.N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]})
    ev = lambda: torch.cuda.Event()
    done_h2d = [[ev() for _ in range(2)] for _ in layers]
    done_comp = [[ev() for _ in range(2)] for _ in layers]
    done_d2h = [[ev() for _ in range(2)] for _ in layers]
    used = [[False, False] for _ in layers]

    def step(i):
        b = i & 1
        for l, L in enumerate(layers):
            B = bufs[l]
            with torch.cuda.stream(h2d):
                if used[l][b]:
                    h2d.wait_event(done_comp[l][b])  # step i-2's compute has read X[b]
                B["X"][b].copy_(hosts[l][i % len(hosts[l])], non_blocking=True)
                done_h2d[l][b].record(h2d)
            with torch.cuda.stream(comp):
                comp.wait_event(done_h2d[l][b])
                if used[l][b]:
                    comp.wait_event(done_d2h[l][b])  # step i-2's output copy has read Y[b]
                cr.cr_w4a4_linear(B["X"][b], L["sets"][0][1], L["sets"][0][2], L["B0"], out=B["Y"][b])
                done_comp[l][b].record(comp)
            with torch.cuda.stream(d2h):
                d2h.wait_event(done_comp[l][b])
                B["Yh"][b].copy_(B["Y"][b], non_blocking=True)
                done_d2h[l][b].record(d2h)
            used[l][b] = True

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(h2d)
    for i in range(steps):
        step(i)
    d2h.wait_stream(h2d)
    d2h.wait_stream(comp)
    e1.record(d2h)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    h2d_bytes = sum(L["w"].M * L["w"].K * 2 for L in layers)
    d2h_bytes = sum(L["w"].M * L["w"].N * 2 for L in layers)

    # the copies' own ceiling on this host link: pinned copies alone, each direction
    def copy_rate(src, dst, n=5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s = torch.cuda.current_stream(device)
        dst.copy_(src, non_blocking=True)
        a.record(s)
        for _ in range(n):
            dst.copy_(src, non_blocking=True)
        b.record(s)
        torch.cuda.synchronize()
        return src.numel() * src.element_size() * n / (a.elapsed_time(b) / 1e3) / 1e9

    big = max(range(len(layers)), key=lambda l: hosts[l][0].numel())
    h2d_gbs = copy_rate(hosts[big][0], bufs[big]["X"][0])
    bigy = max(range(len(layers)), key=lambda l: bufs[l]["Y"][0].numel())
    d2h_gbs = copy_rate(bufs[bigy]["Y"][0], bufs[bigy]["Yh"][0])
    bound_ms = max(h2d_bytes / (h2d_gbs * 1e9), d2h_bytes / (d2h_gbs * 1e9)) * 1e3
    del hosts, bufs
    return ms, h2d_bytes, d2h_bytes, {"h2d_GBps": h2d_gbs, "d2h_GBps": d2h_gbs, "copy_bound_ms_per_step": bound_ms}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args):
    import torch

    rank, world, local_rank = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (there is no CPU path)")
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)

    import w4a8_rotated_quantized_b200 as cr

    env = Env(torch, device)
    names = step_layers(args.workload)
    ops_layers = [2.0 * L.M * L.N * L.K for L in (__import__("w4a8_rotated_quantized_b200.workloads",
                                                             fromlist=["CONFIGS"]).CONFIGS[n] for n in names)]
    ops = sum(ops_layers)
    # rotating sets: the step's inputs, codes, weights and outputs over all its layers
    total_set = 0
    from w4a8_rotated_quantized_b200 import workloads

    for n in names:
        w = workloads.CONFIGS[n]
        total_set += w.M * w.K * 2 + w.M * w.K // 2 + w.M * w.N * 2 + w.N * w.K // 2
    R = rotations(env.l2, total_set)
    layers = [w4a4_layer(env, n, R=R, seed_base=1000 + 100 * i) for i, n in enumerate(names)]
    parts = []
    for n, L in zip(names, layers):
        parts += [(f"{n}.act", L["act"]), (f"{n}.gemm", L["gemm"])]
    t = Timed(torch, env.stream, parts, R, warmup=max(3, args.warmup))

    gpu_uuid = str(torch.cuda.get_device_properties(device).uuid)
    gpu_id = gpu_uuid if gpu_uuid.startswith("GPU-") else f"GPU-{gpu_uuid}"
    with ClockSampler(gpu_id) as clocks:
        barrier(device)
        torch.cuda.synchronize()
        elapsed_ms = t.time_steps(args.steps)  # exactly K steps, per-step graphs, events on the stream
        torch.cuda.synchronize()
        barrier(device)
        sus_steps, sus_ms = t.time_sustained()
        part_us, n_part = t.time_parts()
    status = env.status()
    if status != 0:
        raise SystemExit(f"device status {status}: {cr.cr_status_string(status)}")
    elapsed_ms = max_over_ranks(elapsed_ms, device)
    ms_per_step = elapsed_ms / args.steps
    value = world * ops * args.steps / (elapsed_ms / 1e3) / 1e12
    launches_per_step = t.launches_per_step
    t.release()

    # offline weight packing (reported, not in the step)
    pk0, pk1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream(device)
    pack_us = {}
    for n, L in zip(names, layers):
        cr.cr_pack_weight(L["W0"])
        pk0.record(cur)
        for _ in range(5):
            cr.cr_pack_weight(L["W0"])
        pk1.record(cur)
        torch.cuda.synchronize()
        pack_us[n] = pk0.elapsed_time(pk1) / 5 * 1e3

    e2e_ms, h2d_b, d2h_b, link = e2e_pipelined(env, layers, args.e2e_steps)
    e2e_ms = max_over_ranks(e2e_ms, device)
    e2e_value = world * ops * args.e2e_steps / (e2e_ms / 1e3) / 1e12
    del layers
    torch.cuda.empty_cache()

    peaks, peaks_kind = load_peaks()
    int8_meas = measure_int8_peak(torch, device) if world == 1 else None
    int8_val = int8_meas["value"] if int8_meas else None
    gemm_us = sum(part_us[f"{n}.gemm"] for n in names)
    roof = tensor_roofline("w4a4_gemm_pair (tcgen05 cta_group::2 kind::i8)", ops, gemm_us, peaks, peaks_kind,
                           int8_val, gemm_traffic_per_launch())
    roof["algorithmic"] = (f"2*M*N*K integer ops per launch; the step's {len(names)} GEMM launches "
                           f"({', '.join(names)}) taken together: their ops over the sum of their average durations")
    if roof["traffic"] is not None:
        roof["traffic_note"] = "dram bytes per launch averaged over the step's GEMM launches (ncu)"

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline([("w4a4", n, 1) for n in names], 10.0, 64)
    rows = None
    if not args.no_rows and world == 1:
        only = set(x for x in args.rows.split(",") if x) or None
        rows = bench_rows(env, peaks, peaks_kind, int8_val, not args.no_cpu_baseline, only)
    clk = clocks.summary()

    ws = [workloads.CONFIGS[n] for n in names]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "s4", "data": "synthetic",
        "config": {"workload": f"{args.workload}: " + "; ".join(w.description for w in ws),
                   "layers": [{"name": w.name, "M": w.M, "N": w.N, "K": w.K} for w in ws],
                   "group": 256, "act_scale": "tensorwise dynamic", "weight_scale": "tensorwise",
                   "l2": f"inputs larger than L2: {R} rotating input sets of {total_set / 1e6:.1f} MB "
                         f"({R * total_set / 1e6:.0f} MB vs {env.l2 / 1e6:.0f} MB L2)",
                   "timing": f"exactly {args.steps} steps, one CUDA graph replay per step, between two events on "
                             f"the launching stream; kernel times from {n_part} launches of each kernel in "
                             f"per-kernel graphs with events between them",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "sustained": {"steps": sus_steps, "timed_ms": sus_ms, "ms_per_step": sus_ms / sus_steps,
                      "value": world * ops * sus_steps / (sus_ms / 1e3) / 1e12},
        "roofline": roof,
        "int8_measured_peak": int8_meas,
        "kernels_us": part_us,
        "pack_weight_offline_us": pack_us,
        "act_path_GBps": {n: (2.0 * w.M * w.K + w.M * w.K / 2) / (part_us[f"{n}.act"] * 1e-6) / 1e9
                          for n, w in zip(names, ws)},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d_b, "d2h_bytes_per_step": d2h_b,
                "steps": args.e2e_steps, "api": "cr_w4a4_linear",
                "overlap": "three streams (copy in, compute, copy out), double-buffered device X and Y",
                "host_link": link},
        "gpu_launches": (launches_per_step * args.steps) if launches_per_step is not None else None,
        "gpu_launches_source": "kernel nodes of the captured per-step graph x timed steps"
        if launches_per_step is not None else "unavailable (graph introspection failed)",
        "clocks": clk,
        "rows": rows,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
