"""Benchmark of the TTT layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = one pass of the hot path over one batch.  For the default workload (mixed6084_bf16:
8 images x 6 heads x 78x78 = 6084 tokens, d = 64, bf16, eta = 0.5) that is one ttt_forward_layer call:
the five linear heads and the depthwise-conv head, i.e. the Gram/cross accumulation, the
deterministic merge and update, and the readout of every head.  The other workloads time their own
entry point (linear heads alone, the MLP head, the dense 3x3 conv head, the mini-batch variant, the
backward passes).  Inputs are synthetic (seeded, the pages' shapes and distributions) and already
resident in HBM when the timed region starts; enough input sets are rotated that together they exceed
twice the 126 MB L2, so every step reads cold data.  Steps are replayed from CUDA graphs (each graph
holds a run of consecutive steps over the rotating sets) and timed with CUDA events on the launching
stream; a second pass times single-step replays one by one for the p10 / p50 / p90 spread.

Metric: token*heads per second (B * heads * N per step), whole job over all ranks.  Under torchrun
every rank runs the same per-GPU workload on its own GPU (weak scaling; no data-path collective).

--impl reference times the fp64 CPU oracle (the only reference implementation there is) on this
host's cores for the same workload, metric and unit.
"""
import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from vision_test_token_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

METRIC = "TTT-layer fwd tokens*heads/s at 6084 tokens"
METRIC_BWD = "TTT-layer bwd tokens*heads/s"
UNIT = "token*heads/s"
L2_BYTES = 126 * 2 ** 20

# DRAM traffic per launch (dram__bytes_read.sum, dram__bytes_write.sum) from ncu, keyed by workload,
# with the hash of the kernel sources the capture was taken on (kernel_source_hash below).  An entry
# whose hash differs from the running build's is stale and is not reported.  Captured with
# --cache-control none on the third of three consecutive steps, so that the previous step's Z
# write-back (which lands during the next step) is counted as it is in steady state.
TRAFFIC = {
    "mixed6084_bf16": {"read": 112345856, "write": 38357504, "src_sha": "74d99cca3440ea63"},
    "mixed6084_dot_bf16": {"read": 112343040, "write": 38928384, "src_sha": "74d99cca3440ea63"},
    "lin6400_bf16": {"read": 118186240, "write": 39789312, "src_sha": "18d5da35961c4af8"},
    "lin196_bf16": {"read": 14328576, "write": 824832, "src_sha": "18d5da35961c4af8"},
    "mlp1024_bf16": {"read": 25533440, "write": 6981376, "src_sha": "8628555f505e5694"},
    "conv3x3_6084_bf16": {"read": 18785024, "write": 7295744, "src_sha": "4f937ebd690ee19e"},
    "mb16_6084_bf16": {"read": 112244992, "write": 37442304, "src_sha": "3b0306346188364f"},
    "bwd6084_bf16": {"read": 218148352, "write": 105013504, "src_sha": "41e87f12487cba03"},
    "bwdconv6084_bf16": {"read": 24875776, "write": 16282112, "src_sha": "a4fde4904ecff361"},
    "bwdmlp1024_bf16": {"read": 66835712, "write": 145287168, "src_sha": "3c7fe850a26a981e"},
}

# Kernels of this library launched per step, by workload kind (bf16; fp32 where it differs).
LAUNCHES_PER_STEP = {"linear": 1, "mixed": 2, "mlp": 1, "minibatch": 1, "backward": 4, "backward_conv": 4,
                     "backward_mlp": 7, "conv3x3": 4}
LAUNCHES_PER_STEP_FP32 = {"linear": 2, "mixed": 3, "backward": 3}
SMALL_F32_TOKENS = 384                       # fp32 linear units up to this many tokens: lin_small_f32


# The CUDA sources each workload kind runs: its kernels and their launches, besides the device helpers
# and the host entry points (the layer's SM split) that every kind shares.
KIND_SOURCES = {"linear": ["linear.cu"], "mixed": ["linear.cu", "dwconv.cu"], "mlp": ["mlp.cu"],
                "minibatch": ["minibatch.cu"], "backward": ["backward.cu"], "backward_conv": ["backward_conv.cu"],
                "backward_mlp": ["backward_mlp.cu"], "conv3x3": ["conv3x3.cu"]}
COMMON_SOURCES = ["sm100.cuh", "api.cu"]


def launches_per_step(w):
    """Kernels of this library one step of workload w launches (on all SMs)."""
    n = (LAUNCHES_PER_STEP_FP32 if w.dtype == "fp32" else {}).get(w.kind, LAUNCHES_PER_STEP[w.kind])
    if w.dtype == "fp32" and w.kind in ("linear", "mixed") and w.N <= SMALL_F32_TOKENS:
        n -= 1                               # one cluster kernel instead of the two tile kernels
    return n


def code_of(src):
    """A source file's code for the hash: line comments and blank lines removed (the library's sources
    put no comment marker inside a string literal and use no block comments)."""
    lines = (re.sub(rb"//.*$", b"", line).rstrip() for line in src.split(b"\n"))
    return b"\n".join(line for line in lines if line)


def kernel_source_hash(kind=None):
    """sha256 over the code (code_of) of the CUDA sources a workload kind runs, the device helpers and
    the host entry points (every source of the library when kind is None), sorted by name: a DRAM
    traffic capture stays valid while the code that runs is unchanged."""
    d = os.path.join(ROOT, "vision_test_token_b200", "csrc")
    names = sorted(os.listdir(d)) if kind is None else sorted(COMMON_SOURCES + KIND_SOURCES[kind])
    h = hashlib.sha256()
    for name in names:
        if name.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(d, name), "rb") as f:
                h.update(name.encode() + b"\0" + code_of(f.read()))
    return h.hexdigest()[:16]


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="mixed6084_bf16", choices=sorted(WORKLOADS))
    ap.add_argument("--sets", type=int, default=0,
                    help="rotating input sets (0: enough that together they exceed twice the L2)")
    ap.add_argument("--graph-steps", type=int, default=30, help="consecutive steps captured in one CUDA graph")
    ap.add_argument("--spread-reps", type=int, default=200, help="single-step replays timed one by one")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-oracle", action="store_true", help="skip the CPU-oracle baseline leg")
    return ap.parse_args(argv)


def workload_bytes(w):
    """Algorithmic HBM bytes per step: every input token row read once and every output row written
    once (forward: Q, K, V in, Z out; backward: Q, K, V, dZ in, dQ, dK, dV out)."""
    esz = 2 if w.dtype == "bf16" else 4
    units = w.batch * w.heads
    rows = 7 if w.kind.startswith("backward") else 4
    return rows * units * w.N * w.d * esz


def workload_flops(w):
    """Algorithmic FLOPs per step for the kinds whose bound is arithmetic (None otherwise).
      conv3x3: three 9-tap d x d contractions per token (residual, gradient, readout): 54 d^2.
      mlp: seven d x 4d products per token (five in the inner step, two in the readout).
      backward (linear): 14 d^2 per token (G, C, dW1; dq, dk, dv maps).
      backward_conv: eight 9-tap sums per token and channel (r, g, dW1, dq, dr, two dk terms, dW0).
      backward_mlp: 23 d x 4d products per token (5 in the step, 5 through the readout, 13 back
        through the step), as the chain rule is written out.
      minibatch: 6 d^2 + 4 b d per token."""
    n = w.batch * w.heads * w.N
    d = w.d
    hid = getattr(w, "hidden_ratio", 4) * d
    if w.kind == "conv3x3":
        return n * 54 * d * d
    if w.kind == "mlp":
        return n * 7 * 2 * d * hid
    if w.kind == "backward":
        return n * 14 * d * d
    if w.kind == "backward_conv":
        return n * 8 * 9 * 2 * d
    if w.kind == "backward_mlp":
        return n * 23 * 2 * d * hid
    if w.kind == "minibatch":
        return n * (6 * d * d + 4 * w.mb_tokens * d)
    return None


MAX_SETS = 64


def default_sets(w, cap_bytes=6 << 30):
    """Rotating input sets: at least 3, and enough that together they exceed twice the L2 (within
    cap_bytes of device memory and MAX_SETS).  A workload too small for that (its sets together stay
    within 2 x L2) is timed step by step with the L2 flushed between steps instead."""
    per = max(1, workload_bytes(w))
    return int(max(3, min(math.ceil(2 * L2_BYTES / per), cap_bytes // per, MAX_SETS)))


def needs_flush(w, n_sets):
    return n_sets * workload_bytes(w) <= 2 * L2_BYTES


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------------------------------------
# clocks sampled during the run
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.lines:
            if not (t0 <= ts <= t1):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------------
# distributed plumbing
# ------------------------------------------------------------------------------------------------
def dist_init(gpus, backend="nccl"):
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE).  `backend` is "nccl" on GPUs;
    the CPU tests use "gloo"."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return world, rank, local


def shard_batch(global_batch, rank, world):
    """The contiguous range of images (start, count) that `rank` of `world` processes.  Units are
    independent, so sharding the batch needs no exchange at all; the first global_batch % world ranks
    take one image more."""
    base, extra = divmod(global_batch, world)
    return rank * base + min(rank, extra), base + (1 if rank < extra else 0)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, dev):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------------------------------------
# the CPU oracle leg (cpu_baseline and --impl reference)
# ------------------------------------------------------------------------------------------------
def _np64(t):
    return t.detach().cpu().double().numpy()


def oracle_units(w, x, images, threads, heads=None):
    """Runs the oracle on `images` whole images of the workload (inputs already float64; image i of x
    is used for i < x's batch, then again from the start), on the heads in range `heads` (lo, hi), or
    all heads."""
    import oracle
    lo, hi = heads if heads else (0, w.heads)
    nb = x["Q"].shape[0]
    idx = [i % nb for i in range(images)]
    take = lambda k, a, b: x[k][idx][:, a:b]
    if w.kind == "mixed":
        nl = w.lin_heads
        lin_fn, conv_fn = (oracle.linear_dot, oracle.dwconv_dot) if w.loss == "dot" else (oracle.linear, oracle.dwconv)
        if lo < nl:
            a, b = lo, min(hi, nl)
            lin_fn(take("Q", a, b), take("K", a, b), take("V", a, b), x["W0_lin"][a:b], w.eta, threads=threads)
        if hi > nl:
            a, b = max(lo, nl), hi
            conv_fn(take("Q", a, b), take("K", a, b), take("V", a, b), x["W0_conv"][a - nl:b - nl], w.eta, w.H, w.W,
                    threads=threads)
        return
    Q, K, V = take("Q", lo, hi), take("K", lo, hi), take("V", lo, hi)
    if w.kind == "backward":
        oracle.linear_backward(Q, K, V, x["W0_lin"][lo:hi], w.eta, take("dZ", lo, hi), threads=threads)
    elif w.kind == "backward_conv":
        oracle.dwconv_backward(Q, K, V, x["W0_conv"][lo:hi], w.eta, take("dZ", lo, hi), w.H, w.W, threads=threads)
    elif w.kind == "backward_mlp":
        oracle.mlp_backward(Q, K, V, x["Wa"][lo:hi], x["Wb"][lo:hi], w.eta, take("dZ", lo, hi), threads=threads)
    elif w.kind == "conv3x3":
        oracle.conv3x3(Q, K, V, x["W0_c3"][lo:hi], w.eta, w.H, w.W, threads=threads)
    elif w.kind == "minibatch":
        oracle.linear_minibatch(Q, K, V, x["W0_lin"][lo:hi], w.eta, w.mb_tokens, w.mb_mode, threads=threads)
    elif w.kind == "mlp":
        oracle.mlp(Q, K, V, x["Wa"][lo:hi], x["Wb"][lo:hi], w.eta, threads=threads)
    else:                                                    # linear heads only
        fn = oracle.linear_dot if w.loss == "dot" else oracle.linear
        fn(Q, K, V, x["W0_lin"][lo:hi], w.eta, threads=threads)


def oracle_inputs(w, x, images):
    return {k: _np64(v[:images] if k in ("Q", "K", "V", "dZ") else v) for k, v in x.items()
            if k not in ("Z", "grads")}


def _time_oracle_leg(w, x, images, threads, budget_s):
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle_units(w, x, images, threads)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            return images * w.heads * w.N * reps / el, reps, el


def time_oracle(w, x, budget_s=10.0, single_budget_s=6.0):
    """cpu_baseline: the fp64 oracle on this host's cores.  All-core: enough whole images that their
    (image, head) units occupy every core of os.sched_getaffinity (images of the workload's batch,
    reused when the batch has fewer), OpenMP over the units.  Single-core: one image, one thread."""
    import oracle
    cores = oracle.default_threads()
    if w.kind.startswith("backward"):
        # the backward oracles sum the weight gradients over the images of each head in order: OpenMP
        # over the heads only
        images, used, over = 1, min(cores, w.heads), "heads"
    else:
        images = max(1, math.ceil(cores / w.heads))
        used, over = min(cores, images * w.heads), "(image, head) units"
    xs = oracle_inputs(w, x, min(images, x["Q"].shape[0]))
    v_all, reps, el = _time_oracle_leg(w, xs, images, cores, budget_s)
    v_one, reps1, el1 = _time_oracle_leg(w, xs, 1, 1, single_budget_s)
    return {"value": v_all, "unit": UNIT, "cores": used, "kind": "oracle",
            "sample": f"{images} image(s) of {w.name} ({images * w.heads} (image, head) units of {w.N} tokens) "
                      f"repeated {reps} times in {el:.1f} s, fp64, OpenMP over the {over}: {used} of the "
                      f"{cores} cores of the affinity mask busy",
            "single_core": {"value": v_one, "unit": UNIT, "cores": 1,
                            "sample": f"1 image of {w.name} ({w.heads} units) repeated {reps1} times in "
                                      f"{el1:.1f} s, one thread"}}


def config_of(w, world):
    """The config object of a bench line (the same keys for both arms)."""
    cfg = {"workload": w.name, "batch": w.batch, "global_batch": w.batch * world, "heads": w.heads,
           "lin_heads": w.lin_heads, "conv_heads": w.conv_heads, "grid": [w.H, w.W], "tokens": w.N, "d": w.d,
           "eta": w.eta, "loss": w.loss, "kind": w.kind, "parallelism": f"batch-sharded x{world}"}
    if w.kind == "minibatch":
        cfg.update({"mb_tokens": w.mb_tokens, "mb_mode": w.mb_mode})
    if w.kind in ("mlp", "backward_mlp"):
        cfg["hidden"] = w.hidden_ratio * w.d
    return cfg


def run_reference(args):
    """The reference arm: the fp64 oracle on this host's cores, on the same workload, metric and unit.
    One step = one whole image of the workload (all heads, OpenMP over them), or one (image, head)
    unit per step, heads in turn, when K whole images would not finish within about two and a half
    minutes.  Under torchrun rank 0 alone runs; the other ranks exit without work."""
    import oracle
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    x = oracle_inputs(w, make_inputs(w, seed=0), 1)
    threads = oracle.default_threads()
    t0 = time.perf_counter()
    oracle_units(w, x, 1, threads)                           # warm-up: one whole image
    t_img = time.perf_counter() - t0
    per_image = args.steps * t_img <= 150.0
    step_heads = (lambda i: None) if per_image else (lambda i: (i % w.heads, i % w.heads + 1))
    for i in range(max(0, min(args.warmup, 3) - 1)):
        oracle_units(w, x, 1, threads, step_heads(i))
    t0 = time.perf_counter()
    th = 0
    for i in range(args.steps):
        oracle_units(w, x, 1, threads, step_heads(i))
        th += (w.heads if per_image else 1) * w.N
    el = time.perf_counter() - t0
    value = th / el
    used = min(threads, w.heads) if per_image else 1
    sample = (f"{'one image (' + str(w.heads) + ' heads)' if per_image else 'one (image, head) unit, heads in turn'}"
              f" of {w.name} per step, {args.steps} steps, {el:.1f} s, fp64")
    cb = {"value": value, "unit": UNIT, "kind": "oracle", "cores": used, "sample": sample}
    line = {"impl": "reference", "metric": METRIC_BWD if w.kind.startswith("backward") else METRIC, "value": value,
            "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / max(1, args.steps) * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config_of(w, world), "device": "host CPU",
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------------
def alloc_outputs(w, x, dev):
    """Output buffers of one input set: Z for the forward kinds, the gradient tuple for the backward
    kinds."""
    if w.kind == "backward":
        x["grads"] = (torch.empty_like(x["Q"]), torch.empty_like(x["Q"]), torch.empty_like(x["Q"]),
                      torch.empty((w.heads, w.d, w.d), device=dev), torch.empty(1, device=dev))
    elif w.kind == "backward_conv":
        x["grads"] = (torch.empty_like(x["Q"]), torch.empty_like(x["Q"]), torch.empty_like(x["Q"]),
                      torch.empty((w.heads, w.d, 3, 3), device=dev), torch.empty(1, device=dev))
    elif w.kind == "backward_mlp":
        hid = w.hidden_ratio * w.d
        x["grads"] = (torch.empty_like(x["Q"]), torch.empty_like(x["Q"]), torch.empty_like(x["Q"]),
                      torch.empty((w.heads, hid, w.d), device=dev), torch.empty((w.heads, w.d, hid), device=dev),
                      torch.empty(1, device=dev))
    else:
        x["Z"] = torch.empty_like(x["Q"])


def run_step(w, x, d=None, out=None):
    """One step of the workload through the public Python API: inputs from x (or d, a dict of
    device tensors with the same keys), outputs into x's buffers (or out)."""
    from vision_test_token_b200 import layer
    d = x if d is None else d
    if out is None:
        out = x["grads"] if w.kind.startswith("backward") else x["Z"]
    Q, K, V = d["Q"], d["K"], d["V"]
    if w.kind == "mlp":
        layer.forward_mlp(Q, K, V, d["Wa"], d["Wb"], w.eta, w.H, w.W, Z=out)
    elif w.kind == "minibatch":
        layer.forward_linear_minibatch(Q, K, V, d["W0_lin"], w.eta, w.H, w.W, w.mb_tokens, w.mb_mode, Z=out)
    elif w.kind == "conv3x3":
        layer.forward_conv3x3(Q, K, V, d["W0_c3"], w.eta, w.H, w.W, Z=out)
    elif w.kind == "backward":
        layer.backward_linear(Q, K, V, d["W0_lin"], w.eta, w.H, w.W, d["dZ"], out=out)
    elif w.kind == "backward_conv":
        layer.backward_dwconv(Q, K, V, d["W0_conv"], w.eta, w.H, w.W, d["dZ"], out=out)
    elif w.kind == "backward_mlp":
        layer.backward_mlp(Q, K, V, d["Wa"], d["Wb"], w.eta, w.H, w.W, d["dZ"], out=out)
    elif w.kind == "linear":
        layer.forward_linear(Q, K, V, d["W0_lin"], w.eta, w.H, w.W, Z=out, loss=w.loss)
    else:
        layer.forward_layer(Q, K, V, d, w.eta, w.H, w.W, conv_heads=w.conv_heads, Z=out, loss=w.loss)


def capture(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
        fn()
    return g


def capture_steps(w, xs, first, count, stream):
    """One CUDA graph holding `count` consecutive steps over the rotating input sets, from set
    `first`."""
    def fn():
        for i in range(count):
            run_step(w, xs[(first + i) % len(xs)])
    return capture(fn, stream)


def replay(plan, stream):
    """Replays a list of (graph, times) on `stream` between two CUDA events; returns seconds."""
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for g, times in plan:
            for _ in range(times):
                g.replay()
        end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / 1e3


def time_graphs(graphs, steps, stream):
    return replay([(graphs[i % len(graphs)], 1) for i in range(steps)], stream)


def time_steps(graphs, reps, stream, flush=None):
    """Single-step replays timed one by one (events around each replay, issued back to back, read
    after the last); with `flush` (a device buffer larger than the L2) it is overwritten between
    steps, outside the timed intervals.  Returns the per-step times in microseconds."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    with torch.cuda.stream(stream):
        for i, (a, b) in enumerate(evs):
            if flush is not None:
                flush.fill_(float(i % 7))
            a.record(stream)
            graphs[i % len(graphs)].replay()
            b.record(stream)
    evs[-1][1].synchronize()
    return [a.elapsed_time(b) * 1e3 for a, b in evs]


def spread_of(us):
    us = sorted(us)
    q = lambda f: us[min(len(us) - 1, int(f * len(us)))]
    return {"p10_us": q(0.1), "p50_us": q(0.5), "p90_us": q(0.9), "reps": len(us)}


def time_calls_alone(w, xs, stream, n):
    """Device time per call of the linear heads alone and of the conv heads alone (each on the whole
    GPU), from CUDA-graph replays over the rotating input sets."""
    from vision_test_token_b200 import layer
    nl = w.lin_heads
    out = []
    for which in ("linear", "conv"):
        gs = []
        for x in xs:
            if which == "linear":
                fn = lambda x=x: layer.forward_linear(x["Q"][:, :nl], x["K"][:, :nl], x["V"][:, :nl], x["W0_lin"],
                                                      w.eta, w.H, w.W, Z=x["Z"][:, :nl], loss=w.loss)
            else:
                fn = lambda x=x: layer.forward_dwconv(x["Q"][:, nl:], x["K"][:, nl:], x["V"][:, nl:], x["W0_conv"],
                                                      w.eta, w.H, w.W, Z=x["Z"][:, nl:], loss=w.loss)
            with torch.cuda.stream(stream):
                fn()
            stream.synchronize()
            gs.append(capture(fn, stream))
        time_graphs(gs, 20, stream)
        out.append(time_graphs(gs, n, stream) / n)
    return out[0], out[1]


def traffic_entry(w):
    """The DRAM traffic capture of this workload, if it was taken on the running kernel sources."""
    e = TRAFFIC.get(w.name)
    if not e:
        return None, "no ncu capture for this workload"
    if e["src_sha"] != kernel_source_hash(w.kind):
        return None, f"stale: the capture was taken on kernel sources {e['src_sha']}, not on this build"
    return e, None


def fp32_peak_tflops(mhz):
    return 148 * 128 * 2 * mhz * 1e6 / 1e12


def roofline(w, t_step, pk, clocks, xs, stream, args):
    """The roofline block of the step: HBM-bound kinds against the measured copy bandwidth,
    contractions against the measured bf16 tensor peak, plain FP32 FMA paths against the FP32 peak
    derived from the SM count, the FP32 lanes per SM and the SM clock sampled under load."""
    nbytes, flops = workload_bytes(w), workload_flops(w)
    hbm = nbytes / t_step / 1e9
    tr, tr_note = traffic_entry(w)
    mhz = clocks.get("sm_mhz") or clocks.get("sm_max_mhz") or 1965.0
    common = {"us_per_launch": t_step * 1e6, "algorithmic_bytes": nbytes,
              "traffic": (tr["read"] + tr["write"]) if tr else None}
    if tr:
        common["traffic_read"], common["traffic_write"] = tr["read"], tr["write"]
        common["traffic_src_sha"] = tr["src_sha"]
    else:
        common["traffic_note"] = tr_note
    conv_name = "dw_band<bf16, dot>" if w.loss == "dot" else "dw_band<bf16>"
    if w.kind in ("mixed", "linear"):
        if w.kind == "mixed":
            kern = f"layer step: lin_cluster_bf16 and {conv_name} running at the same time (one ttt_forward_layer call)"
        else:
            kern = "lin_cluster_bf16 (the whole ttt_forward_linear call)" if w.dtype == "bf16" else \
                   "lin_small_f32 (the whole ttt_forward_linear call)" if w.N <= SMALL_F32_TOKENS else \
                   "lin_p1_f32 + lin_p2_f32 (the whole ttt_forward_linear call)"
        roof = {"bound": "hbm", "kernel": kern, "achieved": hbm, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": hbm / pk["hbm_gbs"], "peak_source": pk["source"] + " (copy bandwidth)", **common}
        if w.kind == "mixed":
            esz = 2 if w.dtype == "bf16" else 4
            lin_bytes = 4 * w.batch * w.lin_heads * w.N * w.d * esz
            conv_bytes = 4 * w.batch * w.conv_heads * w.N * w.d * esz
            t_lin, t_conv = time_calls_alone(w, xs, stream, n=max(200, args.steps // 4))
            roof["kernels_alone"] = {
                "lin_cluster_bf16": {"us_per_launch": t_lin * 1e6, "algorithmic_bytes": lin_bytes,
                                     "achieved_gbs": lin_bytes / t_lin / 1e9,
                                     "frac": lin_bytes / t_lin / 1e9 / pk["hbm_gbs"]},
                conv_name: {"us_per_launch": t_conv * 1e6, "algorithmic_bytes": conv_bytes,
                            "achieved_gbs": conv_bytes / t_conv / 1e9,
                            "frac": conv_bytes / t_conv / 1e9 / pk["hbm_gbs"]}}
        return roof
    if w.kind in ("mlp", "conv3x3"):
        kern = "mlp_fused (the whole ttt_forward_mlp call)" if w.kind == "mlp" else \
               "conv3_wprep + conv3_grad + conv3_merge + conv3_readout (the whole ttt_forward_conv3x3 call)"
        tf = flops / t_step / 1e12
        return {"bound": "tensor", "kernel": kern, "achieved": tf, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": tf / pk["bf16_tflops"], "peak_source": pk["source"] + " (bf16 burst)",
                "algorithmic_flops": flops, "hbm_gbs": hbm, "hbm_frac": hbm / pk["hbm_gbs"], **common}
    if w.kind == "backward" and w.dtype == "bf16":
        # two token-streaming phases on the tensor cores: HBM-bound (48 FLOP per byte at most)
        kern = "lin_bwd_p1_tc + lin_bwd_merge_tc + lin_bwd_p2_tc + lin_bwd_sum (the whole ttt_backward_linear call)"
        return {"bound": "hbm", "kernel": kern, "achieved": hbm, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": hbm / pk["hbm_gbs"], "peak_source": pk["source"] + " (copy bandwidth)",
                "algorithmic_flops": flops, "tflops": flops / t_step / 1e12, **common}
    names = {"backward": "lin_bwd_p1 + lin_bwd_p2 + lin_bwd_sum (the whole ttt_backward_linear call)",
             "backward_conv": "cb_reduce + cb_unit + cb_map + cb_final (the whole ttt_backward_dwconv call)",
             "backward_mlp": "mb_prep .. mb_final, 7 kernels (the whole ttt_backward_mlp call)",
             "minibatch": "lin_minibatch (the whole ttt_forward_linear_minibatch call)"}
    peak = fp32_peak_tflops(mhz)
    tf = flops / t_step / 1e12
    return {"bound": "alu", "kernel": names[w.kind], "achieved": tf, "peak": peak, "unit": "TFLOP/s",
            "frac": tf / peak, "peak_source": f"derived: 148 SMs x 128 FP32 lanes x 2 FLOP x {mhz:.0f} MHz "
                                                "(median SM clock under load)",
            "algorithmic_flops": flops, "hbm_gbs": hbm, "hbm_frac": hbm / pk["hbm_gbs"], **common}


def run_ours(args):
    world, rank, local = dist_init(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from vision_test_token_b200 import build as _build, capi
    _build.build()
    capi.lib()
    w = WORKLOADS[args.workload]
    pk = peaks()
    # this rank's images of the global batch (weak scaling: w.batch images per GPU), one input set per
    # seed, with its output buffers
    first, count = shard_batch(w.batch * world, rank, world)
    assert count == w.batch
    n_sets = args.sets or default_sets(w)
    xs = []
    for s in range(n_sets):
        x = make_inputs(w, seed=1000 * first + s, device=dev)
        alloc_outputs(w, x, dev)
        xs.append(x)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for i in range(3):                      # eager warm-up (workspaces, attributes)
            run_step(w, xs[i % n_sets])
    stream.synchronize()
    # graphs: single steps (one per set), and runs of G consecutive steps (G a multiple of the sets)
    singles = [capture_steps(w, xs, i, 1, stream) for i in range(n_sets)]
    G = n_sets * max(1, math.ceil(min(args.graph_steps, max(1, args.steps)) / n_sets))
    run_g = capture_steps(w, xs, 0, G, stream)
    q, r = divmod(args.steps, G)
    plan = [(run_g, q)] + ([(capture_steps(w, xs, 0, r, stream), 1)] if r else [])

    sampler = ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local])
    sampler.start()
    time.sleep(0.3)

    # warm-up (W single-step replays), then exactly K steps in the timed region: runs of G steps, or,
    # for a workload whose sets fit in the L2, single steps with the L2 flushed between them (the
    # flushes outside the timed intervals)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if needs_flush(w, n_sets) else None
    time_graphs(singles, max(3, args.warmup), stream)
    barrier(world)
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    if flush is None:
        el = replay(plan, stream)
    else:
        el = sum(time_steps(singles, args.steps, stream, flush)) / 1e6
    torch.cuda.synchronize(dev)
    barrier(world)
    t_wall1 = time.time()
    el_max = max_over_ranks(el, world, dev)
    spread = spread_of(time_steps(singles, args.spread_reps, stream, flush))
    # keep the GPU loaded a little longer so the clock record covers the load
    if t_wall1 - t_wall0 < 1.0:
        t_est = max((t_wall1 - t_wall0) / max(1, args.steps), 1e-7)
        soak = max(1, min(2000, math.ceil(1.2 / (t_est * G))))
        t_wall0 = time.time()
        replay([(run_g, soak)], stream)
        t_wall1 = time.time()
    time.sleep(0.25)
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1)

    t_step = el_max / args.steps
    value = w.token_heads * world / t_step
    roof = roofline(w, t_step, pk, clocks, xs, stream, args)

    # end to end through the public API: pinned host inputs -> device -> step -> host result
    e2e = run_e2e(w, xs[0], dev, stream, args.e2e_steps, world)

    per_step = launches_per_step(w)
    line = {"metric": METRIC_BWD if w.kind.startswith("backward") else METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": config_of(w, world), "device": torch.cuda.get_device_name(dev),
            "l2": (f"{n_sets} rotating input sets of {workload_bytes(w) / 1e6:.1f} MB "
                   f"({n_sets * workload_bytes(w) / 1e6:.0f} MB in all, > 2 x 126 MB L2)") if flush is None else
                  (f"{n_sets} rotating input sets of {workload_bytes(w) / 1e6:.2f} MB (within the L2): L2 flushed "
                   f"between steps by overwriting a {2 * L2_BYTES / 1e6:.0f} MB buffer, outside the timed intervals"),
            "launch": (f"CUDA graphs of {G} consecutive steps over the rotating sets" if flush is None else
                       "one CUDA graph per step, each timed by its own pair of events")
                      + ("; one ttt_forward_layer call per step: the conv kernel launched behind the linear kernel "
                         "as a programmatic dependent, the two running at the same time" if w.kind == "mixed" else ""),
            "step_spread": spread, "gbs_per_step": workload_bytes(w) / t_step / 1e9,
            "gpu_launches": args.steps * per_step, "gpu_launches_per_step": per_step,
            "kernel_src_sha": kernel_source_hash(w.kind), "clocks": clocks, "e2e": e2e, "roofline": roof}
    if rank == 0 and world == 1 and not args.no_oracle:
        line["cpu_baseline"] = time_oracle(w, xs[0])
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        del singles, run_g, plan
        dist.destroy_process_group()


def run_e2e(w, x, dev, stream, steps, world):
    """The same metric through the public API with the inputs on the host: every step copies its Q, K,
    V (and dZ) and weights from pinned host memory to the device, runs the step and copies its outputs
    (Z, or dQ, dK, dV and the weight gradients) back.  Steps are pipelined over two buffer sets and
    three streams, as a serving loop would run them: the host-to-device copy of step i+1 overlaps the
    compute and the device-to-host copy of step i (PCIe moves both directions at once).  Every step's
    copies are inside the timed region."""
    bwd = w.kind.startswith("backward")
    names = ["Q", "K", "V"] + (["dZ"] if bwd else []) + sorted(k for k in x if k.startswith("W"))
    host = {k: x[k].cpu().pin_memory() for k in names}
    dev_in = [{k: torch.empty_like(x[k]) for k in names} for _ in range(2)]
    outs = list(x["grads"]) if bwd else [x["Z"]]
    o_dev = [[torch.empty_like(t) for t in outs] for _ in range(2)]
    o_host = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs] for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in o_host[0])
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()
    loaded, computed, drained = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    started = [False, False]

    def one(i):
        bsel = i % 2
        d = dev_in[bsel]
        with torch.cuda.stream(s_in):
            if started[bsel]:
                s_in.wait_event(computed[bsel])              # step i-2 has finished reading these inputs
            for k in names:
                d[k].copy_(host[k], non_blocking=True)
            loaded[bsel].record(s_in)
        stream.wait_event(loaded[bsel])
        if started[bsel]:
            stream.wait_event(drained[bsel])                 # step i-2's outputs have left this buffer
        with torch.cuda.stream(stream):
            run_step(w, x, d=d, out=tuple(o_dev[bsel]) if bwd else o_dev[bsel][0])
            computed[bsel].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed[bsel])
            for oh, od in zip(o_host[bsel], o_dev[bsel]):
                oh.copy_(od, non_blocking=True)
            drained[bsel].record(s_out)
        started[bsel] = True

    for i in range(4):
        one(i)
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    s_in.wait_event(a)
    for i in range(steps):
        one(i)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    b.record(stream)
    b.synchronize()
    el = max_over_ranks(a.elapsed_time(b) / 1e3, world, dev)
    return {"value": w.token_heads * world * steps / el, "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": el / steps * 1e3,
            "pipelining": "two buffer sets, three streams: step i+1's host-to-device copy overlaps step i's "
                          "compute and device-to-host copy"}


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
