"""Benchmark of the TTT-layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = one forward of the whole layer over one batch: for the default workload
(mixed6084_bf16: 8 images x 6 heads x 78x78 = 6084 tokens, d = 64, bf16, eta = 0.5) the five linear
heads and the depthwise-conv head, i.e. the Gram/cross accumulation, the deterministic merge and
update, and the readout of every head.  --workload mixed6084_dot_bf16 runs the same layer trained
with the dot-product inner loss (eta = 1.0).  Inputs are synthetic (seeded, the pages' shapes and
distributions) and already resident in HBM when the timed region starts; three input sets of
149.5 MB each (more than the 126 MB L2) are rotated so every step reads cold data.  Steps are replayed
from CUDA graphs (one graph per input set) and timed with CUDA events on the launching stream.

Metric: token*heads per second (B * heads * N per step), whole job over all ranks.  Under torchrun
every rank runs the same per-GPU workload on its own GPU (weak scaling; no data-path collective).

--impl reference times the fp64 CPU oracle (the only reference implementation there is) on this
host's cores for the same workload, metric and unit.
"""
import argparse
import json
import os
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
METRIC_BWD = "TTT-layer bwd (linear heads) tokens*heads/s at 6084 tokens"
UNIT = "token*heads/s"
# dram__bytes_read.sum + dram__bytes_write.sum per launch, from the ncu captures summarised under
# profiles/.  Valid only for the kernel builds those captures were taken on: an entry is removed
# whenever its kernel changes.  Mixed layer: the two kernels of one step, summed.
STEP_TRAFFIC = {"mixed6084_bf16": (93.597184e6 + 3.062272e6) + (18.751488e6 + 0.0),   # profiles/traffic_mixed6084_bf16.md
                "mixed6084_dot_bf16": (93.595904e6 + 4.063488e6) + (18.747392e6 + 0.002816e6)}
                # profiles/layer_kernels_mixed6084_dot_bf16.md
MLP_TRAFFIC = {"mlp1024_bf16": 25.809664e6 + 0.0}                                   # profiles/mlp_fused_mlp1024.md


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="mixed6084_bf16", choices=sorted(WORKLOADS))
    ap.add_argument("--sets", type=int, default=3, help="rotating input sets (total must exceed L2)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-oracle", action="store_true", help="skip the CPU-oracle baseline leg")
    return ap.parse_args()


def workload_bytes(w):
    esz = 2 if w.dtype == "bf16" else 4
    units = w.batch * w.heads
    return 4 * units * w.N * w.d * esz          # read Q, K, V once, write Z once


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


def oracle_units(w, x, units, threads):
    """Runs the oracle on the listed (image, head) units of the workload (inputs already float64)."""
    import oracle
    if w.kind == "backward":
        for (b, h) in units:
            sl = (slice(b, b + 1), slice(h, h + 1))
            oracle.linear_backward(x["Q"][sl], x["K"][sl], x["V"][sl], x["W0_lin"][h:h + 1], w.eta, x["dZ"][sl],
                                   threads=threads)
        return
    if w.kind == "minibatch":
        for (b, h) in units:
            oracle.linear_minibatch(x["Q"][b:b + 1, h:h + 1], x["K"][b:b + 1, h:h + 1], x["V"][b:b + 1, h:h + 1],
                                    x["W0_lin"][h:h + 1], w.eta, w.mb_tokens, w.mb_mode, threads=threads)
        return
    if w.kind == "mlp":
        for (b, h) in units:
            oracle.mlp(x["Q"][b:b + 1, h:h + 1], x["K"][b:b + 1, h:h + 1], x["V"][b:b + 1, h:h + 1],
                       x["Wa"][h:h + 1], x["Wb"][h:h + 1], w.eta, threads=threads)
        return
    nl = w.lin_heads
    imgs = sorted({b for b, _ in units})
    for b in imgs:
        hs = [h for bb, h in units if bb == b]
        lin = [h for h in hs if h < nl]
        conv = [h for h in hs if h >= nl]
        lin_fn, conv_fn = (oracle.linear_dot, oracle.dwconv_dot) if w.loss == "dot" else (oracle.linear, oracle.dwconv)
        if lin:
            lo, hi = min(lin), max(lin) + 1
            lin_fn(x["Q"][b:b + 1, lo:hi], x["K"][b:b + 1, lo:hi], x["V"][b:b + 1, lo:hi],
                   x["W0_lin"][lo:hi], w.eta, threads=threads)
        if conv:
            lo, hi = min(conv), max(conv) + 1
            conv_fn(x["Q"][b:b + 1, lo:hi], x["K"][b:b + 1, lo:hi], x["V"][b:b + 1, lo:hi],
                    x["W0_conv"][lo - nl:hi - nl], w.eta, w.H, w.W, threads=threads)


def oracle_inputs(w, x, images):
    return {k: _np64(v[:images] if k in ("Q", "K", "V", "dZ") else v) for k, v in x.items()
            if k not in ("Z", "grads")}


def time_oracle(w, x, budget_s=12.0):
    """cpu_baseline: whole images of the workload (all heads, OpenMP over units) until budget_s."""
    import oracle
    threads = oracle.default_threads()
    xs = oracle_inputs(w, x, 1)
    units = [(0, h) for h in range(w.heads)]
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle_units(w, xs, units, threads)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": len(units) * w.N * reps / el, "unit": UNIT, "cores": min(threads, len(units)),
            "kind": "oracle",
            "sample": f"image 0 of {w.name} ({w.heads} heads x {w.N} tokens) repeated {reps} times, "
                      f"{el:.1f} s, fp64, OpenMP over the {len(units)} (image, head) units"}


def run_reference(args):
    """The reference arm: the fp64 oracle on this host's cores.  One step = one image of the
    workload (all heads), or one (image, head) unit per step when K whole images would not finish
    within about two and a half minutes."""
    import oracle
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    x = oracle_inputs(w, make_inputs(w, seed=0), 1)
    threads = oracle.default_threads()
    all_units = [(0, h) for h in range(w.heads)]
    t0 = time.perf_counter()
    oracle_units(w, x, all_units, threads)                  # warm-up: one whole image
    t_img = time.perf_counter() - t0
    per_image = args.steps * t_img <= 150.0
    for _ in range(max(0, min(args.warmup, 3) - 1)):
        oracle_units(w, x, all_units if per_image else all_units[:1], threads)
    t0 = time.perf_counter()
    th = 0
    for i in range(args.steps):
        units = all_units if per_image else [all_units[i % len(all_units)]]
        oracle_units(w, x, units, threads)
        th += len(units) * w.N
    el = time.perf_counter() - t0
    value = th / el
    sample = (f"{'one image (' + str(w.heads) + ' heads)' if per_image else 'one (image, head) unit, heads in turn'}"
              f" of {w.name} per step, {args.steps} steps, {el:.1f} s, fp64")
    cb = {"value": value, "unit": UNIT, "kind": "oracle", "cores": min(threads, w.heads if per_image else 1),
          "sample": sample}
    line = {"impl": "reference", "metric": METRIC_BWD if w.kind == "backward" else METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / max(1, args.steps) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "global_batch": w.batch * world, "heads": w.heads, "tokens": w.N, "d": w.d,
                       "eta": w.eta, "loss": w.loss, "device": "host CPU"},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------------
def make_step(w, xs, dev):
    """Returns fn(i) running one layer forward on input set i (all device tensors)."""
    from vision_test_token_b200 import layer
    weights = {k: v for k, v in xs[0].items() if k.startswith("W")}

    def step(i):
        x = xs[i]
        if w.kind == "mlp":
            layer.forward_mlp(x["Q"], x["K"], x["V"], weights["Wa"], weights["Wb"], w.eta, w.H, w.W, Z=x["Z"])
        elif w.kind == "minibatch":
            layer.forward_linear_minibatch(x["Q"], x["K"], x["V"], weights["W0_lin"], w.eta, w.H, w.W, w.mb_tokens,
                                           w.mb_mode, Z=x["Z"])
        elif w.kind == "backward":
            layer.backward_linear(x["Q"], x["K"], x["V"], weights["W0_lin"], w.eta, w.H, w.W, x["dZ"], out=x["grads"])
        else:
            layer.forward_layer(x["Q"], x["K"], x["V"], weights, w.eta, w.H, w.W, conv_heads=w.conv_heads, Z=x["Z"],
                                loss=w.loss)
    return step


def capture(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
        fn()
    return g


def time_graphs(graphs, steps, stream):
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for i in range(steps):
            graphs[i % len(graphs)].replay()
        end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / 1e3


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


def run_ours(args):
    world, rank, local = dist_init(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from vision_test_token_b200 import build as _build, capi, layer
    _build.build()
    capi.lib()
    w = WORKLOADS[args.workload]
    pk = peaks()

    # this rank's images of the global batch (weak scaling: w.batch images per GPU), one input set per
    # seed; Z buffers, workspaces
    first, count = shard_batch(w.batch * world, rank, world)
    assert count == w.batch
    xs = []
    for s in range(args.sets):
        x = make_inputs(w, seed=1000 * first + s, device=dev)
        x["Z"] = torch.empty_like(x["Q"])
        if w.kind == "backward":
            x["grads"] = (torch.empty_like(x["Q"]), torch.empty_like(x["Q"]), torch.empty_like(x["Q"]),
                          torch.empty((w.heads, w.d, w.d), device=dev), torch.empty(1, device=dev))
        xs.append(x)
    stream = torch.cuda.Stream(device=dev)
    step = make_step(w, xs, dev)
    with torch.cuda.stream(stream):
        for i in range(3):                      # eager warm-up (workspaces, attributes)
            step(i % args.sets)
    stream.synchronize()
    graphs = [capture(lambda i=i: step(i), stream) for i in range(args.sets)]

    sampler = ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local])
    sampler.start()
    time.sleep(0.3)

    # warm-up (graph replays), then the timed region
    time_graphs(graphs, max(3, args.warmup), stream)
    barrier(world)
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    el = time_graphs(graphs, args.steps, stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    t_wall1 = time.time()
    el_max = max_over_ranks(el, world, dev)
    # keep the GPU loaded a little longer so the clock record covers the load
    if t_wall1 - t_wall0 < 1.0:
        soak_steps = min(20000, int(args.steps * (1.2 / max(t_wall1 - t_wall0, 1e-3))))
        t_wall0 = time.time()
        time_graphs(graphs, soak_steps, stream)
        t_wall1 = time.time()
    time.sleep(0.25)
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1)

    ms_per_step = el_max / args.steps * 1e3
    th_step = w.token_heads
    value = th_step * world / (el_max / args.steps)

    # roofline.  Mixed layer: one ttt_forward_layer call runs the linear kernel and the conv kernel at
    # the same time (they share HBM), so the bound applies to the layer step as a whole: its
    # algorithmic bytes over its device time.  Each kernel's time when it runs alone on the whole GPU
    # is given beside it.
    roof = None
    if w.kind == "mixed":
        esz = 2 if w.dtype == "bf16" else 4
        lin_bytes = 4 * w.batch * w.lin_heads * w.N * w.d * esz
        conv_bytes = 4 * w.batch * w.conv_heads * w.N * w.d * esz
        t_lin, t_conv = time_calls_alone(w, xs, stream, n=max(200, args.steps // 4))
        step_s = el_max / args.steps
        achieved = workload_bytes(w) / step_s / 1e9
        conv_name = "dw_band<bf16, dot>" if w.loss == "dot" else "dw_band<bf16>"
        roof = {"bound": "hbm",
                "kernel": f"layer step: lin_cluster_bf16 and {conv_name} running at the same time "
                          "(one ttt_forward_layer call)",
                "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": achieved / pk["hbm_gbs"],
                "traffic": STEP_TRAFFIC.get(w.name), "peak_source": pk["source"],
                "algorithmic_bytes": workload_bytes(w), "us_per_launch": step_s * 1e6,
                "kernels_alone": {
                    "lin_cluster_bf16": {"us_per_launch": t_lin * 1e6, "algorithmic_bytes": lin_bytes,
                                         "achieved_gbs": lin_bytes / t_lin / 1e9,
                                         "frac": lin_bytes / t_lin / 1e9 / pk["hbm_gbs"]},
                    conv_name: {"us_per_launch": t_conv * 1e6, "algorithmic_bytes": conv_bytes,
                                       "achieved_gbs": conv_bytes / t_conv / 1e9,
                                       "frac": conv_bytes / t_conv / 1e9 / pk["hbm_gbs"]}}}
    elif w.kind == "backward":
        # plain FP32 FMA kernels: 14 d^2 FLOP per token and head (6 d^2 for G, C, dW1; 8 d^2 for dq, dk,
        # dv); algorithmic bytes: read Q, K, V, dZ and write dQ, dK, dV once (7 N d elements per unit)
        n = max(100, args.steps // 4)
        time_graphs(graphs, 10, stream)
        t_b = time_graphs(graphs, n, stream) / n
        flops = w.batch * w.heads * w.N * 14 * w.d * w.d
        esz = 2 if w.dtype == "bf16" else 4
        nbytes = 7 * w.batch * w.heads * w.N * w.d * esz
        mhz = clocks.get("sm_max_mhz") or 1965.0
        peak = 148 * 128 * 2 * mhz * 1e6 / 1e12
        achieved = flops / t_b / 1e12
        roof = {"bound": "alu", "kernel": "lin_bwd_p1 + lin_bwd_p2 + lin_bwd_sum (the whole ttt_backward_linear call)",
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None,
                "peak_source": f"derived: 148 SMs x 128 FP32 lanes x 2 FLOP x {mhz:.0f} MHz",
                "algorithmic_flops": flops, "algorithmic_bytes": nbytes, "us_per_launch": t_b * 1e6,
                "hbm_gbs": nbytes / t_b / 1e9, "hbm_frac": nbytes / t_b / 1e9 / pk["hbm_gbs"]}
    elif w.kind == "minibatch":
        # a sequential FP32 recurrence: bound by plain FMA issue, not by HBM.  Algorithmic FLOPs per
        # (token, head) are the mini-batch TTT terms 6 d^2 + 4 b d; the peak is 148 SMs x 128 FP32
        # lanes x 2 FLOP per FMA at the SM clock sampled during the run (its maximum if no sample).
        n = max(100, args.steps // 4)
        time_graphs(graphs, 10, stream)
        t_mb = time_graphs(graphs, n, stream) / n
        flops = w.batch * w.heads * w.N * (6 * w.d * w.d + 4 * w.mb_tokens * w.d)
        mhz = clocks.get("sm_max_mhz") or 1965.0
        peak = 148 * 128 * 2 * mhz * 1e6 / 1e12
        achieved = flops / t_mb / 1e12
        roof = {"bound": "alu", "kernel": "lin_minibatch (the whole ttt_forward_linear_minibatch call)",
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None,
                "peak_source": f"derived: 148 SMs x 128 FP32 lanes x 2 FLOP x {mhz:.0f} MHz",
                "algorithmic_flops": flops, "us_per_launch": t_mb * 1e6,
                "hbm_gbs": workload_bytes(w) / t_mb / 1e9}
    elif w.kind == "mlp":
        n = max(100, args.steps // 4)
        time_graphs(graphs, 10, stream)
        t_mlp = time_graphs(graphs, n, stream) / n
        d, hid = w.d, w.hidden_ratio * w.d
        flops = w.batch * w.heads * w.N * (2 * d * hid * 5 + 2 * d * hid * 2)   # 5 products in the step, 2 in the readout
        achieved = flops / t_mlp / 1e12
        roof = {"bound": "tensor", "kernel": "mlp_fused (the whole ttt_forward_mlp call)", "achieved": achieved,
                "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"],
                "traffic": MLP_TRAFFIC.get(w.name),
                "peak_source": pk["source"] + " (bf16 burst)", "algorithmic_flops": flops,
                "us_per_launch": t_mlp * 1e6}

    # end to end through the public API: pinned host inputs -> device -> layer -> host result
    e2e = run_e2e(w, xs[0], dev, stream, args.e2e_steps, world)

    line = {"metric": METRIC_BWD if w.kind == "backward" else METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "global_batch": w.batch * world, "heads": w.heads,
                       "lin_heads": w.lin_heads, "conv_heads": w.conv_heads, "grid": [w.H, w.W],
                       "tokens": w.N, "d": w.d, "eta": w.eta, "loss": w.loss,
                       **({"mb_tokens": w.mb_tokens, "mb_mode": w.mb_mode} if w.kind == "minibatch" else {}),
                       "parallelism": f"batch-sharded x{world}",
                       "l2": f"{args.sets} rotating input sets of {workload_bytes(w) / 1e6:.1f} MB (> 126 MB L2)",
                       "algorithmic_bytes_per_step": workload_bytes(w),
                       "launch": "CUDA graph per input set" + ("; one ttt_forward_layer call per step: the conv kernel "
                                                               "launched behind the linear kernel as a programmatic "
                                                               "dependent, the two running at the same time"
                                                               if w.kind == "mixed" else "")},
            "gbs_per_step": workload_bytes(w) / (el_max / args.steps) / 1e9,
            "gpu_launches": args.steps * (3 if w.kind == "backward" else 2 if (w.kind == "mixed" or w.dtype == "fp32")
                                          else 1),
            "clocks": clocks, "e2e": e2e}
    if roof:
        line["roofline"] = roof
    if rank == 0 and world == 1 and not args.no_oracle:
        line["cpu_baseline"] = time_oracle(w, xs[0], budget_s=12.0)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        del graphs
        dist.destroy_process_group()


def run_e2e(w, x, dev, stream, steps, world):
    """The same metric through the public API with the inputs on the host: every step copies its Q, K,
    V and weights from pinned host memory to the device, runs the layer and copies Z back.  Steps are
    pipelined over two buffer sets and three streams, as a serving loop would run them: the
    host-to-device copy of step i+1 overlaps the compute and the device-to-host copy of step i (PCIe
    moves both directions at once).  Every step's copies are inside the timed region."""
    from vision_test_token_b200 import layer
    names = ["Q", "K", "V"] + (["dZ"] if w.kind == "backward" else []) + sorted(k for k in x if k.startswith("W"))
    host = {k: x[k].cpu().pin_memory() for k in names}
    dev_in = [{k: torch.empty_like(x[k]) for k in names} for _ in range(2)]
    n_out = 3 if w.kind == "backward" else 1                 # dQ, dK, dV, or Z
    z_dev = [[torch.empty_like(x["Q"]) for _ in range(n_out)] for _ in range(2)]
    z_host = [[torch.empty(x["Q"].shape, dtype=x["Q"].dtype).pin_memory() for _ in range(n_out)] for _ in range(2)]
    small = [(torch.empty((w.heads, w.d, w.d), device=dev), torch.empty(1, device=dev)) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in z_host[0])
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
            stream.wait_event(drained[bsel])                 # step i-2's Z has left this buffer
        with torch.cuda.stream(stream):
            if w.kind == "mlp":
                layer.forward_mlp(d["Q"], d["K"], d["V"], d["Wa"], d["Wb"], w.eta, w.H, w.W, Z=z_dev[bsel][0])
            elif w.kind == "minibatch":
                layer.forward_linear_minibatch(d["Q"], d["K"], d["V"], d["W0_lin"], w.eta, w.H, w.W, w.mb_tokens,
                                               w.mb_mode, Z=z_dev[bsel][0])
            elif w.kind == "backward":
                layer.backward_linear(d["Q"], d["K"], d["V"], d["W0_lin"], w.eta, w.H, w.W, d["dZ"],
                                      out=(*z_dev[bsel], *small[bsel]))
            else:
                layer.forward_layer(d["Q"], d["K"], d["V"], d, w.eta, w.H, w.W, conv_heads=w.conv_heads,
                                    Z=z_dev[bsel][0], loss=w.loss)
            computed[bsel].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed[bsel])
            for zh, zd in zip(z_host[bsel], z_dev[bsel]):
                zh.copy_(zd, non_blocking=True)
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
