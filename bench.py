"""Benchmark of the routed-expert MoE layer with decoupled top-k1/top-k2
renormalisation on B200.

Default workload ("decode_b1"): 48 layers, each with its own weights,
d=2048, E=128 experts, I=768, bf16, T=1 token per layer per step, no router
bias; headline condition k1=4, k2=16 (half the trained k of 8, reference
mass of 16 experts), with the other five (k1, k2) conditions of the sweep
reported beside it.  A step is one token through all 48 layers, each layer's
router -> softmax -> top-k -> Eq. 2 weights -> expert FFN -> combine, the
layers chained in one stream (each layer's kernels wait for the previous
layer's) and replayed from one CUDA graph.  value = tokens/s of the 48-layer
stack (T / step time, summed over ranks); us_per_layer = step time / 48.

    python bench.py [--gpus N --steps K --warmup W] [--impl native|reference]
                    [--workload decode_b1|decode_small_batch|prefill|large]
                    [--k1 K1 --k2 K2] [--T T] [--layers L]

N > 1: launched by torch.distributed.run, one rank per GPU, each rank an
independent replica decoding its own tokens (weak scaling, no collective on
the data path; one all-reduce of the elapsed time after the timed region).
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "MoE-layer tokens/s and achieved HBM GB/s (decode) / TFLOP/s (prefill) vs k1,k2"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_PATH = os.path.join(ROOT, "profiles", "traffic.json")

WORKLOADS = {
    "decode_b1": dict(T=1, d=2048, E=128, I=768, layers=48, bias=None,
                      sweep=[(4, 16), (8, 8), (8, 16), (8, 128), (4, 4), (4, 128)]),
    "decode_small_batch": dict(T=8, d=2048, E=128, I=768, layers=48, bias="normal",
                               sweep=[(4, 16), (8, 8)]),
    "prefill": dict(T=4096, d=2048, E=128, I=768, layers=4, bias="zipf", sweep=[(8, 16), (4, 16)]),
    "large": dict(T=1, d=4096, E=512, I=1024, layers=8, bias=None, sweep=[(5, 20), (10, 10)]),
}


# ---------------------------------------------------------------------- helpers
def load_peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def kernel_source_digest():
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "routed_expert_layer_route_b200", "csrc")
    for name in sorted(os.listdir(d)):
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, k1, kernel):
    """ncu DRAM bytes per launch of the dominant kernel, if recorded for the
    current kernel source (null once the source has changed)."""
    try:
        with open(TRAFFIC_PATH) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("source_digest") != kernel_source_digest():
        return None
    return rec.get(kernel, {}).get("%s_k1_%d" % (workload, k1))


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled from before the timed
    region to after it; samples are kept with their host time so the ones
    inside a window can be picked out."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_id):
        self.gpu = gpu_id
        self.proc = None
        self.samples = []  # (host time, sm MHz, max MHz, set of active reasons)
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        t0 = time.time()
        while not self.samples and time.time() - t0 < 5.0:  # let the sampler come up
            time.sleep(0.05)

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.strip().split(",")]
            if len(parts) < 8:
                continue
            try:
                sm, mx = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            reasons = {n for n, v in zip(self.NAMES, parts[4:8]) if v.lower() == "active"}
            self.samples.append((time.time(), sm, mx, reasons))

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)

    def summary(self, t0, t1, min_samples=3):
        sel = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed region"
        if len(sel) < min_samples:
            return None, window
        reasons = set()
        for s in sel:
            reasons |= s[3]
        return {"sm_mhz": statistics.median(s[1] for s in sel),
                "sm_max_mhz": max(s[2] for s in sel), "samples": len(sel),
                "reasons": sorted(reasons), "window": window}, window


def smi_index(local):
    """nvidia-smi's id for this process's CUDA device."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local < len(ids):
            return ids[local]
    return str(local)


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def allreduce_max(v, world, device="cuda"):
    """Max of v over the ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world, cuda=True):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if cuda:
        torch.cuda.synchronize()


def job_rate(units_per_rank, ms_per_rank, world, device="cuda"):
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time (weak scaling: every rank processes the same units)."""
    ms = allreduce_max(ms_per_rank, world, device)
    return world * units_per_rank * 1000.0 / ms, ms


# ---------------------------------------------------------------------- model
class Stack:
    """L layers of seeded synthetic weights and per-layer tokens on the GPU.
    For one-token workloads the down matrices are packed channel-major once,
    at set-up (moe_pack_w_down; the original layout is then freed), and the
    layers run the single-pass decode path."""

    def __init__(self, wl, seed, device, tau=None, router_std=None, keep_frac=None, skip=None):
        from routed_expert_layer_route_b200 import moe, synth
        self.wl = wl
        self.tau = tau  # not None: the variable-k (cascade) route
        self.skip = skip  # not None: (theta_expert, theta_weight) of expert skipping
        self.keep_frac = keep_frac  # not None: channel top-k, this share of k1*I kept
        self.layers = []
        # one token, or up to eight with "cm": the down matrix channel-major and the
        # single-pass decode kernels (k_decode, k_decode_mt)
        self.channel_major = wl["T"] == 1 or (wl.get("cm") == 1 and wl["T"] <= 8)
        # otherwise two or more tokens: the tensor-core grouped GEMMs (what AUTO picks
        # when d and I fill 128-row tiles), named explicitly so the timed kernels are known
        self.grouped = (not self.channel_major and wl["T"] > 1 and wl["d"] % 128 == 0
                        and wl["I"] % 128 == 0)
        self.flags = (moe.MOE_WDOWN_CHANNEL_MAJOR if self.channel_major else
                      moe.MOE_PATH_GROUPED if self.grouped else moe.MOE_PATH_STREAM)
        for l in range(wl["layers"]):
            L = synth.make_layer(wl["T"], wl["d"], wl["E"], wl["I"], seed=seed, layer=l,
                                 device=device, bias=wl["bias"])
            if router_std:  # router logits with this standard deviation (x is RMS-normalised)
                scale = router_std / (0.02 * wl["d"] ** 0.5)
                L.w_router = (L.w_router.float() * scale).to(torch.bfloat16)
            if skip is not None:  # the per-expert table: seeded uniform [0, 1) stand-in values
                g = torch.Generator(device="cpu").manual_seed(1000003 * (seed + 1) + l)
                L.skip_tab = torch.rand(wl["E"], generator=g).to(device)
            if self.channel_major:
                L.w_down = moe.moe_pack_w_down(L.w_down)
                if keep_frac is not None:
                    L.norms = moe.moe_channel_norms(L.w_down, channel_major=True)
            self.layers.append(L)
        torch.cuda.synchronize()

    def keep(self, k1):
        return max(1, int(round(self.keep_frac * k1 * self.wl["I"])))

    def call(self, L, k1, k2, y, ws, stream, idx=None, count=None, x=None, fixed=False):
        """One layer through the public API: moe_layer, or moe_layer_cascade
        when the stack routes with a cascade, or moe_layer_channel_topk with
        channel top-k (unless fixed)."""
        from routed_expert_layer_route_b200 import moe
        x = L.x if x is None else x
        if self.skip is not None and not fixed:
            moe.moe_layer_skip(x, L.w_router, L.bias, L.w_gate, L.w_up, L.w_down, k1, k2,
                               L.skip_tab, self.skip[0], self.skip[1], y, ws, topk_idx_out=idx,
                               topk_count_out=count, flags=self.flags, stream=stream)
        elif self.keep_frac is not None and not fixed:
            moe.moe_layer_channel_topk(x, L.w_router, L.bias, L.w_gate, L.w_up, L.w_down, L.norms,
                                       k1, k2, self.keep(k1), y, ws, topk_idx_out=idx,
                                       stream=stream)
        elif self.tau is None or fixed:
            moe.moe_layer(x, L.w_router, L.bias, L.w_gate, L.w_up, L.w_down, k1, k2, y, ws,
                          topk_idx_out=idx, flags=self.flags, stream=stream)
        else:
            moe.moe_layer_cascade(x, L.w_router, L.bias, L.w_gate, L.w_up, L.w_down, k1, k2,
                                  self.tau, y, ws, topk_idx_out=idx, topk_count_out=count,
                                  flags=self.flags, stream=stream)

    def down_hf(self, L, e):
        """Expert e's down matrix in the [d x I] layout (host copy for the oracle)."""
        from routed_expert_layer_route_b200 import synth
        wd = L.w_down[e].t() if self.channel_major else L.w_down[e]
        return synth.to_numpy(wd.contiguous())


class OracleLayers:
    """The workload's layers for the oracle arm: the same seeded synthetic
    inputs as Stack (synth.make_layer), in the layouts the oracle reads, with
    nothing from the product library (libmoe.so is never loaded on that arm)."""

    def __init__(self, wl, seed, device):
        from routed_expert_layer_route_b200 import synth
        self.wl = wl
        self.layers = [synth.make_layer(wl["T"], wl["d"], wl["E"], wl["I"], seed=seed, layer=l,
                                        device=device, bias=wl["bias"])
                       for l in range(wl["layers"])]

    def down_hf(self, L, e):
        from routed_expert_layer_route_b200 import synth
        return synth.to_numpy(L.w_down[e].contiguous())


def build_graph(stack, k1, k2, ws_list, ys, stream, fixed=False):
    """Capture one step (every layer's layer call) into a CUDA graph."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        # one eager pass first (module attribute set-up happens outside capture)
        for L, ws, y in zip(stack.layers, ws_list, ys):
            stack.call(L, k1, k2, y, ws, stream, fixed=fixed)
        stream.synchronize()
        with torch.cuda.graph(g, stream=stream):
            for L, ws, y in zip(stack.layers, ws_list, ys):
                stack.call(L, k1, k2, y, ws, stream, fixed=fixed)
    return g


def unique_experts(stack, k1, k2, ws_list, ys, stream):
    """Activated experts per layer and the mean experts per token, read back
    from the routing outputs (empty slots of a cascade route excluded)."""
    from routed_expert_layer_route_b200 import moe
    us, ks = [], []
    wl = stack.wl
    for L, ws, y in zip(stack.layers, ws_list, ys):
        idx = torch.empty(wl["T"], k1, dtype=torch.int32, device=L.x.device)
        stack.call(L, k1, k2, y, ws, stream, idx=idx)
        stream.synchronize()
        taken = idx[idx != moe.MOE_EMPTY_SLOT]
        us.append(int(torch.unique(taken).numel()))
        ks.append(taken.numel() / wl["T"])
    return us, statistics.mean(ks)


def graph_time_per_call(calls, stream, reps):
    """Average device time of one call, the calls captured once into a CUDA
    graph (so host-side work between launches is not on the device timeline)
    and the graph replayed `reps` times between CUDA events on its stream."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        for c in calls:  # one eager pass: first-use set-up stays outside capture
            c()
        stream.synchronize()
        with torch.cuda.graph(g, stream=stream):
            for c in calls:
                c()
        g.replay()  # warm
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(reps):
            g.replay()
        e.record(stream)
    e.synchronize()
    ms = s.elapsed_time(e) / (reps * len(calls))
    del g
    return ms


def time_dominant_kernel(stack, k1, k2, ws_list, ys, stream, reps):
    """Average duration of the streaming expert kernel launched alone (no
    programmatic dependent launch), one launch per layer so weights come from
    HBM, not L2 (batches on the CUDA-core streaming path)."""
    from routed_expert_layer_route_b200 import moe
    calls = [(lambda L=L, ws=ws, y=y: moe.moe_test_expert_stream(
        L.x, L.w_gate, L.w_up, L.w_down, k1, k2, y, ws, flags=stack.flags, stream=stream))
        for L, ws, y in zip(stack.layers, ws_list, ys)]
    return graph_time_per_call(calls, stream, reps)


def time_grouped_kernels(stack, k1, ws_list, stream, reps):
    """Average durations (ms) of the token-row gather, the gate/up and the down
    grouped GEMM, each launched alone on the routing tables the layer's last
    moe_layer call left in its workspace, one launch per layer."""
    from routed_expert_layer_route_b200 import moe
    out = []
    for which in (4, 1, 2):
        calls = [(lambda L=L, ws=ws, which=which: moe.moe_test_expert_grouped(
            L.x, L.w_gate, L.w_up, L.w_down, k1, which, ws, stream=stream))
            for L, ws in zip(stack.layers, ws_list)]
        out.append(graph_time_per_call(calls, stream, reps))
    return out


def e2e_tokens_per_s(stack, k1, k2, ws_list, steps, warmup, stream, graph=True):
    """Through the public API with host buffers: per step, pinned-host ->
    device copy of every layer's tokens, every layer's moe_layer call, and a
    device -> pinned-host copy of every layer's output.  graph: the step (the
    two copies and the layer calls, made through moe_layer while capturing)
    is captured once into a CUDA graph and replayed, as a serving loop
    would; else every step issues the calls from Python."""
    wl = stack.wl
    T, d, L_ = wl["T"], wl["d"], wl["layers"]
    host_x = torch.stack([L.x for L in stack.layers]).cpu().pin_memory()
    host_y = torch.empty(L_, T, d, dtype=torch.bfloat16).pin_memory()
    dev_x = torch.empty(L_, T, d, dtype=torch.bfloat16, device="cuda")
    dev_y = torch.empty(L_, T, d, dtype=torch.bfloat16, device="cuda")

    def step():
        dev_x.copy_(host_x, non_blocking=True)
        for l, (L, ws) in enumerate(zip(stack.layers, ws_list)):
            stack.call(L, k1, k2, dev_y[l], ws, stream, x=dev_x[l])
        host_y.copy_(dev_y, non_blocking=True)

    run = step
    g = None
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            step()  # one eager pass: first-use set-up stays outside capture
            stream.synchronize()
            with torch.cuda.graph(g, stream=stream):
                step()
        run = g.replay
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            run()
        stream.synchronize()
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(steps):
            run()
        e.record(stream)
        e.synchronize()
    ms = s.elapsed_time(e) / steps
    del g
    return T * 1000.0 / ms, host_x[0].numel() * 2 * L_, host_y[0].numel() * 2 * L_


# ---------------------------------------------------------------------- CPU oracle
def cpu_oracle_rate(stack, k1, k2, budget_s=12.0, max_tokens=8, stack_layers=None):
    """The oracle as it stands, on the host cores: router logits, routing,
    the k1 experts and the combine, layer after layer until the time budget
    is spent, on the first min(T, max_tokens) tokens of each layer.  Returns
    (tokens/s for a stack of stack_layers layers -- by default the sampled
    stack's own count -- layers run, threads, seconds)."""
    import oracle
    from routed_expert_layer_route_b200 import synth
    wl = stack.wl
    T = min(wl["T"], max_tokens)
    cache = stack.__dict__.setdefault("_oracle_inputs", {})
    prepared = cache.setdefault((k1, k2, T), [])
    # fetch only what the sample needs (router, bias, the routed experts), once
    for L in ([] if prepared else stack.layers):
        x = synth.to_numpy(L.x[:T])
        wr = synth.to_numpy(L.w_router)
        b = synth.to_numpy(L.bias)
        z = oracle.logits(x, wr, b)
        idx, _ = oracle.route_f32(z, k1, k2)
        experts = {int(e): (synth.to_numpy(L.w_gate[int(e)]), synth.to_numpy(L.w_up[int(e)]),
                            stack.down_hf(L, int(e))) for e in np.unique(idx)}
        prepared.append((x, wr, b, experts))
        if len(prepared) >= (6 if wl["T"] == 1 else 2):
            break
    t0 = time.perf_counter()
    n = 0
    while True:
        x, wr, b, experts = prepared[n % len(prepared)]
        z = oracle.logits(x, wr, b)
        oracle.layer_tokens(x, z, lambda e: experts[e], k1, k2)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 1000 * wl["layers"]:
            break
    per_layer = el / n
    return T / (per_layer * (stack_layers or wl["layers"])), n, oracle.num_threads(), el


# ---------------------------------------------------------------------- measurement
def workload_of(args):
    """The workload dict and its (k1, k2) sweep from the command line."""
    wl = dict(WORKLOADS[args.workload])
    if args.T:
        wl["T"] = args.T
    if args.layers:
        wl["layers"] = args.layers
    if getattr(args, "cm", False):
        wl["cm"] = 1
    sweep = list(wl["sweep"])
    if args.k1:
        sweep = [(args.k1, args.k2 or args.k1)]
    elif args.cascade is not None or args.channel_keep is not None or args.skip is not None:
        sweep = [(8, args.k2 or 8)]  # one condition: (cap) k1 = 8, k2 = 8
    return wl, sweep


def workload_config(name, wl, head, world):
    """The line's config: what was run (both arms print this same dict)."""
    T, d, E, I, Ln = wl["T"], wl["d"], wl["E"], wl["I"], wl["layers"]
    k1, k2 = head
    one = T == 1 or wl.get("cm") == 1
    return {"workload": "%s: %d layers, d=%d, E=%d, I=%d, T=%d per rank, k1=%d, k2=%d"
                        % (name, Ln, d, E, I, T, k1, k2),
            "layers": Ln, "d": d, "E": E, "I": I, "T": T, "k1": k1, "k2": k2,
            "bias": wl["bias"],
            "l2": "inputs larger than L2: every step reads the routed experts of all %d layers "
                  "(%.1f GB of expert weights) from HBM" % (Ln, Ln * E * 3 * d * I * 2 / 1e9),
            "timing": "CUDA graph of the %d-layer step, CUDA events, max over ranks" % Ln,
            "w_down_layout": "channel-major [E x I x d], packed once at set-up" if one
            else "[E x d x I]",
            "parallelism": "replicas" if world > 1 else "single GPU"}


def line_config(args, wl, head, world):
    """workload_config plus the variant switches of the command line."""
    c = workload_config(args.workload, wl, head, world)
    c.update({"cascade_tau": args.cascade, "router_logit_std": args.router_std,
              "channel_keep_frac": args.channel_keep,
              "skip_thresholds": list(args.skip) if args.skip is not None else None})
    return c


def timed_graph(graph, steps, warmup, world, stream):
    """Device time of `steps` replays of a CUDA graph, `warmup` replays first,
    barrier + synchronize on both sides; the max over ranks."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            graph.replay()
    stream.synchronize()
    barrier(world)
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    h0 = time.time()
    s.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(steps):
            graph.replay()
    e.record(stream)
    e.synchronize()
    h1 = time.time()
    barrier(world)
    return allreduce_max(s.elapsed_time(e), world) / steps, (h0, h1)


def layer_work(stack, k1, U, mean_k):
    """Algorithmic bytes and FLOPs of one layer: the unique routed experts'
    weights, U*3*d*I*2 bytes, and T*(k*6*d*I + 2*d*E) FLOPs (channel top-k:
    every gate/up row, the norms and the kept down columns)."""
    wl = stack.wl
    T, d, E, I = wl["T"], wl["d"], wl["E"], wl["I"]
    if stack.keep_frac is not None:
        b = U * 2 * d * I * 2 + U * I * 4 + T * stack.keep(k1) * d * 2
        f = T * (mean_k * 4.0 * d * I + 2.0 * stack.keep(k1) * d + 2.0 * d * E)
        return b, f
    return U * 3 * d * I * 2, T * (mean_k * 6.0 * d * I + 2.0 * d * E)


def measure_sweep(stack, sweep, args, world, stream, peaks):
    """Every (k1, k2) condition: one CUDA graph of the whole step each, timed
    by the contract's protocol; unique experts read back from the routing.
    Returns (results, graphs, headline ms, headline window)."""
    from routed_expert_layer_route_b200 import moe
    hbm_peak, bf16_peak, _ = peaks
    wl = stack.wl
    T, d, E, I, Ln = wl["T"], wl["d"], wl["E"], wl["I"], wl["layers"]
    dev = stack.layers[0].x.device
    graphs = {}
    for (k1, k2) in sweep:
        # zeroed on the stream the layers run on (a side stream, which does not
        # wait for the default one by itself)
        ws_list = [moe.workspace(T, d, E, I, k1, device=dev, stream=stream) for _ in range(Ln)]
        ys = [torch.empty(T, d, dtype=torch.bfloat16, device=dev) for _ in range(Ln)]
        stream.wait_stream(torch.cuda.current_stream())
        graphs[(k1, k2)] = (build_graph(stack, k1, k2, ws_list, ys, stream), ws_list, ys)
    results, head_ms, head_win = [], None, None
    for (k1, k2) in sweep:
        g, ws_list, ys = graphs[(k1, k2)]
        ms, win = timed_graph(g, args.steps, args.warmup, world, stream)
        if head_ms is None:
            head_ms, head_win = ms, win
        us, mean_k = unique_experts(stack, k1, k2, ws_list, ys, stream)
        U = statistics.mean(us)
        b, f = layer_work(stack, k1, U, mean_k)
        lay_s = ms / Ln * 1e-3
        results.append({"k1": k1, "k2": k2, "ms_per_step": ms, "us_per_layer": ms * 1000 / Ln,
                        "tokens_per_s": world * T * 1000.0 / ms, "unique_experts_per_layer": U,
                        "mean_experts_per_token": mean_k, "bytes_per_layer": b,
                        "flops_per_layer": f, "expert_GBps": b / lay_s / 1e9,
                        "hbm_frac": b / lay_s / 1e9 / hbm_peak,
                        "layer_TFLOPs": f / lay_s / 1e12,
                        "tensor_frac": f / lay_s / 1e12 / bf16_peak})
    return results, graphs, head_ms, head_win


def k1_ratio(results):
    """Layer time of k1 = 4 over k1 = 8 (same k2 where possible)."""
    by = {(r["k1"], r["k2"]): r for r in results}
    for p4, p8 in (((4, 16), (8, 16)), ((4, 4), (8, 8)), ((4, 16), (8, 8)), ((5, 20), (10, 10))):
        if p4 in by and p8 in by:
            return (round(by[p4]["us_per_layer"] / by[p8]["us_per_layer"], 4),
                    "k1=%d,k2=%d over k1=%d,k2=%d" % (p4 + p8))
    return None, None


def peak_note(kind, what):
    return ("measured (MEASURED_PEAKS.json %s)" % what) if kind == "measured" else \
        "fallback 6650 GB/s, 1590 TFLOP/s"


def roofline_record(stack, workload, head, res, graphs, stream, peaks, variant):
    """Roofline of the dominant kernel of the headline condition.
    One token: the layer is one kernel (router, routing, expert FFN, combine),
    so its average duration in the timed graph is the layer time; bound by
    HBM on the unique routed experts' bytes.  Tensor-core batches: the gate/up
    grouped GEMM alone (and the down GEMM), with the bound that binds for its
    FLOPs and its weight bytes.  CUDA-core streaming batches: that kernel alone."""
    hbm_peak, bf16_peak, kind = peaks
    wl = stack.wl
    T, d, E, I, Ln = wl["T"], wl["d"], wl["E"], wl["I"], wl["layers"]
    k1, k2 = head
    _, ws_list, ys = graphs[head]
    U = res["unique_experts_per_layer"]
    alg_bytes = res["bytes_per_layer"]
    if variant or stack.channel_major:
        lay_s = res["us_per_layer"] * 1e-6
        achieved = alg_bytes / lay_s / 1e9
        dk = "k_decode" if T == 1 else "k_decode_mt"
        kname = ("whole layer (cascade route)" if stack.tau is not None else
                 "whole layer (expert skipping)" if stack.skip is not None else
                 "whole layer (channel top-k: k_logits, k_ctk_gateup, k_ctk_down)"
                 if stack.keep_frac is not None else "moe::" + dk)
        return {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(achieved / hbm_peak, 4),
                "traffic": None if variant else recorded_traffic(
                    workload if T == 1 else "%s_T%d" % (workload, T), k1, dk),
                "frac_of_nominal_8000_GBps": round(achieved / 8000.0, 4),
                "kernel": kname, "kernel_us": round(lay_s * 1e6, 3),
                "launches_per_layer": 1 if not variant or stack.keep_frac is None else 3,
                "algorithmic_bytes_per_launch": int(alg_bytes),
                "duration_from": "the headline's timed CUDA graph (one kernel per layer)",
                "peak_source": peak_note(kind, "hbm_gbs")}
    if stack.grouped:
        gx_ms, g1_ms, g2_ms = time_grouped_kernels(stack, k1, ws_list, stream, reps=3)
        n_slots = T * k1
        # algorithmic work of each GEMM: FLOPs, and the unique experts' weight
        # bytes (the gathered token rows and h are traffic of this design)
        f1 = 2.0 * n_slots * 2 * I * d
        b1 = U * 2 * d * I * 2
        f2 = 2.0 * n_slots * I * d
        b2 = U * d * I * 2

        def bound(f, b, ms):
            t_tensor, t_hbm = f / (bf16_peak * 1e12), b / (hbm_peak * 1e9)
            tf = f / (ms * 1e-3) / 1e12
            gb = b / (ms * 1e-3) / 1e9
            if t_tensor >= t_hbm:
                return "tensor", tf, bf16_peak, "TFLOP/s", tf / bf16_peak
            return "hbm", gb, hbm_peak, "GB/s", gb / hbm_peak

        bd1, a1, p1, u1, fr1 = bound(f1, b1, g1_ms)
        # the gate/up GEMM runs on CTA pairs when I is a multiple of 256
        from routed_expert_layer_route_b200 import moe
        g1_name = "k_gemm1_pair" if I % 256 == 0 and moe.moe_test_grouped_pairs(1) > 0 else "k_gemm1"
        bd2, a2, p2, u2, fr2 = bound(f2, b2, g2_ms)
        return {"bound": bd1, "achieved": round(a1, 1), "peak": p1, "unit": u1,
                "frac": round(fr1, 4), "traffic": recorded_traffic(workload, k1, g1_name),
                "kernel": "moe::" + g1_name, "kernel_us": round(g1_ms * 1000, 2),
                "algorithmic_flops_per_launch": f1, "algorithmic_bytes_per_launch": int(b1),
                "tensor_frac": round(f1 / (g1_ms * 1e-3) / 1e12 / bf16_peak, 4),
                "hbm_frac": round(b1 / (g1_ms * 1e-3) / 1e9 / hbm_peak, 4),
                "second_kernel": {"kernel": "moe::k_gemm2", "kernel_us": round(g2_ms * 1000, 2),
                                  "bound": bd2, "achieved": round(a2, 1), "unit": u2,
                                  "frac": round(fr2, 4), "algorithmic_flops_per_launch": f2,
                                  "algorithmic_bytes_per_launch": int(b2)},
                "gather_kernel": {"kernel": "moe::k_gather_rows",
                                  "kernel_us": round(gx_ms * 1000, 2)},
                "duration_from": "CUDA graph of one launch per layer, kernel alone",
                "peak_source": peak_note(kind, "bf16_tflops burst and hbm_gbs: kernels timed "
                                               "alone")}
    kern_ms = time_dominant_kernel(stack, k1, k2, ws_list, ys, stream, reps=5)
    achieved = alg_bytes / (kern_ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
            "frac": round(achieved / hbm_peak, 4),
            "traffic": recorded_traffic(workload, k1, "k_stream"),
            "kernel": "moe::k_stream", "kernel_us": round(kern_ms * 1000, 2),
            "algorithmic_bytes_per_launch": int(alg_bytes),
            "duration_from": "CUDA graph of one launch per layer, kernel alone",
            "peak_source": peak_note(kind, "hbm_gbs")}


def layer_roofline(res, peaks):
    """The whole layer against its roofline time max(FLOPs / bf16 peak,
    unique expert bytes / HBM bandwidth)."""
    hbm_peak, bf16_peak, _ = peaks
    t_f = res["flops_per_layer"] / (bf16_peak * 1e12)
    t_b = res["bytes_per_layer"] / (hbm_peak * 1e9)
    t = res["us_per_layer"] * 1e-6
    return {"bound": "tensor" if t_f >= t_b else "hbm",
            "roofline_us": round(max(t_f, t_b) * 1e6, 2),
            "frac_of_roofline_time": round(max(t_f, t_b) / t, 4),
            "layer_TFLOPs": round(res["layer_TFLOPs"], 1),
            "tensor_frac": round(res["tensor_frac"], 4), "hbm_frac": round(res["hbm_frac"], 4)}


# workloads timed after the headline in the default run, each a sub-record
# prefill, the small batches on the grouped GEMMs, the large model, then the few-token
# kernel on the channel-major down matrix at the small batches' sizes
EXTRA_WORKLOADS = [
    ("prefill", {}),
    ("decode_small_batch", {"T": 2}), ("decode_small_batch", {"T": 4}),
    ("decode_small_batch", {"T": 8}), ("decode_small_batch", {"T": 32}),
    ("decode_small_batch", {"T": 64}),
    ("large", {"T": 1}), ("large", {"T": 64}),
    ("decode_small_batch", {"T": 2, "cm": 1}), ("decode_small_batch", {"T": 4, "cm": 1}),
    ("decode_small_batch", {"T": 8, "cm": 1}),
]


def extra_record(name, over, args, world, rank, stream, peaks):
    """One more workload, timed like the headline: its sweep, unique experts,
    the k1 ratio and the roofline of its dominant kernel."""
    wl = dict(WORKLOADS[name])
    wl.update(over)
    dev = torch.device("cuda", torch.cuda.current_device())
    stack = Stack(wl, seed=rank, device=dev)
    res, graphs, _, _ = measure_sweep(stack, wl["sweep"], args, world, stream, peaks)
    roof = roofline_record(stack, name, wl["sweep"][0], res[0], graphs, stream, peaks, False)
    ratio, pair = k1_ratio(res)
    rec = {"workload": workload_config(name, wl, wl["sweep"][0], world)["workload"],
           "T": wl["T"], "layers": wl["layers"],
           "conditions": [{k: (round(v, 4) if isinstance(v, float) else v) for k, v in r.items()}
                          for r in res],
           "k1_ratio": ratio, "k1_ratio_conditions": pair, "roofline": roof,
           "layer_roofline": [dict(layer_roofline(r, peaks), k1=r["k1"], k2=r["k2"]) for r in res]}
    for g, _, _ in graphs.values():
        del g
    graphs.clear()
    del stack
    release_memory()
    return rec


def release_memory():
    import gc
    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def run_native(args, world, rank):
    from routed_expert_layer_route_b200 import build as pkg_build
    pkg_build.build()
    wl, sweep = workload_of(args)
    head = sweep[0]
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.Stream()
    peaks = load_peaks()
    hbm_peak, bf16_peak, peak_kind = peaks

    if args.channel_keep is not None and wl["T"] != 1:
        raise SystemExit("--channel-keep: one-token workloads only (T = 1)")
    stack = Stack(wl, seed=rank, device=dev, tau=args.cascade, router_std=args.router_std,
                  keep_frac=args.channel_keep, skip=args.skip)
    variant = stack.tau is not None or stack.keep_frac is not None or stack.skip is not None
    T, d, E, I, Ln = wl["T"], wl["d"], wl["E"], wl["I"], wl["layers"]

    # headline: the timed region of the contract (clocks sampled around it),
    # then every other (k1, k2) condition of the sweep by the same protocol
    clocks = ClockSampler(smi_index(torch.cuda.current_device()))
    clocks.start()
    results, graphs, ms_step, head_win = measure_sweep(stack, sweep, args, world, stream, peaks)
    sweep_t1 = time.time()
    value = world * T * 1000.0 / ms_step

    cascade = None
    channel_topk = None
    if variant:
        # the same stack with the fixed-k1 full layer: compute / bytes saved vs time saved
        k1h_, k2h_ = head
        _, ws_list, ys = graphs[head]
        gf = build_graph(stack, k1h_, k2h_, ws_list, ys, stream, fixed=True)
        graphs[("fixed",) + head] = (gf, ws_list, ys)
        ms_fixed = timed_graph(gf, args.steps, args.warmup, world, stream)[0]
        fixed_us = ms_fixed * 1000 / Ln
        if stack.keep_frac is not None:
            U0 = results[0]["unique_experts_per_layer"]
            channel_topk = {"keep": stack.keep(k1h_), "keep_frac": stack.keep_frac, "k1": k1h_,
                            "k2": k2h_, "channels_per_token": k1h_ * I,
                            "us_per_layer": results[0]["us_per_layer"],
                            "full_layer_us_per_layer": fixed_us,
                            "time_ratio_vs_full": results[0]["us_per_layer"] / fixed_us,
                            "bytes_ratio_vs_full": results[0]["bytes_per_layer"]
                            / (U0 * 3 * d * I * 2)}
        else:
            cascade = {"tau": stack.tau, "skip_thresholds": stack.skip, "k1_cap": k1h_,
                       "k2": k2h_, "mean_experts_per_token": results[0]["mean_experts_per_token"],
                       "us_per_layer": results[0]["us_per_layer"],
                       "fixed_k1_us_per_layer": fixed_us,
                       "time_ratio_vs_fixed": results[0]["us_per_layer"] / fixed_us,
                       "compute_ratio_vs_fixed": results[0]["mean_experts_per_token"] / k1h_}

    clocks.stop()
    clk, _ = clocks.summary(*head_win)
    if clk is None:  # timed region shorter than the sampling period: use the sweep's
        clk, _ = clocks.summary(head_win[0], sweep_t1)
        if clk is not None:
            clk["window"] = "headline and sweep timed regions"

    roofline = roofline_record(stack, args.workload, head, results[0], graphs, stream, peaks,
                               variant)
    k1h, k2h = head
    _, ws_list, ys = graphs[head]

    # end to end through the public API with host buffers: the step captured
    # once into a CUDA graph (as a serving loop would), and issued from Python
    e2e_val, h2d, d2h = e2e_tokens_per_s(stack, k1h, k2h, ws_list, max(3, args.steps // 4),
                                         args.warmup, stream, graph=True)
    e2e_val = world * T * 1000.0 / allreduce_max(T * 1000.0 / e2e_val, world)
    e2e_eager, _, _ = e2e_tokens_per_s(stack, k1h, k2h, ws_list, max(3, args.steps // 4),
                                       args.warmup, stream, graph=False)
    e2e_eager = world * T * 1000.0 / allreduce_max(T * 1000.0 / e2e_eager, world)
    ratio, ratio_pair = k1_ratio(results)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not variant:
        rate, nl, thr, el = cpu_oracle_rate(stack, k1h, k2h)
        cpu = {"value": rate, "unit": "tokens/s", "cores": thr, "kind": "oracle",
               "sample": "%d layers of this workload, first %d token(s) of each (k1=%d, k2=%d), "
                         "in %.1f s; per-layer time scaled to the %d-layer stack"
                         % (nl, min(T, 8), k1h, k2h, el, Ln)}

    # kernels per layer: the one-token layer kernel; router logits, warp router,
    # permutation (2), token-row gather, two grouped GEMMs, finalize (tensor-core
    # path); router logits, top-k, streaming kernel (streaming path)
    per_step_launches = 1 if stack.channel_major else (8 if stack.grouped else 3)
    if stack.keep_frac is not None:
        per_step_launches = 1 + 2 * T  # router logits, then two kernels per token
    config = line_config(args, wl, head, world)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "us_per_layer": round(ms_step * 1000 / Ln, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,0.02) weights, RMS-normalised N(0,1) tokens)",
        "config": config,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_val, 3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "path": "per step: pinned host x -> device, moe_layer (C-ABI) per layer, y -> "
                        "pinned host; the step captured once into a CUDA graph and replayed",
                "eager": {"value": round(e2e_eager, 3), "unit": "tokens/s",
                          "path": "the same step issued from Python every time (ctypes call "
                                  "per layer)"}},
        "gpu_launches": per_step_launches * Ln * args.steps,
        "clocks": clk,
        "sweep": results,
        "cascade": cascade,
        "channel_topk": channel_topk,
        "k1_4_over_k1_8_time_ratio": ratio,
        "k1_ratio_conditions": ratio_pair,
    }
    for g, _, _ in graphs.values():
        del g
    graphs.clear()
    del stack
    release_memory()

    # the other workloads (small batches, prefill, the large model), each a
    # sub-record with its own sweep, unique experts, k1 ratio and roofline
    default = (args.workload == "decode_b1" and not args.k1 and not args.T and not args.layers
               and not getattr(args, "cm", False)
               and not variant and not args.no_extra)
    if default:
        extra = {}
        for name, over in EXTRA_WORKLOADS:
            key = name + "".join("_%s%d" % kv for kv in sorted(over.items()))
            if rank == 0:
                print("bench: workload %s" % key, file=sys.stderr, flush=True)
            extra[key] = extra_record(name, over, args, world, rank, stream, peaks)
        line["workloads"] = extra
        line["k1_ratio_by_batch"] = {
            "T=1": {"ratio": ratio, "conditions": ratio_pair},
            **{"T=%d" % extra[k]["T"]: {"ratio": extra[k]["k1_ratio"],
                                        "conditions": extra[k]["k1_ratio_conditions"]}
               for k in ("decode_small_batch_T8", "decode_small_batch_T32",
                         "decode_small_batch_T64")}}
    return line


def run_reference(args, world, rank):
    """The oracle as it stands on the host cores, on the same workload."""
    if rank != 0:
        return None
    wl, sweep = workload_of(args)
    k1, k2 = sweep[0]
    dev = torch.device("cuda", torch.cuda.current_device())
    small = dict(wl)
    small["layers"] = min(6, wl["layers"])
    stack = OracleLayers(small, seed=0, device=dev)
    rates = []
    # each step a bounded sample: the whole run stays near two minutes at any K
    step_s = max(0.05, min(3.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_oracle_rate(stack, k1, k2, budget_s=step_s, stack_layers=wl["layers"])
    t0 = time.perf_counter()
    for _ in range(args.steps):
        r, nl, thr, el = cpu_oracle_rate(stack, k1, k2, budget_s=step_s, stack_layers=wl["layers"])
        rates.append(r)
    total = time.perf_counter() - t0
    # each rate is already the per-layer time scaled to the full stack
    r_stack = statistics.mean(rates)
    return {
        "impl": "reference", "metric": METRIC, "value": round(r_stack, 4), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1000.0 * wl["T"] / r_stack, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32 (bf16 inputs widened)",
        "data": "synthetic", "config": line_config(args, wl, (k1, k2), world),
        "cpu_baseline": {"value": round(r_stack, 4), "unit": "tokens/s", "cores": thr,
                         "kind": "oracle", "sample": "each step: layers of this workload for "
                                                     "%.2f s, first %d token(s) of each; per-layer "
                                                     "time scaled to the %d-layer stack"
                                                     % (step_s, min(wl["T"], 8), wl["layers"])},
        "e2e": {"value": round(r_stack, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "wall_s": round(total, 2),
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="decode_b1")
    ap.add_argument("--k1", type=int, default=0)
    ap.add_argument("--k2", type=int, default=0)
    ap.add_argument("--T", type=int, default=0)
    ap.add_argument("--layers", type=int, default=0)
    ap.add_argument("--cm", action="store_true",
                    help="2 <= T <= 8: down matrices packed channel-major at set-up, the layers "
                         "on the few-token decode kernel")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only the chosen workload (the default run also times the small "
                         "batches, prefill and the large model as sub-records)")
    ap.add_argument("--cascade", type=float, default=None, metavar="TAU",
                    help="variable experts per token: the first k <= k1 covering mass TAU")
    ap.add_argument("--skip", type=float, nargs=2, default=None, metavar=("TH_E", "TH_W"),
                    help="expert skipping (top-1 kept): skip a slot when its expert's table "
                         "value < TH_E and its weight < TH_W (seeded uniform table)")
    ap.add_argument("--channel-keep", type=float, default=None, metavar="FRAC",
                    help="channel top-k: keep this share of each token's k1*I channels")
    ap.add_argument("--router-std", type=float, default=None,
                    help="scale the router so its logits have this standard deviation")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            line = run_reference(args, world, rank)
        else:
            line = run_native(args, world, rank)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
