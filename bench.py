"""Benchmark of the SLoPe layer step on B200.

One step = the whole hot path over one batch, for every linear of the
workload, through the one-launch calls: prune24_double (the row mask and
compression of prune24 and the transposed backward copy of double_prune),
fwd_fused (XL = X.L and the sparse product with the adapter), bwd_dx_fused
(G = dY.R^T and the sparse input gradient with the adapter) and bwd_dw_fused
(the masked weight gradient with dL and dR); with more than one GPU the gradients (compressed dW, dL, dR) are then summed
across ranks with NCCL (data parallelism: every rank holds the same weights
and its own tokens).

Metric: dense-equivalent TFLOP/s of the layer's fwd+bwd (6*T*in*out per
linear, plus the adapter's 6*T*r*(in+out)) over the device time of the step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C5] [--impl ours|reference]
    python bench.py --fwd-sweep --config C5 [--steps K] [--warmup W]
    python bench.py --adamw-step --config C5 [--steps K] [--warmup W]

The default workload is the largest one that fits one GPU (C5, OPT-66B-shaped
linears, 8192 tokens per GPU).  With `--gpus N` and no WORLD_SIZE in the
environment the script starts its own N ranks (one process per GPU, NCCL);
under torchrun it uses the ranks it is given.  Prints one JSON line (rank 0).
`--impl reference` times the CPU oracle on a bounded sample of the same
workload instead.  `--fwd-sweep` times inference
(adapter_fwd + fwd over the layers) at 1, 16, 128 and 2048 tokens, one line
per token count, against HBM bandwidth.
"""
import argparse
import json
import os
import signal
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

from structured_sparse_pretraining_b200 import dp  # noqa: E402
from structured_sparse_pretraining_b200 import inputs as I  # noqa: E402

METRIC = "SLoPe linear fwd+bwd TFLOP/s and % of 2:4-sparse BF16 peak; speedup vs dense"
UNIT = "TFLOP/s"
L2_FLUSH_BYTES = 256 << 20


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------ flop / byte accounting
def layer_flops(T, inn, out, r):
    """Dense-equivalent flops of one linear's fwd+bwd and of its adapter."""
    dense = 6.0 * T * inn * out
    adapter = 6.0 * T * r * (inn + out)
    return dense, adapter


def kernel_work(op, T, inn, out, r):
    """(dense-equivalent flops, algorithmic bytes) of one launch of `op`."""
    if op == "prune24":
        return 0.0, 3.125 * inn * out
    if op == "double_prune":
        return 0.0, 2.25 * inn * out
    if op == "prune24_double":  # W read once; W^R and (W^{R,C})^T written
        return 0.0, 4.25 * inn * out
    if op == "adapter_fwd":
        return 2.0 * T * inn * r, 2.0 * (T * inn + inn * r + T * r)
    if op == "fwd":  # X, W^R values + codes, XL, R in; Y out
        return (2.0 * T * inn * out + 2.0 * T * r * out,
                2.0 * T * inn + 1.125 * inn * out + 2.0 * r * (T + out) + 2.0 * T * out)
    if op == "adapter_bwd":
        return 2.0 * T * r * (2 * out + inn), 2.0 * (2 * T * out + T * inn) + 8.0 * r * (inn + out)
    if op == "bwd_dx":  # dY, W^{R,C} values + codes, G, L in; dX out
        return (2.0 * T * inn * out + 2.0 * T * r * inn,
                2.0 * T * out + 1.125 * inn * out + 2.0 * r * (T + inn) + 2.0 * T * inn)
    if op == "bwd_dw_masked":
        return 1.0 * T * inn * out, 2.0 * T * (inn + out) + 1.125 * inn * out
    # the fused calls: the same plus the adapter's rank products
    if op == "fwd_fused":  # XL = X.L, then Y; XL written
        return (2.0 * T * inn * out + 2.0 * T * r * (inn + out),
                2.0 * T * inn + 1.125 * inn * out + 2.0 * r * (inn + out) + 2.0 * T * (r + out))
    if op == "bwd_dx_fused":  # G = dY.R^T, then dX; G written
        return (2.0 * T * inn * out + 2.0 * T * r * (inn + out),
                2.0 * T * out + 1.125 * inn * out + 2.0 * r * (inn + out) + 2.0 * T * (r + inn))
    if op == "bwd_dw_fused":  # masked dW (the kept half), dR and dL
        return (1.0 * T * inn * out + 2.0 * T * r * (inn + out),
                2.0 * T * (inn + out + 2 * r) + 1.125 * inn * out + 4.0 * r * (inn + out))
    raise KeyError(op)


OPS = ["prune24_double", "fwd_fused", "bwd_dx_fused", "bwd_dw_fused"]

# The device function each entry point's dominant launch runs (the sparse
# products: see kernel_of).
KERNEL_OF_OP = {"prune24": "prune24_kernel", "double_prune": "double_prune_kernel",
                "prune24_double": "double_prune_kernel", "adapter_fwd": "gemm_kernel",
                "fwd": "sp_pair_kernel", "adapter_bwd": "gemm_kernel", "bwd_dx": "sp_pair_kernel",
                "bwd_dw_masked": "dw_pair_kernel", "fwd_fused": "sp_wide_kernel", "bwd_dx_fused": "sp_wide_kernel",
                "bwd_dw_fused": "dw_pair_kernel"}


def fusable(M, T, K, r, sms=148):
    """The shapes whose fused calls run as one sp_wide_kernel launch (else two
    launches), as the library's planner decides."""
    from structured_sparse_pretraining_b200 import ops
    return ops.fused_launches(M, T, K, r, sms) == 1


def kernel_of(op, T, inn, out, r=0, sms=148):
    """Device function of one launch: the plain sparse products run
    sp_wide_kernel when the planner takes 512-row tiles for their shape, else
    sp_pair_kernel; the fused ones run sp_wide_kernel where fusable."""
    if op in ("fwd", "bwd_dx"):
        from structured_sparse_pretraining_b200 import ops
        M, K = (out, inn) if op == "fwd" else (inn, out)
        return "sp_wide_kernel" if ops.sparse_tile_rows(M, T, K, sms) == 512 else "sp_pair_kernel"
    if op in ("fwd_fused", "bwd_dx_fused") and not (fusable(out, T, inn, r, sms) if op == "fwd_fused"
                                                    else fusable(inn, T, out, r, sms)):
        return kernel_of(op.replace("_fused", ""), T, inn, out, r, sms)
    return KERNEL_OF_OP[op]

# DRAM bytes (read + write) per launch of the dominant kernel, averaged over
# its launches in one step, from an ncu capture of the kernel as it stands,
# keyed by (workload, kernel).  A pair absent here has no capture of the
# current code: the roofline's `traffic` is then null.
TRAFFIC_PER_LAUNCH = {
    # mean over the step's launches of each kernel on the OPT-66B-shaped workload (eager warm-up step)
    ("opt66b-linears-d9216-T8192-r92", "sp_wide_kernel"): 3.490e9,
    ("opt66b-linears-d9216-T8192-r92", "dw_pair_kernel"): 5.798e9,
}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"slope_bench_clocks_rank{index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.send_signal(signal.SIGTERM)
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
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
        busy = sorted(sm)[len(sm) // 2:] if sm else []
        return {"sm_mhz": statistics.median(busy) if busy else None, "sm_max_mhz": mx,
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------------ our arm
class LayerState:
    def __init__(self, w, li, seed, device, gen_tokens):
        from structured_sparse_pretraining_b200 import ops
        self.ops = ops
        lay = w.layers[li]
        self.inn, self.out, self.T, self.r = lay.in_features, lay.out_features, gen_tokens, w.rank_stored
        dev = device
        # weights: identical on every rank; tokens: per rank
        wseed = dp.WEIGHT_SEED
        self.W = I.normal_bf16((self.out, self.inn), w.std_w, wseed, li, "W", dev)
        L = I.normal_bf16((self.inn, w.rank), w.std_l, wseed, li, "L", dev) if w.rank else None
        R = I.normal_bf16((w.rank, self.out), w.std_r, wseed, li, "R", dev) if w.rank else None
        self.L, self.R = I.pad_rank(L, R, self.r)
        self.X = I.normal_bf16((self.T, self.inn), w.std_x, seed, li, "X", dev)
        self.dY = I.normal_bf16((self.T, self.out), w.std_dy, seed, li, "dY", dev)
        e = lambda *s, dt=torch.bfloat16: torch.empty(*s, dtype=dt, device=dev)  # noqa: E731
        self.vals, self.meta = e(self.out, self.inn // 2), e(self.out, self.inn // 16, dt=torch.int16)
        self.vals_t, self.meta_t = e(self.inn, self.out // 2), e(self.inn, self.out // 16, dt=torch.int16)
        self.Y, self.dX = e(self.T, self.out), e(self.T, self.inn)
        self.dW = e(self.out, self.inn // 2)
        if self.r:
            self.XL, self.G = e(self.T, self.r), e(self.T, self.r)
            self.dL, self.dR = e(self.inn, self.r, dt=torch.float32), e(self.r, self.out, dt=torch.float32)
        else:
            self.XL = self.G = self.dL = self.dR = None

    def calls(self, X=None, dY=None, dW=None):
        """The layer's hot-path calls, in order: (label, layer, callable).
        X, dY and dW default to the layer's own buffers."""
        o, r = self.ops, self.r
        X = self.X if X is None else X
        dY = self.dY if dY is None else dY
        dW = self.dW if dW is None else dW
        # both prunings run in one launch, and the adapter's rank products
        # inside the sparse products and the masked gradient (the fused
        # calls): four launches per layer
        c = [
            ("prune24_double", lambda: o.prune24_double(self.W, self.vals, self.meta, self.vals_t, self.meta_t)),
            ("fwd_fused", lambda: o.fwd_fused(X, self.vals, self.meta, self.L, self.R, self.out, self.XL, self.Y)),
            ("bwd_dx_fused", lambda: o.bwd_dx_fused(dY, self.vals_t, self.meta_t, self.R, self.L, self.inn, self.G,
                                                     self.dX)),
            ("bwd_dw_fused", lambda: o.bwd_dw_fused(dY, X, self.meta, self.XL, self.G, dW, self.dL, self.dR)),
        ]
        return [(name, self, fn) for name, fn in c]

    def grads(self, dW=None):
        return dp.replicated_gradients(self.dW if dW is None else dW, self.dL, self.dR)


class Markers:
    """Timing events recorded as external event nodes inside a CUDA graph, so
    that each kernel's device time is read from the replay itself."""

    def __init__(self):
        from cuda.bindings import driver
        self.drv = driver
        self.events = []
        self.labels = []

    def mark(self, label):
        d = self.drv
        rc, ev = d.cuEventCreate(0)
        assert rc == d.CUresult.CUDA_SUCCESS, rc
        st = d.CUstream(torch.cuda.current_stream().cuda_stream)
        rc, = d.cuEventRecordWithFlags(ev, st, d.CUevent_record_flags.CU_EVENT_RECORD_EXTERNAL)
        assert rc == d.CUresult.CUDA_SUCCESS, rc
        self.events.append(ev)
        self.labels.append(label)

    def deltas(self):
        """[(label, ms)] between consecutive markers of the last replay."""
        d = self.drv
        out = []
        for i in range(len(self.events) - 1):
            rc, ms = d.cuEventElapsedTime(self.events[i], self.events[i + 1])
            assert rc == d.CUresult.CUDA_SUCCESS, rc
            out.append((self.labels[i], ms))
        return out


def dense_reference_ms(layers, steps=10):
    """The same shapes as a dense bf16 layer with torch.matmul: Y = X W^T,
    dX = dY W, dW = dY^T X (the comparator of the metric's 'speedup vs dense')."""
    Ws = [l.W for l in layers]

    def step():
        for l, W in zip(layers, Ws):
            torch.matmul(l.X, W.t())
            torch.matmul(l.dY, W)
            torch.matmul(l.dY.t(), l.X)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=Ws[0].device)
    tot = 0.0
    for _ in range(steps):
        flush.fill_(1.0)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        step()
        b.record()
        b.synchronize()
        tot += a.elapsed_time(b)
    return tot / steps


def run_e2e(layers, steps, world, bucket):
    """The same step end to end through the public ops (eager calls): every
    step copies each layer's X and dY in from pinned host memory and its
    compressed dW (summed over ranks when world > 1) back out to pinned host
    memory.  Copies in and out run on two streams of their own, so that they
    overlap the compute of other layers and steps; two device buffer sets per
    layer are used by turns, with events guarding their reuse.  Returns
    (ms per step, H2D bytes per step, D2H bytes per step)."""
    dev = layers[0].X.device
    comp = torch.cuda.current_stream()
    h2d_s, d2h_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    pinned_in = [(l.X.cpu().pin_memory(), l.dY.cpu().pin_memory()) for l in layers]
    pinned_out = [torch.empty(l.dW.shape, dtype=l.dW.dtype).pin_memory() for l in layers]
    h2d = sum(x.numel() * x.element_size() + y.numel() * y.element_size() for x, y in pinned_in)
    d2h = sum(t.numel() * t.element_size() for t in pinned_out)
    sets = [[(l.X, l.dY, l.dW), (torch.empty_like(l.X), torch.empty_like(l.dY), torch.empty_like(l.dW))]
            for l in layers]
    calls = [[l.calls(*sets[i][b]) for b in range(2)] for i, l in enumerate(layers)]

    def events():
        return [[torch.cuda.Event() for _ in range(2)] for _ in layers]

    in_free, in_ready, out_ready, out_free = events(), events(), events(), events()
    for e in in_free + out_free:
        for x in e:
            x.record(comp)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(comp)
    h2d_s.wait_event(start)
    for i in range(steps):
        b = i % 2
        for li in range(len(layers)):
            X, dY, _ = sets[li][b]
            with torch.cuda.stream(h2d_s):
                h2d_s.wait_event(in_free[li][b])
                X.copy_(pinned_in[li][0], non_blocking=True)
                dY.copy_(pinned_in[li][1], non_blocking=True)
                in_ready[li][b].record(h2d_s)
        for li, l in enumerate(layers):
            comp.wait_event(in_ready[li][b])
            comp.wait_event(out_free[li][b])
            for _, _, fn in calls[li][b]:
                fn()
            in_free[li][b].record(comp)
            if world == 1:
                out_ready[li][b].record(comp)
        if world > 1:
            bucket.allreduce([t for li, l in enumerate(layers) for t in l.grads(sets[li][b][2])])
            for li in range(len(layers)):
                out_ready[li][b].record(comp)
        for li in range(len(layers)):
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(out_ready[li][b])
                pinned_out[li].copy_(sets[li][b][2], non_blocking=True)
                out_free[li][b].record(d2h_s)
    comp.wait_stream(d2h_s)
    comp.wait_stream(h2d_s)
    end.record(comp)
    torch.cuda.synchronize()
    return start.elapsed_time(end) / steps, h2d, d2h


def pick_peak(clocks, p_dense, p_dense_sust):
    """The dense bf16 peak that matches the clocks the timed region ran at:
    the sustained figure (measured back to back under the power cap) when the
    run was power-capped or its median SM clock sat well below the maximum,
    else the burst figure."""
    sm, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    capped = "sw_power_cap" in clocks.get("reasons", []) or (sm is not None and mx and sm < 0.9 * mx)
    return (p_dense_sust, "sustained") if capped else (p_dense, "burst")


def run_ours(args, rank, world, local_rank):
    from structured_sparse_pretraining_b200 import ops

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    ops.device_check()
    w = I.WORKLOADS[args.config]
    layers = [LayerState(w, li, seed=dp.token_seed(rank), device=device, gen_tokens=w.tokens)
              for li in range(len(w.layers))]
    # the replicated gradients of every layer, summed over ranks in one fp32 bucket
    bucket = None
    if world > 1:
        bucket = dp.GradBucket([(t.shape, t.dtype) for l in layers for t in l.grads()], device)

    step_calls = [c for l in layers for c in l.calls()]

    def step_eager():
        for _, _, fn in step_calls:
            fn()

    def allreduce_grads():
        bucket.allreduce([t for l in layers for t in l.grads()])

    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    for _ in range(args.warmup):
        step_eager()
        if world > 1:
            allreduce_grads()
    ops.status_sync()
    torch.cuda.synchronize()

    # ---- capture one step (all layers) as a CUDA graph; the replay has no
    # host work between kernels, and consecutive kernels overlap set-up and
    # tail (programmatic dependent launch).  A second graph of the same calls
    # carries an event-record node before every call for the per-kernel times;
    # those nodes cut the overlap, so it is replayed outside the timed region.
    graph = torch.cuda.CUDAGraph()
    ops.launch_count(reset=True)
    with torch.cuda.graph(graph):
        for name, layer, fn in step_calls:
            fn()
    launches_per_step = ops.launch_count(reset=True)
    markers = Markers()
    graph_m = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_m):
        for name, layer, fn in step_calls:
            markers.mark((name, layer.inn, layer.out))
            fn()
        markers.mark(("end", 0, 0))
    ops.launch_count(reset=True)
    graph.replay()
    graph_m.replay()
    torch.cuda.synchronize()
    ops.status_sync()

    # ---- device-timed region: K replays, L2 flushed before each (untimed)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with ClockSampler(local_rank) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush.fill_(float(i))
            starts[i].record()
            graph.replay()
            if world > 1:
                allreduce_grads()
            ends[i].record()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    launches = launches_per_step * args.steps
    ops.status_sync()
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    ms = sum(step_ms) / len(step_ms)

    # ---- per-kernel device times (the marker graph, same flush before each)
    per_kernel = {}
    per_kernel_reps = min(args.steps, 50)
    for i in range(per_kernel_reps):
        flush.fill_(float(i))
        graph_m.replay()
        torch.cuda.synchronize()
        for key, dt in markers.deltas():
            per_kernel.setdefault(key, []).append(dt)
    ops.status_sync()
    del graph, graph_m

    # ---- end to end: host buffers in, gradients out, through the same calls
    e2e_ms, h2d, d2h = run_e2e(layers, args.steps, world, bucket)
    ops.status_sync()

    dense_ms = dense_reference_ms(layers)

    # ---- max over ranks
    t = torch.tensor([ms, e2e_ms, dense_ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms, e2e_ms, dense_ms = t.tolist()

    hbm, p_dense_burst, p_dense_sust, peak_kind = peaks()
    clocks = clk.summary()
    p_dense, regime = pick_peak(clocks, p_dense_burst, p_dense_sust)
    p_sparse = 2.0 * p_dense
    dense_fl = adapter_fl = 0.0
    for l in layers:
        a, b = layer_flops(l.T, l.inn, l.out, w.rank)
        dense_fl += a
        adapter_fl += b
    step_flops = (dense_fl + adapter_fl) * world
    value = step_flops / (ms * 1e-3) / 1e12
    e2e_value = step_flops / (e2e_ms * 1e-3) / 1e12

    # per-kernel roofline from the live events
    kernels = {}
    for (name, inn, out), times in per_kernel.items():
        l = next(x for x in layers if x.inn == inn and x.out == out)
        fl, by = kernel_work(name, l.T, inn, out, l.r)
        avg = sum(times) / len(times)
        key = f"{name}[{inn}x{out}]"
        ent = {"ms": round(avg, 5), "launches": len(times), "kernel": kernel_of(name, l.T, inn, out, l.r)}
        if name in ("fwd", "bwd_dx", "fwd_fused", "bwd_dx_fused"):
            ent.update(bound="tensor", achieved=fl / (avg * 1e-3) / 1e12, peak=p_sparse, unit="TFLOP/s")
        elif name in ("bwd_dw_masked", "bwd_dw_fused"):
            ent.update(bound="tensor", achieved=fl / (avg * 1e-3) / 1e12, peak=p_dense, unit="TFLOP/s")
        else:
            ent.update(bound="hbm", achieved=by / (avg * 1e-3) / 1e9, peak=hbm, unit="GB/s")
        ent["frac"] = ent["achieved"] / ent["peak"]
        ent["total_ms_per_step"] = avg * len(times) / per_kernel_reps
        kernels[key] = ent
    # The dominant kernel is the device function with the most time per step:
    # fwd and bwd_dx of every layer are launches of the same SM-pair sparse
    # product kernel, so they are pooled (work and time summed over launches).
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    groups = {}
    kern_name = {}
    for (name, inn, out), times in per_kernel.items():
        l = next(x for x in layers if x.inn == inn and x.out == out)
        g = kernel_of(name, l.T, inn, out, l.r, sms)
        kern_name[f"{name}[{inn}x{out}]"] = g
        fl, by = kernel_work(name, l.T, inn, out, l.r)
        e = groups.setdefault(g, {"ms": 0.0, "flops": 0.0, "bytes": 0.0, "launches": 0})
        e["ms"] += sum(times) / per_kernel_reps
        e["flops"] += fl * len(times) / per_kernel_reps
        e["bytes"] += by * len(times) / per_kernel_reps
        e["launches"] += len(times) // per_kernel_reps
    top_g = max(groups, key=lambda g: groups[g]["ms"])
    e = groups[top_g]
    if top_g in ("sp_pair_kernel", "sp_wide_kernel"):
        achieved, peak, unit, bound = e["flops"] / (e["ms"] * 1e-3) / 1e12, p_sparse, "TFLOP/s", "tensor"
        burst = 2.0 * p_dense_burst
    elif top_g == "dw_pair_kernel":
        achieved, peak, unit, bound = e["flops"] / (e["ms"] * 1e-3) / 1e12, p_dense, "TFLOP/s", "tensor"
        burst = p_dense_burst
    else:
        achieved, peak, unit, bound = e["bytes"] / (e["ms"] * 1e-3) / 1e9, hbm, "GB/s", "hbm"
        burst = hbm
    roofline = {"kernel": f"{top_g} ({e['launches']} launches/step: "
                          + ", ".join(k for k in kernels if kern_name[k] == top_g) + ")",
                "bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
                "frac": round(achieved / peak, 4), "traffic": TRAFFIC_PER_LAUNCH.get((w.name, top_g)),
                "ms_per_step": round(e["ms"], 5),
                "frac_of_burst_peak": round(achieved / burst, 4),
                "peak_source": (f"{peak_kind} {regime} (MEASURED_PEAKS.json bf16_tflops"
                                f"{'_sustained' if regime == 'sustained' else ''}; 2:4 sparse = 2 x dense bf16): "
                                "the step ran " + ("power-capped" if regime == "sustained" else "at burst clocks"))}
    return dict(ms=ms, value=value, e2e_value=e2e_value, e2e_ms=e2e_ms, h2d=h2d, d2h=d2h, dense_ms=dense_ms,
                kernels=kernels, roofline=roofline, launches=launches, clocks=clocks,
                step_flops=step_flops, dense_fl=dense_fl, adapter_fl=adapter_fl, p_sparse=p_sparse)


# ------------------------------------------------------------------ inference sweep (fwd only)
SWEEP_TOKENS = (1, 16, 128, 2048)


def run_fwd_sweep(args):
    """Inference over the workload's layers at each token count of the sweep:
    per layer XL = X.L (adapter_fwd) and Y = X.(W^R)^T + XL.R (fwd), weights
    pruned and compressed once beforehand.  At a few tokens the step streams
    the compressed weights (values + codes, 1.125 B per dense weight) and is
    bound by HBM; it is reported as algorithmic bytes over device time, as a
    fraction of the measured HBM bandwidth, next to its tensor-core rate.
    One JSON line per token count."""
    from structured_sparse_pretraining_b200 import ops
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    ops.device_check()
    w = I.WORKLOADS[args.config]
    r = w.rank_stored
    hbm, p_dense, _, peak_kind = peaks()
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    layers = []
    for li, lay in enumerate(w.layers):
        W = I.normal_bf16((lay.out_features, lay.in_features), w.std_w, dp.WEIGHT_SEED, li, "W", device)
        vals, meta = ops.prune24(W)
        del W
        L = I.normal_bf16((lay.in_features, w.rank), w.std_l, dp.WEIGHT_SEED, li, "L", device) if w.rank else None
        R = I.normal_bf16((w.rank, lay.out_features), w.std_r, dp.WEIGHT_SEED, li, "R", device) if w.rank else None
        L, R = I.pad_rank(L, R, r)
        layers.append(dict(inn=lay.in_features, out=lay.out_features, vals=vals, meta=meta, L=L, R=R))
    ops.status_sync()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    for T in SWEEP_TOKENS:
        calls = []
        for li, l in enumerate(layers):
            X = I.normal_bf16((T, l["inn"]), w.std_x, dp.token_seed(0), li, "X", device)
            XL = torch.empty(T, r, dtype=torch.bfloat16, device=device) if r else None
            Y = torch.empty(T, l["out"], dtype=torch.bfloat16, device=device)
            # the public fused call: one launch where the shape allows, else adapter_fwd + fwd
            calls.append((("fwd_fused", l["inn"], l["out"]),
                          (lambda X=X, l=l, XL=XL, Y=Y: ops.fwd_fused(X, l["vals"], l["meta"], l["L"], l["R"], l["out"],
                                                                      XL, Y))))
        for _ in range(args.warmup):  # also allocates any split workspace before capture
            for _, fn in calls:
                fn()
        ops.status_sync()
        graph = torch.cuda.CUDAGraph()
        ops.launch_count(reset=True)
        with torch.cuda.graph(graph):
            for _, fn in calls:
                fn()
        launches = ops.launch_count(reset=True)
        markers = Markers()
        graph_m = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_m):
            for key, fn in calls:
                markers.mark(key)
                fn()
            markers.mark(("end", 0, 0))
        graph.replay()
        torch.cuda.synchronize()
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        with ClockSampler(0) as clk:
            for i in range(args.steps):
                flush.fill_(float(i))
                starts[i].record()
                graph.replay()
                ends[i].record()
            torch.cuda.synchronize()
        ops.status_sync()
        ms = sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / args.steps
        per = {}
        reps = min(args.steps, 50)
        for i in range(reps):
            flush.fill_(float(i))
            graph_m.replay()
            torch.cuda.synchronize()
            for key, dt in markers.deltas():
                per.setdefault(key, []).append(dt)
        ops.status_sync()
        tot_bytes = tot_flops = 0.0
        kernels = {}
        for (name, inn, out), times in per.items():
            fl, by = kernel_work(name, T, inn, out, r)
            tot_bytes += by
            tot_flops += fl
            avg = sum(times) / len(times)
            ent = {"ms": round(avg, 5), "gbs": round(by / (avg * 1e-3) / 1e9, 1),
                   "frac_of_hbm": round(by / (avg * 1e-3) / 1e9 / hbm, 4)}
            if name == "fwd_fused":
                bn, sp = ops.sparse_plan(out, T, inn, sms)
                fused_one = fusable(out, T, inn, r, sms)
                ent.update(tflops=round(fl / (avg * 1e-3) / 1e12, 2),
                           frac_of_sparse_peak=round(fl / (avg * 1e-3) / 1e12 / (2 * p_dense), 4),
                           kernel=kernel_of(name, T, inn, out, r, sms),
                           launches=1 if fused_one else 2,
                           token_tile=224 if fused_one else bn, k_splits=1 if fused_one else sp)
            kernels[f"{name}[{inn}x{out}]"] = ent
        gbs = tot_bytes / (ms * 1e-3) / 1e9
        tflops = tot_flops / (ms * 1e-3) / 1e12
        line = {"metric": "SLoPe inference fwd sweep: algorithmic HBM GB/s and % of HBM (adapter_fwd + fwd, "
                          "all layers)",
                "value": round(gbs, 1), "unit": "GB/s", "tokens": T, "n_gpus": 1, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True, "dtype": "bf16",
                "data": "synthetic", "config": {"workload": w.name, "tokens": T, "adapter_rank": w.rank,
                                                "layers": [f"{l['inn']}->{l['out']}" for l in layers],
                                                "l2": "flushed between timed steps (256 MiB write, untimed)"},
                "frac_of_hbm": round(gbs / hbm, 4), "hbm_peak_gbs": hbm, "peak_source": peak_kind,
                "bytes_per_step": tot_bytes, "tflops": round(tflops, 2),
                "frac_of_sparse_peak": round(tflops / (2 * p_dense), 4), "gpu_launches": launches * args.steps,
                "kernels": kernels, "clocks": clk.summary()}
        print(json.dumps(line), flush=True)
        del graph, graph_m


# ------------------------------------------------------------------ one call alone
def run_one_op(args):
    """One call of the step (--op) on one layer (--layer) of the workload,
    launched `warmup` times and then `steps` times back to back (eager), each
    time after an L2 flush; the calls before it in the step run once first so
    that its inputs exist.  Reports the mean device time of the timed calls
    and the call's algorithmic rate.  Meant for profiling one kernel."""
    from structured_sparse_pretraining_b200 import ops
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    ops.device_check()
    w = I.WORKLOADS[args.config]
    l = LayerState(w, args.layer, seed=dp.token_seed(0), device=device, gen_tokens=w.tokens)
    calls = l.calls()
    names = [c[0] for c in calls]
    idx = names.index(args.op)
    for _, _, fn in calls[:idx]:
        fn()
    fn = calls[idx][2]
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    for _ in range(args.warmup):
        fn()
    ops.status_sync()
    times = []
    for i in range(args.steps):
        flush.fill_(float(i))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b))
    ops.status_sync()
    ms = sum(times) / len(times)
    fl, by = kernel_work(args.op, l.T, l.inn, l.out, l.r)
    print(json.dumps({"op": args.op, "layer": f"{l.inn}->{l.out}", "tokens": l.T, "rank": l.r, "workload": w.name,
                      "kernel": kernel_of(args.op, l.T, l.inn, l.out, l.r), "ms": round(ms, 5), "steps": args.steps,
                      "tflops": round(fl / (ms * 1e-3) / 1e12, 2), "gbs": round(by / (ms * 1e-3) / 1e9, 1)}),
          flush=True)


# ------------------------------------------------------------------ compressed AdamW + second pruning
def run_adamw_step(args):
    """The optimizer step of the layers: per layer one fused launch that takes
    an AdamW step on the kept values (fp32 states for the non-zeros only) and
    prunes the updated W^R again into its transposed copy.  Bound by HBM:
    10.125 bytes per dense weight (values, codes, gradient and both states
    read; values, both states, vals_t and meta_t written).  One JSON line."""
    from structured_sparse_pretraining_b200 import ops
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    ops.device_check()
    w = I.WORKLOADS[args.config]
    hbm, _, _, peak_kind = peaks()
    layers = []
    for li, lay in enumerate(w.layers):
        out, inn = lay.out_features, lay.in_features
        W = I.normal_bf16((out, inn), w.std_w, dp.WEIGHT_SEED, li, "W", device)
        vals, meta = ops.prune24(W)
        del W
        g = I.normal_bf16((out, inn // 2), w.std_dy, dp.token_seed(0), li, "dW", device)
        m = torch.zeros(out, inn // 2, dtype=torch.float32, device=device)
        v = torch.zeros_like(m)
        vt = torch.empty(inn, out // 2, dtype=torch.bfloat16, device=device)
        mt = torch.empty(inn, out // 16, dtype=torch.int16, device=device)
        layers.append((out, inn, vals, meta, g, m, v, vt, mt))
    step_no = [1]

    def step():
        for out, inn, vals, meta, g, m, v, vt, mt in layers:
            ops.adamw_double_prune(vals, meta, g, m, v, out, inn, 1e-4, 0.9, 0.999, 1e-8, 0.01, step_no[0], vt, mt)

    for _ in range(args.warmup):
        step()
        step_no[0] += 1
    ops.status_sync()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    ms_list = []
    ops.launch_count(reset=True)
    with ClockSampler(0) as clk:
        for i in range(args.steps):
            flush.fill_(float(i))
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            step()
            b.record()
            b.synchronize()
            step_no[0] += 1
            ms_list.append(a.elapsed_time(b))
    launches = ops.launch_count(reset=True)
    ops.status_sync()
    ms = sum(ms_list) / len(ms_list)
    nbytes = sum(10.125 * out * inn for out, inn, *_ in layers)
    gbs = nbytes / (ms * 1e-3) / 1e9
    line = {"metric": "SLoPe compressed AdamW step + second pruning: algorithmic HBM GB/s and % of HBM",
            "value": round(gbs, 1), "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 5), "higher_is_better": True, "dtype": "f32 states, bf16 weights",
            "data": "synthetic", "config": {"workload": w.name, "layers": [f"{i}->{o}" for o, i, *_ in layers],
                                            "l2": "flushed between timed steps (256 MiB write, untimed)",
                                            "launch": "eager, one launch per layer"},
            "frac_of_hbm": round(gbs / hbm, 4), "hbm_peak_gbs": hbm, "peak_source": peak_kind,
            "bytes_per_step": nbytes, "gpu_launches": launches, "clocks": clk.summary()}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ CPU oracle (reference arm, cpu_baseline)
def oracle_sample_inputs(w, n_tok, band):
    """A bounded sample of the workload for the CPU oracle: per linear, the
    sub-layer of n_tok tokens and the first `band` output features (all input
    features), drawn from the same recipe as the full layer."""
    data = []
    for li, lay in enumerate(w.layers):
        inn, b, r = lay.in_features, min(band, lay.out_features), w.rank
        d = dict(T=n_tok, inn=inn, out=b,
                 X=I.bits(I.normal_bf16((n_tok, inn), w.std_x, 1, li, "X")),
                 W=I.bits(I.normal_bf16((b, inn), w.std_w, 1, li, "W")),
                 dY=I.bits(I.normal_bf16((n_tok, b), w.std_dy, 1, li, "dY")))
        if r:
            d["L"] = I.bits(I.normal_bf16((inn, r), w.std_l, 1, li, "L"))
            d["R"] = I.bits(I.normal_bf16((r, b), w.std_r, 1, li, "R"))
        data.append(d)
    return data


def oracle_sample_step(w, data):
    """The whole hot path of every sampled sub-layer on the CPU oracle: prune24,
    double_prune, adapter_fwd, fwd, adapter_bwd (G, dR, dL), bwd_dx and
    bwd_dw_masked.  Returns the dense-equivalent flops of the sample, counted
    like the metric (6*T*in*out + 6*T*r*(in+out) per sub-layer)."""
    import oracle
    fl = 0.0
    for d in data:
        T, inn, out, r = d["T"], d["inn"], d["out"], w.rank
        vals, meta, _ = oracle.prune24(d["W"])
        vt, mt = oracle.double_prune(vals, meta, out, inn)
        XL = oracle.adapter_fwd(d["X"], d["L"]) if r else None
        oracle.fwd(d["X"], vals, meta, XL, d.get("R"), out)
        G = oracle.adapter_g(d["dY"], d["R"]) if r else None
        if r:
            oracle.adapter_dr(XL, d["dY"])
            oracle.adapter_dl(d["X"], G)
        oracle.bwd_dx(d["dY"], vt, mt, G, d.get("L"), inn)
        oracle.bwd_dw_masked(d["dY"], d["X"], meta)
        a, b = layer_flops(T, inn, out, r)
        fl += a + b
    return fl


REF_SAMPLE = (128, 128)        # tokens x output features per linear, per reference-arm step
CPU_BASELINE_SAMPLE = (256, 256)   # per cpu_baseline repetition


def run_reference(args):
    import oracle
    w = I.WORKLOADS[args.config]
    cores = oracle.threads(len(os.sched_getaffinity(0)))
    n_tok, band = REF_SAMPLE
    data = oracle_sample_inputs(w, n_tok, band)
    for _ in range(args.warmup):
        oracle_sample_step(w, data)
    times, fl = [], 0.0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        fl = oracle_sample_step(w, data)
        times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    v = fl / sec / 1e12
    sample = (f"per step and linear: the whole hot path (prune24, double_prune, adapter_fwd, fwd, adapter_bwd, "
              f"bwd_dx, bwd_dw_masked) of the sub-layer of {n_tok} tokens x the first {band} output features "
              f"(all input features); flops counted like the metric")
    return dict(value=v, sec=sec, cores=cores, sample=sample)


def cpu_baseline(w):
    import oracle
    cores = oracle.threads(len(os.sched_getaffinity(0)))
    n_tok, band = CPU_BASELINE_SAMPLE
    data = oracle_sample_inputs(w, n_tok, band)
    t0 = time.perf_counter()
    fl = 0.0
    reps = 0
    while True:
        fl += oracle_sample_step(w, data)
        reps += 1
        if time.perf_counter() - t0 > 12.0 or reps >= 400:  # about 12 s of CPU work
            break
    sec = time.perf_counter() - t0
    return {"value": fl / sec / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": (f"{reps} x (per linear: the whole hot path of the sub-layer of {n_tok} tokens x the first "
                       f"{band} output features, all input features); {sec:.1f} s of CPU work, dense-equivalent "
                       f"flops counted like the metric")}


# ------------------------------------------------------------------ launching ranks
def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_entry(rank, world, port, argv):
    """One spawned rank: the torchrun environment, then the same main()."""
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), LOCAL_WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.argv = [sys.argv[0]] + list(argv)
    main()


def launch_ranks(n, argv):
    """Start n ranks of this script (one process per GPU, rank = local GPU
    index), as torchrun would, and wait for them; a failing rank fails the run."""
    import torch.multiprocessing as mp
    mp.start_processes(_rank_entry, args=(n, _free_port(), argv), nprocs=n, start_method="spawn", join=True)


def plumbing_check(rank, world):
    """The multi-rank plumbing alone, on CPU with gloo (no GPU): every rank
    fills a replicated-gradient set (bf16 dW, fp32 dL and dR) with rank + 1,
    sums it through the same fp32 bucket the GPU run uses, and rank 0 prints
    one JSON line with the world size and whether every sum came out right."""
    dist.init_process_group("gloo")
    try:
        grads = [torch.full((64, 32), rank + 1.0).bfloat16(), torch.full((64, 8), rank + 1.0),
                 torch.full((8, 64), rank + 1.0)]
        bucket = dp.GradBucket([(t.shape, t.dtype) for t in grads], "cpu")
        bucket.allreduce(grads)
        want = world * (world + 1) / 2
        ok = all(bool(torch.all(t.float() == want)) for t in grads)
        flag = torch.tensor([1 if ok else 0])
        dist.all_reduce(flag, op=dist.ReduceOp.MIN)
        if rank == 0:
            print(json.dumps({"plumbing_check": "ok" if int(flag) == 1 else "wrong sums", "n_gpus": world,
                              "ranks": world, "backend": "gloo"}), flush=True)
    finally:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="C5", choices=sorted(I.WORKLOADS),
                    help="workload (default C5: the largest that fits one GPU, the headline)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fwd-sweep", action="store_true",
                    help="inference sweep (fwd only) over 1, 16, 128, 2048 tokens; one line per token count")
    ap.add_argument("--adamw-step", action="store_true",
                    help="the fused compressed AdamW step + second pruning over the layers, against HBM")
    ap.add_argument("--plumbing-check", action="store_true",
                    help="launch the ranks and sum a gradient set over them with gloo on CPU (no GPU work)")
    ap.add_argument("--op", default=None, choices=OPS,
                    help="time one call of the step alone (eager, after the calls before it in the step) on one "
                         "layer of the workload; one JSON line")
    ap.add_argument("--layer", type=int, default=0, help="with --op: the layer of the workload")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    if "WORLD_SIZE" not in os.environ and args.gpus > 1 and args.impl == "ours":
        # not under torchrun: start the ranks here (the reference arm runs on rank 0 alone)
        launch_ranks(args.gpus, sys.argv[1:])
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.plumbing_check:
        if world == 1:
            print(json.dumps({"plumbing_check": "ok", "n_gpus": 1, "ranks": 1, "backend": "none"}), flush=True)
        else:
            plumbing_check(rank, world)
        return
    w = I.WORKLOADS[args.config]
    config = {"workload": w.name, "layers": [f"{l.in_features}->{l.out_features}" for l in w.layers],
              "tokens_per_gpu": w.tokens, "global_tokens": w.tokens * max(world, 1), "adapter_rank": w.rank,
              "adapter_rank_stored": w.rank_stored, "parallelism": f"dp{world}",
              "l2": "flushed between timed steps (256 MiB write, untimed)"}

    if args.op:
        if args.impl == "ours" and rank == 0:
            run_one_op(args)
        return
    if args.fwd_sweep:
        if args.impl == "ours" and rank == 0:
            run_fwd_sweep(args)
        return
    if args.adamw_step:
        if args.impl == "ours" and rank == 0:
            run_adamw_step(args)
        return

    if args.impl == "reference":
        if rank != 0:
            return
        ref = run_reference(args)
        line = {"metric": METRIC, "value": round(ref["value"], 6), "unit": UNIT, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ref["sec"] * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config, "impl": "reference",
                "cpu_baseline": {"value": round(ref["value"], 6), "unit": UNIT, "cores": ref["cores"],
                                 "kind": "oracle", "sample": ref["sample"]},
                "e2e": {"value": round(ref["value"], 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    res = run_ours(args, rank, world, local_rank)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    dense_flops_rate = res["dense_fl"] * world / (res["dense_ms"] * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": round(res["value"], 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(res["ms"], 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config,
        "frac_of_sparse_peak": round(res["value"] / world / res["p_sparse"], 4),
        "dense_torch_matmul": {"ms_per_step": round(res["dense_ms"], 5), "tflops": round(dense_flops_rate, 3),
                               "speedup": round(res["dense_ms"] / res["ms"], 4),
                               "note": "Y=XW^T, dX=dY W, dW=dY^T X in bf16 torch.matmul, same shapes, no adapter"},
        "e2e": {"value": round(res["e2e_value"], 3), "unit": UNIT, "h2d_bytes_per_step": res["h2d"],
                "d2h_bytes_per_step": res["d2h"], "ms_per_step": round(res["e2e_ms"], 5),
                "how": "eager public ops; X, dY in from pinned host memory and dW out every step, on copy "
                       "streams overlapping the compute"},
        "gpu_launches": res["launches"], "roofline": res["roofline"], "clocks": res["clocks"],
        "kernels": {k: {kk: (round(vv, 5) if isinstance(vv, float) else vv) for kk, vv in v.items()}
                    for k, v in res["kernels"].items()},
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
