"""Benchmark: layer-wise 4-bit GPTQ + RTN of a whole model's weight layers.

A step runs the complete per-layer path on every layer of the workload:
H = 2 X^T X, damping + dead columns + U (H^-1 = U^T U), GPTQ, RTN, and the
reconstruction error of both quantised layers.  Default workload: the
three Llama-2-70B-shaped layers (8192 -> 8192, 8192 -> 28672, 28672 -> 8192;
fp16 weights) with 262144 calibration tokens each, symmetric 4-bit, group
128, block 128, damp 0.01.  Workload 2 is the 49 weight-bearing layers of
GPT-2 small with 2560 tokens each.  Inputs are seeded synthetic data (no
dataset or trained weights), resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 5|1|2|3|4]
                    [--impl reference]

Prints one JSON line (rank 0).  Under torchrun every rank quantises its own
copy of the workload (layers are independent: weak scaling, no collective
on the data path); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = ("GPTQ layers/s & Mweights/s; XᵀX TFLOP/s; RTN GB/s (vs B200 roofline)")
WORKLOAD_NAMES = {
    1: "gpt2-small c_proj 768x768, 2048 tokens (single layer)",
    2: "gpt2-small 49 weight layers, 2560 tokens each",
    3: "gpt2-style 1.3B, block 0 (4 layers: 2048->6144, 2048->2048, 2048->8192, 8192->2048), "
       "262144 tokens each",
    4: "llama-7b-shaped 7 layers, 262144 tokens, affine g128 act-order",
    5: "llama-2-70b-shaped 3 layers, 262144 tokens, sym g128",
}


# ----------------------------------------------------------------------------- helpers

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, world: int) -> float:
    """Max of a float over all ranks (identity for a single process)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64)
    if dist.get_backend() == "nccl":
        t = t.cuda()
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        # nvidia-smi takes a moment to start: wait (at most 5 s) for its first
        # sample so that the timed region that follows is covered
        t0 = time.time()
        while self.proc is not None and time.time() - t0 < 5.0:
            self.file.flush()
            if os.path.getsize(self.file.name) > 0:
                break
            time.sleep(0.02)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        self.file.flush()
        self.file.seek(0)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.file:
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx.append(float(p[2]))
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.file.name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ----------------------------------------------------------------------------- GPU arm

# token chunks of a layer's X in the end-to-end run (copied in one after another;
# the Hessian accumulates over each as it lands)
E2E_CHUNKS = 8

class LayerRun:
    """Device buffers of one layer and the calls of one step on it."""

    def __init__(self, spec, dev, W, X, recon_route="hessian"):
        import torch
        from post_weight_quantization_27_b200 import gq
        self.spec = spec
        self.W, self.X = W, X
        self.route = recon_route
        d_in, d_out, n = spec.d_in, spec.d_out, spec.n_tok
        f = dict(device=dev)
        self.H0 = torch.empty((d_in, d_in), dtype=torch.float32, **f)   # undamped, kept
        self.H = torch.empty((d_in, d_in), dtype=torch.float32, **f)    # the solve's scratch
        self.U = torch.empty((d_in, d_in), dtype=torch.float32, **f)
        self.n_chunks = E2E_CHUNKS if n % E2E_CHUNKS == 0 and n >= 8192 * E2E_CHUNKS else 1
        self.ws_h = gq.workspace(max(gq.hessian_workspace_size(n, d_in),
                                     gq.hessian_workspace_size(n // self.n_chunks, d_in)), dev)
        self.ws_c = gq.workspace(gq.damp_cholesky_workspace_size(d_in), dev)
        self.ws_g = gq.workspace(gq.gptq_workspace_size(d_out, d_in, spec.block_size), dev)
        self.ws_r = gq.workspace(gq.recon_workspace_size(d_out, d_in, n) if recon_route == "direct"
                                 else gq.recon_error_hessian_workspace_size(d_out, d_in), dev)
        self.q_gptq = gq._outputs(d_out, d_in, spec.group_size, spec.sym, dev, spec.act_order)
        self.q_rtn = gq._outputs(d_out, d_in, spec.group_size, spec.sym, dev, False)
        self.perm = torch.empty(d_in, dtype=torch.int32, **f) if spec.act_order else None
        self.dead = torch.empty(d_in, dtype=torch.uint8, **f)
        self.info = torch.empty(1, dtype=torch.int32, **f)
        self.sse = torch.empty(2, dtype=torch.float64, **f)

    def hessian(self):
        from post_weight_quantization_27_b200 import gq
        L, s = gq.lib(), gq._stream(None)
        gq._check(L.gq_hessian_compute(gq._p(self.X), self.spec.n_tok, self.spec.d_in,
                                       gq._p(self.H0), gq._p(self.ws_h), self.ws_h.numel(), s),
                  "hessian")

    def hessian_part(self, c):
        """H0 over token chunk c of n_chunks: := for the first, += after
        (the end-to-end run accumulates H while the later chunks of X are
        still being copied in)."""
        from post_weight_quantization_27_b200 import gq
        L, s = gq.lib(), gq._stream(None)
        n = self.spec.n_tok // self.n_chunks
        x = gq._p(self.X) + c * n * self.spec.d_in * 2
        fn = L.gq_hessian_compute if c == 0 else L.gq_hessian_accumulate
        gq._check(fn(x, n, self.spec.d_in, gq._p(self.H0), gq._p(self.ws_h), self.ws_h.numel(),
                     s), "hessian")

    def solve(self):
        from post_weight_quantization_27_b200 import gq
        L, s, sp = gq.lib(), gq._stream(None), self.spec
        self.H.copy_(self.H0)            # the solve uses its H as scratch; H0 stays for the error
        gq._check(L.gq_damp_cholesky_inverse(
            gq._p(self.H), sp.d_in, sp.damp, int(sp.act_order), gq._p(self.perm),
            gq._p(self.dead), gq._p(self.U), gq._p(self.info), None, gq._p(self.ws_c),
            self.ws_c.numel(), s), "damp_cholesky")

    def gptq(self):
        from post_weight_quantization_27_b200 import gq
        L, s, sp, o = gq.lib(), gq._stream(None), self.spec, self.q_gptq
        gq._check(L.gq_gptq_quantize_layer(
            gq._p(self.W), gq._DTYPES[self.W.dtype], sp.d_out, sp.d_in, gq._p(self.U), 4,
            sp.group_size, sp.block_size, int(sp.sym), gq._p(self.perm), gq._p(self.dead),
            gq._p(o["qpacked"]), gq._p(o["scales"]), gq._p(o["zeros"]), gq._p(o["g_idx"]),
            gq._p(self.ws_g), self.ws_g.numel(), s), "gptq")

    def rtn(self):
        from post_weight_quantization_27_b200 import gq
        L, s, sp, o = gq.lib(), gq._stream(None), self.spec, self.q_rtn
        gq._check(L.gq_rtn_quantize_pack(gq._p(self.W), gq._DTYPES[self.W.dtype], sp.d_out,
                                         sp.d_in, 4, sp.group_size, int(sp.sym),
                                         gq._p(o["qpacked"]), gq._p(o["scales"]),
                                         gq._p(o["zeros"]), s), "rtn")

    def recon(self):
        from post_weight_quantization_27_b200 import gq
        L, s, sp = gq.lib(), gq._stream(None), self.spec
        for k, o in enumerate((self.q_gptq, self.q_rtn)):
            if self.route == "hessian":
                gq._check(L.gq_recon_error_hessian(
                    gq._p(self.W), gq._DTYPES[self.W.dtype], gq._p(o["qpacked"]),
                    gq._p(o["scales"]), gq._p(o["zeros"]), gq._p(o.get("g_idx")), sp.d_out,
                    sp.d_in, 4, sp.group_size, int(sp.sym), gq._p(self.H0), sp.n_tok,
                    self.sse.data_ptr() + 8 * k, None, None, gq._p(self.ws_r),
                    self.ws_r.numel(), s), "recon")
                continue
            gq._check(L.gq_recon_error(
                gq._p(self.W), gq._DTYPES[self.W.dtype], gq._p(o["qpacked"]),
                gq._p(o["scales"]), gq._p(o["zeros"]), gq._p(o.get("g_idx")), sp.d_out,
                sp.d_in, 4, sp.group_size, int(sp.sym), gq._p(self.X), sp.n_tok,
                self.sse.data_ptr() + 8 * k, None, None, gq._p(self.ws_r),
                self.ws_r.numel(), s), "recon")

    STAGES = ("hessian", "solve", "gptq", "rtn", "recon")


def build_layers(workload: int, dev, generate_on_device: bool, recon_route: str = "hessian"):
    import torch
    from post_weight_quantization_27_b200 import inputs as I
    runs = []
    layers = I.workload_layers(workload)
    if workload == 3:
        # the 96 layers' resident X would need 168 GB; one block's four shapes
        # (7.5 GB of X) stand for the stack, every layer of which has one of them
        layers = layers[:4]
    for spec in layers:
        W = I.make_weights(spec).to(dev)
        X = I.make_x_device(spec, dev) if generate_on_device else I.make_x(spec).to(dev)
        runs.append(LayerRun(spec, dev, W, X, recon_route))
    torch.cuda.synchronize()
    return runs


def schedule(runs, n_streams):
    """Layers to streams, largest first onto the least-loaded stream."""
    order = sorted(range(len(runs)), key=lambda i: -runs[i].spec.d_out * runs[i].spec.d_in
                   - runs[i].spec.d_in ** 2)
    load = [0] * n_streams
    lists = [[] for _ in range(n_streams)]
    for i in order:
        k = min(range(n_streams), key=lambda j: load[j])
        lists[k].append(i)
        sp = runs[i].spec
        load[k] += sp.d_out * sp.d_in + 4 * sp.d_in ** 2
    return lists


def make_streams(n_streams):
    """The capture stream and the layer streams of the step (reused by every
    capture, so that helper streams the library creates for a stream in an
    eager pass serve it inside the graphs too)."""
    import torch
    return torch.cuda.Stream(), [torch.cuda.Stream() for _ in range(n_streams)]


def warm_streams(runs, sides):
    """One eager pass of every layer on the stream it is scheduled on: the
    Cholesky call creates its helper stream for a caller stream only outside
    a capture, and uses it inside one (its inverse chain then runs beside
    the factorisation in the graph)."""
    import torch
    for si, idxs in enumerate(schedule(runs, len(sides))):
        with torch.cuda.stream(sides[si]):
            for i in idxs:
                for st in LayerRun.STAGES:
                    getattr(runs[i], st)()
    torch.cuda.synchronize()


def capture_step(runs, n_streams, timed=False, host=None, kernel=None, capacity=0,
                 streams=None, serial=()):
    """One whole step (every layer, every stage) captured as a CUDA graph:
    the layers run on ``n_streams`` streams forked from and joined back to
    one capture stream.  ``timed`` adds timing event nodes around each
    stage call; ``kernel`` (a name or a list of names) adds the library's per-launch
    event pairs around every launch of that kernel (read with gq.kernel_timer_read after the
    replays); ``host`` adds the pinned host <-> device copies of the
    end-to-end run; stages named in ``serial`` run one layer at a time
    across the streams (each waits for the previous layer's, in issue
    order).  Returns (graph, stream, stage events, launches/step)."""
    import torch
    from post_weight_quantization_27_b200 import gq
    main, sides = streams if streams is not None else make_streams(n_streams)
    sched = schedule(runs, n_streams)
    if host is not None:
        # the inputs come in on their own stream, in the order the layers
        # run, so that a layer's copy overlaps the compute of the layers
        # before it; the results go back on another
        h2d_st, d2h_st = torch.cuda.Stream(), torch.cuda.Stream()
        order = [i for pos in range(max(len(x) for x in sched))
                 for x in sched if pos < len(x) for i in [x[pos]]]
    g = torch.cuda.CUDAGraph()
    events = []
    n0 = gq.launch_count()
    if kernel is not None:
        gq.kernel_timer_start(list(kernel) if isinstance(kernel, (list, tuple)) else [kernel],
                              capacity)
    with torch.cuda.graph(g, stream=main):
        fork = torch.cuda.Event()
        fork.record(main)
        for sd in sides:
            sd.wait_event(fork)
        ready, last = {}, {}
        if host is not None:
            h2d_st.wait_event(fork)
            d2h_st.wait_event(fork)
            with torch.cuda.stream(h2d_st):
                for i in order:
                    r, nc = runs[i], runs[i].n_chunks
                    r.W.copy_(host[i]["W"], non_blocking=True)
                    ready[i] = []
                    rows = r.spec.n_tok // nc
                    for c in range(nc):
                        r.X[c * rows:(c + 1) * rows].copy_(host[i]["X"][c * rows:(c + 1) * rows],
                                                           non_blocking=True)
                        ready[i].append(torch.cuda.Event())
                        ready[i][-1].record(h2d_st)
        for si, idxs in enumerate(sched):
            sd = sides[si]
            with torch.cuda.stream(sd):
                for i in idxs:
                    r = runs[i]
                    stages = LayerRun.STAGES
                    if host is not None:
                        # H over the chunks of X as they land, then the rest
                        if "hessian" in serial and "hessian" in last:
                            sd.wait_event(last["hessian"])
                        for c, ev in enumerate(ready[i]):
                            sd.wait_event(ev)
                            r.hessian_part(c)
                        if "hessian" in serial:
                            last["hessian"] = torch.cuda.Event()
                            last["hessian"].record(sd)
                        stages = stages[1:]
                    for st in stages:
                        if st in serial and st in last:
                            sd.wait_event(last[st])
                        if timed:
                            e0 = torch.cuda.Event(enable_timing=True, external=True)
                            e1 = torch.cuda.Event(enable_timing=True, external=True)
                            e0.record(sd)
                        getattr(r, st)()
                        if st in serial:
                            last[st] = torch.cuda.Event()
                            last[st].record(sd)
                        if timed:
                            e1.record(sd)
                            events.append((i, st, e0, e1))
                    if host is not None:
                        done = torch.cuda.Event()
                        done.record(sd)
                        d2h_st.wait_event(done)
                        h = host[i]
                        with torch.cuda.stream(d2h_st):
                            h["q"].copy_(r.q_gptq["qpacked"], non_blocking=True)
                            h["s"].copy_(r.q_gptq["scales"], non_blocking=True)
                            h["qr"].copy_(r.q_rtn["qpacked"], non_blocking=True)
                            h["sse"].copy_(r.sse, non_blocking=True)
        for sd in sides + ([h2d_st, d2h_st] if host is not None else []):
            j = torch.cuda.Event()
            j.record(sd)
            main.wait_event(j)
    if kernel is not None:
        gq.kernel_timer_stop()
    return g, main, events, gq.launch_count() - n0


def replay(graph, stream, n, timed=False):
    """Launch the captured step ``n`` times on ``stream`` (the stream it was
    captured from, so the timing events below bracket the replays); with
    ``timed`` returns the mean ms per replay from events on that stream,
    synchronising on both sides."""
    import torch
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(n):
            graph.replay()
        t1.record(stream)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / max(n, 1) if timed else None


def kernel_shares(runs):
    """Per kernel (total ms, launches, work) over one step, timed inside a
    captured graph of the step on one fresh stream (the library's per-launch
    event pairs on every launch: device time with no host gaps, and no
    helper stream, since none is created during a capture, so the kernels
    run one after another as in an ncu launch list); picks the dominant
    kernel."""
    import torch
    from post_weight_quantization_27_b200 import gq
    n0 = gq.launch_count()
    for r in runs:
        for st in LayerRun.STAGES:
            getattr(r, st)()
    torch.cuda.synchronize()
    cap = int(1.2 * (gq.launch_count() - n0)) + 64
    graph, gstream, _, _ = capture_step(runs, 1, kernel=list(gq.KERNELS), capacity=cap,
                                        streams=make_streams(1))
    try:
        replay(graph, gstream, 2)
        torch.cuda.synchronize()
        recs = gq.kernel_timer_read()
    finally:
        gq.kernel_timer_release()
        del graph
    tot = {}
    for k, ms, w in recs:
        t, n, wk = tot.get(k, (0.0, 0, 0.0))
        tot[k] = (t + ms, n + 1, wk + w)
    return tot


def stage_work(spec, recon_route="hessian"):
    """Algorithmic work per call of each stage (bytes or flops)."""
    wb = {"f32": 4, "f16": 2, "bf16": 2}[spec.w_dtype]
    n_groups = 1 if spec.group_size == -1 else spec.d_in // spec.group_size
    zero_bytes = 0 if spec.sym else 2 * spec.d_out * n_groups
    return {
        # symmetric half of X^T X: N d (d + 1) flops
        "hessian_flops": spec.n_tok * spec.d_in * (spec.d_in + 1),
        # read W, write codes + fp16 scales (+ zeros)
        "rtn_bytes": spec.d_out * spec.d_in * (wb + 0.5) + 2 * spec.d_out * n_groups + zero_bytes,
        # two reconstruction errors: 2 N d_out d_in each (direct), or the
        # lower triangle of dW^T dW, d_out d_in (d_in + 1) each, from the Hessian
        "recon_flops": (2 * 2 * spec.n_tok * spec.d_out * spec.d_in if recon_route == "direct"
                        else 2 * spec.d_out * spec.d_in * (spec.d_in + 1)),
        "weights": spec.d_out * spec.d_in,
    }


def gpu_arm(args, world, rank, local):
    import torch
    from post_weight_quantization_27_b200 import gq
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    gq.lib()
    big = args.workload >= 3
    runs = build_layers(args.workload, dev, generate_on_device=big, recon_route=args.recon)
    peaks = measured_peaks()
    n_streams = max(1, min(args.streams, len(runs)))

    # eager passes (set kernel attributes; per-kernel shares), then the
    # captured step with the dominant kernel's launches timed
    streams = make_streams(n_streams)
    warm_streams(runs, streams[1])
    shares = kernel_shares(runs)
    dom_kernel = max(shares, key=lambda k: shares[k][0])
    serial = tuple(x for x in args.serial_stages.split(",") if x)
    graph, gstream, events, launches_per_step = capture_step(
        runs, n_streams, timed=True, kernel=dom_kernel, capacity=shares[dom_kernel][1] + 64,
        streams=streams, serial=serial)

    replay(graph, gstream, args.warmup)
    torch.cuda.synchronize()
    barrier(world)

    # ---------------- timed region: inputs resident in HBM
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        barrier(world)
        w0 = time.perf_counter()
        ms_local = replay(graph, gstream, args.steps, timed=True)
        wall_ms = (time.perf_counter() - w0) * 1e3 / args.steps
        barrier(world)
    ms = reduce_max(ms_local, world)
    clocks = clk.summary()

    # per-call stage durations of the last timed step (event nodes in the graph)
    calls = {st: [] for st in LayerRun.STAGES}
    for i, st, e0, e1 in events:
        calls[st].append(e0.elapsed_time(e1))
    stage_ms = {st: sum(v) for st, v in calls.items()}
    work = [stage_work(r.spec, args.recon) for r in runs]
    tot = {k: sum(w[k] for w in work) for k in work[0]}
    n_layers = len(runs)
    value = world * n_layers / (ms / 1e3)

    recs = [r for r in gq.kernel_timer_read() if r[0] == dom_kernel]
    gq.kernel_timer_release()
    roof = roofline(dom_kernel, recs, peaks, args.workload, ms)
    del graph

    e2e = e2e_run(runs, args, dev, world, n_streams, streams)

    out = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "layers/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "wall_ms_per_step": round(wall_ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 X, fp32 H/U/GPTQ, int4 codes",
        "data": "synthetic (seeded; random-init weights of the named layer shapes)",
        "config": {"workload": WORKLOAD_NAMES[args.workload], "layers": n_layers,
                   "recon_route": args.recon,
                   "weights_per_step": tot["weights"], "parallelism": f"layers x{world} (weak)",
                   "streams": n_streams, "serial_stages": args.serial_stages,
                   "cuda_graph": True,
                   "l2": "inputs larger than L2 (%.0f MB of W and X per step)" % (
                       sum(r.W.numel() * r.W.element_size() + r.X.numel() * 2 for r in runs) / 1e6)},
        "mweights_per_s": round(world * tot["weights"] / (ms / 1e3) / 1e6, 2),
        "stage_ms_sum_of_calls": {k: round(v, 4) for k, v in stage_ms.items()},
        "kernel_share": {k: {"ms": round(t, 3), "launches": n,
                             "share": round(t / sum(v[0] for v in shares.values()), 4)}
                         for k, (t, n, _) in sorted(shares.items(), key=lambda x: -x[1][0])},
        # per-kernel rates from the serialised graph pass (work / event time)
        "xtx_tflops": rate(shares, "hessian_mma", 1e12),
        "rtn_gbs": rate(shares, "rtn", 1e9),
        "recon_tflops": rate(shares, "recon_mma" if args.recon == "direct" else "syrk_bf16", 1e12),
        "tf32x3_gemm_tflops": rate(shares, "gemm_tf32x3", 1e12),
        "gptq_block_gbs": rate(shares, "gptq_block", 1e9),
        "roofline": roof,
        "gpu_launches": int(launches_per_step * args.steps),
        "clocks": clocks,
        "e2e": e2e,
    }
    return out


def rate(shares, kernel, scale):
    if kernel not in shares or shares[kernel][0] <= 0:
        return None
    t, _, w = shares[kernel]
    return round(w / (t / 1e3) / scale, 2)


# Roofline ceiling per kernel: (bound, dtype of its arithmetic, tensor-core
# passes per algorithmic product).  The peak is the measured one of the
# kernel's own arithmetic: bf16 for the bf16 contractions, TF32 (the
# measured bf16 rate x the nominal dense TF32 / bf16 ratio of B200, 1.1 /
# 2.25) for the 3 x TF32 GEMM, the fp32 FMA rate of the SMs (148 SMs x 128
# lanes x 2 flops x the maximum SM clock) for the SIMT factor kernels, the
# measured copy bandwidth for the memory-bound ones.  The fraction is
# algorithmic work / time / that peak; the tensor pipe's own utilisation is
# that fraction times the passes (the bf16 hi + lo split runs two products,
# the 3 x TF32 split three), reported beside it.
KERNEL_BOUND = {
    "hessian_mma": ("tensor", "bf16", 1),
    "recon_mma": ("tensor", "bf16", 2),
    "gemm_tf32x3": ("tensor", "tf32", 3),
    "potrf_trsm": ("alu", "fp32 FMA", 1),
    "block_inverse": ("alu", "fp32 FMA", 1),
    "gptq_block": ("hbm", "HBM copy", 1),
    "rtn": ("hbm", "HBM copy", 1),
    "qlinear": ("tensor", "bf16", 2),
    "syrk_bf16": ("tensor", "bf16", 3),
}


def kernel_peak(kernel, peaks, sustained=True):
    """(peak, unit, description) for the kernel's own arithmetic.  Kernels
    timed inside a long step take the sustained bf16 figure."""
    bf16 = (peaks["bf16_tflops_sustained"] if sustained else None) or peaks["bf16_tflops"]
    which = "sustained" if sustained and peaks["bf16_tflops_sustained"] else "burst"
    src = peaks["source"]
    _, dtype, _ = KERNEL_BOUND[kernel]
    if dtype == "bf16":
        return bf16, "TFLOP/s", f"{src} bf16 dense {which}"
    if dtype == "tf32":
        return bf16 * 1.1 / 2.25, "TFLOP/s", f"{src} bf16 dense {which} x 1.1/2.25 (tf32)"
    if dtype == "fp32 FMA":
        mhz = peaks.get("sm_max_mhz") or 1965.0
        return 148 * 128 * 2 * mhz * 1e6 / 1e12, "TFLOP/s", f"148 SMs x 128 FMA x 2 x {mhz:.0f} MHz"
    return peaks["hbm_gbs"], "GB/s", f"{src} HBM copy"


def profiled_traffic(kernel, workload):
    """DRAM bytes per launch of ``kernel`` on ``workload`` from the committed
    ncu summary (profiles/traffic.txt: kernel, workload, bytes per launch),
    or None when no capture of the current kernel is recorded."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 3 and not line.startswith("#") and parts[0] == kernel \
                    and parts[1] == str(workload):
                return float(parts[2])
    return None


def roofline(kernel, recs, peaks, workload, ms_per_step):
    """Roofline of the dominant kernel: its launches' algorithmic work (flops
    or bytes, as the library counts them per launch) over their CUDA-event
    durations in the last timed replay."""
    bound, dtype, passes = KERNEL_BOUND[kernel]
    peak, unit, src = kernel_peak(kernel, peaks)
    work = sum(w for _, _, w in recs)
    sec = sum(ms for _, ms, _ in recs) / 1e3
    scale = 1e12 if unit == "TFLOP/s" else 1e9
    a = work / sec / scale if sec > 0 else 0.0
    out = {"kernel": kernel, "bound": bound, "achieved": round(a, 3), "peak": round(peak, 1),
           "unit": unit, "frac": round(a / peak, 4), "traffic": profiled_traffic(kernel, workload),
           "launches": len(recs), "avg_launch_us": round(sec / max(len(recs), 1) * 1e6, 2),
           "kernel_ms_per_step": round(sec * 1e3, 3), "step_ms": round(ms_per_step, 3),
           "work_per_launch": work / max(len(recs), 1), "arith": dtype, "peak_source": src}
    if bound == "tensor":
        out["tensor_passes"] = passes
        out["tensor_pipe_frac"] = round(a * passes / peak, 4)
    return out


def e2e_run(runs, args, dev, world, n_streams, streams=None):
    """Same metric through the C-ABI with host buffers: every step copies
    each layer's W and X from pinned host memory and reads back the packed
    codes, scales and both SSEs (copies and compute in one captured graph;
    the copies on their own streams, each layer's compute waiting for its
    inputs only)."""
    import torch
    host = []

    def pinned_copy(t):  # one pinned host copy (no pageable intermediate)
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        return h

    for r in runs:
        host.append(dict(W=pinned_copy(r.W), X=pinned_copy(r.X),
                         q=torch.empty(r.q_gptq["qpacked"].shape, dtype=torch.int32).pin_memory(),
                         s=torch.empty(r.q_gptq["scales"].shape, dtype=torch.float16).pin_memory(),
                         qr=torch.empty(r.q_rtn["qpacked"].shape, dtype=torch.int32).pin_memory(),
                         sse=torch.empty(2, dtype=torch.float64).pin_memory()))
    h2d = sum(h["W"].numel() * h["W"].element_size() + h["X"].numel() * 2 for h in host)
    d2h = sum(h["q"].numel() * 4 + h["s"].numel() * 2 + h["qr"].numel() * 4 + 16 for h in host)
    graph, gstream, _, _ = capture_step(runs, n_streams, timed=False, host=host,
                                        streams=streams,
                                        serial=tuple(x for x in args.serial_stages.split(",")
                                                     if x))
    steps = max(1, min(args.steps, 5))
    replay(graph, gstream, 1)
    torch.cuda.synchronize()
    barrier(world)
    ms = reduce_max(replay(graph, gstream, steps, timed=True), world)
    del graph
    return {"value": round(world * len(runs) / (ms / 1e3), 3), "unit": "layers/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps}


# ----------------------------------------------------------------------------- CPU oracle

def oracle_sample_step(workload: int):
    """One bounded sample of the workload on the CPU oracle: every layer of
    transformer block 0 (the four GPT-2 shapes) through the whole path.
    Returns (layers done, seconds)."""
    import numpy as np
    import oracle as O
    from post_weight_quantization_27_b200 import inputs as I
    layers = I.workload_layers(workload)
    sample = layers[:4] if workload == 2 else layers[:1]
    data = [(s, I.make_weights(s).float().numpy(), I.make_x(s).float().numpy()) for s in sample]
    t0 = time.perf_counter()
    for s, W, X in data:
        res, H0, U, perm, dead = O.gptq_layer(W, X, group_size=s.group_size, sym=s.sym,
                                              block_size=s.block_size, damp_percent=s.damp,
                                              act_order=s.act_order)
        rtn = O.rtn_quantize(W, s.group_size, s.sym)
        Wr = O.dequantize_packed(rtn["qpacked"], rtn["scales"], rtn["zeros"], s.d_in,
                                 s.group_size, s.sym)
        O.recon_sse(W, res.W_hat, X)
        O.recon_sse(W, Wr, X)
    del np
    return len(data), time.perf_counter() - t0


# Sampled units of the oracle for the full-size layers (the whole fp64 path
# of one 28672-wide layer would take hours on the host): tokens, rows and
# tiles per layer, and the width of the Cholesky sample.
SAMPLE_TOKENS, SAMPLE_ROWS, SAMPLE_TILES, SAMPLE_TILE, SAMPLE_U = 8192, 128, 16, 256, 1024


def oracle_sampled_layer(spec, rng):
    """Times the oracle on sampled units of one full-size layer and
    extrapolates to the whole layer.  Units: H on SAMPLE_TILES random
    SAMPLE_TILE^2 tiles of the upper triangle over the first SAMPLE_TOKENS
    tokens (scaled to all tiles and all tokens); U on the damped Hessian of
    the first SAMPLE_U channels (scaled by (d_in / SAMPLE_U)^3); GPTQ, RTN
    and both reconstruction errors on SAMPLE_ROWS random rows at full width
    (GPTQ given a d_in x d_in factor; errors over the sampled tokens, scaled
    to all rows and tokens).  Returns (extrapolated seconds, measured
    seconds)."""
    import numpy as np
    import oracle as O
    from post_weight_quantization_27_b200 import inputs as I
    d, n_rows = spec.d_in, min(SAMPLE_ROWS, spec.d_out)
    ntok = min(SAMPLE_TOKENS, spec.n_tok)
    X = I.make_x(spec, rows=ntok).float().numpy()
    rows = np.sort(rng.choice(spec.d_out, size=n_rows, replace=False))
    W = I.make_weights(spec)[torch_index(rows)].float().numpy()
    nt = (d + SAMPLE_TILE - 1) // SAMPLE_TILE
    tri = [(a, b) for a in range(nt) for b in range(a, nt)]
    pick = [tri[i] for i in rng.choice(len(tri), size=min(SAMPLE_TILES, len(tri)), replace=False)]
    uw = min(SAMPLE_U, d)
    U_full = np.eye(d)
    t_meas = 0.0
    # H tiles
    t0 = time.perf_counter()
    for a, b in pick:
        ra = np.arange(a * SAMPLE_TILE, min(d, (a + 1) * SAMPLE_TILE))
        rb = np.arange(b * SAMPLE_TILE, min(d, (b + 1) * SAMPLE_TILE))
        O.hessian_entries(X[:, np.concatenate([ra, rb])], np.arange(len(ra)),
                          np.arange(len(ra), len(ra) + len(rb)))
    t_h = time.perf_counter() - t0
    # U of the leading uw channels
    Hs = O.hessian_entries(X[:, :uw], np.arange(uw), np.arange(uw))
    t0 = time.perf_counter()
    Hd, _ = O.damp_hessian(Hs, spec.damp)
    O.upper_factor_of_inverse(Hd)
    t_u = time.perf_counter() - t0
    # GPTQ, RTN, both reconstruction errors on the sampled rows
    t0 = time.perf_counter()
    res = O.gptq_quantize(W, U_full, group_size=spec.group_size, block_size=spec.block_size,
                          sym=spec.sym)
    t_g = time.perf_counter() - t0
    t0 = time.perf_counter()
    rtn = O.rtn_quantize(W, spec.group_size, spec.sym)
    Wr = O.dequantize_packed(rtn["qpacked"], rtn["scales"], rtn["zeros"], d, spec.group_size,
                             spec.sym)
    t_r = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.recon_sse(W, res.W_hat, X)
    O.recon_sse(W, Wr, X)
    t_m = time.perf_counter() - t0
    t_meas = t_h + t_u + t_g + t_r + t_m
    tok = spec.n_tok / ntok
    est = (t_h * len(tri) / len(pick) * tok + t_u * (d / uw) ** 3
           + (t_g + t_r + t_m * tok) * spec.d_out / n_rows)
    return est, t_meas


def torch_index(rows):
    import torch
    return torch.from_numpy(rows)


def oracle_sampled_step(workload: int, layer_ids, seed: int):
    """The sampled oracle on the given layers of a full-size workload;
    returns (layers, extrapolated seconds, measured seconds)."""
    import numpy as np
    from post_weight_quantization_27_b200 import inputs as I
    layers = I.workload_layers(workload)
    rng = np.random.default_rng(seed)
    est = meas = 0.0
    for i in layer_ids:
        e, m = oracle_sampled_layer(layers[i], rng)
        est += e
        meas += m
    return len(layer_ids), est, meas


SAMPLED_DESC = ("per layer: H on %d random %dx%d upper-triangle tiles over the first %d tokens, "
                "U of the leading %d channels, GPTQ + RTN + both reconstruction errors on %d "
                "random rows at full width; each unit timed and scaled to the whole layer "
                "(extrapolated)" % (SAMPLE_TILES, SAMPLE_TILE, SAMPLE_TILE, SAMPLE_TOKENS,
                                    SAMPLE_U, SAMPLE_ROWS))


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def reference_arm(args, world, rank):
    if rank != 0:
        return None
    from post_weight_quantization_27_b200 import inputs as I
    cores = cpu_threads()
    if args.workload in (1, 2):
        for _ in range(args.warmup):
            oracle_sample_step(args.workload)
        n, sec = 0, 0.0
        for _ in range(args.steps):
            k, s = oracle_sample_step(args.workload)
            n += k
            sec += s
        value = n / sec
        sample = ("block 0 of the 49-layer workload (768->2304, 768->768, 768->3072, "
                  "3072->768), full path per layer" if args.workload == 2 else "the single layer")
        ms_step = sec / args.steps * 1e3
    else:
        # one layer's sampled units per step, cycling over the workload's shapes
        n_layers = len(I.workload_layers(args.workload))
        shapes = list(range(n_layers if args.workload != 3 else 4))
        for w in range(args.warmup):
            oracle_sampled_step(args.workload, [shapes[w % len(shapes)]], 1000 + w)
        n, est, meas = 0, 0.0, 0.0
        for k in range(args.steps):
            a, e, m = oracle_sampled_step(args.workload, [shapes[k % len(shapes)]], k)
            n += a
            est += e
            meas += m
        value = n / est
        sample = SAMPLED_DESC + "; one layer per step, cycling over the workload's shapes"
        ms_step = est / args.steps * 1e3
    return {"metric": METRIC, "value": round(value, 6), "unit": "layers/s", "impl": "reference",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_step, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
            "data": "synthetic (seeded)",
            "config": {"workload": WORKLOAD_NAMES[args.workload]},
            "cpu_baseline": {"value": round(value, 6), "unit": "layers/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "layers/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def cpu_baseline(workload: int) -> dict:
    """The oracle on a bounded sample, timed on the host cores (rank 0, N=1)."""
    if workload in (1, 2):
        n, sec = oracle_sample_step(workload)
        sample = ("block 0 of the workload (4 layers: 768->2304, 768->768, 768->3072, "
                  "3072->768), full path each; the lm_head is not in the sample"
                  if workload == 2 else "first layer of the workload")
        return {"value": round(n / sec, 4), "unit": "layers/s", "cores": cpu_threads(),
                "kind": "oracle", "sample": sample, "seconds": round(sec, 2)}
    from post_weight_quantization_27_b200 import inputs as I
    ids = list(range(len(I.workload_layers(workload)) if workload != 3 else 4))
    n, est, meas = oracle_sampled_step(workload, ids, 7)
    return {"value": round(n / est, 6), "unit": "layers/s", "cores": cpu_threads(),
            "kind": "oracle", "sample": SAMPLED_DESC + "; every layer shape of the workload once",
            "seconds_measured": round(meas, 2), "seconds_extrapolated": round(est, 1)}


# ----------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 10 for the full-size workloads, 50 otherwise)")
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", type=int, default=5, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--impl", default="gq", choices=["gq", "reference"])
    ap.add_argument("--streams", type=int, default=None,
                    help="concurrent streams (default: one per layer up to 32 for the small "
                         "workloads; 1 for the full-size ones, whose layers each fill the GPU)")
    ap.add_argument("--recon", default="hessian", choices=["hessian", "direct"],
                    help="reconstruction error route: from the Hessian (tr(dW H0 dW^T) / 2) "
                         "or directly (||dW X^T||^2)")
    ap.add_argument("--serial-stages", default="",
                    help="stages (comma-separated, e.g. hessian) that run one layer at a time "
                         "across the streams")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.steps is None:
        args.steps = 10 if args.workload >= 3 else 50
    if args.streams is None:
        args.streams = 1 if args.workload >= 3 else 32
    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "gq" else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    try:
        if args.impl == "reference":
            out = reference_arm(args, world, rank)
        else:
            out = gpu_arm(args, world, rank, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = cpu_baseline(args.workload)
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
