"""Benchmark: layer-wise 4-bit GPTQ + RTN of a whole model's weight layers.

A step runs the complete per-layer path on every layer of the workload:
H = 2 X^T X, damping + dead columns + U (H^-1 = U^T U), GPTQ, RTN, and the
reconstruction error of both quantised layers.  Default workload: the 49
weight-bearing layers of GPT-2 small (768 -> 2304 / 768 / 3072, 3072 -> 768
per block, x12, plus the 768 -> 50257 head) with 2560 calibration tokens
per layer, per-channel symmetric 4-bit, block 128, damp 0.01.  Inputs are
seeded synthetic data (no dataset or trained weights), resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 2|1|3|4|5]
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
    3: "gpt2-style 1.3B, 96 layers, 262144 tokens each",
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
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
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

class LayerRun:
    """Device buffers of one layer and the calls of one step on it."""

    def __init__(self, spec, dev, W, X):
        import torch
        from post_weight_quantization_27_b200 import gq
        self.spec = spec
        self.W, self.X = W, X
        d_in, d_out, n = spec.d_in, spec.d_out, spec.n_tok
        f = dict(device=dev)
        self.H = torch.empty((d_in, d_in), dtype=torch.float32, **f)
        self.U = torch.empty((d_in, d_in), dtype=torch.float32, **f)
        self.ws_h = gq.workspace(gq.hessian_workspace_size(n, d_in), dev)
        self.ws_c = gq.workspace(gq.damp_cholesky_workspace_size(d_in), dev)
        self.ws_g = gq.workspace(gq.gptq_workspace_size(d_out, d_in, spec.block_size), dev)
        self.ws_r = gq.workspace(gq.recon_workspace_size(d_out, d_in, n), dev)
        self.q_gptq = gq._outputs(d_out, d_in, spec.group_size, spec.sym, dev, spec.act_order)
        self.q_rtn = gq._outputs(d_out, d_in, spec.group_size, spec.sym, dev, False)
        self.perm = torch.empty(d_in, dtype=torch.int32, **f) if spec.act_order else None
        self.dead = torch.empty(d_in, dtype=torch.uint8, **f)
        self.info = torch.empty(1, dtype=torch.int32, **f)
        self.sse = torch.empty(2, dtype=torch.float64, **f)

    def hessian(self):
        from post_weight_quantization_27_b200 import gq
        L, s = gq.lib(), gq._stream(None)
        self.H.zero_()
        gq._check(L.gq_hessian_accumulate(gq._p(self.X), self.spec.n_tok, self.spec.d_in,
                                          gq._p(self.H), gq._p(self.ws_h), self.ws_h.numel(), s),
                  "hessian")

    def solve(self):
        from post_weight_quantization_27_b200 import gq
        L, s, sp = gq.lib(), gq._stream(None), self.spec
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
            gq._check(L.gq_recon_error(
                gq._p(self.W), gq._DTYPES[self.W.dtype], gq._p(o["qpacked"]),
                gq._p(o["scales"]), gq._p(o["zeros"]), gq._p(o.get("g_idx")), sp.d_out,
                sp.d_in, sp.group_size, int(sp.sym), gq._p(self.X), sp.n_tok,
                self.sse.data_ptr() + 8 * k, None, None, gq._p(self.ws_r),
                self.ws_r.numel(), s), "recon")

    STAGES = ("hessian", "solve", "gptq", "rtn", "recon")


def build_layers(workload: int, dev, generate_on_device: bool):
    import torch
    from post_weight_quantization_27_b200 import inputs as I
    runs = []
    for spec in I.workload_layers(workload):
        W = I.make_weights(spec).to(dev)
        X = I.make_x_device(spec, dev) if generate_on_device else I.make_x(spec).to(dev)
        runs.append(LayerRun(spec, dev, W, X))
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


def capture_step(runs, n_streams, timed=False, host=None):
    """One whole step (every layer, every stage) captured as a CUDA graph:
    the layers run on ``n_streams`` streams forked from and joined back to
    one capture stream.  ``timed`` adds timing event nodes around each
    stage call; ``host`` adds the pinned host <-> device copies of the
    end-to-end run.  Returns (graph, stream, stage events, launches/step)."""
    import torch
    from post_weight_quantization_27_b200 import gq
    main = torch.cuda.Stream()
    sides = [torch.cuda.Stream() for _ in range(n_streams)]
    g = torch.cuda.CUDAGraph()
    events = []
    n0 = gq.launch_count()
    with torch.cuda.graph(g, stream=main):
        fork = torch.cuda.Event()
        fork.record(main)
        for sd in sides:
            sd.wait_event(fork)
        for si, idxs in enumerate(schedule(runs, n_streams)):
            sd = sides[si]
            with torch.cuda.stream(sd):
                for i in idxs:
                    r = runs[i]
                    if host is not None:
                        r.W.copy_(host[i]["W"], non_blocking=True)
                        r.X.copy_(host[i]["X"], non_blocking=True)
                    for st in LayerRun.STAGES:
                        if timed:
                            e0 = torch.cuda.Event(enable_timing=True, external=True)
                            e1 = torch.cuda.Event(enable_timing=True, external=True)
                            e0.record(sd)
                        getattr(r, st)()
                        if timed:
                            e1.record(sd)
                            events.append((i, st, e0, e1))
                    if host is not None:
                        h = host[i]
                        h["q"].copy_(r.q_gptq["qpacked"], non_blocking=True)
                        h["s"].copy_(r.q_gptq["scales"], non_blocking=True)
                        h["qr"].copy_(r.q_rtn["qpacked"], non_blocking=True)
                        h["sse"].copy_(r.sse, non_blocking=True)
        for sd in sides:
            j = torch.cuda.Event()
            j.record(sd)
            main.wait_event(j)
    return g, main, events, gq.launch_count() - n0


def stage_work(spec):
    """Algorithmic work per call of each stage (bytes or flops)."""
    wb = {"f32": 4, "f16": 2, "bf16": 2}[spec.w_dtype]
    n_groups = 1 if spec.group_size == -1 else spec.d_in // spec.group_size
    zero_bytes = 0 if spec.sym else 2 * spec.d_out * n_groups
    return {
        # symmetric half of X^T X: N d (d + 1) flops
        "hessian_flops": spec.n_tok * spec.d_in * (spec.d_in + 1),
        # read W, write codes + fp16 scales (+ zeros)
        "rtn_bytes": spec.d_out * spec.d_in * (wb + 0.5) + 2 * spec.d_out * n_groups + zero_bytes,
        # two reconstruction GEMMs, 2 N d_out d_in each
        "recon_flops": 2 * 2 * spec.n_tok * spec.d_out * spec.d_in,
        "weights": spec.d_out * spec.d_in,
    }


def gpu_arm(args, world, rank, local):
    import torch
    from post_weight_quantization_27_b200 import gq
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    gq.lib()
    big = args.workload >= 3
    runs = build_layers(args.workload, dev, generate_on_device=big)
    peaks = measured_peaks()
    n_streams = max(1, min(args.streams, len(runs)))

    # one eager pass (sets kernel attributes), then the captured step
    for r in runs:
        for st in LayerRun.STAGES:
            getattr(r, st)()
    torch.cuda.synchronize()
    graph, gstream, events, launches_per_step = capture_step(runs, n_streams, timed=True)

    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    barrier(world)

    # ---------------- timed region: inputs resident in HBM
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        barrier(world)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(gstream)
        for _ in range(args.steps):
            graph.replay()
        t1.record(gstream)
        torch.cuda.synchronize()
        barrier(world)
    ms_local = t0.elapsed_time(t1) / args.steps
    ms = reduce_max(ms_local, world)
    clocks = clk.summary()

    # per-call stage durations of the last timed step (event nodes in the graph)
    calls = {st: [] for st in LayerRun.STAGES}
    for i, st, e0, e1 in events:
        calls[st].append(e0.elapsed_time(e1))
    stage_ms = {st: sum(v) for st, v in calls.items()}
    work = [stage_work(r.spec) for r in runs]
    tot = {k: sum(w[k] for w in work) for k in work[0]}
    n_layers = len(runs)
    value = world * n_layers / (ms / 1e3)

    dom = max(stage_ms, key=stage_ms.get)
    roof = roofline(dom, stage_ms, tot, peaks)
    del graph

    e2e = e2e_run(runs, args, dev, world, n_streams)

    out = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "layers/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 X, fp32 H/U/GPTQ, int4 codes",
        "data": "synthetic (seeded; random-init weights of the named layer shapes)",
        "config": {"workload": WORKLOAD_NAMES[args.workload], "layers": n_layers,
                   "weights_per_step": tot["weights"], "parallelism": f"layers x{world} (weak)",
                   "streams": n_streams, "cuda_graph": True,
                   "l2": "inputs larger than L2 (%.0f MB of W and X per step)" % (
                       sum(r.W.numel() * r.W.element_size() + r.X.numel() * 2 for r in runs) / 1e6)},
        "mweights_per_s": round(world * tot["weights"] / (ms / 1e3) / 1e6, 2),
        "stage_ms_sum_of_calls": {k: round(v, 4) for k, v in stage_ms.items()},
        "xtx_tflops": round(tot["hessian_flops"] / (stage_ms["hessian"] / 1e3) / 1e12, 2),
        "rtn_gbs": round(tot["rtn_bytes"] / (stage_ms["rtn"] / 1e3) / 1e9, 2),
        "recon_tflops": round(tot["recon_flops"] / (stage_ms["recon"] / 1e3) / 1e12, 2),
        "roofline": roof,
        "gpu_launches": int(launches_per_step * args.steps),
        "clocks": clocks,
        "e2e": e2e,
    }
    return out


def roofline(dom, stage_ms, tot, peaks):
    """Roofline of the dominant stage, from its algorithmic work and its
    CUDA-event time inside the timed region."""
    t = stage_ms[dom] / 1e3          # sum over the step's calls of this stage
    if dom == "hessian":
        a = tot["hessian_flops"] / t / 1e12
        return {"stage": dom, "bound": "tensor", "achieved": round(a, 2),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(a / peaks["bf16_tflops"], 4), "traffic": None,
                "peak_source": peaks["source"] + " (burst bf16)"}
    if dom == "recon":
        a = tot["recon_flops"] / t / 1e12
        return {"stage": dom, "bound": "tensor", "achieved": round(a, 2),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(a / peaks["bf16_tflops"], 4), "traffic": None,
                "peak_source": peaks["source"] + " (burst bf16)"}
    if dom == "rtn":
        a = tot["rtn_bytes"] / t / 1e9
        return {"stage": dom, "bound": "hbm", "achieved": round(a, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(a / peaks["hbm_gbs"], 4), "traffic": None,
                "peak_source": peaks["source"]}
    # gptq / solve: report the fp32 weight traffic of the stage against HBM
    a = tot["weights"] * 4 * 2 / t / 1e9
    return {"stage": dom, "bound": "hbm", "achieved": round(a, 1), "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": round(a / peaks["hbm_gbs"], 4), "traffic": None,
            "peak_source": peaks["source"], "note": "fp32 working-copy bytes (read+write W once)"}


def e2e_run(runs, args, dev, world, n_streams):
    """Same metric through the C-ABI with host buffers: every step copies
    each layer's W and X from pinned host memory and reads back the packed
    codes, scales and both SSEs (copies and compute in one captured graph,
    on the same streams)."""
    import torch
    host = []
    for r in runs:
        host.append(dict(W=r.W.cpu().pin_memory(), X=r.X.cpu().pin_memory(),
                         q=torch.empty(r.q_gptq["qpacked"].shape, dtype=torch.int32).pin_memory(),
                         s=torch.empty(r.q_gptq["scales"].shape, dtype=torch.float16).pin_memory(),
                         qr=torch.empty(r.q_rtn["qpacked"].shape, dtype=torch.int32).pin_memory(),
                         sse=torch.empty(2, dtype=torch.float64).pin_memory()))
    h2d = sum(h["W"].numel() * h["W"].element_size() + h["X"].numel() * 2 for h in host)
    d2h = sum(h["q"].numel() * 4 + h["s"].numel() * 2 + h["qr"].numel() * 4 + 16 for h in host)
    graph, gstream, _, _ = capture_step(runs, n_streams, timed=False, host=host)
    steps = max(1, min(args.steps, 5))
    graph.replay()
    torch.cuda.synchronize()
    barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(gstream)
    for _ in range(steps):
        graph.replay()
    t1.record(gstream)
    torch.cuda.synchronize()
    ms = reduce_max(t0.elapsed_time(t1) / steps, world)
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
    if args.workload != 2 and args.workload != 1:
        return {"impl": "reference", "unavailable": "oracle reference arm is sized for workloads 1-2"}
    for _ in range(args.warmup):
        oracle_sample_step(args.workload)
    n, sec = 0, 0.0
    for _ in range(args.steps):
        k, s = oracle_sample_step(args.workload)
        n += k
        sec += s
    value = n / sec
    sample = ("block 0 of the 49-layer workload (768->2304, 768->768, 768->3072, 3072->768), "
              "full path per layer" if args.workload == 2 else "the single layer")
    cores = cpu_threads()
    return {"metric": METRIC, "value": round(value, 4), "unit": "layers/s", "impl": "reference",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(sec / args.steps * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
            "data": "synthetic (seeded)",
            "config": {"workload": WORKLOAD_NAMES[args.workload]},
            "cpu_baseline": {"value": round(value, 4), "unit": "layers/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "layers/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def cpu_baseline(workload: int) -> dict:
    """The oracle on a bounded sample, timed on the host cores (rank 0, N=1)."""
    n, sec = oracle_sample_step(workload)
    sample = ("block 0 of the workload (4 layers: 768->2304, 768->768, 768->3072, 3072->768), "
              "full path each; the lm_head is not in the sample" if workload == 2
              else "first layer of the workload")
    return {"value": round(n / sec, 4), "unit": "layers/s", "cores": cpu_threads(),
            "kind": "oracle", "sample": sample, "seconds": round(sec, 2)}


# ----------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", type=int, default=2, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--impl", default="gq", choices=["gq", "reference"])
    ap.add_argument("--streams", type=int, default=16)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
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
            if rank == 0 and world == 1 and not args.no_cpu_baseline and args.workload in (1, 2):
                out["cpu_baseline"] = cpu_baseline(args.workload)
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
