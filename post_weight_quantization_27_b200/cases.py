"""Run the path on one layer of a workload once, on the GPU, through the
C-ABI library -- a fixed, small case for profilers (ncu) and for timing one
stage by hand.

    python -m post_weight_quantization_27_b200.cases --workload 2 --layer 3
           [--tokens N] [--repeat R]
           [--stages hessian,solve,gptq,rtn,recon,trace,awq,w4a16,qlinear]

The stages always run in path order (H -> damp/U -> GPTQ -> RTN -> recon),
each as many times as --repeat says; a stage that is not listed still runs
once if a listed stage needs its output.  Prints one line per stage with its
CUDA-event time.  "recon" is the direct error ||(W - W^) X^T||^2 of the GPTQ
and RTN layers; "trace" is the error from the Hessian (tr(dW H dW^T) / 2) of
the GPTQ layer (of the RTN layer when GPTQ is not listed); "awq" is the
activation-aware scaling search before RTN (20 values of alpha), which needs
only H; "w4a16" multiplies the RTN layer with the first (at most 8192)
tokens; "qlinear" applies it to them (token-major bf16 output, GELU).
"""
from __future__ import annotations

import argparse

import torch

from . import gq
from . import inputs as I

ORDER = ("hessian", "solve", "gptq", "rtn", "recon", "trace", "awq", "w4a16", "qlinear")


def run(workload: int, layer: int, tokens: int | None, stages, repeat: int = 1) -> dict:
    spec = I.workload_layers(workload)[layer]
    if tokens is not None:
        spec = spec.with_tokens(tokens)
    W = I.make_weights(spec).cuda()
    X = I.make_x_device(spec, "cuda")
    # what each stage needs run before it
    deps = {"hessian": set(), "solve": {"hessian"}, "gptq": {"hessian", "solve"}, "rtn": set(),
            "recon": {"hessian", "solve", "gptq", "rtn"}, "awq": {"hessian"},
            "trace": {"hessian"} | ({"solve", "gptq"} if "gptq" in stages else {"rtn"}),
            "w4a16": {"rtn"}, "qlinear": {"rtn"}}
    need = set(stages)
    for st in stages:
        need |= deps[st]
    times = {}

    def timed(name, fn):
        n = repeat if name in stages else 1
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        out = None
        e0.record()
        for _ in range(n):
            out = fn()
        e1.record()
        torch.cuda.synchronize()
        times[name] = e0.elapsed_time(e1) / n
        return out

    H = U = perm = dead = q = None
    if "hessian" in need:
        H = timed("hessian", lambda: gq.hessian(X))
    if "solve" in need:
        Hs = H.clone()
        U, perm, dead, _ = timed("solve", lambda: gq.damp_cholesky_inverse(
            Hs.copy_(H), spec.damp, act_order=spec.act_order))
    if "gptq" in need:
        q = timed("gptq", lambda: gq.gptq_quantize_layer(
            W, U, 4, spec.group_size, spec.block_size, spec.sym, perm=perm, dead=dead))
    r = None
    if "rtn" in need:
        r = timed("rtn", lambda: gq.rtn_quantize_pack(W, 4, spec.group_size, spec.sym))
    if "recon" in need:
        timed("recon", lambda: gq.recon_error(W, q, X, spec.group_size, spec.sym))
    if "trace" in need:
        timed("trace", lambda: gq.recon_error_hessian(W, q if q is not None else r, H,
                                                      X.shape[0], spec.group_size, spec.sym))
    if "awq" in need:
        timed("awq", lambda: gq.awq_rtn_search(W, H, X, 4, spec.group_size, spec.sym, 20))
    if "w4a16" in need:  # the RTN layer times the first (at most 8192) tokens
        Xs = X[:min(X.shape[0], 8192) // 4 * 4]
        timed("w4a16", lambda: gq.w4a16_matmul(r, spec.d_in, Xs, spec.group_size, spec.sym))
    if "qlinear" in need:
        Xs = X[:min(X.shape[0], 8192)]
        timed("qlinear", lambda: gq.qlinear_bf16(Xs, spec.d_out, q=r, group_size=spec.group_size,
                                                 sym=spec.sym, act="gelu"))
    return {"spec": spec, "ms": times}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", type=int, default=2, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--layer", type=int, default=0)
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--repeat", type=int, default=1)
    ap.add_argument("--stages", default=",".join(ORDER))
    a = ap.parse_args()
    stages = [s for s in a.stages.split(",") if s]
    for s in stages:
        if s not in ORDER:
            raise SystemExit(f"unknown stage {s!r}; stages are {', '.join(ORDER)}")
    r = run(a.workload, a.layer, a.tokens, stages, a.repeat)
    sp = r["spec"]
    print(f"workload {a.workload} layer {a.layer} ({sp.name}: {sp.d_in} -> {sp.d_out}, "
          f"{sp.n_tok} tokens)")
    for k, v in r["ms"].items():
        print(f"  {k:8s} {v:10.3f} ms")


if __name__ == "__main__":
    main()
