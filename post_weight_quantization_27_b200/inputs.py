"""Seeded synthetic layer inputs (weights W and calibration activations X).

This module holds no quantisation arithmetic: it only draws random numbers.
It is the one module that both the CUDA path's tests / bench and the CPU
oracle's checks use, so both sides see identical bytes.

Workloads (shapes from the pages: GPT-2 small's 49 weight-bearing layers in
"GPT-2 Quantization Reconstruction Error"; the 1.3B GPT-2-style model of
"Quantization sweep: perplexity vs compression"; 128 x 2048 calibration
tokens and the Llama-2-70B example of "GPTQ: Post-Training INT4").  None of
the pages' datasets or pretrained weights are available, so:

* W ~ N(0, std^2) in the layer's dtype, with the outlier structure of the
  workload (a few input columns scaled up, or sparse Student-t(3) entries).
* X[t, c] = N(0, 1) * sigma_c with sigma_c ~ LogNormal(0, 0.5) per input
  channel and a few outlier channels scaled up, rounded to bf16 once.

Seeds: numpy PCG64 seeded by SeedSequence([workload, layer, tensor]).  For
the largest workloads the N(0, 1) part of X can also be drawn on the GPU
with torch's CUDA generator (``make_x_device``): same per-channel scales,
different noise stream; those runs check the oracle on sampled entries
copied back from the device.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np
import torch

T_W, T_XNOISE, T_XSCALE, T_WOUT = 0, 1, 2, 3


@dataclass(frozen=True)
class LayerSpec:
    workload: int          # 1..5
    index: int             # layer index inside the workload
    name: str
    d_in: int
    d_out: int
    w_dtype: str           # "f32" | "f16" | "bf16"
    w_std: float
    w_outlier: str         # "none" | "cols:<frac>:<factor>" | "t3:<frac>:<scale>"
    n_tok: int
    x_out_channels: int
    x_out_factor: float
    group_size: int        # -1 = per channel
    sym: bool
    act_order: bool
    damp: float = 0.01
    block_size: int = 128

    def with_tokens(self, n_tok: int) -> "LayerSpec":
        return replace(self, n_tok=n_tok)


TORCH_DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def workload_layers(k: int) -> list[LayerSpec]:
    """Layer list of workload ``k`` (1..5)."""
    if k == 1:
        return [LayerSpec(1, 0, "gpt2.h0.attn.c_proj", 768, 768, "f32", 0.02,
                          "cols:0.01:8", 2048, 4, 20.0, -1, True, False)]
    if k == 2:
        out = []
        i = 0
        for blk in range(12):
            for nm, di, do, std in (("attn.c_attn", 768, 2304, 0.02),
                                    ("attn.c_proj", 768, 768, 0.02),
                                    ("mlp.c_fc", 768, 3072, 0.02),
                                    ("mlp.c_proj", 3072, 768, 0.02 / np.sqrt(24.0))):
                out.append(LayerSpec(2, i, f"h.{blk}.{nm}", di, do, "f32", float(std),
                                     "none", 2560, 4, 20.0, -1, True, False))
                i += 1
        out.append(LayerSpec(2, i, "lm_head", 768, 50257, "f32", 0.02, "none",
                             2560, 4, 20.0, -1, True, False))
        return out
    if k == 3:
        out = []
        i = 0
        for blk in range(24):
            for nm, di, do in (("attn.qkv", 2048, 6144), ("attn.proj", 2048, 2048),
                               ("mlp.fc", 2048, 8192), ("mlp.proj", 8192, 2048)):
                out.append(LayerSpec(3, i, f"h.{blk}.{nm}", di, do, "f16", 0.02,
                                     "t3:0.001:0.02", 262144, 0, 1.0, 128, True, False))
                i += 1
        return out
    if k == 4:
        shapes = ([("attn.q", 4096, 4096), ("attn.k", 4096, 4096), ("attn.v", 4096, 4096),
                   ("attn.o", 4096, 4096), ("mlp.gate", 4096, 11008),
                   ("mlp.up", 4096, 11008), ("mlp.down", 11008, 4096)])
        return [LayerSpec(4, i, nm, di, do, "bf16", 0.015, "cols:0.005:10", 262144,
                          4, 20.0, 128, False, True) for i, (nm, di, do) in enumerate(shapes)]
    if k == 5:
        shapes = [("attn.o", 8192, 8192), ("mlp.up", 8192, 28672), ("mlp.down", 28672, 8192)]
        return [LayerSpec(5, i, nm, di, do, "f16", 0.01, "cols:0.005:10", 262144,
                          8, 50.0, 128, True, False) for i, (nm, di, do) in enumerate(shapes)]
    raise ValueError(f"unknown workload {k}")


def _rng(spec: LayerSpec, tensor: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(
        np.random.SeedSequence([spec.workload, spec.index, tensor, spec.d_in, spec.d_out])))


def make_weights(spec: LayerSpec) -> torch.Tensor:
    """W [d_out, d_in] as a CPU tensor of the layer's dtype."""
    rng = _rng(spec, T_W)
    W = rng.standard_normal((spec.d_out, spec.d_in), dtype=np.float32) * np.float32(spec.w_std)
    if spec.w_outlier.startswith("cols:"):
        _, frac, fac = spec.w_outlier.split(":")
        k = max(1, int(round(float(frac) * spec.d_in)))
        cols = _rng(spec, T_WOUT).choice(spec.d_in, size=k, replace=False)
        W[:, cols] *= np.float32(fac)
    elif spec.w_outlier.startswith("t3:"):
        _, frac, sc = spec.w_outlier.split(":")
        r2 = _rng(spec, T_WOUT)
        k = max(1, int(round(float(frac) * spec.d_in * spec.d_out)))
        pos = r2.choice(spec.d_in * spec.d_out, size=k, replace=False)
        W.reshape(-1)[pos] = (r2.standard_t(3.0, size=k) * float(sc)).astype(np.float32)
    return torch.from_numpy(W).to(TORCH_DTYPES[spec.w_dtype])


def channel_scales(spec: LayerSpec) -> np.ndarray:
    """Per-input-channel activation scale sigma_c (float32)."""
    rng = _rng(spec, T_XSCALE)
    sig = rng.lognormal(0.0, 0.5, size=spec.d_in).astype(np.float32)
    if spec.x_out_channels:
        ch = rng.choice(spec.d_in, size=spec.x_out_channels, replace=False)
        sig[ch] *= np.float32(spec.x_out_factor)
    return sig


def make_x(spec: LayerSpec, rows: int | None = None) -> torch.Tensor:
    """X [n_tok, d_in] (or its first ``rows`` tokens) as a CPU bf16 tensor."""
    n = spec.n_tok if rows is None else rows
    rng = _rng(spec, T_XNOISE)
    sig = channel_scales(spec)
    out = torch.empty((n, spec.d_in), dtype=torch.bfloat16)
    step = max(1, (1 << 24) // spec.d_in)
    for r0 in range(0, n, step):
        r1 = min(n, r0 + step)
        z = rng.standard_normal((r1 - r0, spec.d_in), dtype=np.float32) * sig[None, :]
        out[r0:r1] = torch.from_numpy(z).to(torch.bfloat16)
    return out


def make_x_device(spec: LayerSpec, device, rows: int | None = None) -> torch.Tensor:
    """X drawn on ``device`` with torch's generator (large workloads)."""
    n = spec.n_tok if rows is None else rows
    gen = torch.Generator(device=device)
    gen.manual_seed(int(np.random.SeedSequence(
        [spec.workload, spec.index, T_XNOISE, spec.d_in, spec.d_out]).generate_state(1)[0]))
    sig = torch.from_numpy(channel_scales(spec)).to(device)
    out = torch.empty((n, spec.d_in), dtype=torch.bfloat16, device=device)
    step = max(1, (1 << 26) // spec.d_in)
    for r0 in range(0, n, step):
        r1 = min(n, r0 + step)
        z = torch.randn((r1 - r0, spec.d_in), generator=gen, device=device, dtype=torch.float32)
        out[r0:r1] = (z * sig[None, :]).to(torch.bfloat16)
    return out


def random_layer(seed: int, d_in: int, d_out: int, n_tok: int, w_dtype: str = "f32",
                 w_std: float = 0.02) -> tuple[torch.Tensor, torch.Tensor]:
    """Small random (W, X) pair for parity tests of arbitrary shapes."""
    spec = LayerSpec(0, seed, "rand", d_in, d_out, w_dtype, w_std, "none", n_tok,
                     min(2, d_in), 10.0, -1, True, False)
    return make_weights(spec), make_x(spec)
