"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
import numpy as np
import torch


def u32(t: torch.Tensor) -> np.ndarray:
    """Device int32 tensor of uint32 bit patterns -> numpy uint32."""
    return t.cpu().numpy().view(np.uint32)


def f16(t: torch.Tensor) -> np.ndarray:
    """Device fp16 tensor -> numpy float16 (bit-exact)."""
    return t.cpu().numpy().astype(np.float16)


def np_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
