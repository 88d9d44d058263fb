"""W4A16 product Y = W^ X^T from the packed format on the GPU against the
oracle (fp64 from the dequantised weights)."""
import numpy as np
import pytest
import torch

import oracle as O
from post_weight_quantization_27_b200 import gq, inputs as I
from tests.gpu_util import f16, rel_fro, u32

pytestmark = pytest.mark.gpu


def _check(q, d_in, X, group_size, sym, g_idx=None):
    Y = gq.w4a16_matmul(q, d_in, X.cuda(), group_size, sym)
    torch.cuda.synchronize()
    ref = O.w4a16_matmul(u32(q["qpacked"]), f16(q["scales"]),
                         None if sym else f16(q["zeros"]), d_in, group_size, sym,
                         X.float().numpy(), g_idx)
    got = Y.cpu().numpy().astype(np.float64)
    assert got.shape == ref.shape
    # The products s (c - z) x are exact (W^ is held exactly by the bf16 pair
    # and X is bf16); the error is the tensor core's fp32 accumulation over
    # the d_in terms, about sqrt(d_in) * 2^-24 relative: 1e-5 bounds it for
    # d_in up to a few thousand.
    assert rel_fro(got, ref) <= 1e-5
    assert np.max(np.abs(got - ref)) <= 1e-4 * np.max(np.abs(ref))


@pytest.mark.parametrize("d_out,d_in,n_tok,group_size,sym,dt", [
    (96, 256, 512, -1, True, "f32"),
    (130, 768, 300, 128, False, "bf16"),       # ragged rows and tokens
    (300, 512, 1028, 32, True, "f16"),
    (64, 384, 64, 0, False, "f32"),            # per-tensor scale
])
def test_w4a16_rtn_layers(d_out, d_in, n_tok, group_size, sym, dt):
    spec = I.LayerSpec(0, d_out + d_in, "w", d_in, d_out, dt, 0.02, "none", n_tok, 4, 20.0,
                       group_size, sym, False)
    W, X = I.make_weights(spec), I.make_x(spec)
    q = gq.rtn_quantize_pack(W.cuda(), 4, group_size, sym)
    _check(q, d_in, X, group_size, sym)


def test_w4a16_gptq_act_order():
    """GPTQ output with act-order (g_idx maps each column to its group)."""
    spec = I.workload_layers(4)[0].with_tokens(2048)
    spec = I.LayerSpec(spec.workload, spec.index, spec.name, 512, 192, spec.w_dtype, spec.w_std,
                       spec.w_outlier, 2048, spec.x_out_channels, spec.x_out_factor, 128, False,
                       True)
    W, X = I.make_weights(spec).cuda(), I.make_x(spec)
    H = gq.hessian(X.cuda())
    U, perm, dead, _ = gq.damp_cholesky_inverse(H, 0.01, act_order=True)
    q = gq.gptq_quantize_layer(W, U, 4, 128, 128, False, perm=perm, dead=dead)
    _check(q, 512, X, 128, False, q["g_idx"].cpu().numpy())
