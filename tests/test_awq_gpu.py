"""Activation-aware per-channel scaling before RTN on the GPU against the
oracle: the error curve over alpha, the chosen alpha, the channel scales, and
the codes of the chosen alpha bit for bit (the oracle's RTN applied to the
GPU's fp32 scales, so that both sides round the same products)."""
import numpy as np
import pytest
import torch

import oracle as O
from post_weight_quantization_27_b200 import gq, inputs as I
from tests.gpu_util import f16, u32

pytestmark = pytest.mark.gpu


def _outlier_layer(seed, d_out, d_in, n_tok):
    g = torch.Generator().manual_seed(seed)
    X = torch.randn((n_tok, d_in), generator=g)
    X[:, 3] *= 50.0
    X[:, 17] *= 20.0
    W = torch.randn((d_out, d_in), generator=g) * 0.02
    return W, X.to(torch.bfloat16)


def _run(W, X, group_size, sym, n_grid):
    Wd, Xd = W.cuda(), X.cuda()
    H = gq.hessian(Xd)
    out = gq.awq_rtn_search(Wd, H, Xd, 4, group_size, sym, n_grid)
    torch.cuda.synchronize()
    Wn = W.float().numpy()
    Xn = X.float().numpy()
    ref = O.awq_rtn_search(Wn, Xn, group_size=group_size, sym=sym, n_grid=n_grid)
    # error curve and choice
    assert np.allclose(out["mse"], ref["mse"], rtol=1e-3, atol=0)
    srt = np.sort(ref["mse"])
    if n_grid == 1 or srt[1] > srt[0] * (1 + 2e-3):
        assert out["best"] == ref["best"]
    else:
        assert ref["mse"][out["best"]] <= srt[0] * (1 + 2e-3)
    # scales of the chosen alpha
    s_gpu = out["col_scale"].cpu().numpy()
    hd = 2.0 * np.sum(Xn.astype(np.float64) ** 2, axis=0)
    s_ref = O.awq_channel_scales(hd, out["best"] / n_grid)
    assert np.allclose(s_gpu, s_ref, rtol=1e-5, atol=0)
    # codes, scales, zeros of RTN(W diag(s)) bit for bit
    r, _ = O.awq_apply(Wn, s_gpu, group_size, sym)
    assert np.array_equal(u32(out["qpacked"]), r["qpacked"])
    assert np.array_equal(f16(out["scales"]).view(np.uint16), r["scales"].view(np.uint16))
    if not sym:
        assert np.array_equal(f16(out["zeros"]).view(np.uint16), r["zeros"].view(np.uint16))
    return out, ref


@pytest.mark.parametrize("group_size,sym", [(-1, True), (32, False), (128, True)])
def test_awq_outlier_channels(group_size, sym):
    W, X = _outlier_layer(11, 96, 256, 1024)
    out, ref = _run(W, X, group_size, sym, 10)
    assert ref["best"] > 0 and out["mse"][out["best"]] < out["mse"][0]


@pytest.mark.parametrize("workload,idx,group_size,sym", [(1, 0, -1, True), (2, 1, 128, False)])
def test_awq_workload_layers(workload, idx, group_size, sym):
    spec = I.workload_layers(workload)[idx]
    W = I.make_weights(spec)
    X = I.make_x(spec)
    _run(W, X, group_size, sym, 20)


def test_awq_single_point_is_rtn():
    """n_grid = 1 tries alpha = 0 only: the output is plain RTN."""
    W, X = _outlier_layer(5, 64, 128, 512)
    out, _ = _run(W, X, 32, True, 1)
    rtn = gq.rtn_quantize_pack(W.cuda(), 4, 32, True)
    assert torch.equal(out["qpacked"], rtn["qpacked"])
    assert torch.allclose(out["col_scale"], torch.ones(128, device="cuda"))
