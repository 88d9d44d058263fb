"""Reconstruction error ||(W - W^) X^T||^2 on the GPU against the oracle
(relative error <= 1e-3), fed the oracle's own quantised layers."""
import numpy as np
import pytest
import torch

import oracle as O
from post_weight_quantization_27_b200 import gq, inputs as I

pytestmark = pytest.mark.gpu
TOL = 1e-3


def _q_from_oracle(res, sym, act_order=False):
    q = dict(qpacked=torch.from_numpy(res["qpacked"].view(np.int32)).cuda(),
             scales=torch.from_numpy(res["scales"]).cuda(),
             zeros=None if sym else torch.from_numpy(res["zeros"]).cuda())
    if act_order:
        q["g_idx"] = torch.from_numpy(res["g_idx"]).cuda()
    return q


@pytest.mark.parametrize("d_out,d_in,n_tok,gs,sym,dt", [
    (96, 256, 512, -1, True, torch.float32),
    (130, 136, 300, 8, False, torch.float16),
    (768, 768, 2048, -1, True, torch.float32),
    (300, 1024, 700, 128, False, torch.bfloat16),
    (1, 64, 1, -1, True, torch.float32),
])
def test_recon_rtn_layers(d_out, d_in, n_tok, gs, sym, dt):
    spec = I.LayerSpec(0, d_in + n_tok, "r", d_in, d_out, "f32", 0.02, "none", n_tok, 2, 20.0,
                       gs, sym, False)
    W = I.make_weights(spec).to(dt)
    X = I.make_x(spec)
    Wn = W.float().numpy()
    ref = O.rtn_quantize(Wn, gs, sym)
    Wh = O.dequantize_packed(ref["qpacked"], ref["scales"], ref["zeros"], d_in, gs, sym)
    sse_ref = O.recon_sse(Wn, Wh, X.float().numpy())
    sse, mse = gq.recon_error(W.cuda(), _q_from_oracle(ref, sym), X.cuda(), gs, sym)
    assert abs(sse - sse_ref) <= TOL * sse_ref
    assert abs(mse - sse_ref / (n_tok * d_out)) <= TOL * sse_ref / (n_tok * d_out)


def test_recon_gptq_act_order_layer():
    rng = np.random.default_rng(3)
    d_out, d_in, n_tok = 64, 256, 600
    X = (rng.standard_normal((n_tok, d_in)) * rng.lognormal(0, 0.5, d_in)).astype(np.float32)
    Xb = torch.from_numpy(X).to(torch.bfloat16)
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float32)
    res, *_ = O.gptq_layer(W, Xb.float().numpy(), group_size=128, sym=False, act_order=True)
    sse_ref = O.recon_sse(W, res.W_hat, Xb.float().numpy())
    q = dict(qpacked=res.qpacked, scales=res.scales, zeros=res.zeros, g_idx=res.g_idx)
    sse, _ = gq.recon_error(torch.from_numpy(W).cuda(), _q_from_oracle(q, False, True), Xb.cuda(),
                            128, False)
    assert abs(sse - sse_ref) <= TOL * sse_ref


def test_recon_empty_and_deterministic():
    spec = I.LayerSpec(0, 9, "r", 256, 100, "f32", 0.02, "none", 1000, 2, 20.0, -1, True, False)
    W, X = I.make_weights(spec).cuda(), I.make_x(spec).cuda()
    q = gq.rtn_quantize_pack(W, 4, -1, True)
    sse0, _ = gq.recon_error(W, q, X[:0], -1, True)
    assert sse0 == 0.0
    a, _ = gq.recon_error(W, q, X, -1, True)
    b, _ = gq.recon_error(W, q, X, -1, True)
    assert a == b and a > 0


# ---------------------------------------------------------------- trace route

@pytest.mark.parametrize("d_out,d_in,n_tok,gs,sym,dt", [
    (96, 256, 512, -1, True, torch.float32),
    (130, 136, 300, 8, False, torch.float16),      # ragged tiles in both directions
    (300, 1024, 2000, 128, False, torch.bfloat16),
    (1, 64, 100, -1, True, torch.float32),
    (520, 776, 1500, 8, True, torch.float16),      # d_in not a multiple of the K step
])
def test_recon_hessian_route_matches_oracle(d_out, d_in, n_tok, gs, sym, dt):
    """tr(dW H0 dW^T) / 2 on the GPU, with the oracle's H0 (rounded to fp32,
    as the Hessian call returns it) and the oracle's RTN layer, against the
    oracle's direct ||dW X^T||^2 (relative 1e-3)."""
    spec = I.LayerSpec(0, d_in + 3 * n_tok, "r", d_in, d_out, "f32", 0.02, "none", n_tok, 2,
                       20.0, gs, sym, False)
    W = I.make_weights(spec).to(dt)
    X = I.make_x(spec)
    Wn, Xn = W.float().numpy(), X.float().numpy()
    ref = O.rtn_quantize(Wn, gs, sym)
    Wh = O.dequantize_packed(ref["qpacked"], ref["scales"], ref["zeros"], d_in, gs, sym)
    sse_ref = O.recon_sse(Wn, Wh, Xn)
    H0 = torch.from_numpy(O.hessian(Xn).astype(np.float32)).cuda()
    sse, mse = gq.recon_error_hessian(W.cuda(), _q_from_oracle(ref, sym), H0, n_tok, gs, sym)
    assert abs(sse - sse_ref) <= TOL * sse_ref, (sse, sse_ref)
    assert abs(mse - sse_ref / (n_tok * d_out)) <= TOL * sse_ref / (n_tok * d_out)
    # and the GPU's own direct route, bit-for-bit deterministic on a second call
    sse_d, _ = gq.recon_error(W.cuda(), _q_from_oracle(ref, sym), X.cuda(), gs, sym)
    assert abs(sse - sse_d) <= TOL * sse_d
    again, _ = gq.recon_error_hessian(W.cuda(), _q_from_oracle(ref, sym), H0, n_tok, gs, sym)
    assert again == sse


def test_recon_hessian_route_gptq_act_order():
    """The trace route on a GPTQ layer (its error is shaped by H, the hard
    case for a quadratic form) with act-order group indices, using the
    GPU's own Hessian."""
    rng = np.random.default_rng(4)
    d_out, d_in, n_tok = 200, 512, 3000
    X = (rng.standard_normal((n_tok, d_in)) * rng.lognormal(0, 0.5, d_in)).astype(np.float32)
    X[:, 7] *= 50.0
    Xb = torch.from_numpy(X).to(torch.bfloat16)
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float32)
    res, *_ = O.gptq_layer(W, Xb.float().numpy(), group_size=128, sym=False, act_order=True)
    sse_ref = O.recon_sse(W, res.W_hat, Xb.float().numpy())
    q = _q_from_oracle(dict(qpacked=res.qpacked, scales=res.scales, zeros=res.zeros,
                            g_idx=res.g_idx), False, True)
    H0 = gq.hessian(Xb.cuda())
    sse, _ = gq.recon_error_hessian(torch.from_numpy(W).cuda(), q, H0, n_tok, 128, False)
    assert abs(sse - sse_ref) <= TOL * sse_ref, (sse, sse_ref)
