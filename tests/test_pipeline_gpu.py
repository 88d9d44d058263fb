"""The quantised layer applied to its input (gq_qlinear_bf16: dequantising
inside the GEMM, token-major bf16 output with activation and residual) and
the sequential pipeline (gq_gptq_sequential: each layer calibrated on the
output of the quantised layers before it) against the oracle.

bf16 outputs: the GPU sums in fp32, the oracle in fp64, and both round once
to bf16, so an output may differ by one bf16 step where the exact value
lies within the fp32 sum's error of a rounding boundary; the bound used is
one step of the value plus 2^-20 of sum |x| |w| (the fp32 accumulation
error, with room)."""
import numpy as np
import pytest
import torch

import oracle as O
from post_weight_quantization_27_b200 import gq, inputs as I
from tests.gpu_util import f16, rel_fro, u32
from tests.test_gptq_gpu import check_gptq

pytestmark = pytest.mark.gpu


def _bf16_close(got, ref, X, W_hat, min_exact=0.99):
    got = np.asarray(got, dtype=np.float64)
    step = np.ldexp(1.0, np.frexp(np.abs(ref))[1] - 8)          # one bf16 step at |ref|
    bound = step + 2.0 ** -20 * (np.abs(X) @ np.abs(W_hat).T)
    assert np.all(np.abs(got - ref) <= bound), float(np.max(np.abs(got - ref) - bound))
    assert np.mean(got == ref) >= min_exact, np.mean(got == ref)


def _x(n, d, seed):
    return I.random_layer(seed, d, 8, n)[1]


@pytest.mark.parametrize("bits,group_size,sym", [(4, -1, True), (4, 128, False), (4, 32, True),
                                                 (8, 64, True), (3, 128, False), (2, -1, True)])
@pytest.mark.parametrize("act", ["none", "relu", "gelu"])
def test_qlinear_packed_matches_oracle(bits, group_size, sym, act):
    n, d_in, d_out = 700, 256, 200
    X = _x(n, d_in, bits + group_size)
    W = torch.randn(d_out, d_in, generator=torch.Generator().manual_seed(3)) * 0.05
    ref = O.rtn_quantize(W.numpy(), group_size, sym, bits)
    Wh = O.dequantize_packed(ref["qpacked"], ref["scales"], ref["zeros"], d_in, group_size, sym,
                             bits=bits)
    q = dict(qpacked=torch.from_numpy(ref["qpacked"].view(np.int32)).cuda(),
             scales=torch.from_numpy(ref["scales"]).cuda(),
             zeros=None if sym else torch.from_numpy(ref["zeros"]).cuda(), bits=bits)
    Xn = X.float().numpy()
    R = None
    if act == "none":                       # with a residual of the output's width
        R = _x(n, d_out, 77)
    Z = gq.qlinear_bf16(X.cuda(), d_out, q=q, group_size=group_size, sym=sym, act=act,
                        R=None if R is None else R.cuda())
    Zref = O.apply_layer(Xn, Wh, act, None if R is None else R.float().numpy())
    _bf16_close(Z.float().cpu().numpy(), Zref, Xn, Wh)


@pytest.mark.parametrize("dt", [torch.float32, torch.float16, torch.bfloat16])
def test_qlinear_dense_weights(dt):
    """Without codes the same kernel applies the full-precision layer."""
    n, d_in, d_out = 300, 200, 136          # ragged tiles in every direction
    X = _x(n, d_in, 5)
    W = (torch.randn(d_out, d_in, generator=torch.Generator().manual_seed(4)) * 0.05).to(dt)
    Z = gq.qlinear_bf16(X.cuda(), d_out, W=W.cuda(), act="gelu")
    Wn, Xn = W.float().numpy(), X.float().numpy()
    _bf16_close(Z.float().cpu().numpy(), O.apply_layer(Xn, Wn, "gelu"), Xn, Wn)


def test_qlinear_act_order_groups():
    """Group indices of an act-ordered layer are honoured per column."""
    rng = np.random.default_rng(6)
    n, d_in, d_out = 512, 256, 96
    X = _x(n, d_in, 6)
    Xn = X.float().numpy()
    W = rng.standard_normal((d_out, d_in)) * 0.02
    res, *_ = O.gptq_layer(W, Xn, group_size=64, sym=False, act_order=True)
    q = dict(qpacked=torch.from_numpy(res.qpacked.view(np.int32)).cuda(),
             scales=torch.from_numpy(res.scales).cuda(), zeros=torch.from_numpy(res.zeros).cuda(),
             g_idx=torch.from_numpy(res.g_idx).cuda(), bits=4)
    Z = gq.qlinear_bf16(X.cuda(), d_out, q=q, group_size=64, sym=False)
    _bf16_close(Z.float().cpu().numpy(), O.apply_layer(Xn, res.W_hat), Xn, res.W_hat)


def _chain(seed, d=256, n=2048):
    rng = np.random.default_rng(seed)
    shapes = [(512, d, "gelu", None), (d, 512, "none", 0), (384, d, "relu", None),
              (d, 384, "none", 2)]
    layers = []
    for d_out, d_in, act, r in shapes:
        W = (rng.standard_normal((d_out, d_in)) * (0.5 / np.sqrt(d_in))).astype(np.float32)
        layers.append(dict(W=W, act=act, residual_from=r))
    X0 = _x(n, d, seed)
    return X0, layers


def _u_err(x: torch.Tensor) -> float:
    """Relative Frobenius error of the GPU's U (from its H of the bf16 input
    x) against the oracle's U of the same input."""
    U, _, _, _ = gq.damp_cholesky_inverse(gq.hessian(x.contiguous()), 0.01)
    Hd, _ = O.damp_hessian(O.hessian(x.float().cpu().numpy()), 0.01)
    return rel_fro(U.cpu().numpy(), O.upper_factor_of_inverse(Hd))


@pytest.mark.parametrize("bits,group_size,sym", [(4, 128, True), (4, -1, False), (8, 64, True)])
def test_sequential_pipeline_matches_oracle(bits, group_size, sym):
    """The whole chain against the oracle's: each layer's codes to the GPTQ
    bar, its error to 1e-3, and every intermediate input bit for bit, with
    the oracle replaying the GPU's choices at rounding ties of codes and of
    the bf16 activations only (at a tie both roundings are correct; the
    replay keeps the two chains on the same inputs)."""
    X0, layers = _chain(10 + bits)
    glayers = [dict(W=torch.from_numpy(L["W"]).cuda(), act=L["act"],
                    residual_from=L["residual_from"]) for L in layers]
    outs, sse, xs_gpu = gq.gptq_sequential(X0.cuda(), glayers, bits=bits, group_size=group_size,
                                           sym=sym)
    torch.cuda.synchronize()
    X0n = X0.float().numpy()
    follow = []
    for o, L in zip(outs, layers):
        d_in = L["W"].shape[1]
        follow.append(dict(codes=O.unpack_nibbles(u32(o["qpacked"]), d_in, sym, bits),
                           scales=f16(o["scales"]),
                           zeros=None if sym else f16(o["zeros"])))
    fx = [x.float().cpu().numpy() for x in xs_gpu[1:]]
    # each layer's GPTQ decisions are taken with the GPU's fp32 U of its own
    # input: its measured error widens the tie windows (as end to end in
    # test_configs_gpu)
    tie_rel = [max(O.TIE_REL, _u_err(x)) for x in xs_gpu[:-1]]
    # the GPU multiplies with W^ held as a bf16 pair (16 significant bits):
    # exact for symmetric codes of <= 5 bits (an fp16 scale times a small
    # integer), within 2^-16 relative per weight otherwise (8-bit codes, an
    # fp16 zero-point), which widens the activations' window by 2^-16 |X||W^|
    x_tie = O.TIE_REL + (0.0 if sym and bits <= 5 else 2.0 ** -16)
    res, sse_ref, xs = O.gptq_sequential(X0n, layers, bits=bits, group_size=group_size, sym=sym,
                                         follow=follow, follow_x=fx, tie_rel=tie_rel,
                                         x_tie_rel=x_tie)
    for li, (o, L) in enumerate(zip(outs, layers)):
        d_in = L["W"].shape[1]
        got = follow[li]["codes"]
        agree = np.mean(got == res[li].codes)
        diff = np.argwhere(got != res[li].codes)
        print(f"[pipeline {bits}-bit layer {li}] codes agree {agree:.6f} ({len(diff)} differ, "
              f"rows {sorted(set(diff[:, 0].tolist()))[:8]}), ties followed "
              f"{res[li].n_followed}, expected {res[li].expected_ties:.1f}, tie_rel "
              f"{tie_rel[li]:.2e}, X equal {np.mean(fx[li] == xs[li + 1]):.6f}")
        assert agree >= 0.999 and np.max(np.abs(got - res[li].codes)) <= 1, (li, agree)
        assert abs(sse[li] - sse_ref[li]) <= 1e-3 * sse_ref[li], (li, sse[li], sse_ref[li])
        assert np.array_equal(fx[li], xs[li + 1]), (li, np.mean(fx[li] == xs[li + 1]))


def test_sequential_errors_compound():
    """Calibrating on the quantised upstream output is what the pipeline
    does: its later layers' inputs differ from the full-precision chain's,
    and its per-layer errors are measured on those inputs (the oracle's
    full-precision-input run is the comparison)."""
    X0, layers = _chain(3)
    glayers = [dict(W=torch.from_numpy(L["W"]).cuda(), act=L["act"],
                    residual_from=L["residual_from"]) for L in layers]
    outs, sse, xs_gpu = gq.gptq_sequential(X0.cuda(), glayers, bits=4, group_size=128, sym=True)
    _, sse_fp, xs_fp = O.gptq_sequential(X0.float().numpy(), layers, group_size=128, sym=True,
                                         quantized_inputs=False)
    assert abs(sse[0] - sse_fp[0]) <= 1e-3 * sse_fp[0]          # same first input
    assert not np.allclose(xs_gpu[-1].float().cpu().numpy(), xs_fp[-1])
    print("[pipeline] per-layer SSE, quantised inputs:", np.round(sse, 4).tolist(),
          "full-precision inputs:", np.round(sse_fp, 4).tolist())
