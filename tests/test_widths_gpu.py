"""Code widths other than 4 bits (2, 3 and 8: "GPT-2 Quantization
Reconstruction Error", "Possible extensions", 4-bit against 8-bit; INT8 and
INT4 in "Quantization sweep: perplexity vs compression") through every
kernel that reads or writes codes, against the oracle: RTN bit for bit,
GPTQ to the parity bar of test_gptq_gpu, GPTQ == RTN on a diagonal Hessian
bit for bit, both reconstruction-error routes and the dequantising product
to their tolerances."""
import numpy as np
import pytest
import torch

import oracle as O
from post_weight_quantization_27_b200 import gq, inputs as I
from tests.gpu_util import f16, u32
from tests.test_gptq_gpu import check_gptq, e2e_tie_rel

pytestmark = pytest.mark.gpu
DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def _layer(d_out, d_in, n_tok, seed, dtype="f32"):
    spec = I.LayerSpec(0, seed, "w", d_in, d_out, dtype, 0.02, "cols:0.02:8", n_tok,
                       min(4, d_in), 20.0, -1, True, False)
    return I.make_weights(spec), I.make_x(spec)


@pytest.mark.parametrize("bits", [2, 3, 8])
@pytest.mark.parametrize("group_size", [-1, 0, 32, 128])
@pytest.mark.parametrize("sym", [True, False])
@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_rtn_widths_bit_exact(bits, group_size, sym, dt):
    W, _ = _layer(67, 256, 8, bits * 100 + group_size + 7 * sym, dt)
    out = gq.rtn_quantize_pack(W.cuda(), bits, group_size, sym)
    torch.cuda.synchronize()
    ref = O.rtn_quantize(W.float().numpy(), group_size, sym, bits)
    assert out["qpacked"].shape[1] == bits * 256 // 32
    assert np.array_equal(u32(out["qpacked"]), ref["qpacked"])
    assert np.array_equal(f16(out["scales"]).view(np.uint16), ref["scales"].view(np.uint16))
    if not sym:
        assert np.array_equal(f16(out["zeros"]).view(np.uint16), ref["zeros"].view(np.uint16))


@pytest.mark.parametrize("bits", [2, 3, 8])
def test_rtn_widths_wide_rows(bits):
    """Per-channel rows wider than the lanes of one warp pass (several
    32-column chunks per lane) and a single-row matrix."""
    W, _ = _layer(40, 4096, 8, 5 + bits, "f16")
    for Wx in (W, W[:1].contiguous()):
        out = gq.rtn_quantize_pack(Wx.cuda(), bits, -1, True)
        ref = O.rtn_quantize(Wx.float().numpy(), -1, True, bits)
        assert np.array_equal(u32(out["qpacked"]), ref["qpacked"])


@pytest.mark.parametrize("bits", [2, 3, 8])
@pytest.mark.parametrize("group_size,sym", [(-1, True), (128, False), (64, True), (32, False),
                                            (0, True)])
def test_gptq_widths(bits, group_size, sym):
    W, X = _layer(96, 384, 1500, 17 * bits + group_size, "f16")
    Wd, Xd = W.cuda(), X.cuda()
    H = gq.hessian(Xd)
    U, perm, dead, info = gq.damp_cholesky_inverse(H, 0.01)
    out = gq.gptq_quantize_layer(Wd, U, bits, group_size, 128, sym, dead=dead)
    torch.cuda.synchronize()
    Wn, Xn = W.float().numpy(), X.float().numpy()
    tr = e2e_tie_rel(U, Xn)
    check_gptq(out, lambda f: O.gptq_layer(Wn, Xn, bits=bits, group_size=group_size, sym=sym,
                                           follow=f, tie_rel=tr)[0], 384, sym, bits=bits)


@pytest.mark.parametrize("bits", [3, 8])
def test_gptq_widths_act_order(bits):
    W, X = _layer(64, 256, 1200, 40 + bits, "bf16")
    Wd, Xd = W.cuda(), X.cuda()
    U, perm, dead, info = gq.damp_cholesky_inverse(gq.hessian(Xd), 0.01, act_order=True)
    out = gq.gptq_quantize_layer(Wd, U, bits, 128, 128, False, perm=perm, dead=dead)
    torch.cuda.synchronize()
    Wn, Xn = W.float().numpy(), X.float().numpy()
    Hd, dead_o = O.damp_hessian(O.hessian(Xn), 0.01)
    pref, _ = O.act_order_perm(Hd, follow=perm.cpu().numpy())
    assert np.array_equal(perm.cpu().numpy(), pref)
    Uo = O.upper_factor_of_inverse(Hd[np.ix_(pref, pref)])
    tr = e2e_tie_rel(U, Xn, perm=pref)
    check_gptq(out, lambda f: O.gptq_quantize(Wn, Uo, bits=bits, group_size=128, sym=False,
                                              perm=pref, dead=dead_o, follow=f, tie_rel=tr),
               256, False, bits=bits)


@pytest.mark.parametrize("bits", [2, 3, 8])
def test_gptq_widths_diagonal_hessian_is_rtn(bits):
    """Orthogonal inputs: GPTQ equals RTN bit for bit at every width."""
    d_in = 256
    X = torch.zeros((d_in, d_in), dtype=torch.bfloat16)
    X[torch.arange(d_in), torch.arange(d_in)] = torch.linspace(0.5, 3.0, d_in).to(torch.bfloat16)
    W, _ = _layer(48, d_in, 10, 60 + bits)
    for gs, sym in ((-1, True), (128, False), (32, True), (0, False)):
        U, perm, dead, info = gq.damp_cholesky_inverse(gq.hessian(X.cuda()), 0.01)
        out = gq.gptq_quantize_layer(W.cuda(), U, bits, gs, 128, sym, dead=dead)
        rtn = gq.rtn_quantize_pack(W.cuda(), bits, gs, sym)
        torch.cuda.synchronize()
        assert np.array_equal(u32(out["qpacked"]), u32(rtn["qpacked"])), (gs, sym)
        assert torch.equal(out["scales"], rtn["scales"])


@pytest.mark.parametrize("bits", [2, 3, 8])
@pytest.mark.parametrize("group_size,sym", [(-1, True), (64, False)])
def test_recon_and_product_widths(bits, group_size, sym):
    """Both reconstruction-error routes (relative 1e-3) and the dequantising
    product (relative Frobenius 1e-5) read the packed codes of every width."""
    W, X = _layer(130, 512, 700, 70 + bits + group_size, "f16")
    Wn, Xn = W.float().numpy(), X.float().numpy()
    ref = O.rtn_quantize(Wn, group_size, sym, bits)
    Wh = O.dequantize_packed(ref["qpacked"], ref["scales"], ref["zeros"], 512, group_size, sym,
                             bits=bits)
    sse_ref = O.recon_sse(Wn, Wh, Xn)
    q = dict(qpacked=torch.from_numpy(ref["qpacked"].view(np.int32)).cuda(),
             scales=torch.from_numpy(ref["scales"]).cuda(),
             zeros=None if sym else torch.from_numpy(ref["zeros"]).cuda(), bits=bits)
    sse, _ = gq.recon_error(W.cuda(), q, X.cuda(), group_size, sym)
    assert abs(sse - sse_ref) <= 1e-3 * sse_ref
    H0 = gq.hessian(X.cuda())
    sse_h, _ = gq.recon_error_hessian(W.cuda(), q, H0, 700, group_size, sym)
    assert abs(sse_h - sse_ref) <= 1e-3 * sse_ref
    Y = gq.w4a16_matmul(q, 512, X[:696].cuda(), group_size, sym).cpu().numpy()
    Yref = O.w4a16_matmul(ref["qpacked"], ref["scales"], ref["zeros"], 512, group_size, sym,
                          Xn[:696], bits=bits)
    assert np.linalg.norm(Y - Yref) <= 1e-5 * np.linalg.norm(Yref)


def test_eight_bit_error_is_far_below_four_bit():
    """On the GPU as in the oracle: 8-bit RTN per channel has about
    (7/127)^2 of the 4-bit reconstruction error."""
    W, X = _layer(256, 1024, 2048, 99, "f32")
    sse = {}
    for bits in (4, 8):
        q = gq.rtn_quantize_pack(W.cuda(), bits, -1, True)
        sse[bits], _ = gq.recon_error(W.cuda(), q, X.cuda(), -1, True)
    assert 0.5 * (7 / 127) ** 2 < sse[8] / sse[4] < 2.0 * (7 / 127) ** 2
