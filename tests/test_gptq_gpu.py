"""GPTQ on the GPU against the oracle: at least 99.9% of the int codes
identical and every mismatch exactly one level.

GPTQ feeds every rounding decision forward along the row, so a decision
that is a rounding tie at the GPU's precision (the oracle's w/s within the
decision's tie window of k + 1/2: max(1e-6, 2^-18 E / s) steps with E the
accumulated magnitude of the updates the weight received, or its scale
that close to an fp16 rounding boundary) can legitimately go either way in
fp32 and fp64, after which the row follows a different valid trajectory.
Each check therefore runs the oracle twice: plain (the raw agreement is
reported) and replaying the GPU's choices at such ties only, against which
every code must agree to 99.9%, no mismatch may exceed one level, and the
number of adopted ties must be what the windows predict."""
import numpy as np
import pytest
import torch

import oracle as O
from post_weight_quantization_27_b200 import gq, inputs as I
from tests.gpu_util import f16, rel_fro, u32

pytestmark = pytest.mark.gpu
DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def _codes(out, d_in, sym, bits=4):
    return O.unpack_nibbles(u32(out["qpacked"]), d_in, sym, bits)


def code_agreement(got, ref):
    diff = np.abs(got.astype(np.int64) - ref.astype(np.int64))
    return float(np.mean(diff == 0)), int(diff.max(initial=0))


def check_gptq(out, oracle_run, d_in, sym, min_agree=0.999, bits=4):
    """oracle_run(follow) -> GptqResult.  Asserts the parity bar (module
    docstring) on the oracle run that replays the GPU's choices at rounding
    ties, and that the number of adopted ties is what the tie windows
    predict (a Poisson count: at most 3x its mean + 4).  Returns (raw
    agreement, replayed agreement, ties)."""
    got = _codes(out, d_in, sym, bits)
    raw = oracle_run(None)
    raw_agree, raw_max = code_agreement(got, raw.codes)
    follow = dict(codes=got, scales=f16(out["scales"]),
                  zeros=None if sym else f16(out["zeros"]))
    rep = oracle_run(follow)
    agree, maxdiff = code_agreement(got, rep.codes)
    print(f"[gptq parity] raw {raw_agree:.6f} replayed {agree:.6f} followed {rep.n_followed} "
          f"(expected {rep.expected_ties:.2f}) max tie distance {rep.max_follow_dist:.3g}")
    assert agree >= min_agree and maxdiff <= 1, (raw_agree, agree, maxdiff, rep.n_followed)
    assert rep.n_followed <= 3.0 * rep.expected_ties + 4, (rep.n_followed, rep.expected_ties)
    return raw_agree, agree, rep.n_followed


def _layer(d_out, d_in, n_tok, seed, dtype="f32", outlier="cols:0.02:8"):
    spec = I.LayerSpec(0, seed, "g", d_in, d_out, dtype, 0.02, outlier, n_tok, min(4, d_in),
                       20.0, -1, True, False)
    return I.make_weights(spec), I.make_x(spec)


def e2e_tie_rel(U_gpu, X, damp=0.01, perm=None):
    """Scale of the tie windows for an end-to-end comparison.  There the GPU
    runs GPTQ with its own fp32 U, whose relative error against the
    oracle's fp64 U perturbs every update term as the column loop's own
    rounding does: the window scale is the larger of TIE_REL and that
    measured error (relative Frobenius)."""
    Hd, _ = O.damp_hessian(O.hessian(X), damp)
    if perm is not None:
        Hd = Hd[np.ix_(perm, perm)]
    Uo = O.upper_factor_of_inverse(Hd)
    return max(O.TIE_REL, rel_fro(U_gpu.cpu().numpy(), Uo))


def _run_gpu(W, X, group_size, sym, act_order=False, block_size=128, damp=0.01, bits=4):
    """The whole GPU path; returns (quantised layer, perm, end-to-end tie
    window scale)."""
    Wd, Xd = W.cuda(), X.cuda()
    H = gq.hessian(Xd)
    U, perm, dead, info = gq.damp_cholesky_inverse(H, damp, act_order=act_order)
    out = gq.gptq_quantize_layer(Wd, U, bits, group_size, block_size, sym, perm=perm, dead=dead)
    torch.cuda.synchronize()
    p = None if perm is None else perm.cpu().numpy()
    if p is not None:   # the order the oracle takes (reading 15)
        p, _ = O.act_order_perm(O.damp_hessian(O.hessian(X.float().numpy()), damp)[0], follow=p)
    return out, perm, e2e_tie_rel(U, X.float().numpy(), damp, p)


@pytest.mark.parametrize("d_out,d_in,n_tok,group_size,sym,dt", [
    (96, 256, 512, -1, True, "f32"),
    (7, 136, 300, -1, False, "f16"),
    (130, 768, 2048, 128, True, "bf16"),
    (64, 384, 1000, 128, False, "f32"),
    (33, 200, 800, -1, True, "f32"),          # ragged last block (72 columns)
    (50, 512, 1500, 64, True, "f16"),
    (40, 512, 1500, 32, False, "f32"),
    (96, 256, 512, 0, True, "f32"),           # per-tensor scale
    (64, 384, 1000, 0, False, "bf16"),
])
def test_gptq_end_to_end(d_out, d_in, n_tok, group_size, sym, dt):
    W, X = _layer(d_out, d_in, n_tok, d_out + d_in, dt)
    out, _, tr = _run_gpu(W, X, group_size, sym)
    Wn, Xn = W.float().numpy(), X.float().numpy()
    check_gptq(out, lambda f: O.gptq_layer(Wn, Xn, group_size=group_size, sym=sym,
                                           follow=f, tie_rel=tr)[0], d_in, sym)


@pytest.mark.parametrize("block_size,group_size", [(64, -1), (64, 64), (32, 32), (128, 32)])
def test_gptq_block_sizes(block_size, group_size):
    W, X = _layer(80, 320, 900, block_size + group_size)
    out, _, tr = _run_gpu(W, X, group_size, True, block_size=block_size)
    Wn, Xn = W.numpy(), X.float().numpy()
    check_gptq(out, lambda f: O.gptq_layer(Wn, Xn, group_size=group_size,
                                           block_size=block_size, follow=f, tie_rel=tr)[0],
               320, True)


def test_gptq_with_oracle_u_is_near_exact():
    """Given the oracle's own U (rounded to fp32), the GPU column loop and
    trailing updates reproduce the oracle's codes."""
    W, X = _layer(256, 512, 2000, 5)
    H0 = O.hessian(X.float().numpy())
    Hd, dead = O.damp_hessian(H0, 0.01)
    U = O.upper_factor_of_inverse(Hd)
    Wn = W.numpy()
    for gs, sym in ((-1, True), (128, False)):
        out = gq.gptq_quantize_layer(W.cuda(), torch.from_numpy(U.astype(np.float32)).cuda(), 4,
                                     gs, 128, sym)
        raw, agree, ties = check_gptq(
            out, lambda f: O.gptq_quantize(Wn, U, group_size=gs, sym=sym, follow=f), 512, sym,
            min_agree=0.9995)
        # the scales (and zeros) too, against the replayed run: the fp16
        # scale is an integer decision like a code
        got = dict(codes=O.unpack_nibbles(u32(out["qpacked"]), 512, sym),
                   scales=f16(out["scales"]), zeros=None if sym else f16(out["zeros"]))
        ref = O.gptq_quantize(Wn, U, group_size=gs, sym=sym, follow=got)
        s = f16(out["scales"]).view(np.uint16)
        assert np.mean(s == ref.scales.view(np.uint16)) >= 0.999
        if not sym:
            z = f16(out["zeros"]).view(np.uint16)
            assert np.mean(z == ref.zeros.view(np.uint16)) >= 0.999


def test_gptq_act_order_affine():
    W, X = _layer(64, 384, 1200, 11, "bf16", "cols:0.02:10")
    out, perm, tr = _run_gpu(W, X, 128, False, act_order=True)
    Wn, Xn = W.float().numpy(), X.float().numpy()
    Hd, dead = O.damp_hessian(O.hessian(Xn), 0.01)
    pref, _ = O.act_order_perm(Hd, follow=perm.cpu().numpy())     # reading 15
    assert np.array_equal(perm.cpu().numpy(), pref)
    Uo = O.upper_factor_of_inverse(Hd[np.ix_(pref, pref)])
    ref = O.gptq_quantize(Wn, Uo, group_size=128, sym=False, perm=pref, dead=dead)
    assert np.array_equal(out["g_idx"].cpu().numpy(), ref.g_idx)
    check_gptq(out, lambda f: O.gptq_quantize(Wn, Uo, group_size=128, sym=False, perm=pref,
                                              dead=dead, follow=f, tie_rel=tr), 384, False)


def test_gptq_dead_columns():
    W, X = _layer(32, 256, 600, 12)
    X[:, [3, 77]] = 0
    out, _, tr = _run_gpu(W, X, -1, True)
    codes = _codes(out, 256, True)
    assert np.all(codes[:, [3, 77]] == 0)
    Wn, Xn = W.numpy(), X.float().numpy()
    check_gptq(out, lambda f: O.gptq_layer(Wn, Xn, group_size=-1, follow=f, tie_rel=tr)[0],
               256, True)


def test_gptq_diagonal_hessian_is_rtn():
    """Orthogonal inputs: GPTQ must equal RTN bit for bit."""
    d_in = 256
    X = torch.zeros((d_in, d_in), dtype=torch.bfloat16)
    X[torch.arange(d_in), torch.arange(d_in)] = torch.linspace(0.5, 3.0, d_in).to(torch.bfloat16)
    W, _ = _layer(48, d_in, 10, 13)
    for gs, sym in ((-1, True), (128, False), (32, True), (0, True), (0, False)):
        out, _, _ = _run_gpu(W, X, gs, sym)
        rtn = gq.rtn_quantize_pack(W.cuda(), 4, gs, sym)
        torch.cuda.synchronize()
        assert np.array_equal(u32(out["qpacked"]), u32(rtn["qpacked"]))
        assert torch.equal(out["scales"], rtn["scales"])


@pytest.mark.parametrize("workload,idx", [(1, 0), (2, 1), (2, 3)])
def test_gptq_workload_layers(workload, idx):
    spec = I.workload_layers(workload)[idx]
    W, X = I.make_weights(spec), I.make_x(spec)
    out, _, tr = _run_gpu(W, X, spec.group_size, spec.sym)
    Wn, Xn = W.float().numpy(), X.float().numpy()
    check_gptq(out, lambda f: O.gptq_layer(Wn, Xn, group_size=spec.group_size, sym=spec.sym,
                                           follow=f, tie_rel=tr)[0], spec.d_in, spec.sym)


def test_gptq_division_matches_ieee_at_midpoints():
    """The column loop divides by a reciprocal plus one FMA correction; with
    a diagonal Hessian GPTQ must still reproduce RTN (IEEE division) bit for
    bit, on weights packed with exact rounding midpoints k + 1/2 of the
    row's step and their fp32 neighbours."""
    d_in, d_out = 512, 2048
    g = torch.Generator().manual_seed(31)
    W = torch.randn((d_out, d_in), generator=g) * 0.02
    amax = W.abs().amax(1, keepdim=True)
    s16 = (amax / 7).to(torch.float16).float()
    k = torch.randint(-7, 7, (d_out, d_in), generator=g).float()
    mid = (k + 0.5) * s16
    pick = torch.randint(0, 4, (d_out, d_in), generator=g)
    W = torch.where(pick == 0, mid, W)
    W = torch.where(pick == 1, torch.nextafter(mid, torch.full_like(mid, 1e9)), W)
    W = torch.where(pick == 2, torch.nextafter(mid, torch.full_like(mid, -1e9)), W)
    W = torch.clamp(W, -amax, amax)
    X = torch.zeros((d_in, d_in), dtype=torch.bfloat16)
    X[torch.arange(d_in), torch.arange(d_in)] = torch.linspace(0.5, 2.0, d_in).to(torch.bfloat16)
    for gs, sym in ((-1, True), (128, True), (64, False)):
        out, _, _ = _run_gpu(W, X, gs, sym)
        rtn = gq.rtn_quantize_pack(W.cuda(), 4, gs, sym)
        torch.cuda.synchronize()
        assert np.array_equal(u32(out["qpacked"]), u32(rtn["qpacked"])), (gs, sym)
