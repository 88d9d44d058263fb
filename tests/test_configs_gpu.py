"""Every layer shape of the five workloads, at full width, against the oracle.

For each shape the GPU runs the whole per-layer path (Hessian, damping and
act-order, U, GPTQ, RTN, reconstruction error) and the oracle recomputes it
from the same seeded inputs:

* H: the oracle's fp64 H = 2 X^T X over the calibration tokens, compared in
  full (relative Frobenius <= 1e-5).  For the widest layers the oracle's
  fp64 Hessian over all 262144 tokens would take the host tens of minutes,
  so these cases calibrate on fewer tokens (still more tokens than input
  channels, so H keeps full rank); the Hessian kernel itself is compared at
  262144 tokens on sampled tiles in test_hessian_gpu.py.
* act-order: the oracle's stable descending sort of the damped diagonal;
  where two keys tie at fp32 precision (relative 1e-6) either order is
  correct and the oracle follows the GPU's (``act_order_perm(follow=...)``).
* U: the oracle's factor (Cholesky, inverse, Cholesky of the inverse) against
  the GPU's, relative Frobenius <= 1e-3 (fp32 against fp64 on a damped H
  whose condition number reaches ~1e5).
* GPTQ, two ways, on sampled rows (rows are independent given U):
  - the GPTQ stage alone: the GPU column loop and trailing updates given the
    oracle's U (rounded to fp32) against the oracle's GPTQ with its fp64 U;
  - end to end: the GPU's codes from its own H and U against the oracle's.
  Both to the bar of test_gptq_gpu.check_gptq (>= 99.9% identical codes,
  mismatches one level, rounding ties replayed inside the windows of
  reading 11; end to end the windows also cover the GPU's fp32 U, whose
  measured relative error widens them).
* RTN of the whole layer bit for bit (codes, scales, zeros, packed words).
* reconstruction error: the GPU's, over all 262144 tokens, of the oracle's
  GPTQ rows against the oracle's fp64 ||(W - W^) X^T||^2 (relative 1e-3);
  and where the oracle's trace route is cheap, the whole layer's RTN error
  at the calibration tokens against tr(dW H0 dW^T) / 2.
"""
import time

import numpy as np
import pytest
import torch

import oracle as O
from post_weight_quantization_27_b200 import gq, inputs as I
from tests.gpu_util import f16, rel_fro, u32
from tests.test_gptq_gpu import check_gptq

pytestmark = pytest.mark.gpu

# (workload, layer, calibration tokens for the oracle path (None = the
# workload's own), sampled GPTQ rows)
CASES = [
    (2, 0, None, 256), (2, 1, None, 256), (2, 2, None, 256), (2, 3, None, 256),
    (2, 48, None, 512),
    (3, 0, None, 128), (3, 1, None, 128), (3, 2, None, 128), (3, 3, 65536, 128),
    (4, 0, None, 128), (4, 4, None, 128), (4, 6, 32768, 96),
    (5, 0, 65536, 64), (5, 1, 65536, 128),
    pytest.param(5, 2, 32768, 48, marks=pytest.mark.slow),
]


def _oracle_hessian(X: torch.Tensor) -> np.ndarray:
    """Oracle H = 2 X^T X of a device bf16 X, summed over token chunks."""
    d = X.shape[1]
    H = np.zeros((d, d))
    step = max(1, (1 << 31) // (8 * d))
    for r0 in range(0, X.shape[0], step):
        H += O.hessian(X[r0:r0 + step].float().cpu().numpy())
    return H


def _oracle_sse(W: np.ndarray, W_hat: np.ndarray, X: torch.Tensor) -> float:
    """Oracle ||(W - W^) X^T||^2 over all tokens of a device X, in chunks."""
    step = max(1, (1 << 30) // (8 * X.shape[1]))
    return sum(O.recon_sse(W, W_hat, X[r0:r0 + step].float().cpu().numpy())
               for r0 in range(0, X.shape[0], step))


def _rows(q, rows):
    return dict(qpacked=q["qpacked"][rows], scales=q["scales"][rows],
                zeros=None if q["zeros"] is None else q["zeros"][rows])


def _as_device(res, act_order):
    return dict(qpacked=torch.from_numpy(res.qpacked.view(np.int32)).cuda(),
                scales=torch.from_numpy(res.scales).cuda(),
                zeros=torch.from_numpy(res.zeros).cuda(),
                g_idx=torch.from_numpy(res.g_idx).cuda() if act_order else None)


@pytest.mark.parametrize("workload,idx,n_cal,n_rows", CASES)
def test_config_layer(workload, idx, n_cal, n_rows):
    t_start = time.time()
    spec = I.workload_layers(workload)[idx]
    sp = spec.with_tokens(n_cal) if n_cal is not None else spec
    W = I.make_weights(spec).cuda()
    X = I.make_x_device(spec, "cuda") if spec.n_tok > 8192 else I.make_x(spec).cuda()
    Xc = X[:sp.n_tok]
    g, sym, B = spec.group_size, spec.sym, spec.block_size

    # ---------------- GPU: the whole path on the calibration tokens
    H = gq.hessian(Xc)
    Hg = H.cpu().numpy()
    U, perm, dead, info = gq.damp_cholesky_inverse(H, spec.damp, act_order=spec.act_order)
    q = gq.gptq_quantize_layer(W, U, 4, g, B, sym, perm=perm, dead=dead)
    rtn = gq.rtn_quantize_pack(W, 4, g, sym)
    torch.cuda.synchronize()

    # ---------------- oracle: H, damping, act-order, U
    H0 = _oracle_hessian(Xc)
    assert rel_fro(Hg, H0) <= 1e-5
    del Hg
    Hd, dead_o = O.damp_hessian(H0, spec.damp)
    assert np.array_equal(dead.cpu().numpy().astype(bool), dead_o)
    perm_o = None
    if spec.act_order:
        perm_o, _ = O.act_order_perm(Hd, follow=perm.cpu().numpy())
        assert np.array_equal(perm.cpu().numpy(), perm_o)
        Hd = Hd[np.ix_(perm_o, perm_o)]
    Uo = O.upper_factor_of_inverse(Hd)
    del Hd
    u_err = rel_fro(U.cpu().numpy(), Uo)
    assert u_err <= 1e-3

    rng = np.random.default_rng(1000 * workload + idx)
    rows = np.sort(rng.choice(spec.d_out, size=min(n_rows, spec.d_out), replace=False))
    rows_t = torch.from_numpy(rows).cuda()
    Wn = W[rows_t].float().cpu().numpy()

    def oracle_gptq(follow, tie_rel=O.TIE_REL):
        return O.gptq_quantize(Wn, Uo, group_size=g, block_size=B, sym=sym, perm=perm_o,
                               dead=dead_o, follow=follow, tie_rel=tie_rel)

    # ---------------- GPTQ stage alone: the oracle's U on both sides
    U32 = torch.from_numpy(Uo.astype(np.float32)).cuda()
    perm_t = None if perm_o is None else torch.from_numpy(perm_o.astype(np.int32)).cuda()
    dead_t = torch.from_numpy(dead_o.astype(np.uint8)).cuda()
    q_stage = gq.gptq_quantize_layer(W[rows_t].contiguous(), U32, 4, g, B, sym, perm=perm_t,
                                     dead=dead_t)
    torch.cuda.synchronize()
    check_gptq(q_stage, oracle_gptq, spec.d_in, sym)
    del U32

    # ---------------- end to end: the GPU's own H and U (its fp32 U's measured
    # error widens the tie windows, reading 11)
    check_gptq(_rows(q, rows_t), lambda f: oracle_gptq(f, max(O.TIE_REL, u_err)), spec.d_in, sym)
    if spec.act_order:
        assert np.array_equal(q["g_idx"].cpu().numpy(),
                              (np.argsort(perm_o) // g).astype(np.int32))

    # ---------------- RTN, whole layer, bit for bit
    ref = O.rtn_quantize(W.float().cpu().numpy(), g, sym)
    assert np.array_equal(u32(rtn["qpacked"]), ref["qpacked"])
    assert np.array_equal(f16(rtn["scales"]).view(np.uint16), ref["scales"].view(np.uint16))
    if not sym:
        assert np.array_equal(f16(rtn["zeros"]).view(np.uint16), ref["zeros"].view(np.uint16))

    # ---------------- reconstruction error of the oracle's GPTQ rows, all tokens
    res = oracle_gptq(None)
    sse_ref = _oracle_sse(Wn, res.W_hat, X)
    sse, _ = gq.recon_error(W[rows_t].contiguous(), _as_device(res, spec.act_order), X, g, sym)
    assert abs(sse - sse_ref) <= 1e-3 * sse_ref, (sse, sse_ref)

    # ---------------- whole-layer RTN error by the trace route (cheap cases)
    if spec.d_out * spec.d_in ** 2 <= 4e12:
        Wf = W.float().cpu().numpy()
        Wr = O.dequantize_packed(ref["qpacked"], ref["scales"], ref["zeros"], spec.d_in, g, sym)
        sse_tr = O.recon_sse_trace(Wf, Wr, H0)
        sse_g, _ = gq.recon_error(W, rtn, Xc, g, sym)
        assert abs(sse_g - sse_tr) <= 1e-3 * sse_tr, (sse_g, sse_tr)
        # and the GPU's own Hessian route on the GPU's H of the same tokens
        sse_h, _ = gq.recon_error_hessian(W, rtn, gq.hessian(Xc), Xc.shape[0], g, sym)
        assert abs(sse_h - sse_tr) <= 1e-3 * sse_tr, (sse_h, sse_tr)
    print(f"[config {workload}.{idx} {spec.d_in}->{spec.d_out}] {time.time() - t_start:.1f} s")
    del X, Xc, H, U, q, rtn
    torch.cuda.empty_cache()
