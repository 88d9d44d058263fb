"""Damping, dead columns, act-order and the upper factor U (H^-1 = U^T U)
on the GPU against the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from post_weight_quantization_27_b200 import gq, inputs as I
from tests.gpu_util import rel_fro

pytestmark = pytest.mark.gpu


def _H(n_tok, d, seed, dead=()):
    spec = I.LayerSpec(0, seed, "c", d, 8, "f32", 0.02, "none", n_tok, min(4, d), 20.0, -1,
                       True, False)
    X = I.make_x(spec).float().numpy()
    X[:, list(dead)] = 0.0
    return O.hessian(X).astype(np.float32)


# (the last case's trailing updates are large enough to run on CTA pairs)
@pytest.mark.parametrize("n_tok,d", [(64, 8), (300, 136), (2048, 768), (1500, 1032), (4000, 3072),
                                     (8192, 6144)])
def test_upper_factor_matches_oracle(n_tok, d):
    H32 = _H(n_tok, d, d)
    U, perm, dead, info = gq.damp_cholesky_inverse(torch.from_numpy(H32).cuda(), 0.01)
    Ug = U.cpu().numpy()
    Hd, dref = O.damp_hessian(H32.astype(np.float64), 0.01)
    Uref = O.upper_factor_of_inverse(Hd)
    assert int(info.item()) == -1
    assert np.all(np.tril(Ug, -1) == 0)
    assert rel_fro(Ug, Uref) < 2e-4
    # property: U^T U H = I
    R = Ug.astype(np.float64).T @ Ug.astype(np.float64) @ Hd - np.eye(d)
    assert np.linalg.norm(R) / np.sqrt(d) < 2e-3
    assert np.array_equal(dead.cpu().numpy().astype(bool), dref)


def test_dead_columns_and_act_order():
    d = 264
    H32 = _H(900, d, 3, dead=(5, 100, 263))
    U, perm, dead, info = gq.damp_cholesky_inverse(torch.from_numpy(H32).cuda(), 0.01,
                                                   act_order=True)
    Hd, dref = O.damp_hessian(H32.astype(np.float64), 0.01)
    assert np.array_equal(dead.cpu().numpy().astype(bool), dref)
    pref = O.act_order_perm(Hd)
    pg = perm.cpu().numpy()
    keys = np.diag(Hd)
    # identical except possibly among keys equal to fp32 rounding
    mism = np.nonzero(pg != pref)[0]
    for i in mism:
        assert abs(keys[pg[i]] - keys[pref[i]]) <= 1e-6 * abs(keys[pref[i]])
    Uref = O.upper_factor_of_inverse(Hd[np.ix_(pref, pref)])
    if len(mism) == 0:
        assert rel_fro(U.cpu().numpy(), Uref) < 2e-4


def test_not_positive_definite_reported():
    d = 64
    H = -torch.eye(d, device="cuda")
    with pytest.raises(gq.GQError) as e:
        gq.damp_cholesky_inverse(H, 0.01)
    assert e.value.name == "GQ_ERR_NOT_PD"
    # an indefinite entry at a known column: the reported column is that one
    H = torch.eye(d, device="cuda")
    H[40, 40] = -5.0
    U, perm, dead, info = gq.damp_cholesky_inverse(H, 0.0, check=False)
    assert int(info.item()) == 40
