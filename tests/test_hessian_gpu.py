"""H += 2 X^T X on the tensor cores against the fp64 oracle (relative
Frobenius error <= 1e-5 on the same bf16 X), exact symmetry, determinism
and additivity."""
import numpy as np
import pytest
import torch

import oracle as O
from post_weight_quantization_27_b200 import gq, inputs as I
from tests.gpu_util import rel_fro

pytestmark = pytest.mark.gpu
TOL = 1e-5


def _x(n_tok, d_in, seed):
    spec = I.LayerSpec(0, seed, "h", d_in, 8, "f32", 0.02, "none", n_tok, min(4, d_in), 20.0,
                       -1, True, False)
    return I.make_x(spec)


# ragged tiles in both directions (136, 264, 520, 1032, 1304); 20000 x 1304
# splits the tokens over few tiles; 70000 x 256 runs several waves
@pytest.mark.parametrize("n_tok,d_in", [(64, 8), (100, 136), (2048, 768), (1000, 264),
                                        (4097, 520), (2560, 3072), (300, 1032), (70000, 256),
                                        (20000, 1304)])
def test_hessian_matches_oracle(n_tok, d_in):
    X = _x(n_tok, d_in, n_tok + d_in)
    H = gq.hessian(X.cuda()).cpu().numpy()
    ref = O.hessian(X.float().numpy())
    assert rel_fro(H, ref) <= TOL
    assert np.array_equal(H, H.T)


def test_hessian_empty_and_additive():
    X = _x(513, 136, 5)
    Xd = X.cuda()
    H = torch.zeros((136, 136), dtype=torch.float32, device="cuda")
    gq.hessian_accumulate(Xd[:0], H)                   # n_tok = 0: nothing added
    assert torch.count_nonzero(H) == 0
    gq.hessian_accumulate(Xd[:200], H)
    gq.hessian_accumulate(Xd[200:], H)
    ref = O.hessian(X.float().numpy())
    assert rel_fro(H.cpu().numpy(), ref) <= TOL
    # the incoming upper triangle is what counts
    H2 = torch.zeros_like(H)
    H2.tril_(-1).add_(torch.tril(torch.ones_like(H), -1) * 5.0)
    gq.hessian_accumulate(Xd, H2)
    assert rel_fro(H2.cpu().numpy(), ref) <= TOL


def test_hessian_deterministic():
    X = _x(5000, 1032, 9).cuda()
    a = gq.hessian(X)
    b = gq.hessian(X)
    assert torch.equal(a, b)


@pytest.mark.parametrize("workload,idx", [(3, 3), (5, 2)])
def test_hessian_full_size_sampled(workload, idx):
    """262144 tokens at the workloads' widths; the oracle computes sampled
    256 x 256 tiles (one on the diagonal) and 512 diagonal entries."""
    spec = I.workload_layers(workload)[idx]
    X = I.make_x_device(spec, "cuda")
    H = gq.hessian(X)
    torch.cuda.synchronize()
    d = spec.d_in
    rng = np.random.default_rng(idx)
    got, ref = [], []
    tiles = [(0, 0), (int(rng.integers(0, d // 256)) * 256, int(rng.integers(0, d // 256)) * 256)]
    for r0, c0 in tiles:
        rows = np.arange(r0, r0 + 256)
        cols = np.arange(c0, c0 + 256)
        Xr = X[:, r0:r0 + 256].float().cpu().numpy()
        Xc = X[:, c0:c0 + 256].float().cpu().numpy()
        ref.append(2.0 * (Xr.astype(np.float64).T @ Xc.astype(np.float64)))
        got.append(H[r0:r0 + 256, c0:c0 + 256].cpu().numpy())
    diag_idx = np.sort(rng.choice(d, 512, replace=False))
    Xdg = X[:, torch.from_numpy(diag_idx).cuda()].float().cpu().numpy().astype(np.float64)
    ref.append(2.0 * np.sum(Xdg * Xdg, axis=0))
    got.append(torch.diagonal(H).cpu().numpy()[diag_idx])
    for g_, r_ in zip(got, ref):
        assert rel_fro(g_, r_) <= TOL
    del X, H
    torch.cuda.empty_cache()


def test_compute_overwrites_without_reading():
    """gq_hessian_compute ignores what H holds (NaN here) and gives exactly
    what accumulating onto zeros gives; with no tokens it gives zeros."""
    X = I.random_layer(21, 200, 8, 777)[1].cuda()
    H_nan = torch.full((200, 200), float("nan"), device="cuda")
    a = gq.hessian(X, H=H_nan)
    b = gq.hessian_accumulate(X, torch.zeros(200, 200, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    z = gq.hessian(X[:0], H=torch.full((200, 200), 3.0, device="cuda"))
    assert torch.count_nonzero(z).item() == 0
