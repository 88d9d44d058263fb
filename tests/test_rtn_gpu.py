"""RTN quantize + pack on the GPU against the oracle: codes, scales, zeros
and packed bytes bit for bit."""
import numpy as np
import pytest
import torch

import oracle as O
from post_weight_quantization_27_b200 import gq, inputs as I
from tests.gpu_util import f16, u32

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def _check(W: torch.Tensor, group_size: int, sym: bool, rows=None):
    Wd = W.cuda()
    out = gq.rtn_quantize_pack(Wd, 4, group_size, sym)
    torch.cuda.synchronize()
    Wn = W.float().numpy()
    if rows is not None:
        Wn = Wn[rows]
    ref = O.rtn_quantize(Wn, group_size, sym)
    q = u32(out["qpacked"])
    s = f16(out["scales"])
    if rows is not None:
        q, s = q[rows], s[rows]
    assert np.array_equal(q, ref["qpacked"])
    assert np.array_equal(s.view(np.uint16), ref["scales"].view(np.uint16))
    if not sym:
        z = f16(out["zeros"])
        if rows is not None:
            z = z[rows]
        assert np.array_equal(z.view(np.uint16), ref["zeros"].view(np.uint16))


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("group_size,sym", [(-1, True), (-1, False), (128, True), (128, False),
                                            (32, True), (8, False), (64, True), (256, False),
                                            (0, True), (0, False)])
@pytest.mark.parametrize("shape", [(7, 256), (33, 768), (130, 1024)])
def test_rtn_bit_exact(dt, group_size, sym, shape):
    d_out, d_in = shape
    if group_size > 0 and d_in % group_size:
        pytest.skip("group does not divide d_in")
    g = torch.Generator().manual_seed(d_out * 1000 + d_in + (group_size % 97))
    W = (torch.randn(shape, generator=g) * 0.02).to(DT[dt])
    W[0, :8] = 0                                        # zero words
    if d_out > 2:
        W[2] = 0                                        # an all-zero row
    _check(W, group_size, sym)


@pytest.mark.parametrize("d_in", [8, 2048, 2056, 4096, 28672])
def test_rtn_per_channel_long_rows(d_in):
    g = torch.Generator().manual_seed(d_in)
    W = (torch.randn((5, d_in), generator=g) * 0.01).to(torch.float16)
    _check(W, -1, True)
    _check(W, -1, False)


def test_rtn_rounding_ties():
    """Values exactly half-way between two levels round to even."""
    s = 0.25
    row = np.array([7 * s, -1.5 * s, 2.5 * s, 0.5 * s, -0.5 * s, 3.5 * s, -2.5 * s, 6.5 * s],
                   dtype=np.float32)
    W = torch.from_numpy(np.tile(row, (3, 2)))
    _check(W, -1, True)
    _check(W, 8, True)
    _check(W, 16, False)


@pytest.mark.parametrize("workload,idx", [(2, 48), (3, 3), (4, 6), (5, 1)])
def test_rtn_full_size_layers(workload, idx):
    """Full-size layers of the workloads; the oracle checks every row of the
    GPT-2 lm_head and 96 sampled rows of the larger layers."""
    spec = I.workload_layers(workload)[idx]
    W = I.make_weights(spec)
    rows = None
    if spec.d_out * spec.d_in > 50_000_000:
        rows = np.sort(np.random.default_rng(idx).choice(spec.d_out, 96, replace=False))
    _check(W, spec.group_size, spec.sym, rows)


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("group_size,sym", [(-1, True), (128, True), (128, False), (32, False)])
def test_rtn_dense_midpoints(dt, group_size, sym):
    """Weights packed with exact rounding midpoints (k + 1/2) s of each
    group's step and their neighbours one ulp away, where a division that
    is not correctly rounded would change the code."""
    d_out, d_in = 1024, 512
    g = torch.Generator().manual_seed(77 + group_size)
    W = (torch.randn((d_out, d_in), generator=g) * 0.02).to(DT[dt]).float()
    gs = d_in if group_size == -1 else group_size
    Wg = W.view(d_out, d_in // gs, gs)
    amax = Wg.abs().amax(2, keepdim=True)
    s16 = (amax / 7).to(torch.float16).float() if sym else \
        ((Wg.amax(2, keepdim=True).clamp(min=0) - Wg.amin(2, keepdim=True).clamp(max=0)) / 15).to(torch.float16).float()
    k = torch.randint(-6, 6, Wg.shape, generator=g).float()
    mid = ((k + 0.5) * s16).to(DT[dt]).float()
    pick = torch.randint(0, 4, Wg.shape, generator=g)
    up = torch.nextafter(mid, torch.full_like(mid, 1e9))
    dn = torch.nextafter(mid, torch.full_like(mid, -1e9))
    Wm = torch.where(pick == 0, mid, torch.where(pick == 1, up, torch.where(pick == 2, dn, Wg)))
    if sym:
        Wm = torch.maximum(torch.minimum(Wm, amax), -amax)
        keep = [Wg.abs().argmax(2, keepdim=True)]
    else:
        Wm = torch.maximum(torch.minimum(Wm, Wg.amax(2, keepdim=True)), Wg.amin(2, keepdim=True))
        keep = [Wg.argmax(2, keepdim=True), Wg.argmin(2, keepdim=True)]
    for idx in keep:                                        # the group's extremes stay,
        Wm.scatter_(2, idx, Wg.gather(2, idx))               # so its step is s16 above
    _check(Wm.reshape(d_out, d_in).to(DT[dt]), group_size, sym)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("group_size,sym", [(-1, True), (-1, False), (32, True), (32, False),
                                            (128, True), (128, False)])
def test_rtn_extreme_scales(dt, group_size, sym):
    """Rows whose fp16 scale is subnormal, saturates at 65504, or is zero
    (all-zero rows and rows that underflow), next to ordinary rows: the
    kernels' short path for groups with small quotients and their general
    path must both match the oracle."""
    d_out, d_in = 60, 256
    g = torch.Generator().manual_seed(5 + group_size + (0 if sym else 1))
    W = torch.randn((d_out, d_in), generator=g)
    mags = torch.tensor([1e-30, 1e-9, 3e-7, 2e-6, 1e-5, 0.02, 1.0, 3e5, 1e6, 1e9, 0.0, 6e4])
    W = W * mags[torch.arange(d_out) % len(mags)][:, None]
    W[5, :128] *= 1e-12                     # one row mixing tiny and ordinary groups
    _check(W.to(DT[dt]), group_size, sym)


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("shape", [(1, 8), (3, 16), (2048, 4096)])
def test_rtn_per_tensor(dt, shape):
    """One scale for the whole matrix (group_size 0): a one-block path for
    small matrices and block partials for large ones."""
    g = torch.Generator().manual_seed(shape[0] + shape[1])
    W = (torch.randn(shape, generator=g) * 0.02).to(DT[dt])
    W.view(-1)[shape[0] * shape[1] // 2] = 0.3      # the extreme sits in the middle
    _check(W, 0, True)
    _check(W, 0, False)


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("group_size,sym", [(-1, True), (-1, False), (128, True), (128, False)])
def test_rtn_nan_weight_keeps_the_other_codes(dt, group_size, sym):
    """A NaN weight has no defined code.  The group statistic passes over it
    (as fminf / fmaxf do), and it must not disturb any other code of its word
    or group: with the NaN positions set to 0 (inside every group's range
    already, since the range includes 0) the oracle's scales, zeros and the
    codes of every other position are the GPU's."""
    d_out, d_in = 16, 512
    g = torch.Generator().manual_seed(77 + group_size + int(sym))
    W = (torch.randn((d_out, d_in), generator=g) * 0.02).to(DT[dt])
    nan_at = [(r, (37 * r + 5) % d_in) for r in range(0, d_out, 2)]
    Wn, W0 = W.clone(), W.float().numpy().copy()
    for r, c in nan_at:
        Wn[r, c] = float("nan")
        W0[r, c] = 0.0
    out = gq.rtn_quantize_pack(Wn.cuda(), 4, group_size, sym)
    torch.cuda.synchronize()
    ref = O.rtn_quantize(W0, group_size, sym)
    assert np.array_equal(f16(out["scales"]).view(np.uint16), ref["scales"].view(np.uint16))
    if not sym:
        assert np.array_equal(f16(out["zeros"]).view(np.uint16), ref["zeros"].view(np.uint16))
    mask = np.full(ref["qpacked"].shape, 0xFFFFFFFF, dtype=np.uint32)
    for r, c in nan_at:
        mask[r, c // 8] &= np.uint32(~(0xF << (4 * (c % 8))) & 0xFFFFFFFF)
    assert np.array_equal(u32(out["qpacked"]) & mask, ref["qpacked"] & mask)
