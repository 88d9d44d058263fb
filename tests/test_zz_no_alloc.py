"""gq_damp_cholesky_inverse_noalloc: the damp / act-order / upper-factor step
for callers that cannot allocate device memory (for instance code whose
device memory belongs to a host framework's pool or fixed budget, or that
must not stall on cudaMalloc / cudaFree), so cannot pass a workspace.

Its scratch is a fixed array inside the library, shared by every call and
keeping the previous call's contents; two calls in a row must each give the
same result as the workspace entry point.  This file is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from post_weight_quantization_27_b200 import gq

pytestmark = pytest.mark.gpu


def _H(d, seed, n_tok=None):
    g = torch.Generator(device="cuda").manual_seed(seed)
    n = n_tok or 2 * d
    sig = torch.exp(0.5 * torch.randn(d, generator=g, device="cuda"))
    X = (torch.randn(n, d, generator=g, device="cuda") * sig).to(torch.bfloat16)
    return gq.hessian(X)


def _noalloc(H, damp, act_order):
    """Direct C-ABI call of the no-allocation entry point."""
    d = H.shape[0]
    U = torch.empty((d, d), dtype=torch.float32, device="cuda")
    perm = torch.empty(d, dtype=torch.int32, device="cuda") if act_order else None
    dead = torch.empty(d, dtype=torch.uint8, device="cuda")
    info = torch.empty(1, dtype=torch.int32, device="cuda")
    info_host = ctypes.c_int32(-7)
    st = gq.lib().gq_damp_cholesky_inverse_noalloc(
        H.data_ptr(), d, damp, int(act_order), gq._p(perm), dead.data_ptr(), U.data_ptr(),
        info.data_ptr(), ctypes.byref(info_host), torch.cuda.current_stream().cuda_stream)
    return st, U, perm, dead, info, info_host.value


@pytest.mark.parametrize("d,act_order", [(768, False), (3072, True), (136, False)])
def test_noalloc_matches_workspace_entry_point(d, act_order):
    for call in range(2):                       # two calls in a row share the scratch
        H = _H(d, 100 * call + d)
        H[5, :] = 0.0
        H[:, 5] = 0.0                           # a dead column
        U_ref, perm_ref, dead_ref, info_ref = gq.damp_cholesky_inverse(H.clone(), 0.01, act_order)
        st, U, perm, dead, info, info_host = _noalloc(H.clone(), 0.01, act_order)
        assert st == 0, gq.lib().gq_last_error()
        assert info_host == -1 and int(info.item()) == -1 == int(info_ref.item())
        # the same kernels in the same order on the same input, none with
        # atomics or order-dependent sums: bit-identical
        assert torch.equal(U, U_ref)
        assert torch.equal(dead, dead_ref)
        if act_order:
            assert torch.equal(perm, perm_ref)


def test_noalloc_reports_not_pd_then_recovers():
    d = 256
    H = torch.eye(d, device="cuda")
    H[100, 100] = -3.0
    st, U, perm, dead, info, info_host = _noalloc(H, 0.0, False)
    assert st == 5 and info_host == 100          # GQ_ERR_NOT_PD at that column
    good = _H(d, 7)
    U_ref, *_ = gq.damp_cholesky_inverse(good.clone(), 0.01)
    st, U, *_rest, info_host = _noalloc(good.clone(), 0.01, False)
    assert st == 0 and info_host == -1           # leftovers of the failed call do not leak
    assert torch.equal(U, U_ref)


def test_noalloc_rejects_sizes_beyond_its_limit():
    H = torch.empty((4104, 4104), dtype=torch.float32, device="cuda")
    st, *_ = _noalloc(H, 0.01, False)
    assert st == 2                               # GQ_ERR_SHAPE, nothing launched
    assert b"no-allocation limit" in gq.lib().gq_last_error()
