"""Device-side failure reporting: every wait inside a kernel is bounded and
a wait that gives up is reported as GQ_ERR_TIMEOUT through the call's
device status word, leaving the CUDA context usable.

The failure is made without faulting or hanging anything: the library's
self-test kernel waits on a shared-memory barrier that nothing arrives on,
with a 1 ms limit (no copy engine, no tensor-core work involved)."""
import pytest
import torch

from post_weight_quantization_27_b200 import gq

pytestmark = pytest.mark.gpu

GQ_ERR_TIMEOUT = 7


def test_bounded_wait_reports_timeout_and_context_survives():
    assert gq.selftest_bounded_wait(True, 1_000_000) == 0          # arrived: no timeout
    assert gq.selftest_bounded_wait(False, 1_000_000) == GQ_ERR_TIMEOUT
    assert b"gave up" in gq.lib().gq_last_error()
    assert gq.selftest_bounded_wait(False, 0) == GQ_ERR_TIMEOUT
    # the context is still usable: a real call runs and reports no failure
    X = torch.randn(512, 64, device="cuda").to(torch.bfloat16)
    ws = gq.workspace(gq.hessian_workspace_size(512, 64), X.device)
    H = torch.zeros(64, 64, device="cuda")
    gq.hessian_accumulate(X, H, ws=ws)
    assert gq.workspace_status(ws) == 0
    ref = 2.0 * (X.double().T @ X.double())
    assert torch.allclose(H.double(), ref, rtol=1e-5, atol=1e-3)


def test_selftest_rejects_long_limits_and_small_workspaces():
    L = gq.lib()
    ws = gq.workspace(256, torch.device("cuda"))
    s = torch.cuda.current_stream().cuda_stream
    assert L.gq_selftest_bounded_wait(0, 2_000_000_000, gq._p(ws), 256, s) == 1   # GQ_ERR_ARG
    assert L.gq_selftest_bounded_wait(0, 1000, gq._p(ws), 128, s) == 4           # GQ_ERR_WORKSPACE


def test_status_word_clean_after_gptq():
    d_out, d_in = 64, 256
    X = torch.randn(1024, d_in, device="cuda").to(torch.bfloat16)
    W = torch.randn(d_out, d_in, device="cuda") * 0.02
    H = gq.hessian(X)
    U, perm, dead, info = gq.damp_cholesky_inverse(H, 0.01)
    ws = gq.workspace(gq.gptq_workspace_size(d_out, d_in, 128), W.device)
    gq.gptq_quantize_layer(W, U, 4, 128, 128, True, dead=dead, ws=ws)
    assert gq.workspace_status(ws) == 0
