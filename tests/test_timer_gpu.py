"""Per-launch kernel timing: records appear for the timed kernels only,
durations are positive, the work figures follow the launch shapes, and a
captured graph re-records them on replay."""
import pytest
import torch

from post_weight_quantization_27_b200 import gq, inputs as I

pytestmark = pytest.mark.gpu


def test_timer_eager_and_graph():
    W, X = I.random_layer(1, 512, 384, n_tok=1024)
    W, X = W.cuda(), X.to(torch.bfloat16).cuda()
    gq.kernel_timer_start(["hessian_mma", "rtn"], 64)
    try:
        H = gq.hessian(X)
        q = gq.rtn_quantize_pack(W, 4, 128, True)
        torch.cuda.synchronize()
        recs = gq.kernel_timer_read()
        assert [r[0] for r in recs] == ["hessian_mma", "rtn"]
        assert all(r[1] > 0 for r in recs)
        n, d = X.shape
        assert recs[0][2] == n * d * (d + 1)
        d_out, d_in = W.shape
        assert recs[1][2] == d_out * d_in * (4 + 0.5) + 2 * d_out * (d_in // 128)

        # captured: the same slots are recorded by every replay
        s = torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        out = gq._outputs(d_out, d_in, 128, True, W.device, False)
        with torch.cuda.graph(g, stream=s):
            gq.rtn_quantize_pack(W, 4, 128, True, out=out)
        gq.kernel_timer_stop()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        recs = gq.kernel_timer_read()
        assert len(recs) == 3 and recs[2][0] == "rtn" and recs[2][1] > 0
        assert torch.equal(out["qpacked"], q["qpacked"])
        del g
    finally:
        gq.kernel_timer_release()
    assert gq.kernel_timer_read() == []
