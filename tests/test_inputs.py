"""The seeded input generators: shapes, dtypes, determinism, structure."""
import numpy as np
import torch

from post_weight_quantization_27_b200 import inputs as I


def test_workload_shapes():
    assert len(I.workload_layers(1)) == 1
    w2 = I.workload_layers(2)
    assert len(w2) == 49 and w2[-1].d_out == 50257 and w2[-1].d_in == 768
    assert len(I.workload_layers(3)) == 96
    assert [(l.d_in, l.d_out) for l in I.workload_layers(5)] == [(8192, 8192), (8192, 28672), (28672, 8192)]
    assert all(l.act_order and not l.sym for l in I.workload_layers(4))


def test_deterministic_and_dtypes():
    spec = I.workload_layers(1)[0]
    a, b = I.make_weights(spec), I.make_weights(spec)
    assert a.dtype == torch.float32 and torch.equal(a, b)
    x1, x2 = I.make_x(spec, rows=64), I.make_x(spec, rows=64)
    assert x1.dtype == torch.bfloat16 and torch.equal(x1, x2)
    assert torch.equal(I.make_x(spec)[:64], x1)


def test_outlier_structure():
    spec = I.workload_layers(1)[0]
    W = I.make_weights(spec).numpy()
    col_std = W.std(0)
    assert (col_std > 4 * np.median(col_std)).sum() == 8          # 1% of 768 columns x8
    X = I.make_x(spec).float().numpy()
    xs = X.std(0)
    assert (xs > 8 * np.median(xs)).sum() >= 4                      # 4 channels x20
