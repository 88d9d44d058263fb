"""Host-side logic of bench.py that needs no GPU: the layer-to-stream
schedule, the roofline arithmetic of the dominant kernel, the per-kernel
ceilings, the committed traffic table, and the per-kernel rates."""
import types

import pytest

import bench
from post_weight_quantization_27_b200 import inputs as I


def _runs(workload):
    return [types.SimpleNamespace(spec=s) for s in I.workload_layers(workload)]


@pytest.mark.parametrize("n_streams", [1, 7, 32, 64])
def test_schedule_covers_every_layer_once(n_streams):
    runs = _runs(2)
    lists = bench.schedule(runs, n_streams)
    assert len(lists) == n_streams
    flat = sorted(i for l in lists for i in l)
    assert flat == list(range(len(runs)))


def test_schedule_balances_the_largest_layers():
    """With as many streams as there are big layers, the twelve 3072-wide
    layers (the heaviest by d_out d_in + 4 d_in^2) and the lm_head land on
    different streams."""
    runs = _runs(2)
    lists = bench.schedule(runs, 16)
    heavy = {i for i, r in enumerate(runs) if r.spec.d_in == 3072 or r.spec.d_out == 50257}
    owner = {i: k for k, l in enumerate(lists) for i in l}
    assert len({owner[i] for i in heavy}) == len(heavy)


PEAKS = {"hbm_gbs": 6546.9, "bf16_tflops": 1676.5, "bf16_tflops_sustained": 1374.1,
         "sm_max_mhz": 1965.0, "source": "measured"}


def test_roofline_arithmetic():
    # two launches of 1e9 flop in 1 ms each: 1 TFLOP/s
    recs = [("gemm_tf32x3", 1.0, 1e9), ("gemm_tf32x3", 1.0, 1e9)]
    r = bench.roofline("gemm_tf32x3", recs, PEAKS, 99, 10.0)
    assert r["achieved"] == pytest.approx(1.0)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    # the peak of the kernel's own arithmetic (tf32), not divided by passes
    assert r["peak"] == pytest.approx(1374.1 * 1.1 / 2.25, rel=1e-3)
    assert r["frac"] == pytest.approx(1.0 / r["peak"], rel=1e-2)
    assert r["tensor_passes"] == 3
    assert r["tensor_pipe_frac"] == pytest.approx(3 * r["frac"], rel=1e-2)
    assert r["launches"] == 2 and r["avg_launch_us"] == pytest.approx(1000.0)
    assert r["kernel_ms_per_step"] == pytest.approx(2.0) and r["step_ms"] == 10.0
    # a bf16 contraction against the sustained bf16 peak itself
    r = bench.roofline("recon_mma", [("recon_mma", 1.0, 1374.1e9)], PEAKS, 99, 1.0)
    assert r["frac"] == pytest.approx(1.0, rel=1e-4) and r["tensor_pipe_frac"] == pytest.approx(2.0, rel=1e-4)
    # bytes: 6.5469e9 bytes in 1 ms -> the copy bandwidth
    r = bench.roofline("rtn", [("rtn", 1.0, 6.5469e9)], PEAKS, 99, 1.0)
    assert r["bound"] == "hbm" and r["frac"] == pytest.approx(1.0, rel=1e-4)
    # fp32 ALU ceiling from the SM count, lanes and clock
    r = bench.roofline("potrf_trsm", [("potrf_trsm", 1.0, 1e9)], PEAKS, 99, 1.0)
    assert r["bound"] == "alu"
    assert r["peak"] == pytest.approx(148 * 128 * 2 * 1965e6 / 1e12, rel=1e-3)


def test_every_timed_kernel_has_a_ceiling():
    from post_weight_quantization_27_b200 import gq
    for k in gq.KERNELS:
        bound, _, _ = bench.KERNEL_BOUND[k]
        peak, unit, _ = bench.kernel_peak(k, PEAKS)
        assert peak > 0 and unit in ("TFLOP/s", "GB/s")
        assert (unit == "GB/s") == (bound == "hbm")


def test_traffic_table_parses():
    t = bench.profiled_traffic("hessian_mma", 5)
    assert t is not None and t > 0
    assert bench.profiled_traffic("hessian_mma", 99) is None
    assert bench.profiled_traffic("no_such_kernel", 5) is None


def test_rate():
    shares = {"rtn": (2.0, 5, 4e9)}
    assert bench.rate(shares, "rtn", 1e9) == pytest.approx(2000.0)
    assert bench.rate(shares, "hessian_mma", 1e12) is None
