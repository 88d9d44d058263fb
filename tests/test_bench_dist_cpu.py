"""The bench's multi-rank plumbing (max over ranks, barrier) on 2 gloo
ranks on the CPU: layers are independent, so the only cross-rank step is the
max of the step time."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, l = bench.dist_env()
        assert (w, r, l) == (world, rank, rank)
        bench.barrier(world)
        got = bench.reduce_max(10.0 + rank * 5.0, world)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_reduce_max_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert res == [(0, 15.0), (1, 15.0)]


def test_single_process_identity():
    import bench
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.stage_work(__import__("post_weight_quantization_27_b200.inputs",
                                       fromlist=["x"]).workload_layers(1)[0])["weights"] == 768 * 768
