"""Host-side logic of the multi-GPU bench path on CPU: world-size-2 gloo ranks take the
max of their elapsed times and report whole-job throughput (weak scaling: every rank
runs the same per-GPU workload; no collective touches the data path)."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed = [12.0, 15.0][rank]                 # ms over the timed steps on this rank
        t = bench.reduce_max(elapsed, dist)
        agg = bench.aggregate([t] * world, 1.374e11, 100)
        q.put((rank, t, agg))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, agg in res:
        assert t == 15.0                             # max over ranks
        assert agg["ms_per_step"] == pytest.approx(0.15)
        # both ranks' flops over the slowest rank's time
        assert agg["tflops"] == pytest.approx(2 * 100 * 1.374e11 / 15e-3 / 1e12)


def test_single_rank_reduce_is_identity():
    import bench
    assert bench.reduce_max(3.5, None) == 3.5
    agg = bench.aggregate([10.0], 2e12, 10)
    assert agg["tflops"] == pytest.approx(2e12 * 10 / 10e-3 / 1e12)
