"""Host logic of the multi-rank benchmark, on CPU with the gloo backend and
two ranks: the max-over-ranks reduction of the elapsed time and the whole-job
(weak scaling) throughput."""

import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        mine = 1.0 + rank * 0.25          # rank 1 is the slow one
        t = bench.reduce_max(mine, dist)
        dist.barrier()
        q.put((rank, t, bench.weak_scaling_value(6.6e12, world, t)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=60) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, value in out:
        assert t == 1.25
        assert value == pytest.approx(2 * 6.6e12 / 1.25 / 1e12)


def test_single_process_helpers():
    assert bench.reduce_max(3.5, None) == 3.5
    assert bench.weak_scaling_value(1e12, 1, 0.5) == 2.0
    assert bench.dense_equivalent_ops(1, 12, 32768, 128) == 4.0 * 12 * 32768 ** 2 * 128
    qk, pv = bench.critical_ops(1, 12, 32768, 128, 128, 26)
    assert qk == pv == 12 * 256 * 26 * 2.0 * 128 * 128 * 128
    peak, _ = bench.attn_roofline(qk, pv, {"bf16_tflops": 1000.0})
    assert peak == pytest.approx(2 / (1 / 2000.0 + 1 / 1000.0))
