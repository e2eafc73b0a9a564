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
    import numpy as np

    # every block full: 2 * block^2 * d per kept pair, for QK^T and for PV
    idx = np.tile(np.arange(26, dtype=np.int32), (1, 12, 256, 1))
    qk, pv = bench.critical_ops(idx, 32768, 128, 128)
    assert qk == pv == 12 * 256 * 26 * 2.0 * 128 * 128 * 128
    peak, _ = bench.attn_roofline(qk, pv, {"bf16_tflops": 1000.0})
    assert peak == pytest.approx(2 / (1 / 2000.0 + 1 / 1000.0))
    # a partial last block (N = 300, block 128: sizes 128, 128, 44) counts its valid rows and keys
    idx = np.array([[[[0, 2], [1, 2], [0, 1]]]], dtype=np.int32)
    qk, _ = bench.critical_ops(idx, 300, 64, 128)
    assert qk == 2.0 * 64 * (128 * (128 + 44) + 128 * (128 + 44) + 44 * (128 + 128))
    # the whole-call roofline takes the slower of the tensor and HBM bounds
    r = bench.call_roofline(2e12, 1e12, 6.5e9, 2.0, {"bf16_tflops": 1000.0, "hbm_gbs": 6500.0})
    assert r["bound"] == "tensor" and r["t_roof_ms"] == pytest.approx(2.0) and r["frac"] == pytest.approx(1.0)
    r = bench.call_roofline(2e9, 1e9, 6.5e9, 2.0, {"bf16_tflops": 1000.0, "hbm_gbs": 6500.0})
    assert r["bound"] == "hbm" and r["t_roof_ms"] == pytest.approx(1.0) and r["frac"] == pytest.approx(0.5)
    assert bench.algorithmic_bytes(1, 12, 32768, 128, 256, 26) == (
        12 * 32768 * 128 * 12 + 2 * 12 * 256 * (128 * 128 + 128) * 4)
    assert bench.algorithmic_bytes(1, 12, 32768, 128, 256, 256) == 12 * 32768 * 128 * 12


def test_bench_helpers_for_the_extended_workloads():
    """Lists shorter than the pitch (-1 entries) count no work; the metric
    strings name the three-class, finer-granularity and W8A8 workloads."""
    import numpy as np

    from synth import CONFIGS

    idx = np.array([[[[0, 1, -1], [2, -1, -1], [0, 1, 2]]]], dtype=np.int32)
    qk, pv = bench.critical_ops(idx, 384, 64, 128)
    assert qk == pv == 2.0 * 64 * 128 * 128 * (2 + 1 + 3)
    m = bench.metric_for(CONFIGS["480p_classes"])
    assert "per head" in m and "skip 50%" in m
    assert "scale per 32 tokens" in bench.metric_for(CONFIGS["480p_gran32"])
    assert bench.metric_for(CONFIGS["480p"]) == bench.METRIC
    assert bench.algorithmic_bytes(1, 12, 32768, 128, 256, 52, linear=False) == 12 * 32768 * 128 * 12


def test_w8a8_oracle_legs_of_the_bench_run_on_the_cpu():
    """The W8A8 workloads' CPU baseline and reference arm (plain C++ oracle)."""
    import argparse

    from synth.linear import LINEAR_CONFIGS, make_linear_workload

    w = LINEAR_CONFIGS["w8a8_small"]
    dt, rows = bench.linear_oracle_sample(w, make_linear_workload(w), 0.05)
    assert dt > 0 and 0 < rows <= w.M
    args = argparse.Namespace(workload="w8a8_small", steps=3, warmup=3)
    line = bench.run_reference_linear(args, bench.Dist(1))
    assert line["impl"] == "reference" and line["value"] > 0
    assert "plain C++" in line["cpu_baseline"]["sample"]
