"""Host side of the multi-GPU bench on CPU: world size 2 over gloo.

The path shards by sequence (each rank runs its own independent sequence, no
data-path collective); the only collectives are the barrier and the max over
ranks of the step time. These tests run those pieces on CPU processes.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from long_context_sparse_07_b200 import workloads as W  # noqa: E402


def _rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 1.0 + rank          # rank 1 is the slower one
        rate, ms = bench.job_rate(local_ms, 4096, world, dist, "cpu")
        e2e_rate, e2e_ms = bench.job_rate(10.0 - rank, 4096, world, dist, "cpu")
        dist.barrier()
        with open(os.path.join(out_dir, "r%d.txt" % rank), "w") as f:
            f.write("%r %r %r %r\n" % (rate, ms, e2e_rate, e2e_ms))
    finally:
        dist.destroy_process_group()


def test_job_rate_takes_the_slowest_rank_over_gloo(tmp_path):
    world = 2
    port = 29500 + (os.getpid() % 1000)
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    got = [open(tmp_path / ("r%d.txt" % r)).read().split() for r in range(world)]
    for rate, ms, e2e_rate, e2e_ms in got:
        assert float(ms) == 2.0                      # max of 1.0 and 2.0
        assert float(rate) == pytest.approx(4096 * 2 / 2e-3)
        assert float(e2e_ms) == 10.0                 # max of 10.0 and 9.0
        assert float(e2e_rate) == pytest.approx(4096 * 2 / 10e-3)


def test_job_rate_without_a_process_group_is_the_local_rate():
    rate, ms = bench.job_rate(0.5, 4096, 1, None, "cpu")
    assert ms == 0.5 and rate == pytest.approx(4096 / 0.5e-3)


def test_rank_workloads_are_independent_sequences():
    w = W.scaled(W.WORKLOADS["csa_fp32_n256"], n=64)
    w0, w1 = bench.rank_workload(w, 0), bench.rank_workload(w, 1)
    assert w0 is w and w1.seed != w0.seed
    assert (w1.n, w1.c, w1.k, w1.h) == (w0.n, w0.c, w0.k, w0.h)
    a0, a1 = W.csa_operands(w0), W.csa_operands(w1)
    assert not np.array_equal(np.asarray(a0["Ca"]), np.asarray(a1["Ca"]))
    assert np.array_equal(np.asarray(a0["Ca"]), np.asarray(W.csa_operands(w)["Ca"]))


def test_reference_arm_on_a_nonzero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, env=env, timeout=300, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == ""
