"""The N>1 path of the bench on CPU: world-size-2 `gloo` process groups.

Decode at batch 1 has no exchange step, so ranks are independent replicas:
each draws its own weights and activations, and the only collectives are the
barrier before the timed region and the max-over-ranks of its duration.
These tests run that host logic with two gloo ranks (no GPU), and the
reference arm under torchrun, where rank 0 alone prints the line.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _replica_rank(rank, world, port, out_dir):
    import datetime

    import torch.distributed as tdist

    sys.path.insert(0, ROOT)
    import bench
    import kqgen

    tdist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                             timeout=datetime.timedelta(seconds=60))
    try:
        tdist.barrier()
        my_ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        ms = bench.max_over_ranks(my_ms, "cpu")
        seed = bench.rank_seed(rank)
        W = kqgen.matrix("q4_k", kqgen.tensor_seed(seed, 0, 0), 2, 256)
        res = {"ms": ms, "seed": seed, "w": W.tobytes().hex(),
               "rate": bench.job_rate(1000.0, 4, world, ms)}
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump(res, f)
        tdist.barrier()
    finally:
        tdist.destroy_process_group()


def test_two_gloo_ranks_take_slowest_time_and_distinct_replicas(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_replica_rank, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r = [json.load(open(tmp_path / f"r{i}.json")) for i in range(world)]
    # every rank ends with the slowest rank's time
    assert r[0]["ms"] == r[1]["ms"] == 15.0
    # whole-job rate: units of all ranks over that time
    assert r[0]["rate"] == pytest.approx(1000.0 * 4 * 2 / 15e-3)
    # replicas: distinct seeds, distinct weights
    assert r[0]["seed"] != r[1]["seed"]
    assert r[0]["w"] != r[1]["w"]


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.job_rate(10.0, 5, 1, 1000.0) == pytest.approx(50.0)
    assert np.isclose(bench.job_rate(10.0, 5, 8, 1000.0), 400.0)


def test_reference_arm_under_torchrun_prints_on_rank0_only():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--workload", "gemv_q4k_4096"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    p = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["value"] == line["cpu_baseline"]["value"] == line["e2e"]["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
