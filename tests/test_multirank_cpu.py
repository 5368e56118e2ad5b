"""Host logic of the multi-GPU bench path, run as world-size-2 gloo ranks on
the CPU: every rank streams its own replica batch (weak scaling, no
collective on the data path); the job's time is the slowest rank's and its
throughput counts every rank's bytes; only rank 0 reports.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    from head_latent_attention_02_b200.workloads import WORKLOADS, make_inputs

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank times its own replica; the slower one sets the job time
        times = [1.0 + rank, 5.0 - 2 * rank]
        got = bench.max_over_ranks(times, "cpu", world)
        # replicas draw distinct inputs of the same shape (seed = rank)
        wl = WORKLOADS["tiny_f32"]
        inp = make_inputs(wl, seed=rank)
        nbytes = bench._cache_bytes(wl, inp.n_rows)
        sizes = bench.max_over_ranks([nbytes, -nbytes], "cpu", world)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": got, "bytes": nbytes, "sizes": sizes,
                       "q0": float(inp.q_nope.reshape(-1)[0])}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_replica_inputs_two_gloo_ranks(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(world)]
    # max over ranks: [max(1, 2), max(5, 3)] on both ranks
    assert r[0]["max"] == [2.0, 5.0] and r[1]["max"] == [2.0, 5.0]
    # same per-rank bytes (max of b and of -b agree), different input draws
    assert r[0]["bytes"] == r[1]["bytes"]
    assert r[0]["sizes"] == [r[0]["bytes"], -r[0]["bytes"]]
    assert r[0]["q0"] != r[1]["q0"]


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.job_throughput(75497472, 1, 0.05)
    assert one == pytest.approx(75497472 / 0.05e-3 / 1e9)
    assert bench.job_throughput(75497472, 8, 0.05) == pytest.approx(8 * one)
    assert bench.max_over_ranks([3, 4.5], "cpu", 1) == [3.0, 4.5]


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "1"], env=env, capture_output=True,
                         text=True, timeout=300)
    assert res.returncode == 0, res.stderr
    assert res.stdout.strip() == ""
