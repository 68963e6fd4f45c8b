"""The multi-rank path of the benchmark on CPU: two `gloo` ranks, each on its own shard of
sequences, reduce their timings to the slowest rank and report the whole job's rate. No data
crosses ranks (every (sequence, head) recurrence is independent)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    from workloads import WORKLOADS, decode_inputs

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        wl = bench.shard_workload(WORKLOADS["gdn-mid"].with_(B=2, H=2, T=3), rank)
        q = decode_inputs(wl, "cpu")["q"].float()
        qs = [torch.empty_like(q) for _ in range(world)]
        dist.all_gather(qs, q)
        ms = 10.0 + 5.0 * rank
        slowest = bench.max_over_ranks(ms, world, "cpu")
        rate = bench.whole_job_rate(wl.heads * wl.T, world, slowest)
        res = {"seed": wl.seed, "slowest": slowest, "rate": rate,
               "same_as_other": bool(torch.equal(qs[0], qs[1]))}
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(world)]
    assert r[0]["seed"] != r[1]["seed"]
    assert not r[0]["same_as_other"]                 # disjoint sequences per rank
    assert r[0]["slowest"] == r[1]["slowest"] == 15.0  # max over ranks on every rank
    heads_steps = 2 * 2 * 3
    assert r[0]["rate"] == pytest.approx(heads_steps * world / 0.015)


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"], env=env, cwd=ROOT,
                       capture_output=True, text=True, timeout=120)
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""
