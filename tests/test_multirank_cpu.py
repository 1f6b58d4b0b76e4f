"""The multi-rank host logic of bench.py on CPU: two gloo ranks (no GPU).

Quantization shards without communication: every rank takes its own matrices, and the only
collective is the max-over-ranks of the timings.  These tests check that the stack's 224
matrices are split so that every one lands on exactly one rank, that the timing reduction
returns the maximum on every rank, and that the reference arm runs on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as tmp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out_dir):
    import datetime

    import bench
    from free_weight_quantization_b200 import workloads as wl
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        keys = [(l, i) for l in range(wl.STACK_LAYERS) for i in range(len(wl.STACK_SHAPES))]
        mine = bench.shard(keys, rank, ws)
        everyone = [None] * ws
        dist.all_gather_object(everyone, mine)
        got = bench.max_over_ranks([10.0 * (rank + 1), 5.0 - rank], "cpu", ws)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"mine": mine, "everyone": everyone, "max": got, "n": len(keys)}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_the_stack_and_reduce_timings(tmp_path):
    ws = 2
    tmp.spawn(_rank_main, args=(ws, _free_port(), str(tmp_path)), nprocs=ws, join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(ws)]
    for r in res:
        assert r["max"] == [20.0, 5.0]                      # max over ranks, on every rank
    shards = [[tuple(k) for k in part] for part in res[0]["everyone"]]
    flat = [k for part in shards for k in part]
    assert len(flat) == res[0]["n"] == 224                  # no matrix lost or repeated
    assert len(set(flat)) == 224
    assert abs(len(shards[0]) - len(shards[1])) <= 1       # balanced


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, WORLD_SIZE="2", MASTER_ADDR="127.0.0.1")
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
           "small", "--steps", "1", "--warmup", "1"]
    r1 = subprocess.run(cmd, env=dict(env, RANK="1", LOCAL_RANK="1"), capture_output=True,
                        text=True, timeout=300)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = subprocess.run(cmd, env=dict(env, RANK="0", LOCAL_RANK="0"), capture_output=True,
                        text=True, timeout=300)
    assert r0.returncode == 0, r0.stderr
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["n_gpus"] == 2
