"""Host logic of the multi-GPU bench path, on CPU: two ranks in a gloo process
group (127.0.0.1), as ``bench.py --gpus 2`` runs them under torchrun.

The path shards with no data exchange: each rank runs its own workload, and the
ranks meet only in the barriers around the timed region and in the max-over-ranks
reduction of the time. These tests check those pieces: the slowest rank's time
wins on every rank, the ranks' workloads differ, the whole-job value counts all
ranks' tokens, and the reference arm does no work off rank 0.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import bench
    from kimi_delta_attention_27_b200.inputs import CONFIGS, make_inputs
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        # each rank reports a different time; all must see the largest
        t = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        # per-rank workloads: a small slice of the varlen config, seeded per rank
        seed = bench.rank_seed(CONFIGS["t256_h1"]["seed"], rank)
        inp = make_inputs("t256_h1", device="cpu", seed=seed, T=64)
        digest = float(inp["q"].float().sum())
        bench.barrier(world)
        q.put((rank, t, seed, digest))
    finally:
        dist.destroy_process_group()


def test_two_rank_barrier_and_max_over_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [15.0, 15.0]        # the slowest rank's time on both ranks
    assert res[0][2] != res[1][2]                      # distinct seeds ...
    assert res[0][3] != res[1][3]                      # ... hence distinct data


def test_reference_arm_is_rank0_only(tmp_path):
    """Under torchrun, ranks other than 0 exit 0 at once without running the oracle."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=120, cwd=str(tmp_path))
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_whole_job_value_counts_every_rank():
    import bench
    # 4 ranks of 1M tokens each, slowest step 50 ms: 4M tokens per 50 ms
    assert bench.whole_job_value(4, 1 << 20, 50.0) == pytest.approx(83886080.0)
    assert bench.whole_job_value(1, 1 << 20, 50.0) == pytest.approx(20971520.0)
    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_gpus_flag_starts_that_many_ranks(tmp_path):
    """``bench.py --gpus 2`` without torchrun starts two ranks itself (torchrun on
    127.0.0.1) and prints one line, for two GPUs; here through the reference arm, which
    runs on the host cores (rank 0 works, rank 1 exits at once)."""
    import json
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "t256_h1",
                        "--ref-tokens", "64"],
                       env=env, capture_output=True, text=True, timeout=300, cwd=str(tmp_path))
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    assert json.loads(lines[0])["n_gpus"] == 2


def test_rank_count_must_match_gpus_flag(tmp_path):
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=120, cwd=str(tmp_path))
    assert r.returncode == 2
    assert r.stdout.strip() == ""


def test_head_split_covers_every_head_once():
    import bench
    for H, world in [(32, 8), (32, 3), (5, 4), (1, 1), (32, 32)]:
        seen = []
        for rank in range(world):
            h0, h1 = bench.head_range(H, world, rank)
            assert 0 <= h0 <= h1 <= H
            seen += list(range(h0, h1))
        assert seen == list(range(H))
        sizes = [bench.head_range(H, world, r)[1] - bench.head_range(H, world, r)[0] for r in range(world)]
        assert max(sizes) - min(sizes) <= 1
