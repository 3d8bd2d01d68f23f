"""Host logic of bench.py's multi-GPU path, on CPU with gloo ranks.

The step does not shard, so `--gpus N` runs N independent replicas; the only
cross-rank work is the max over ranks of the timed region and the whole-job
rate built from it.  Two gloo ranks check both, and that the reference arm
prints from rank 0 alone.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = [120.0, 250.0, 80.0, 10.0][rank]  # per-rank timed totals
        m = bench.max_over_ranks(ms)
        v = bench.whole_job_rate(1000, 4, world, m)
        q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_max_over_ranks_and_rate_gloo(world):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    expect_ms = max([120.0, 250.0, 80.0, 10.0][:world])
    for rank, m, v in got:
        assert m == expect_ms
        # 1000 units per step per rank, 4 steps, all ranks, over the slowest time
        assert v == pytest.approx(1000 * 4 * world / (expect_ms / 1e3))


def test_max_over_ranks_without_group_is_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5


def _run_reference(env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
         "tiny", "--steps", "1", "--warmup", "0", "--ref-budget", "0.5", "--gpus", "2"],
        capture_output=True, text=True, env=env, timeout=300)


def test_reference_arm_rank_nonzero_exits_quietly():
    r = _run_reference({"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_line():
    r = _run_reference({"RANK": "0", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["config"]["parallelism"] == "replicas2"
