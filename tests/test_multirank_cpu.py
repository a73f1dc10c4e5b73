"""The multi-process (N > 1) path of bench.py, on CPU with the gloo backend.

bench.py --gpus N runs one process per GPU under torchrun; every rank runs
its own replica of the workload (independent matrices, no data-path
collective), and the job's time is the max over ranks of each rank's
device-timed region.  These tests drive the same rank logic (RankContext:
env parsing, barrier, max-over-ranks, teardown) with world size 2 on gloo,
and check that the reference arm runs on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    R = bench.RankContext("gloo", timeout_s=60)
    assert (R.rank, R.world, R.local) == (rank, world, rank)
    R.barrier()
    # each rank's "device-timed" value; the job reports the max over ranks
    got = R.max(10.0 * rank + 3.5)
    got2 = R.max(-1.0 if rank == 0 else -7.0)
    R.close()
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump({"max": got, "max2": got2, "root": R.is_root}, f)


def test_rank_context_max_over_ranks_gloo(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    assert [r["max"] for r in res] == [13.5, 13.5]
    assert [r["max2"] for r in res] == [-1.0, -1.0]
    assert [r["root"] for r in res] == [True, False]


def test_single_rank_context_needs_no_process_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    sys.path.insert(0, ROOT)
    import bench
    R = bench.RankContext("gloo")
    assert R.world == 1 and R.is_root and R.dist is None
    assert R.max(4.25) == 4.25
    R.barrier()
    R.close()


@pytest.mark.parametrize("rank", [1])
def test_reference_arm_runs_on_rank_zero_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--gpus", "2"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_prints_one_line_on_rank_zero():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "single_256x1024", "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "ms" and d["higher_is_better"] is False
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
