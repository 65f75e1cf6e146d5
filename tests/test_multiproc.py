"""The N > 1 host logic of bench.py on CPU: two ranks over gloo (127.0.0.1).

The benchmark runs independent replicas (no exchange step in the op); its only
cross-rank logic is the barrier around the timed region, the max over ranks of
the timed total, the weak-scaling aggregate, and the reference arm's rule that
rank 0 alone works and prints."""
import contextlib
import datetime
import io
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, port):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60))


def _timing_worker(rank, port, out_dir):
    import torch.distributed as dist
    import bench
    _init(rank, port)
    try:
        world, r, local = bench.dist_env()
        bench.barrier(world)
        # Each rank's timed total differs; every rank must see the slowest.
        mx = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        bench.barrier(world)
        value = bench.replica_throughput(world, 1000, 4, mx)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"world": world, "rank": r, "local": local, "max": mx, "value": value}, f)
    finally:
        dist.destroy_process_group()


def _reference_worker(rank, port, out_dir):
    import bench
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    # The oracle's own cost is not under test: a stand-in result marks who ran it.
    bench.run_reference = lambda args: {"impl": "reference", "ran_on": rank}
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--gpus", str(WORLD), "--steps", "1",
                         "--warmup", "3"])
    with open(os.path.join(out_dir, f"ref{rank}.json"), "w") as f:
        json.dump({"rc": rc, "stdout": buf.getvalue()}, f)


def test_max_over_ranks_and_replica_throughput(tmp_path):
    mp.start_processes(_timing_worker, args=(_free_port(), str(tmp_path)), nprocs=WORLD,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(WORLD)]
    for r, x in enumerate(res):
        assert (x["world"], x["rank"], x["local"]) == (WORLD, r, r)
        assert x["max"] == 15.0                       # the slowest rank's total
        # Two replicas of 1000 units x 4 steps in 15 ms: 8000 units / 0.015 s.
        assert x["value"] == pytest.approx(WORLD * 1000 * 4 / 0.015)


def test_reference_arm_runs_on_rank_zero_only(tmp_path):
    mp.start_processes(_reference_worker, args=(_free_port(), str(tmp_path)), nprocs=WORLD,
                       join=True, start_method="spawn")
    r0 = json.load(open(tmp_path / "ref0.json"))
    r1 = json.load(open(tmp_path / "ref1.json"))
    assert r0["rc"] == 0 and r1["rc"] == 0
    assert json.loads(r0["stdout"].strip()) == {"impl": "reference", "ran_on": 0}
    assert r1["stdout"] == ""
