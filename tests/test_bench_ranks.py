"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the timing
is the maximum over ranks and the throughput counts every rank's work; the
reference arm runs on rank 0 only."""
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
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    local_ms = [12.5, 40.25][rank]
    t = bench.max_over_ranks(local_ms, torch.device("cpu"), world)
    v = bench.whole_job_tops(world, 10, 1e12, t)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"t": t, "v": v}, f)
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_throughput(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["t"] == 40.25                      # the slowest rank's time
        assert r["v"] == pytest.approx(world * 10 * 1e12 / 40.25e-3 / 1e12)


def test_single_rank_is_local():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, None, 1) == 3.5


@pytest.mark.parametrize("rank", [1])
def test_reference_arm_other_ranks_exit_quietly(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""
