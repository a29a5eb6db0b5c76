"""The multi-GPU path of bench.py (independent replicas, no data-path
collective) on CPU: two gloo ranks run its process-group set-up, the
max-over-ranks step time, the barrier, the whole-job throughput and the
rank-0-only oracle arm."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, ws: int, port: int, out: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(ws),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench

    ws_, rank_, local = bench.dist_setup()
    assert (ws_, rank_, local) == (ws, rank, rank)
    assert torch.distributed.get_backend() == "gloo"
    # per-rank step times: the reported time is the slowest rank's
    step_ms = 1.0 + rank
    t = bench.allmax(step_ms, ws_)
    bench.barrier(ws_)
    units_per_rank = 8192
    value = units_per_rank * ws_ / (t * 1e-3)
    with open(f"{out}.{rank}", "w") as f:
        json.dump({"max_ms": t, "value": value}, f)
    torch.distributed.destroy_process_group()


def test_two_gloo_ranks_max_time_and_weak_scaling(tmp_path):
    ws, port = 2, _free_port()
    out = str(tmp_path / "r")
    mp.start_processes(_rank_main, args=(ws, port, out), nprocs=ws, join=True,
                       start_method="spawn")
    res = [json.load(open(f"{out}.{r}")) for r in range(ws)]
    for r in res:
        assert r["max_ms"] == 2.0                     # slowest rank's time on every rank
        assert r["value"] == 8192 * 2 / 2.0e-3        # all ranks' units over that time


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun the oracle arm runs on rank 0 alone; another rank exits
    at once, without output."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""
