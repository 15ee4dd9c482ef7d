"""The benchmark's multi-rank plumbing on the host: two gloo ranks (CPU, no GPU).

bench.py runs one process per GPU; each rank times the same independent problem, the
step time is the maximum over ranks and the value is every rank's work over that time.
Checked here: the rank reduction returns the slowest rank's time on every rank, the
whole-job rate counts all ranks' units, the barrier releases, and the reference arm does
its work (and prints) on rank 0 only.
"""
import contextlib
import io
import json
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    try:
        got_ws, got_rank, got_local = bench.dist_info()
        ms = [3.0, 5.0][rank]                      # rank 1 is the slow one
        slowest = bench.max_over_ranks(ms, ws)
        bench.barrier(ws)
        rate = bench.whole_job_rate(1e9, slowest, ws)

        class Args:
            steps, warmup, gpus = 1, 0, ws
        buf = io.StringIO()
        calls = []
        real = bench.cpu_baseline
        bench.cpu_baseline = lambda w, budget, seed=0: (calls.append(budget) or
                                                        (0.5, 2, "stub sample", 0.01))
        with contextlib.redirect_stdout(buf):
            bench.arm_reference(Args, ws, rank)
        bench.cpu_baseline = real
        bench.barrier(ws)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ws": got_ws, "rank": got_rank, "local": got_local,
                       "slowest": slowest, "rate": rate, "printed": buf.getvalue(),
                       "calls": len(calls)}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    ws, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(ws, port, str(tmp_path)), nprocs=ws, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(ws)]
    for r, d in enumerate(res):
        assert (d["ws"], d["rank"], d["local"]) == (ws, r, r)
        assert d["slowest"] == 5.0                 # max over ranks, on every rank
        assert d["rate"] == pytest.approx(2 * 1e9 / 5e-3)
    # the reference arm ran and printed its line on rank 0 only
    assert res[0]["calls"] == 1 and res[1]["calls"] == 0
    assert res[1]["printed"] == ""
    line = json.loads(res[0]["printed"].strip())
    assert line["impl"] == "reference" and line["n_gpus"] == ws and line["value"] == 0.5
