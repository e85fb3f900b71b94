"""The multi-rank plumbing of the bench on CPU (gloo, world size 2): replicas
run independently, the job time is the slowest rank's, the job throughput
counts every rank's tokens, only rank 0 reports, and the reference arm runs on
rank 0 alone.  (The data path has no collective: replicas only.)"""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out_q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from datetime import timedelta

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    t = bench.max_over_ranks(times[rank], world, "cpu")
    tok_s = bench.job_throughput(640, world, t)
    dist.barrier()
    dist.destroy_process_group()
    out_q.put((rank, t, tok_s))


def test_max_over_ranks_and_job_throughput_gloo_world2():
    world, port = 2, _free_port()
    times = [12.5, 17.25]  # ms: rank 1 is the slow one
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, tok_s in res:
        assert t == pytest.approx(17.25)          # every rank agrees on the slowest time
        assert tok_s == pytest.approx(640 * 2 / 17.25e-3)  # all ranks' tokens / job time


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.0, 1, "cpu") == 3.0
    assert bench.job_throughput(64, 1, 2.0) == pytest.approx(32000.0)


def test_reference_arm_runs_on_rank_0_only(capsys, monkeypatch):
    """Under torchrun, ranks other than 0 exit 0 at once without output (the
    oracle is a CPU program; one rank times it)."""
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    args = type("A", (), dict(gpus=2, steps=1, warmup=0, seed=0))()
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line(capsys, monkeypatch):
    """Rank 0 prints one JSON line with the reference fields the contract asks."""
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    args = type("A", (), dict(gpus=1, steps=1, warmup=0, seed=0))()
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference"
    assert line["unit"] == "tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"
