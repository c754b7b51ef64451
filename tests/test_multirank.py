"""The multi-GPU launch path of bench.py, on CPU: two gloo ranks.

Each rank runs its own replica on its own token batch (the layer's work
splits into independent token batches, so no collective is on the data path).
The only cross-rank steps are the barrier and the max-over-ranks of the timed
regions; the job's throughput is every rank's tokens over the slowest rank's
time.  Under torchrun the reference arm runs on rank 0 alone.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import bench
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        torch.distributed.barrier()
        ms = bench.max_over_ranks(times[rank], world, "cpu")
        e2e = bench.max_over_ranks(2 * times[rank], world, "cpu")
        out[rank] = (ms, e2e, bench.job_throughput(4096, 20, world, ms))
    finally:
        torch.distributed.destroy_process_group()


def test_two_ranks_agree_on_the_slowest_time_and_the_job_throughput():
    world, port = 2, _free_port()
    times = [3.25, 7.5]
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, times, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        ms, e2e, tput = res[r]
        assert ms == 7.5 and e2e == 15.0
        assert tput == pytest.approx(2 * 4096 * 20 / 7.5e-3)


def test_one_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.0, 1, "cpu") == 4.0
    assert bench.job_throughput(64, 10, 1, 2.0) == pytest.approx(64 * 10 / 2e-3)


def test_reference_arm_runs_on_rank_zero_only(capsys, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
                                      "--warmup", "3"])
    called = []
    monkeypatch.setattr(bench, "run_reference", lambda args, world: called.append((args, world)) or {})
    bench.main()
    assert called == [] and capsys.readouterr().out == ""


def test_reference_arm_line_on_rank_zero(capsys, monkeypatch):
    """Rank 0 prints the reference line: the oracle on a token sample, with the
    workload config the GPU arm prints for the same workload and world size."""
    sys.path.insert(0, ROOT)
    import json
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("LOCAL_RANK", "0")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2", "--workload", "tiny",
                                      "--tokens", "16", "--steps", "1", "--warmup", "3", "--ref-sample", "2"])
    bench.main()
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    cfg = line["config"]
    assert cfg["workload"] == "tiny T=16" and cfg["T_per_gpu"] == 16
    assert cfg["parallelism"] == "replicas x2 (token batches)"
    assert set(cfg) == {"workload", "H", "I", "E", "k", "activation", "T_per_gpu", "parallelism", "l2"}
