"""Host logic of bench.py's multi-rank (replica) runs, on CPU with gloo:
the slowest rank's time is every rank's, and the job rate counts the units
of all ranks."""
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(times[rank], dist, device="cpu")
        out[rank] = (ms, bench.job_rate(100, world, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_slowest_rank_sets_the_time_world2():
    world = 2
    times = [12.5, 20.0]
    with mp.Manager() as man:
        out = man.dict()
        mp.spawn(_rank, args=(world, _free_port(), times, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        ms, rate = res[r]
        assert ms == 20.0
        assert rate == pytest.approx(100 * world / 0.020)


def test_single_rank_passthrough():
    assert bench.max_over_ranks(3.0) == 3.0
    assert bench.job_rate(10, 1, 1000.0) == pytest.approx(10.0)


def test_reference_arm_silent_on_other_ranks(capsys, monkeypatch):
    # under torchrun only rank 0 runs and prints the oracle line
    monkeypatch.setenv("RANK", "1")
    import synth
    args = type("A", (), {"cpu_sample": 3, "warmup": 3, "steps": 1, "gpus": 2, "copies": 8,
                          "small": True})()
    bench.run_reference(args, synth.TINY)
    assert capsys.readouterr().out == ""


def test_reference_arm_line_tiny(capsys, monkeypatch):
    # rank 0 prints one JSON line: the oracle timed on the host cores
    import json
    import synth
    monkeypatch.setenv("RANK", "0")
    args = type("A", (), {"cpu_sample": 3, "warmup": 3, "steps": 2, "gpus": 1, "copies": 8,
                          "small": True})()
    bench.run_reference(args, synth.TINY)
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == bench.UNIT
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0
