"""Host logic of bench.py's multi-process path, on CPU with the gloo backend
(world size 2): the barrier, the max over ranks that sets the step time,
and the reference arm's rank handling.  No GPU is used."""

import io
import contextlib
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        # each rank times its own steps; the job time is the slowest rank
        m = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        bench.barrier(world)
        q.put((rank, m))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q))
             for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got == {0: 15.0, 1: 15.0}


def test_single_rank_passes_through():
    assert bench.max_over_ranks(3.25, 1) == 3.25
    bench.barrier(1)                     # no process group needed


def test_reference_arm_runs_on_rank0_only(monkeypatch):
    """Under torchrun, ranks other than 0 exit without work or output."""
    monkeypatch.setenv("RANK", "1")
    called = []
    monkeypatch.setattr(bench, "cpu_baseline",
                        lambda *a, **k: called.append(1))
    args = type("A", (), dict(workload="layer4k", steps=2, warmup=1,
                              gpus=2))()
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.reference_arm(args)
    assert buf.getvalue() == "" and not called


def test_reference_arm_line(monkeypatch):
    """Rank 0 prints one JSON line with the reference keys; warm-up samples
    are not timed."""
    import json
    monkeypatch.setenv("RANK", "0")
    calls = []

    def fake(name, budget_s=15.0):
        calls.append(budget_s)
        return {"value": 100.0 + len(calls), "unit": "encoded KV vecs/s",
                "cores": 4, "kind": "oracle", "sample": "s"}
    monkeypatch.setattr(bench, "cpu_baseline", fake)
    args = type("A", (), dict(workload="layer4k", steps=2, warmup=3,
                              gpus=1))()
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.reference_arm(args)
    lines = buf.getvalue().strip().splitlines()
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["steps"] == 2 and j["warmup"] == 3
    assert len(calls) == 5
    assert j["value"] == pytest.approx((104.0 + 105.0) / 2)
    assert j["e2e"]["h2d_bytes_per_step"] == 0
    assert j["cpu_baseline"]["kind"] == "oracle"
    assert j["metric"] == bench.METRIC


def test_clock_parsing():
    """Median SM clock, max clock and active throttle reasons from
    nvidia-smi CSV lines."""
    c = bench.Clocks(0)
    c.proc = type("P", (), dict(terminate=lambda s: None,
                                wait=lambda s, timeout=None: 0))()
    c.lines = [
        "1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "1900, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "1950, 1965, 980.0, 0x4, Not Active, Not Active, Not Active, Active",
        "garbage",
    ]
    r = c.stop()
    assert r["sm_mhz"] == 1950 and r["sm_max_mhz"] == 1965
    assert r["reasons"] == ["sw_power_cap"] and r["samples"] == 3
