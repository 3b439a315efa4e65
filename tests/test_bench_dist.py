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

    def fake_sampler(name):
        def run(budget_s):
            calls.append(budget_s)
            return {"value": 100.0 + len(calls), "unit": bench.ENCODE_UNIT,
                    "cores": 4, "kind": "oracle", "sample": "s"}
        return run
    monkeypatch.setattr(bench, "oracle_sampler", fake_sampler)
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
    # the same unit and config as the sdk arm prints for this workload
    assert j["unit"] == bench.ENCODE_UNIT
    assert j["config"] == bench.workload_config("layer4k", args)


def test_reference_arm_default_line_carries_prefill(monkeypatch):
    """The default workload's reference line has the decode unit and
    config and a prefill-encode sub-record in the encode unit."""
    import json
    monkeypatch.setenv("RANK", "0")

    def fake_sampler(name):
        unit = bench.DECODE_UNIT if name == "decode256k" else bench.ENCODE_UNIT
        return lambda budget_s: {"value": 7.0, "unit": unit, "cores": 4,
                                 "kind": "oracle", "sample": "s"}
    monkeypatch.setattr(bench, "oracle_sampler", fake_sampler)
    args = type("A", (), dict(workload="decode256k", steps=2, warmup=1, gpus=1,
                              no_prefill=False, full_softmax=False,
                              int_softmax=False, context_shard=False,
                              layers=None))()
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.reference_arm(args)
    j = json.loads(buf.getvalue().strip())
    assert j["unit"] == bench.DECODE_UNIT and j["config"]["workload"] == "decode256k"
    assert j["config"] == bench.workload_config("decode256k", args)
    assert j["prefill_encode"]["unit"] == bench.ENCODE_UNIT
    assert j["prefill_encode"]["config"]["workload"] == "prefill256k_vec"


def test_clock_parsing():
    """Median SM clock, max clock and active throttle reasons from
    nvidia-smi CSV lines."""
    c = bench.Clocks(0)
    c.proc = type("P", (), dict(terminate=lambda s: None,
                                wait=lambda s, timeout=None: 0))()
    c.lines = [(float(i), ln) for i, ln in enumerate([
        "1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "1900, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "1950, 1965, 980.0, 0x4, Not Active, Not Active, Not Active, Active",
        "garbage",
    ])]
    r = c.stop()
    assert r["sm_mhz"] == 1950 and r["sm_max_mhz"] == 1965
    assert r["reasons"] == ["sw_power_cap"] and r["samples"] == 3
    # only the samples inside the marked timed region count; a region
    # shorter than the sampling period takes its neighbours
    c.t0, c.t1 = 0.5, 1.5
    r = c.stop()
    assert r["sm_mhz"] == 1900 and r["samples"] == 1
    c.t0, c.t1 = 1.2, 1.3
    r = c.stop()
    assert r["samples"] == 2 and r["sm_mhz"] == 1925


def test_profiled_traffic_only_for_the_captured_source(tmp_path, monkeypatch):
    """roofline.traffic comes from a committed ncu summary only while the
    kernel's source file still has the sha256 the summary records."""
    import hashlib
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    (tmp_path / "profiles").mkdir()
    sha = hashlib.sha256(b"kernel v1").hexdigest()
    (tmp_path / "profiles" / "attend_kernel_w.md").write_text(
        "traffic_bytes_per_launch: 123456789\nsource_sha256: %s k.cu\n" % sha)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    t, note = bench.profiled_traffic("attend_kernel", "w")
    assert t == 123456789.0 and "attend_kernel_w.md" in note
    src.write_text("kernel v2")
    t, note = bench.profiled_traffic("attend_kernel", "w")
    assert t is None and "changed" in note
    assert bench.profiled_traffic("attend_kernel", "other")[0] is None
