"""The exchange driver of the context-sharded decode (sharded.run_exchanges)
on CPU with the gloo backend, world size 2: the sums and rank-major gathers
each stage asks for.  No GPU is used; the stages are stand-ins that yield
tensors with rank-dependent contents in the order the real stages do."""

import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _fake_stages(rank, world, R, seen):
    hist1 = torch.arange(R * 8, dtype=torch.int32) + 100 * rank
    yield ("sum", hist1, None)
    seen["hist1"] = hist1.clone()
    hist2 = torch.full((R * 8,), rank + 1, dtype=torch.int32)
    yield ("sum", hist2, None)
    seen["hist2"] = hist2.clone()
    ties = torch.full((R,), 10 * rank + 1, dtype=torch.int32)
    ties_all = torch.zeros(world * R, dtype=torch.int32)
    yield ("gather", ties, ties_all)
    seen["ties_all"] = ties_all.clone()
    mz = torch.tensor([float(rank), 1.0 + rank] * R, dtype=torch.float32)
    mz_all = torch.zeros(world * 2 * R, dtype=torch.float32)
    yield ("gather", mz, mz_all)
    seen["mz_all"] = mz_all.clone()
    out = torch.full((R, 4), 0.5 * (rank + 1))
    yield ("sum", out, None)
    seen["out"] = out.clone()


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from sparse_dictionary_coded_b200.sharded import run_exchanges
        seen = {}
        run_exchanges(_fake_stages(rank, world, 3, seen))
        q.put((rank, {k: v.tolist() for k, v in seen.items()}))
    finally:
        dist.destroy_process_group()


def test_exchanges_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = dict(q.get(timeout=5) for _ in range(2))
    R = 3
    for rank in (0, 1):
        s = got[rank]
        assert s["hist1"] == [2 * i + 100 for i in range(R * 8)]
        assert s["hist2"] == [3] * (R * 8)
        assert s["ties_all"] == [1] * R + [11] * R          # rank-major
        assert s["mz_all"] == [0.0, 1.0] * R + [1.0, 2.0] * R
        assert s["out"] == [[1.5] * 4] * R
