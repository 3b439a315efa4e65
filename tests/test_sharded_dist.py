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


# ---------------------------------------------------------------------------
# The real host logic of the context-sharded decode (sharded.ShardPlan,
# shard_stages, run_exchanges) over gloo with two processes.  Only the C-ABI
# stage call is replaced: _StageEmulator writes into the exchanged workspace
# regions what each stage of sdk_decode_attn_shard writes there (include/
# sdk.h: histograms of the order-preserving keys, tie counts, softmax
# statistics, partial outputs), from given per-token scores, logits and
# value vectors.  The scores hold many ties, some straddling the shard
# boundary, so the split of the ties (lower ranks first) and the merge of
# the softmax statistics across processes decide the result, which must
# equal the whole-context selection and softmax.

def _keys_of(scores):
    import numpy as np
    b = np.asarray(scores, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = np.where((b << 1) & 0xFFFFFFFF == 0, 0, b)          # -0 -> +0
    return np.where(b & 0x80000000, ~b & 0xFFFFFFFF, b | 0x80000000).astype(np.uint64)


def _find_desc(hist, k):
    """Bin of the k-th element from the top, and the count above it."""
    above = 0
    for b in range(len(hist) - 1, -1, -1):
        if above + hist[b] >= k:
            return b, above
        above += hist[b]
    raise AssertionError("k beyond the histogram")


class _StageEmulator:
    def __init__(self, real, plan_ref, data):
        self.real, self.plan_ref, self.data = real, plan_ref, data
        self.st = {}

    def sdk_decode_workspace_bytes(self, *a):
        return self.real.sdk_decode_workspace_bytes(*a)

    def sdk_decode_layout_of(self, *a):
        return self.real.sdk_decode_layout_of(*a)

    def sdk_decode_attn_shard(self, stage, rank, world, gathered, *rest):
        import numpy as np
        p = self.plan_ref[0]
        R, B, Hq = p.R, p.B, p.Hq
        d = self.data
        if stage == 1:
            self.st["keys"] = [_keys_of(d["score"][r]) for r in range(R)]
            h1 = p.region("hist1", R * 4096, torch.int32).view(R, 4096)
            for r in range(R):
                h1[r] = torch.from_numpy(np.bincount((self.st["keys"][r] >> 20).astype(np.int64),
                                                     minlength=4096).astype(np.int32))
        elif stage == 2:
            h1 = p.region("hist1", R * 4096, torch.int32).view(R, 4096).numpy()
            h2 = p.region("hist2", R * 4096, torch.int32).view(R, 4096)
            self.st["b1"], self.st["k1"] = [], []
            for r in range(R):
                k = d["k"][r // Hq]
                b1, above = _find_desc(h1[r], k)
                self.st["b1"].append(b1)
                self.st["k1"].append(k - above)
                key = self.st["keys"][r]
                c = key[(key >> 20) == b1]
                h2[r] = torch.from_numpy(np.bincount(((c >> 8) & 0xFFF).astype(np.int64),
                                                     minlength=4096).astype(np.int32))
        elif stage == 3:
            h2 = p.region("hist2", R * 4096, torch.int32).view(R, 4096).numpy()
            h3 = p.region("hist1", R * 256, torch.int32).view(R, 256)
            self.st["pre"], self.st["k2"] = [], []
            for r in range(R):
                b2, above = _find_desc(h2[r], self.st["k1"][r])
                pre = (self.st["b1"][r] << 12) | b2
                self.st["pre"].append(pre)
                self.st["k2"].append(self.st["k1"][r] - above)
                key = self.st["keys"][r]
                c = key[(key >> 8) == pre]
                h3[r] = torch.from_numpy(np.bincount((c & 0xFF).astype(np.int64),
                                                     minlength=256).astype(np.int32))
        elif stage == 4:
            h3 = p.region("hist1", R * 256, torch.int32).view(R, 256).numpy()
            ties = p.region("hist2", R, torch.int32)
            self.st["T"], self.st["take"] = [], []
            for r in range(R):
                b3, above = _find_desc(h3[r], self.st["k2"][r])
                T = (self.st["pre"][r] << 8) | b3
                self.st["T"].append(T)
                self.st["take"].append(self.st["k2"][r] - above)
                ties[r] = int((self.st["keys"][r] == T).sum())
        elif stage == 5:
            assert gathered == p.ties_all.data_ptr()
            tall = p.ties_all.view(world, R).numpy()
            mz = p.region("hist2", 2 * R, torch.float32, 4 * R).view(R, 2)
            self.st["sel"] = []
            for r in range(R):
                key, T = self.st["keys"][r], self.st["T"][r]
                before = int(tall[:rank, r].sum())             # ties of lower ranks
                mine = max(0, min(int(tall[rank, r]), self.st["take"][r] - before))
                tie_idx = np.flatnonzero(key == T)[:mine]      # lowest tokens first
                sel = np.concatenate([np.flatnonzero(key > T), tie_idx])
                self.st["sel"].append(sel)
                lg = d["logit"][r][sel]
                m = float(lg.max()) if sel.size else -np.inf
                mz[r, 0] = m
                mz[r, 1] = float(np.exp(lg - m).sum()) if sel.size else 0.0
        elif stage == 6:
            assert gathered == p.mz_all.data_ptr()
            mz = p.mz_all.view(world, R, 2).numpy()
            for r in range(R):
                m = mz[:, r, 0].max()
                z = sum(float(zw) * np.exp(mw - m) for mw, zw in mz[:, r] if zw > 0)
                sel = self.st["sel"][r]
                pr = np.exp(d["logit"][r][sel] - m) / z
                p.out.view(R, -1)[r] = torch.from_numpy(
                    (pr[:, None] * d["V"][r][sel]).sum(axis=0).astype(np.float32))
        return 0


def _case(world):
    """Per rank: scores (ties across the boundary), logits, values."""
    import numpy as np
    rng = np.random.default_rng(7)
    B, Hq, N, dv = 2, 2, 90, 4
    R = B * Hq
    score = np.floor(rng.random((R, N)) * 6.0)              # 6 values: many ties
    score[:, 40:50] = 4.0                                   # around the shard boundary
    logit = rng.standard_normal((R, N)) * 0.5
    V = rng.standard_normal((R, N, dv))
    bounds = [N * r // world for r in range(world + 1)]
    k = [-(-N // 5)] * B                                    # top 20 %: 18 of 90
    return dict(B=B, Hq=Hq, N=N, dv=dv, score=score, logit=logit, V=V,
                bounds=bounds, k=k)


def _shard_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from sparse_dictionary_coded_b200 import sharded, _capi
        c = _case(world)
        lo, hi = c["bounds"][rank], c["bounds"][rank + 1]
        R = c["B"] * c["Hq"]
        data = dict(k=c["k"], score=c["score"][:, lo:hi], logit=c["logit"][:, lo:hi],
                    V=c["V"][:, lo:hi])
        plan_ref = []
        fake = _StageEmulator(_capi.load(), plan_ref, data)
        sharded.load = lambda: fake
        store = type("S", (), dict(Hkv=1, cap=hi - lo, lens=[hi - lo] * c["B"],
                                   k_lo=torch.zeros(1), k_full=torch.zeros(1),
                                   v_full=torch.zeros(1)))()
        qv = torch.zeros(c["B"], c["Hq"], 64)
        dk = torch.zeros(1024, 64, dtype=torch.bfloat16)
        plan = sharded.ShardPlan(qv, dk, dk, store, [c["N"]] * c["B"], rank, world,
                                 top_num=1, top_den=5,
                                 out=torch.zeros(c["B"], c["Hq"], c["dv"]))
        plan_ref.append(plan)
        sharded.run_exchanges(sharded.shard_stages(plan, stream=0))
        q.put((rank, plan.out.numpy().tolist()))
    finally:
        dist.destroy_process_group()


def test_shard_stages_host_logic_gloo_world2():
    import numpy as np
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs)
    got = dict(q.get(timeout=5) for _ in range(2))
    c = _case(2)
    R = c["B"] * c["Hq"]
    for r in range(R):
        sel = oracle.select_top(c["score"][r], c["k"][r // c["Hq"]])
        lg = c["logit"][r][sel]
        pr = np.exp(lg - lg.max())
        pr /= pr.sum()
        ref = (pr[:, None] * c["V"][r][sel]).sum(axis=0)
        for rank in (0, 1):
            out = np.asarray(got[rank]).reshape(R, -1)[r]
            assert np.allclose(out, ref, rtol=0, atol=1e-5), (rank, r, out, ref)
