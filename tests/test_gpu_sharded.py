"""Context-sharded decode (sdk_decode_attn_shard) against the whole-context
decode and the oracle.  The ranks are emulated in one process on one GPU:
each shard runs its stages on its own workspace, and the exchanges between
stages (histogram sums, gathers of tie counts and softmax statistics, the
sum of `out`) are done with torch operations over the shards' buffers.
Kernels of different shards never wait on one another: they run one after
the other on one stream."""

import math

import numpy as np
import pytest
import torch

import oracle
import workloads
import sparse_dictionary_coded_b200 as sdk
from sparse_dictionary_coded_b200 import sharded
from parity import OUT_TOL, words_np

pytestmark = pytest.mark.gpu


def _emulate(plans):
    """Runs every shard's stages, doing each exchange across the shards."""
    gens = [sharded.shard_stages(p) for p in plans]
    for items in zip(*gens):
        kind = items[0][0]
        assert all(it[0] == kind for it in items)
        if kind == "sum":
            tot = items[0][1].clone()
            for _, t, _ in items[1:]:
                tot += t
            for _, t, _ in items:
                t.copy_(tot)
        else:
            cat = torch.cat([t for _, t, _ in items])
            for _, _, into in items:
                into.copy_(cat)


def _shard_store(kw, vw, lens, lo, hi):
    """Code store of tokens [lo[b], hi[b]) of each sequence, at positions
    0 .. hi[b]-lo[b]-1."""
    B = kw.shape[0]
    n = max(h - l for l, h in zip(lo, hi))
    ks = torch.zeros(B, kw.shape[1], n, 16, dtype=kw.dtype)
    vs = torch.zeros_like(ks)
    for b in range(B):
        ks[b, :, :hi[b] - lo[b]] = kw[b, :, lo[b]:hi[b]]
        vs[b, :, :hi[b] - lo[b]] = vw[b, :, lo[b]:hi[b]]
    k_lo, k_full, v_full = workloads.layout(ks, vs)
    return sdk.CodeStore.from_tensors(k_lo.cuda(), k_full.cuda(), v_full.cuda(),
                                      [h - l for l, h in zip(lo, hi)])


def _check(q, DK, DV, kw, vw, lens, cuts, klow=3, khigh=16, top_num=1, top_den=10,
           oracle_heads=2):
    """cuts[s][b]: first token of shard s in sequence b (cuts[0] all 0)."""
    B, Hq, d = q.shape
    R = B * Hq
    world = len(cuts)
    qd, DKd, DVd = q.cuda(), DK.cuda(), DV.cuda()
    # the whole context in one call
    k_lo, k_full, v_full = workloads.layout(kw, vw)
    full = sdk.CodeStore.from_tensors(k_lo.cuda(), k_full.cuda(), v_full.cuda(), lens)
    ws = sdk.new_workspace(sdk.sdk_decode_workspace_bytes(B, Hq, d, DK.shape[0], max(lens)))
    ref = sdk.sdk_decode_attn(qd, DKd, DVd, full, klow=klow, khigh=khigh, top_num=top_num,
                              top_den=top_den, workspace=ws)
    torch.cuda.synchronize()
    assert sdk.sdk_check_status(ws)[0] == 0
    lay = sdk.sdk_decode_layout_of(B, Hq, d, DK.shape[0], max(lens))
    ks = [oracle.topk_count(lens[r // Hq], top_num, top_den) for r in range(R)]
    lst = ws[lay["list"]:lay["list"] + R * lay["row"] * 4].view(torch.int32)
    lst = lst.view(R, lay["row"]).cpu().numpy()
    ref_sets = [set(lst[r, :ks[r]].tolist()) for r in range(R)]
    # the shards
    plans = []
    for s in range(world):
        lo = cuts[s]
        hi = cuts[s + 1] if s + 1 < world else lens
        store = _shard_store(kw, vw, lens, lo, hi)
        plans.append(sharded.ShardPlan(qd, DKd, DVd, store, lens, s, world, klow, khigh,
                                       top_num, top_den))
    _emulate(plans)
    torch.cuda.synchronize()
    for p in plans:
        rc, hdr = sdk.sdk_check_status(p.ws)
        assert rc == 0, (rc, [hex(h) for h in hdr])
        assert torch.equal(p.out, plans[0].out)
    # the union of the shards' selected lists is the whole-context set
    for r in range(R):
        got = []
        for s, p in enumerate(plans):
            st = sdk.read_select_state(p.ws, p.layout, R)
            n_sel = int(st["n_sel"][r])
            pl = p.ws[p.layout["list"]:p.layout["list"] + R * p.layout["row"] * 4]
            pl = pl.view(torch.int32).view(R, p.layout["row"]).cpu().numpy()
            got += (pl[r, :n_sel] + cuts[s][r // Hq]).tolist()
        assert len(got) == ks[r] and set(got) == ref_sets[r], r
    out = plans[0].out.cpu().double()
    refo = ref.cpu().double()
    assert torch.max(torch.abs(out - refo)) <= 1e-5 * max(1.0, float(refo.abs().max()))
    # and against the oracle for a few heads
    qn = q.double().numpy()
    kwn, vwn = words_np(kw), words_np(vw)
    DKn, DVn = DK.float().double().numpy(), DV.float().double().numpy()
    g = Hq // kw.shape[1]
    for r in list(range(R))[:: max(1, R // oracle_heads)]:
        b, h = divmod(r, Hq)
        o = oracle.decode_head_ref(qn[b, h], kwn[b, h // g, :lens[b]], vwn[b, h // g, :lens[b]],
                                   DKn, DVn, klow, khigh, top_num, top_den,
                                   force_set=sorted(ref_sets[r]))
        assert np.max(np.abs(out[b, h].numpy() - o["out"])) <= OUT_TOL


def _unit(q):
    return q / q.norm(dim=-1, keepdim=True)


def _case(seed, B, Hq, Hkv, N, d, n):
    g = workloads.make_gen(seed)
    DK = workloads.gaussian_dictionary(n, d, g)
    DV = workloads.gaussian_dictionary(n, d, g)
    kw = workloads.random_codes((B, Hkv, N), n, g)
    vw = workloads.random_codes((B, Hkv, N), n, g)
    q = _unit(workloads.queries(B, Hq, d, g))
    return q, DK, DV, kw, vw


@pytest.mark.parametrize("cuts", [[[0], [2048]], [[0], [1000], [2500]], [[0], [1], [4000], [4095]]],
                         ids=["2-even", "3-uneven", "4-with-1-token-shards"])
def test_layer4k_shape_sharded(cuts):
    """32 q / 8 KV heads, d=128, 32768 atoms, 4096 tokens split 2, 3 and 4
    ways (one shard of a single token)."""
    q, DK, DV, kw, vw = _case(91, 1, 32, 8, 4096, 128, 32768)
    _check(q, DK, DV, kw, vw, [4096], cuts)


def test_ragged_batch_sharded():
    """B=3 with lengths 40, 333 and 1000 over 2 ranks (each rank at least one
    token of every sequence), GQA 6/2, d=64, 1000 atoms, Klow/Khigh 5/12,
    top 3/10."""
    q, DK, DV, kw, vw = _case(92, 3, 6, 2, 1000, 64, 1000)
    lens = [40, 333, 1000]
    _check(q, DK, DV, kw, vw, lens, [[0, 0, 0], [7, 300, 512]], klow=5, khigh=12,
           top_num=3, top_den=10)


@pytest.mark.parametrize("world", [2, 3])
def test_ties_across_shards(world):
    """Every token carries the same key code: the k lowest global indices
    are selected, so the first shards take all their ties and a later one
    part or none; then half the tokens tied at the threshold."""
    g = workloads.make_gen(93)
    n, d, N = 512, 64, 1000
    DK = workloads.gaussian_dictionary(n, d, g)
    DV = workloads.gaussian_dictionary(n, d, g)
    one = workloads.random_codes((1, 1, 1), n, g)
    kw = one.expand(1, 1, N, 16).contiguous()
    vw = workloads.random_codes((1, 1, N), n, g)
    q = _unit(workloads.queries(1, 2, d, g))
    cuts = [[0], [37], [90]][:world] if world == 3 else [[0], [60]]
    _check(q, DK, DV, kw, vw, [N], cuts)
    kw = workloads.random_codes((1, 1, N), n, g)
    kw[0, 0, 1::2] = kw[0, 0, 7]
    _check(q, DK, DV, kw, vw, [N], [[0], [333], [700]][:world])


def test_full_size_decode256k_two_ranks():
    """One layer of the 256K workload (32 q / 8 KV heads, 262,144 tokens)
    split over two ranks at an uneven cut: every head's selected set equals
    the whole-context one; outputs against the whole-context decode, and
    two sampled heads against the oracle."""
    lay = workloads.decode_layer("decode256k", 0)
    q = _unit(lay["q"])
    N = lay["n_tokens"]
    _check(q, lay["DK"], lay["DV"], lay["kwords"], lay["vwords"], [N],
           [[0], [100_003]], oracle_heads=2)
