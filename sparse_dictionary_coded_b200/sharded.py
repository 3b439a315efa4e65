"""Context-sharded decode attention (sdk_decode_attn_shard, include/sdk.h).

Every sequence's context is split over the ranks of a process group, rank r
holding a contiguous token range (ranks in token order).  Each rank runs the
six stages of sdk_decode_attn_shard on its own shard and workspace; between
stages the ranks combine small workspace regions: the sums of the three
radix histograms of the selection, gathers of the per-head tie counts and
softmax statistics, and the sum of ``out``.  ``shard_stages`` runs the
stages of one rank and yields each exchange; ``run_exchanges`` performs
them with torch.distributed collectives (NCCL on GPUs).  The selected set is
the exact global top k of the whole context, so the result equals
sdk_decode_attn over the whole context up to the order of fp32 additions.
"""

import ctypes
import math

import torch

from . import _capi
from ._capi import load


class ShardPlan:
    """One rank's inputs and buffers for a sharded decode call.

    q [B, Hq, d] fp32 (the same on every rank), dict_k / dict_v bf16
    [n_atoms, d], store: this rank's CodeStore (its tokens at positions
    0 .. lens[b]-1), glens: every sequence's whole length."""

    def __init__(self, q, dict_k, dict_v, store, glens, rank, world, klow=3,
                 khigh=16, top_num=1, top_den=10, scale=None, out=None,
                 workspace=None):
        self.q, self.dict_k, self.dict_v, self.store = q, dict_k, dict_v, store
        self.rank, self.world = rank, world
        B, Hq, d = q.shape
        self.B, self.Hq, self.d = B, Hq, d
        self.R = B * Hq
        self.n_atoms = dict_k.shape[0]
        self.klow, self.khigh, self.top_num, self.top_den = klow, khigh, top_num, top_den
        self.scale = 1.0 / math.sqrt(d) if scale is None else scale
        self.lens = list(store.lens)
        self.glens = list(glens)
        if len(self.glens) != B or any(g < l for g, l in zip(self.glens, self.lens)):
            raise ValueError("glens must hold every sequence's whole length")
        lib = load()
        max_len = max(self.lens)
        if workspace is None:
            workspace = torch.zeros(
                lib.sdk_decode_workspace_bytes(B, Hq, d, self.n_atoms, max_len),
                dtype=torch.uint8, device=q.device)
        self.ws = workspace
        lay = _capi.DecodeLayout()
        rc = lib.sdk_decode_layout_of(B, Hq, d, self.n_atoms, max_len, ctypes.byref(lay))
        if rc != 0:
            raise RuntimeError("sdk_decode_layout_of: status %d" % rc)
        self.layout = {f: getattr(lay, f) for f, _ in _capi.DecodeLayout._fields_}
        self.out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device) \
            if out is None else out
        self.ties_all = torch.zeros(world * self.R, dtype=torch.int32, device=q.device)
        self.mz_all = torch.zeros(world * self.R * 2, dtype=torch.float32, device=q.device)

    def region(self, name, count, dtype, byte_offset=0):
        o = self.layout[name] + byte_offset
        size = torch.tensor([], dtype=dtype).element_size()
        return self.ws[o:o + count * size].view(dtype)


def shard_stages(plan, stream=None):
    """Runs the six stages for one rank.  After each it yields the exchange
    that must follow, as ("sum", tensor, None): sum over ranks in place, or
    ("gather", tensor, into): gather every rank's tensor, rank-major, into
    ``into``.  Resume the generator once the exchange is done."""
    lib = load()
    p = plan
    st = torch.cuda.current_stream().cuda_stream if stream is None else stream
    lens = (ctypes.c_int32 * p.B)(*p.lens)
    glens = (ctypes.c_int32 * p.B)(*p.glens)
    s = p.store
    for stage in range(1, 7):
        gathered = p.ties_all if stage == 5 else (p.mz_all if stage == 6 else None)
        rc = lib.sdk_decode_attn_shard(
            stage, p.rank, p.world, None if gathered is None else gathered.data_ptr(),
            p.q.data_ptr(), p.B, p.Hq, s.Hkv, p.d, p.dict_k.data_ptr(), p.dict_v.data_ptr(),
            p.n_atoms, s.k_lo.data_ptr(), s.k_full.data_ptr(), s.v_full.data_ptr(), s.cap,
            lens, glens, p.klow, p.khigh, p.top_num, p.top_den, 0, float(p.scale),
            p.out.data_ptr(), p.ws.data_ptr(), p.ws.numel(), st)
        if rc != 0:
            raise RuntimeError("sdk_decode_attn_shard stage %d: %s" % (
                stage, _capi.STATUS_NAMES.get(rc, rc)))
        if stage == 1:
            yield ("sum", p.region("hist1", p.R * 4096, torch.int32), None)
        elif stage == 2:
            yield ("sum", p.region("hist2", p.R * 4096, torch.int32), None)
        elif stage == 3:
            yield ("sum", p.region("hist1", p.R * 256, torch.int32), None)
        elif stage == 4:
            yield ("gather", p.region("hist2", p.R, torch.int32), p.ties_all)
        elif stage == 5:
            yield ("gather", p.region("hist2", 2 * p.R, torch.float32, 4 * p.R), p.mz_all)
        else:
            yield ("sum", p.out, None)


def run_exchanges(stages, group=None):
    """Drives a stage generator, doing each exchange with torch.distributed
    collectives on ``group``."""
    import torch.distributed as dist
    for kind, t, into in stages:
        if kind == "sum":
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
        else:
            dist.all_gather_into_tensor(into, t, group=group)


def sdk_decode_attn_sharded(q, dict_k, dict_v, store, glens, group=None, klow=3,
                            khigh=16, top_num=1, top_den=10, scale=None,
                            out=None, workspace=None):
    """One layer of decode attention over a context split across the ranks
    of ``group`` (this rank's tokens in ``store``, whole lengths in
    ``glens``).  Returns out [B, Hq, d] fp32, the same on every rank."""
    import torch.distributed as dist
    plan = ShardPlan(q, dict_k, dict_v, store, glens, dist.get_rank(group),
                     dist.get_world_size(group), klow, khigh, top_num, top_den,
                     scale, out, workspace)
    run_exchanges(shard_stages(plan), group)
    return plan.out
