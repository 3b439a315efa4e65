"""Benchmark of the dictionary-coded KV cache hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sdk|reference]
                    [--workload decode256k|decode32k_b4|prefill256k_vec|layer4k|
                                append_token_b1|append_token_b4]

Default workload 'decode256k': one decode step of a 32-layer Llama-3.1-8B KV
shape at batch 1 over 262,144 context tokens (32 q / 8 KV heads, d=128,
32768-atom bf16 K and V dictionaries per layer, 16-atom codes), the 32 layer
calls (sdk_decode_attn) replayed as one CUDA graph; the headline value is
context tokens attended per second per decode step.  The same line carries
the prefill encode of 16384 tokens x 8 KV heads x 2 streams = 262,144
vectors (sdk_encode, greedy pursuit over one layer's dictionaries) as the
keyed sub-record "prefill_encode" (encoded vectors/s, tensor roofline, its
own e2e); --no-prefill leaves it out.  Other workloads: 'decode32k_b4' (32
layers, batch 4, 32K tokens), 'prefill256k_vec' alone, 'layer4k' (encode +
append 65,536 vectors of one layer, then one decode step over 4096 tokens),
'append_token_b1' / 'append_token_b4' (one generated token appended to all
32 layers).

Timing: W untimed warm-up steps, then K steps, each timed with CUDA events on
the launching stream.  Encode workloads flush the L2 (256 MiB memset)
between steps, outside the events; the decode workloads' inputs exceed the
L2 (every layer's working set is larger than it), so they run unflushed.  Multi-GPU (torchrun): every rank runs its own
independent copy of the workload (weak scaling, no collective on the data
path); the time is the max over ranks.  Rank 0 prints one JSON line.
"""

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("decode ctx tokens/s/step & encoded KV vecs/s (1 B200), "
          "% HBM/tensor roofline")
# algorithmic encode work per vector: 16 greedy steps x n_atoms x head_dim
# multiply-adds (134,217,728 FLOP at 32768 atoms, d=128)
def enc_flop_per_vector(n_atoms, head_dim):
    return 16 * n_atoms * head_dim * 2


# kernels of one decode layer: qd, klow, pass2, final, attend, out
DEC_KERNELS_PER_LAYER = 6
DECODE_UNIT = "ctx tokens/s/step"
ENCODE_UNIT = "encoded KV vecs/s"


def _sha256(path):
    import hashlib
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def profiled_traffic(kernel, workload):
    """DRAM bytes (read + write) per launch of `kernel` on `workload` from
    the committed ncu summary profiles/<kernel>_<workload>.md, whose lines
    'traffic_bytes_per_launch: T' and 'source_sha256: H' record the capture
    and the sha256 of the kernel's source file when it was taken.  None
    when no summary exists or the source has changed since (the counters
    then describe another kernel).  Returns (bytes or None, note)."""
    import re
    path = os.path.join(ROOT, "profiles", "%s_%s.md" % (kernel, workload))
    if not os.path.exists(path):
        return None, "no ncu summary for this kernel and workload"
    txt = open(path).read()
    mt = re.search(r"^traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt, re.M)
    ms = re.search(r"^source_sha256:\s*([0-9a-f]{64})\s+(\S+)", txt, re.M)
    if not mt or not ms:
        return None, "summary holds no traffic line"
    src = os.path.join(ROOT, ms.group(2))
    if not os.path.exists(src) or _sha256(src) != ms.group(1):
        return None, "kernel source changed since the capture in %s" % os.path.relpath(path, ROOT)
    return float(mt.group(1)), ("dram__bytes_read.sum + dram__bytes_write.sum per launch, "
                                "from %s" % os.path.relpath(path, ROOT))
ENC_DTYPE = ("f32 (residuals and re-scoring; tensor-core operands fp16 with "
             "fp32 accumulation; bf16 dictionaries; fp16 coefficients)")


def tensor_roofline(tflops, pk, kernel):
    """Encode roofline: the correlation GEMM on the tensor cores.  Its
    operands are fp16, whose nominal dense rate equals bf16's (ratio 1), so
    the peak is the measured bf16 GEMM rate (burst: the step is timed as a
    short burst of launches); the sustained figure is reported beside it."""
    return {"bound": "tensor", "kernel": kernel, "achieved": tflops,
            "peak": pk["bf16"], "unit": "TFLOP/s", "frac": tflops / pk["bf16"],
            "frac_of_sustained": tflops / pk["bf16_sus"], "traffic": None,
            "peak_note": "measured bf16 dense GEMM x 1 (fp16/bf16 nominal "
                         "ratio)"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="sdk", choices=["sdk", "reference"])
    ap.add_argument("--workload", default="decode256k",
                    choices=["decode256k", "layer4k", "decode32k_b4",
                             "prefill256k_vec", "append_token_b1",
                             "append_token_b4"])
    ap.add_argument("--layers", type=int, default=None,
                    help="decode workloads: layers to instantiate (default: "
                         "the workload's 32); fewer layers make small ncu "
                         "captures and are recorded in config.layers")
    ap.add_argument("--int-softmax", action="store_true",
                    help="decode workloads: integer softmax (token-wise INT16 "
                         "logits, integer exponential); recorded in config")
    ap.add_argument("--full-softmax", action="store_true",
                    help="decode workloads: softmax over every token")
    ap.add_argument("--context-shard", action="store_true",
                    help="decode workloads: split every sequence's context "
                         "over the ranks (sdk_decode_attn_shard with NCCL "
                         "exchanges; strong scaling of one context) instead "
                         "of running one independent copy per rank")
    ap.add_argument("--kv-layout", default="separate",
                    choices=["separate", "interleaved"],
                    help="decode workloads: key and value records in two "
                         "arrays, or interleaved (a token's K and V records "
                         "in one 128-byte line)")
    ap.add_argument("--no-prefill", action="store_true",
                    help="decode256k: leave out the prefill-encode sub-record")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return dict(hbm=j["hbm_gbs"], bf16=j["bf16_tflops"],
                    bf16_sus=j["bf16_tflops_sustained"],
                    sm_max=j.get("sm_max_mhz", 1965.0), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, sm_max=1965.0,
                src="fallback")


# ----------------------------------------------------------------- clocks

class Clocks:
    """nvidia-smi samples (every 20 ms) of one GPU.  start() returns once
    the first sample has arrived, so the sampler is running when the timed
    region begins; mark(True/False) brackets the timed region, and stop()
    summarises the samples taken inside it (or, when the region is shorter
    than the sampling period, the last sample before it and the first one
    after it)."""

    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []          # (monotonic time, line)
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, ValueError):
            self.proc = None
            return
        deadline = time.monotonic() + 5.0
        while not self.lines and time.monotonic() < deadline:
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def mark(self, begin):
        if begin:
            self.t0 = time.monotonic()
        else:
            self.t1 = time.monotonic()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        t0 = self.t0 if self.t0 is not None else -1e30
        t1 = self.t1 if self.t1 is not None else 1e30
        inside = [ln for t, ln in self.lines if t0 <= t <= t1]
        if not inside:
            before = [ln for t, ln in self.lines if t < t0][-1:]
            after = [ln for t, ln in self.lines if t > t1][:1]
            inside = before + after
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        for ln in inside:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                smax.append(float(f[1]))
            except ValueError:
                continue
            for nm, v in zip(names, f[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "timed_region_ms": ((t1 - t0) * 1e3 if self.t0 is not None
                                    and self.t1 is not None else None)}


# ---------------------------------------------------------- distributed

def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "sdk":
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif args.impl == "sdk":
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """The largest x over all ranks (every rank gets it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
    return float(t.item())


# ------------------------------------------------------------ helpers

def timed_steps(step, steps, warmup, flush, world, clocks=None):
    """Runs warm-up steps, then `steps` steps each between CUDA events on
    the current stream with an L2 flush before each (outside the events).
    Returns (per-step ms list, total device ms)."""
    import torch
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
        torch.cuda.synchronize()
        clocks.mark(True)
    evs = []
    for _ in range(steps):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        step()
        b.record()
        evs.append((a, b))
    torch.cuda.synchronize()
    if clocks:
        clocks.mark(False)
    barrier(world)
    torch.cuda.synchronize()
    ck = clocks.stop() if clocks else None
    ms = [a.elapsed_time(b) for a, b in evs]
    return ms, ck


def no_flush():
    pass


def make_flush():
    import torch
    buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def flush():
        buf.zero_()
    return flush


def union_bytes(sdk, ws_list, lay, B, Hq, Hkv, N, k, full):
    """Algorithmic code bytes of one decode layer from the selected sets in
    the workspaces: 12 B per token per KV head (Klow scan) + 52 B per token
    of the GQA-group union U (Khigh rescore beyond the first 3 words) + 64 B
    per value code read (U, or every token with the full-softmax flag)."""
    import torch
    g = Hq // Hkv
    total = 0
    usum = 0
    for ws in ws_list:
        row = lay["row"]                 # per-head stride of the list
        lst = ws[lay["list"]:lay["list"] + B * Hq * row * 4].view(torch.int32)
        lst = lst.view(B, Hkv, g, row)[..., :k].long()
        mark = torch.zeros(B, Hkv, N, dtype=torch.bool, device=lst.device)
        mark.scatter_(2, lst.reshape(B, Hkv, g * k), True)
        U = int(mark.sum())
        usum += U
        total += 12 * N * B * Hkv + 52 * U + (64 * N * B * Hkv if full else 64 * U)
    return total, usum


# ---------------------------------------------------------- workloads

def workload_config(name, args):
    """The `config` object of a workload's line, shared by both arms."""
    import workloads
    if name == "prefill256k_vec":
        return {"workload": name, "n_vectors": 262144, "tokens": 16384,
                "Hkv": 8, "streams": 2, "head_dim": 128, "n_atoms": 32768,
                "k_atoms": 16, "vectors": "dense Student-t (nu=4), 4 outlier "
                "channels x10; correlated dictionaries",
                "l2": "flushed between steps (256 MiB memset)"}
    if name == "layer4k":
        return {"workload": name, "B": 1, "Hq": 32, "Hkv": 8, "head_dim": 128,
                "n_atoms": 32768, "n_tokens": 4096, "k_atoms": 16, "klow": 3,
                "khigh": 16, "top": "1/10",
                "l2": "flushed between steps (256 MiB memset)"}
    if name in APPEND_WORKLOADS:
        W = workloads.WORKLOADS[APPEND_WORKLOADS[name]]
        L = W["L"] if args.layers is None else max(1, min(W["L"], args.layers))
        return {"workload": name, "layers": L, "B": W["B"], "Hkv": W["Hkv"],
                "head_dim": W["d"], "n_atoms": W["n_atoms"], "k_atoms": 16,
                "n_new": 1, "l2": "flushed between steps; the layers' "
                "dictionaries (%.0f MB) exceed L2" % (L * 2 * W["n_atoms"] * W["d"] * 2 / 1e6)}
    W = workloads.WORKLOADS[name]
    L = W["L"] if args.layers is None else max(1, min(W["L"], args.layers))
    return {"workload": name, "layers": L, "B": W["B"], "Hq": W["Hq"],
            "Hkv": W["Hkv"], "head_dim": W["d"], "n_atoms": W["n_atoms"],
            "n_tokens": W["n_tokens"], "klow": 3, "khigh": 16, "top": "1/10",
            "softmax": ("integer (INT16 logits)" if args.int_softmax else "fp32")
                       + (", all tokens" if args.full_softmax else ", selected set"),
            "kv_layout": getattr(args, "kv_layout", "separate"),
            "l2": "not flushed: inputs larger than L2 (codes %.1f GB; every layer's "
                  "working set exceeds the 126 MB L2)"
                  % (L * W["B"] * W["Hkv"] * W["n_tokens"] * 140 / 1e9)}


def bench_layer4k(args, world, rank, pk):
    import torch
    import workloads
    import sparse_dictionary_coded_b200 as sdk
    w = workloads.layer4k(device="cuda")
    d, n, N, Hkv, Hq = w["d"], w["n_atoms"], w["n_tokens"], w["Hkv"], w["Hq"]
    if rank:
        # every rank encodes its own independent sequence (weak scaling)
        w["xk"] = torch.roll(w["xk"], shifts=rank * 7, dims=2).contiguous()
        w["xv"] = torch.roll(w["xv"], shifts=rank * 7, dims=2).contiguous()
    DK, DV, xk, xv = w["DK"], w["DV"], w["xk"], w["xv"]
    q = (w["q"] / w["q"].norm(dim=-1, keepdim=True)).contiguous()
    store = sdk.CodeStore(1, Hkv, N)
    aws = sdk.new_workspace(sdk.sdk_append_workspace_bytes(1, Hkv, N, d, n))
    dws = sdk.new_workspace(sdk.sdk_decode_workspace_bytes(1, Hq, d, n, N))
    out = torch.empty(1, Hq, d, device="cuda")
    n_vec = 2 * Hkv * N
    ev = {"enc": [], "dec": []}

    def step(record=False):
        store.lens = [0]
        if record:
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            e0.record()
        sdk.sdk_append(store, xk, xv, DK, DV, workspace=aws)
        if record:
            e1.record()
        sdk.sdk_decode_attn(q, DK, DV, store, out=out, workspace=dws)
        if record:
            e2.record()
            ev["enc"].append((e0, e1))
            ev["dec"].append((e1, e2))

    flush = make_flush()
    clocks = Clocks(torch.cuda.current_device())
    ms, ck = timed_steps(lambda: step(True), args.steps, args.warmup, flush,
                         world, clocks)
    ev["enc"] = ev["enc"][args.warmup:]
    ev["dec"] = ev["dec"][args.warmup:]
    rc, hdr = sdk.sdk_check_status(aws)
    assert rc == 0, "device check failed in append"
    rc, _ = sdk.sdk_check_status(dws)
    assert rc == 0, "device check failed in decode"
    enc_ms = statistics.mean(a.elapsed_time(b) for a, b in ev["enc"])
    dec_ms = statistics.mean(a.elapsed_time(b) for a, b in ev["dec"])
    step_ms = max_over_ranks(statistics.mean(ms), world)
    lay = sdk.sdk_decode_layout_of(1, Hq, d, n, N)
    k = (N + 9) // 10
    dec_bytes, U = union_bytes(sdk, [dws], lay, 1, Hq, Hkv, N, k, False)
    dec_bytes += 2 * n * d * 2
    flops = n_vec * enc_flop_per_vector(n, d)
    enc_tflops = flops / (enc_ms * 1e-3) / 1e12
    res = {
        "value": world * n_vec / (step_ms * 1e-3),
        "unit": ENCODE_UNIT,
        "unit_note": "whole step: encode+append 65,536 vectors, then one "
                     "decode step over 4096 tokens",
        "ms_per_step": step_ms,
        "encode": {"value": n_vec / (enc_ms * 1e-3), "unit": "vecs/s",
                   "ms": enc_ms, "tflops": enc_tflops},
        "decode": {"value": N / (dec_ms * 1e-3), "unit": "ctx tokens/s/step",
                   "ms": dec_ms, "alg_bytes": dec_bytes, "union_tokens": U,
                   "gbs": dec_bytes / (dec_ms * 1e-3) / 1e9,
                   "frac_hbm": dec_bytes / (dec_ms * 1e-3) / 1e9 / pk["hbm"]},
        "roofline": tensor_roofline(enc_tflops, pk,
                                    "encode (sdk_append: 2 x encode_tc_kernel"
                                    " + dictionary prep + scatter)"),
        "clocks": ck,
        "config": workload_config("layer4k", args),
        "dtype": ENC_DTYPE,
        # kernels per step: append = 2 x (dictionary statistics + fp16
        # dictionary copy) + one encoder over both streams + 2 scatters;
        # decode = DEC_KERNELS_PER_LAYER
        "gpu_launches": args.steps * (2 * 2 + 1 + 2 + DEC_KERNELS_PER_LAYER),
        "enc_fallback_rows": hdr[2],
    }
    if not args.no_e2e:
        res["e2e"] = e2e_layer4k(args, sdk, store, aws, dws, xk, xv, q, DK, DV,
                                 out, world, n_vec)
    return res


def e2e_layer4k(args, sdk, store, aws, dws, xk, xv, q, DK, DV, out, world,
                n_vec):
    """Same step through the public API with inputs copied from pinned host
    memory every step and the decode output read back."""
    import torch
    hxk = xk.cpu().pin_memory()
    hxv = xv.cpu().pin_memory()
    hq = q.cpu().pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    dxk, dxv, dq = torch.empty_like(xk), torch.empty_like(xv), torch.empty_like(q)

    def step():
        dxk.copy_(hxk, non_blocking=True)
        dxv.copy_(hxv, non_blocking=True)
        dq.copy_(hq, non_blocking=True)
        store.lens = [0]
        sdk.sdk_append(store, dxk, dxv, DK, DV, workspace=aws)
        sdk.sdk_decode_attn(dq, DK, DV, store, out=out, workspace=dws)
        hout.copy_(out, non_blocking=True)

    flush = make_flush()
    ms, _ = timed_steps(step, max(2, args.steps // 2), 1, flush, world)
    t = max_over_ranks(statistics.mean(ms), world)
    return {"value": world * n_vec / (t * 1e-3), "unit": ENCODE_UNIT,
            "h2d_bytes_per_step": hxk.numel() * 4 + hxv.numel() * 4 + hq.numel() * 4,
            "d2h_bytes_per_step": hout.numel() * 4, "ms_per_step": t}


def bench_decode_sharded(args, world, rank, pk, name):
    """One decode step whose every sequence is split over the ranks (rank r
    holds tokens [r N / world, (r + 1) N / world)); the exchanges between
    the stages are NCCL collectives.  Layers run one after the other (no
    CUDA graph)."""
    import torch
    import workloads
    import sparse_dictionary_coded_b200 as sdk
    from sparse_dictionary_coded_b200 import sharded
    W = workloads.WORKLOADS[name]
    L, B, Hq, Hkv, d, n, N = (W["L"], W["B"], W["Hq"], W["Hkv"], W["d"],
                              W["n_atoms"], W["n_tokens"])
    if args.layers is not None:
        L = max(1, min(L, args.layers))
    lo, hi = N * rank // world, N * (rank + 1) // world
    plans = []
    for l in range(L):
        lay = workloads.decode_layer(name, l, device="cuda")
        k_lo, k_full, v_full = workloads.layout(lay["kwords"][:, :, lo:hi].contiguous(),
                                                lay["vwords"][:, :, lo:hi].contiguous())
        del lay["kwords"], lay["vwords"]
        store = sdk.CodeStore.from_tensors(k_lo, k_full, v_full, [hi - lo] * B)
        q = (lay["q"] / lay["q"].norm(dim=-1, keepdim=True)).contiguous()
        plans.append(sharded.ShardPlan(q, lay["DK"], lay["DV"], store, [N] * B, rank, world))
    torch.cuda.synchronize()

    def step():
        for plan in plans:
            gen = sharded.shard_stages(plan)
            if world > 1:
                sharded.run_exchanges(gen)
            else:
                # one rank: a sum over ranks is the identity, a gather a copy
                for kind, t, into in gen:
                    if kind == "gather":
                        into.copy_(t)

    flush = no_flush      # inputs larger than L2, as for the unsharded decode
    timed = step
    graph = None
    if world == 1:
        # one rank: every exchange is the identity, so the stages of all
        # layers are replayed as one CUDA graph (as the unsharded step is);
        # with several ranks the NCCL exchanges run between host-driven
        # stages
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            step()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        timed = graph.replay
    clocks = Clocks(torch.cuda.current_device())
    ms, ck = timed_steps(timed, args.steps, args.warmup, flush, world, clocks)
    ms_nog = None
    if graph is not None:
        ms_nog, _ = timed_steps(step, max(2, args.steps // 2), 1, flush, world)
        del graph
    for plan in plans:
        rc, _ = sdk.sdk_check_status(plan.ws)
        assert rc == 0, "device check failed in sharded decode"
    step_ms = max_over_ranks(statistics.mean(ms), world)
    k = (N + 9) // 10
    # algorithmic bytes of the whole step (all ranks): 12 B per token per KV
    # head, 116 B per selected (token, query head) record pair, and every
    # rank reads both dictionaries
    alg = L * (12 * N * B * Hkv + 116 * k * B * Hq + world * 2 * n * d * 2)
    gbs = alg / (step_ms * 1e-3) / 1e9
    return {
        "value": B * N / (step_ms * 1e-3),
        "unit": DECODE_UNIT,
        "unit_note": "%d layers, context split over %d GPUs%s" % (
            L, world, " (one CUDA graph)" if world == 1 else ""),
        "ms_per_step": step_ms,
        **({"ms_per_step_no_graph": statistics.mean(ms_nog)} if ms_nog else {}),
        "scaling": "strong",
        "roofline": {"bound": "hbm", "kernel": "context-sharded decode step "
                     "(all stages, %d layers)" % L, "achieved": gbs,
                     "peak": world * pk["hbm"], "unit": "GB/s",
                     "frac": gbs / (world * pk["hbm"]), "traffic": None,
                     "alg_bytes_per_step": alg,
                     "note": "selected records counted per query head (no "
                             "union); peak = ranks x measured HBM copy"},
        "clocks": ck,
        "config": {"workload": name, "layers": L, "B": B, "Hq": Hq,
                   "Hkv": Hkv, "head_dim": d, "n_atoms": n, "n_tokens": N,
                   "klow": 3, "khigh": 16, "top": "1/10",
                   "parallelism": "context split over %d ranks" % world,
                   "l2": "flushed between steps"},
        "dtype": "f32 (bf16 dictionaries, fp16 coefficients)",
        # per layer: qd, klow, pass2, 3 selection stages, attend x2, out
        "gpu_launches": args.steps * L * 9,
    }


def bench_decode(args, world, rank, pk, name):
    import torch
    import workloads
    import sparse_dictionary_coded_b200 as sdk
    W = workloads.WORKLOADS[name]
    L, B, Hq, Hkv, d, n, N = (W["L"], W["B"], W["Hq"], W["Hkv"], W["d"],
                              W["n_atoms"], W["n_tokens"])
    if args.layers is not None:
        L = max(1, min(L, args.layers))
    layers = []
    for l in range(L):
        lay = workloads.decode_layer(name, l + 1000 * rank, device="cuda")
        k_lo, k_full, v_full = workloads.layout(
            lay["kwords"], lay["vwords"], interleaved=args.kv_layout == "interleaved")
        del lay["kwords"], lay["vwords"]
        store = sdk.CodeStore.from_tensors(k_lo, k_full, v_full, [N] * B)
        q = (lay["q"] / lay["q"].norm(dim=-1, keepdim=True)).contiguous()
        ws = sdk.new_workspace(sdk.sdk_decode_workspace_bytes(B, Hq, d, n, N))
        layers.append(dict(DK=lay["DK"], DV=lay["DV"], store=store, q=q, ws=ws,
                           out=torch.empty(B, Hq, d, device="cuda")))
    torch.cuda.synchronize()

    def step():
        for ly in layers:
            sdk.sdk_decode_attn(ly["q"], ly["DK"], ly["DV"], ly["store"],
                                out=ly["out"], workspace=ly["ws"],
                                full_softmax=args.full_softmax,
                                int_softmax=args.int_softmax)

    # capture the 32 layer calls in one CUDA graph
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    # no L2 flush: every layer's working set (codes, lists, QD: about 150
    # MB) and the step's codes (gigabytes) exceed the 126 MB L2, so a step
    # never finds the previous one's data there; a memset flush would
    # only leave dirty lines whose write-back lands in the timed step
    flush = no_flush
    clocks = Clocks(torch.cuda.current_device())
    ms, ck = timed_steps(g.replay, args.steps, args.warmup, flush, world, clocks)
    # serialised-layer variant without the graph, for reference
    ms_nog, _ = timed_steps(step, max(2, args.steps // 2), 1, flush, world)
    e2e = None
    if not args.no_e2e:
        # through the public API with host buffers: every layer's queries
        # copied in from pinned memory, the step replayed, every layer's
        # output read back
        hq = [ly["q"].cpu().pin_memory() for ly in layers]
        hout = torch.empty(len(layers), B, Hq, d).pin_memory()

        def e2e_step():
            for ly, h in zip(layers, hq):
                ly["q"].copy_(h, non_blocking=True)
            g.replay()
            for l, ly in enumerate(layers):
                hout[l].copy_(ly["out"], non_blocking=True)

        ms_e, _ = timed_steps(e2e_step, max(2, args.steps // 2), 1, flush, world)
        t = max_over_ranks(statistics.mean(ms_e), world)
        e2e = {"value": world * B * N / (t * 1e-3), "unit": DECODE_UNIT,
               "ms_per_step": t,
               "h2d_bytes_per_step": sum(h.numel() * 4 for h in hq),
               "d2h_bytes_per_step": hout.numel() * 4}
    # the dominant kernel (attend_kernel: Khigh rescore, softmax, value
    # scatter), timed live: a second capture of the step in which the
    # library brackets every attention launch with CUDA events on the
    # launching stream (sdk_timing_enable), replayed with the L2 flushed
    # before each replay; the headline step time above has no events in it
    sdk.sdk_timing_enable(True)
    gt = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gt):
        step()
    sdk.sdk_timing_enable(False)
    att = []
    for _ in range(max(3, args.steps // 2)):
        flush()
        gt.replay()
        torch.cuda.synchronize()
        att += sdk.sdk_timing_read(L)
    del gt
    att_ms = max_over_ranks(statistics.mean(att), world)
    for ly in layers:
        rc, _ = sdk.sdk_check_status(ly["ws"])
        assert rc == 0, "device check failed in decode"
    step_ms = max_over_ranks(statistics.mean(ms), world)
    lay = sdk.sdk_decode_layout_of(B, Hq, d, n, N)
    k = (N + 9) // 10
    code_bytes, U = union_bytes(sdk, [ly["ws"] for ly in layers], lay, B, Hq,
                                Hkv, N, k, args.full_softmax)
    alg = code_bytes + L * 2 * n * d * 2
    gbs = alg / (step_ms * 1e-3) / 1e9
    # attend's algorithmic bytes per launch: the code bytes of the layer
    # without the Klow scan's 12 B per token per KV head
    att_alg = (code_bytes - L * 12 * N * B * Hkv) / L
    att_gbs = att_alg / (att_ms * 1e-3) / 1e9
    traffic, traffic_note = (profiled_traffic("attend_kernel", name)
                             if not (args.full_softmax or args.int_softmax)
                             else (None, "no ncu summary for this flag"))
    return {
        "value": world * B * N / (step_ms * 1e-3),
        "unit": DECODE_UNIT,
        "ms_per_step": step_ms,
        "ms_per_step_no_graph": statistics.mean(ms_nog),
        "roofline": {"bound": "hbm",
                     "kernel": "attend_kernel (Khigh rescore, softmax and "
                               "value scatter; the step's largest kernel)",
                     "achieved": att_gbs, "peak": pk["hbm"], "unit": "GB/s",
                     "frac": att_gbs / pk["hbm"],
                     "traffic": traffic,
                     "traffic_source": traffic_note,
                     "alg_bytes_per_launch": att_alg,
                     "ms_per_launch": att_ms, "launches_timed": len(att),
                     "step": {"kernels": "all %d per layer, %d layers"
                                         % (DEC_KERNELS_PER_LAYER, L),
                              "achieved": gbs, "frac": gbs / pk["hbm"],
                              "alg_bytes_per_step": alg,
                              "union_tokens_per_step": U}},
        "clocks": ck,
        "config": workload_config(name, args),
        "dtype": "f32 (bf16 dictionaries, fp16 coefficients)",
        "gpu_launches": args.steps * L * DEC_KERNELS_PER_LAYER,
        **({"e2e": e2e} if e2e else {}),
    }


def bench_prefill(args, world, rank, pk):
    """The prefill encode: 16384 tokens x 8 KV heads of keys and values
    (262,144 vectors) encoded against one layer's K and V dictionaries and
    written into an empty code store, through one sdk_append call (both
    streams' row tiles in one tensor-core launch)."""
    import torch
    import workloads
    import sparse_dictionary_coded_b200 as sdk
    w = workloads.prefill(device="cuda")
    d, n, Hkv, N = w["d"], w["n_atoms"], w["Hkv"], w["n_tokens"]
    xk, xv = w["xk"].contiguous(), w["xv"].contiguous()
    if rank:
        xk, xv = xv.flip(2).contiguous(), xk.flip(2).contiguous()
    nv = Hkv * N
    store = sdk.CodeStore(1, Hkv, N)
    ws = sdk.new_workspace(sdk.sdk_append_workspace_bytes(1, Hkv, N, d, n))

    def step():
        store.lens = [0]
        sdk.sdk_append(store, xk, xv, w["DK"], w["DV"], workspace=ws)

    flush = make_flush()
    clocks = Clocks(torch.cuda.current_device())
    ms, ck = timed_steps(step, args.steps, args.warmup, flush, world, clocks)
    rc, hdr = sdk.sdk_check_status(ws)
    assert rc == 0
    step_ms = max_over_ranks(statistics.mean(ms), world)
    e2e = None
    if not args.no_e2e:
        # host vectors in (pinned), the appended code records back out
        hxk, hxv = xk.cpu().pin_memory(), xv.cpu().pin_memory()
        hck = torch.empty(store.k_full.shape, dtype=torch.int32).pin_memory()
        hcv = torch.empty(store.v_full.shape, dtype=torch.int32).pin_memory()
        dxk, dxv = torch.empty_like(xk), torch.empty_like(xv)

        def e2e_step():
            dxk.copy_(hxk, non_blocking=True)
            dxv.copy_(hxv, non_blocking=True)
            store.lens = [0]
            sdk.sdk_append(store, dxk, dxv, w["DK"], w["DV"], workspace=ws)
            hck.copy_(store.k_full, non_blocking=True)
            hcv.copy_(store.v_full, non_blocking=True)

        ms_e, _ = timed_steps(e2e_step, max(2, args.steps // 2), 1, flush, world)
        t = max_over_ranks(statistics.mean(ms_e), world)
        e2e = {"value": world * 2 * nv / (t * 1e-3), "unit": ENCODE_UNIT,
               "ms_per_step": t,
               "h2d_bytes_per_step": (hxk.numel() + hxv.numel()) * 4,
               "d2h_bytes_per_step": (hck.numel() + hcv.numel()) * 4}
    # the dominant kernel (encode_tc_kernel: both streams' row tiles in one
    # launch), timed live with the library's event hook on its stream
    sdk.sdk_timing_enable(True)
    kms = []
    for _ in range(3):
        flush()
        step()
        torch.cuda.synchronize()
        kms += sdk.sdk_timing_read(4)
    sdk.sdk_timing_enable(False)
    k_ms = max_over_ranks(statistics.mean(kms), world)
    flops = 2 * nv * enc_flop_per_vector(n, d)
    tfl = flops / (k_ms * 1e-3) / 1e12
    tfl_step = flops / (step_ms * 1e-3) / 1e12
    roof = tensor_roofline(tfl, pk, "encode_tc_kernel (one launch over both streams' "
                           "row tiles), timed live with CUDA events")
    roof.update({"ms_per_launch": k_ms, "launches_timed": len(kms),
                 "alg_flop_per_launch": flops,
                 "step": {"kernels": "sdk_append: dictionary statistics and fp16 "
                                     "copy per stream, the encoder, one code "
                                     "scatter per stream",
                          "achieved": tfl_step, "frac": tfl_step / pk["bf16"]}})
    return {
        "value": world * 2 * nv / (step_ms * 1e-3), "unit": ENCODE_UNIT,
        "ms_per_step": step_ms,
        "roofline": roof,
        "clocks": ck,
        "config": workload_config("prefill256k_vec", args),
        "dtype": ENC_DTYPE,
        # dictionary statistics + fp16 copy per stream, one encoder, one
        # scatter per stream
        "gpu_launches": args.steps * (2 * 2 + 1 + 2),
        "enc_fallback_rows": hdr[2],
        **({"e2e": e2e} if e2e else {}),
    }


APPEND_WORKLOADS = {"append_token_b1": "decode256k",
                    "append_token_b4": "decode32k_b4"}


def bench_append(args, world, rank, pk, name):
    """One generated token's append over all layers of a 32-layer decode
    workload: per layer, B x 8 new K and 8 new V vectors encoded against
    that layer's own dictionaries and written into its code store
    (sdk_append with n_new = 1, one call per layer)."""
    import torch
    import workloads
    import sparse_dictionary_coded_b200 as sdk
    base = APPEND_WORKLOADS[name]
    W = workloads.WORKLOADS[base]
    L, B, Hkv, d, n = W["L"], W["B"], W["Hkv"], W["d"], W["n_atoms"]
    if args.layers is not None:
        L = max(1, min(L, args.layers))
    cap = 4
    layers = []
    for l in range(L):
        a = workloads.append_token(base, l + 1000 * rank, device="cuda")
        layers.append(dict(DK=a["DK"], DV=a["DV"], xk=a["xk"].contiguous(),
                           xv=a["xv"].contiguous(),
                           store=sdk.CodeStore(B, Hkv, cap)))
    aws = sdk.new_workspace(sdk.sdk_append_workspace_bytes(B, Hkv, 1, d, n))
    n_vec = L * 2 * B * Hkv
    torch.cuda.synchronize()

    def step():
        for ly in layers:
            ly["store"].lens = [cap - 1] * B
            sdk.sdk_append(ly["store"], ly["xk"], ly["xv"], ly["DK"], ly["DV"],
                           workspace=aws)

    flush = make_flush()
    clocks = Clocks(torch.cuda.current_device())
    ms, ck = timed_steps(step, args.steps, args.warmup, flush, world, clocks)
    rc, _ = sdk.sdk_check_status(aws)
    assert rc == 0, "device check failed in append"
    step_ms = max_over_ranks(statistics.mean(ms), world)
    flops = n_vec * enc_flop_per_vector(n, d)
    tfl = flops / (step_ms * 1e-3) / 1e12
    res = {
        "value": world * n_vec / (step_ms * 1e-3),
        "unit": ENCODE_UNIT,
        "unit_note": "one token appended to all %d layers" % L,
        "ms_per_step": step_ms,
        "us_per_token": step_ms * 1e3,
        "us_per_layer": step_ms * 1e3 / L,
        # the correlation GEMM runs on the tensor cores; a call is 16
        # dependent greedy steps, each ending in a grid-wide exchange, so the
        # fraction is small: the step latency, not the FLOP rate, bounds it
        "roofline": dict(tensor_roofline(tfl, pk, "encode_small_kernel (%d "
                                         "launches)" % L),
                         note="latency-bound: 16 dependent steps per call, "
                              "%.1f us per step" % (step_ms * 1e3 / L / 16),
                         hbm_floor_us=L * 2 * n * d * 2 / (pk["hbm"] * 1e9) * 1e6),
        "clocks": ck,
        "config": workload_config(name, args),
        "dtype": ("f32 (residuals, exact re-scoring; tensor-core operands "
                  "bf16 with fp32 accumulation; fp16 coefficients)"),
        # per layer one kernel (the exchange words are cleared by a runtime
        # memset, not counted)
        "gpu_launches": args.steps * L,
    }
    if not args.no_e2e:
        hx = [(ly["xk"].cpu().pin_memory(), ly["xv"].cpu().pin_memory())
              for ly in layers]
        hout = torch.empty(L, 2, B, Hkv, 16, dtype=torch.int32).pin_memory()

        def e2e_step():
            for l, ly in enumerate(layers):
                ly["xk"].copy_(hx[l][0], non_blocking=True)
                ly["xv"].copy_(hx[l][1], non_blocking=True)
                ly["store"].lens = [cap - 1] * B
                sdk.sdk_append(ly["store"], ly["xk"], ly["xv"], ly["DK"],
                               ly["DV"], workspace=aws)
                hout[l, 0].copy_(ly["store"].k_full[:, :, cap - 1], non_blocking=True)
                hout[l, 1].copy_(ly["store"].v_full[:, :, cap - 1], non_blocking=True)

        ms_e, _ = timed_steps(e2e_step, max(2, args.steps // 2), 1, flush, world)
        t = max_over_ranks(statistics.mean(ms_e), world)
        res["e2e"] = {"value": world * n_vec / (t * 1e-3),
                      "unit": ENCODE_UNIT, "ms_per_step": t,
                      "h2d_bytes_per_step": sum(a.numel() * 4 + b.numel() * 4
                                                for a, b in hx),
                      "d2h_bytes_per_step": hout.numel() * 4}
    return res


# ------------------------------------------------------ oracle timings

def oracle_sampler(name):
    """The fp64 oracle on this host's cores, prepared for a bounded sample
    of the workload: returns run(budget_s) -> {value, unit, cores, kind,
    sample}, the oracle's rate scaled to the metric's unit.  The sample's
    inputs are generated once, outside every timing."""
    import numpy as np
    import torch
    import oracle
    import workloads
    cores = len(os.sched_getaffinity(0))
    torch.set_num_threads(cores)

    def encode_runner(xs, Dn, per_step, what, extra=None):
        def run(budget_s):
            t0 = time.perf_counter()
            nvec = 0
            while (time.perf_counter() - t0 < budget_s * 0.8 or nvec == 0) \
                    and nvec < xs.shape[0]:
                oracle.encode_ref(xs[nvec:nvec + 4], Dn)
                nvec += 4
            t_vec = (time.perf_counter() - t0) / nvec
            t_step = t_vec * per_step
            sample = "%d %s encoded by the oracle" % (nvec, what)
            if extra is not None:
                t_extra, note = extra()
                t_step += t_extra
                sample += note
            return {"value": per_step / t_step, "unit": ENCODE_UNIT,
                    "cores": cores, "kind": "oracle",
                    "sample": sample + "; rate scaled to the whole step"}
        return run

    if name in APPEND_WORKLOADS:
        base = APPEND_WORKLOADS[name]
        W = workloads.WORKLOADS[base]
        a = workloads.append_token(base, 0)
        xs = a["xk"].reshape(-1, a["d"]).double().numpy()
        Dn = a["DK"].float().double().numpy()
        per_step = W["L"] * 2 * W["B"] * W["Hkv"]
        return encode_runner(xs, Dn, per_step, "of the %d vectors of one token's "
                             "append" % per_step)
    if name == "layer4k":
        w = workloads.layer4k()
        xs = w["xk"].reshape(-1, w["d"]).double().numpy()
        Dn = w["DK"].float().double().numpy()
        per_step = 2 * w["Hkv"] * w["n_tokens"]
        g = workloads.make_gen(5)
        kw = workloads.random_codes((4096,), 32768, g).numpy().view(np.uint32)
        vw = workloads.random_codes((4096,), 32768, g).numpy().view(np.uint32)
        qh = np.random.default_rng(0).standard_normal(128)

        def dec():
            t1 = time.perf_counter()
            oracle.decode_head_ref(qh, kw, vw, Dn, Dn)
            return (time.perf_counter() - t1) * 32, " + 1 of 32 decode heads (4096 tokens)"
        return encode_runner(xs, Dn, per_step, "vectors", dec)
    if name == "prefill256k_vec":
        w = workloads.prefill(n_tokens=64)
        xs = w["xk"].reshape(-1, w["d"]).double().numpy()
        Dn = w["DK"].float().double().numpy()
        return encode_runner(xs, Dn, 2 * 8 * 16384, "of the 262,144 vectors")
    # decode workloads: one head of one layer, x (L*B*Hq)
    W = workloads.WORKLOADS[name]
    lay = workloads.decode_layer(name, 0, B=1)
    kw = lay["kwords"][0, 0].numpy().view(np.uint32).copy()
    vw = lay["vwords"][0, 0].numpy().view(np.uint32).copy()
    qn = lay["q"][0, 0].double().numpy()
    Dk = lay["DK"].float().double().numpy()
    Dv = lay["DV"].float().double().numpy()
    del lay
    heads = W["L"] * W["B"] * W["Hq"]

    def run(budget_s):
        t0 = time.perf_counter()
        oracle.decode_head_ref(qn, kw, vw, Dk, Dv)
        t_step = (time.perf_counter() - t0) * heads
        return {"value": W["B"] * W["n_tokens"] / t_step, "unit": DECODE_UNIT,
                "cores": cores, "kind": "oracle",
                "sample": "1 query head of 1 layer (%d tokens), time x%d for the "
                          "whole step" % (W["n_tokens"], heads)}
    return run


def cpu_baseline(name, budget_s=15.0):
    """One bounded oracle sample of the workload (see oracle_sampler)."""
    return oracle_sampler(name)(budget_s)


def reference_arm(args):
    """The oracle as the reference implementation, timed on the host cores
    with the same metric, unit and config as the sdk arm; with the default
    workload it also carries the prefill-encode sub-record."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    name = args.workload

    def arm(nm, steps, warmup):
        run = oracle_sampler(nm)
        for _ in range(warmup):
            run(0.2)
        vals = []
        t0 = time.perf_counter()
        for _ in range(max(1, steps)):
            vals.append(run(min(20.0, 90.0 / max(1, steps))))
        wall = time.perf_counter() - t0
        v = statistics.mean(x["value"] for x in vals)
        cb = dict(vals[0])
        cb["value"] = v
        return v, vals[0]["unit"], wall * 1e3 / max(1, steps), cb

    v, unit, ms, cb = arm(name, args.steps, args.warmup)
    line = {"impl": "reference", "metric": METRIC, "value": v,
            "unit": unit, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": workload_config(name, args), "cpu_baseline": cb,
            "e2e": {"value": v, "unit": unit,
                    "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    if with_prefill(args):
        pv, pu, pms, pcb = arm("prefill256k_vec", max(1, args.steps // 4), 1)
        line["prefill_encode"] = {
            "value": pv, "unit": pu, "ms_per_step": pms,
            "config": workload_config("prefill256k_vec", args),
            "cpu_baseline": pcb,
            "e2e": {"value": pv, "unit": pu, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def with_prefill(args):
    """The default decode256k line carries the prefill-encode sub-record."""
    return (args.workload == "decode256k" and not args.no_prefill and not
            (args.full_softmax or args.int_softmax or args.context_shard))


def main():
    args = parse()
    if args.impl == "reference":
        reference_arm(args)
        return
    import torch
    world, rank, local = dist_setup(args)
    import sparse_dictionary_coded_b200 as sdk
    sdk.load()
    pk = peaks()
    if args.workload == "layer4k":
        res = bench_layer4k(args, world, rank, pk)
    elif args.workload == "prefill256k_vec":
        res = bench_prefill(args, world, rank, pk)
    elif args.workload in APPEND_WORKLOADS:
        res = bench_append(args, world, rank, pk, args.workload)
    elif args.context_shard:
        res = bench_decode_sharded(args, world, rank, pk, args.workload)
    else:
        res = bench_decode(args, world, rank, pk, args.workload)
    if with_prefill(args):
        pre = bench_prefill(args, world, rank, pk)
        pre["roofline"]["peak_source"] = pk["src"]
        if world == 1 and not args.no_cpu_baseline:
            pre["cpu_baseline"] = cpu_baseline("prefill256k_vec")
        res["prefill_encode"] = pre
    if rank == 0:
        line = {"metric": METRIC, "value": res.pop("value"),
                "unit": res.pop("unit"), "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": res.pop("ms_per_step"),
                "higher_is_better": True, "scaling": res.pop("scaling", "weak"),
                "vs_baseline": None, "dtype": res.pop("dtype"),
                "data": "synthetic (seeded; shapes of the Llama-3.1-8B KV "
                        "workloads, no model or dataset)"}
        line.update(res)
        line["roofline"]["peak_source"] = pk["src"]
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args.workload)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
