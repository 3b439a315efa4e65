"""GPU parity of decode attention (sdk_decode_attn through the C ABI) against
the fp64 oracle, on identical codes (oracle-encoded or drawn by the input
generator; never produced by the CUDA path)."""

import math

import numpy as np
import pytest
import torch

import oracle
import workloads
import sparse_dictionary_coded_b200 as sdk
from parity import (OUT_TOL, check_selection, words_np)

pytestmark = pytest.mark.gpu


def _store(kw, vw, lens=None, cap=None):
    """Code store on the GPU from [B, Hkv, N, 16] int32 word tensors."""
    k_lo, k_full, v_full = workloads.layout(kw, vw, cap)
    B = kw.shape[0]
    lens = [kw.shape[2]] * B if lens is None else lens
    return sdk.CodeStore.from_tensors(k_lo.cuda(), k_full.cuda(),
                                      v_full.cuda(), lens)


def _unit(q):
    return q / q.norm(dim=-1, keepdim=True)


def _run(q, DK, DV, store, **kw):
    """One decode call; every token's Klow key is kept in the workspace
    (SDK_DECODE_KEEP_KEYS) so the tests can compare s_lo for all tokens."""
    kw.setdefault("keep_keys", True)
    B, Hq, d = q.shape
    ws = sdk.new_workspace(sdk.sdk_decode_workspace_bytes(
        B, Hq, d, DK.shape[0], max(store.lens)))
    out = sdk.sdk_decode_attn(q.cuda(), DK.cuda(), DV.cuda(), store,
                              workspace=ws, **kw)
    torch.cuda.synchronize()
    rc, hdr = sdk.sdk_check_status(ws)
    lay = sdk.sdk_decode_layout_of(B, Hq, d, DK.shape[0], max(store.lens))
    return out.cpu().double().numpy(), ws, lay, rc


def _gpu_sets(ws, lay, R, L, ks):
    row = lay["row"]                     # per-head stride (>= L, multiple of 4)
    lst = ws[lay["list"]:lay["list"] + R * row * 4].view(torch.int32)
    lst = lst.view(R, row).cpu().numpy()
    return [lst[r, :ks[r]] for r in range(R)]


def _gpu_keys(ws, lay, R, L):
    row = lay["row"]
    k = ws[lay["keys"]:lay["keys"] + R * row * 4].view(torch.int32)
    return k.view(R, row)[:, :L].cpu().numpy().view(np.uint32)


def _key_to_float(keys):
    keys = keys.astype(np.uint32)
    neg = (keys & 0x80000000) == 0
    b = np.where(neg, ~keys, keys & 0x7FFFFFFF).astype(np.uint32)
    return b.view(np.float32)


def _isoft_logits(ws, lay, r, k, n_b, full, keys_r, scale):
    """The fp32 logits the kernel fed its integer softmax for head r: the
    rescored selected entries (sel_score) and, with the full flag, scale *
    s_lo of the others (from their keys, in fp32 like the kernel)."""
    row = lay["row"]
    ss = ws[lay["sel_score"]:lay["sel_score"] + (r + 1) * row * 4].view(torch.float32)
    sel = ss.view(r + 1, row)[r, :k].cpu().numpy()
    if not full:
        return sel
    lst = ws[lay["list"]:lay["list"] + (r + 1) * row * 4].view(torch.int32)
    lst = lst.view(r + 1, row)[r].cpu().numpy()
    comp = lst[k:n_b]                                # the back of the list
    lo = _key_to_float(keys_r[comp])
    return np.concatenate([sel, np.float32(scale) * lo])


def _compare(q, DK, DV, kw, vw, lens, klow=3, khigh=16, top_num=1, top_den=10,
             full=False, heads=None, isoft=False, select=None):
    """Runs GPU decode and checks sets, s_lo and outputs against the oracle
    for the given (b, h) heads (all if None).  isoft: integer softmax on
    both sides, and the kernel's integer sum and guard shift recomputed
    exactly from its own fp32 logits."""
    B, Hq, d = q.shape
    store = _store(kw, vw, lens)
    out, ws, lay, rc = _run(q, DK, DV, store, klow=klow, khigh=khigh,
                            top_num=top_num, top_den=top_den,
                            full_softmax=full, int_softmax=isoft, select=select)
    assert rc == 0, "device check failed"
    L = max(lens)
    R = B * Hq
    ks = [oracle.topk_count(lens[r // Hq], top_num, top_den) for r in range(R)]
    sets = _gpu_sets(ws, lay, R, L, ks)
    keys = _gpu_keys(ws, lay, R, L)
    st = sdk.read_select_state(ws, lay, R)
    qn = q.double().numpy()
    kwn, vwn = words_np(kw), words_np(vw)
    DKn, DVn = DK.float().double().numpy(), DV.float().double().numpy()
    Hkv = kw.shape[1]
    g = Hq // Hkv
    ndiff = 0
    for r in range(R):
        b, h = divmod(r, Hq)
        if heads is not None and (b, h) not in heads:
            continue
        n_b = lens[b]
        kvh = h // g
        assert int(st["n_sel"][r]) == ks[r]
        # full softmax or select="radix": radix selection (0); select=
        # "bracket": the sampled bracket (1); the library's default: either
        path = int(st["select_path"][r])
        if full or select == "radix":
            assert path == 0, path
        elif select == "bracket":
            assert path == 1, path
        else:
            assert path in (0, 1), path
        ref = oracle.decode_head_ref(qn[b, h], kwn[b, kvh, :n_b],
                                     vwn[b, kvh, :n_b], DKn, DVn, klow, khigh,
                                     top_num, top_den, full, int_softmax=isoft)
        if isoft:
            lg = _isoft_logits(ws, lay, r, ks[r], n_b, full, keys[r],
                               1.0 / math.sqrt(d))
            _, E, sh = oracle.integer_softmax(lg)
            assert int(st["isoft_sum"][r]) == E, (r, int(st["isoft_sum"][r]), E)
            assert int(st["isoft_shift"][r]) == sh
        # s_lo of the GPU within fp32 rounding of the oracle's
        s_gpu = _key_to_float(keys[r, :n_b]).astype(np.float64)
        scale_lo = np.max(np.abs(ref["s_lo"])) + 1e-30
        assert np.max(np.abs(s_gpu - ref["s_lo"])) <= 1e-5 * scale_lo
        nd = check_selection(sets[r], ref["s_lo"], ks[r])
        ndiff += nd
        if nd:
            ref = oracle.decode_head_ref(qn[b, h], kwn[b, kvh, :n_b],
                                         vwn[b, kvh, :n_b], DKn, DVn, klow,
                                         khigh, top_num, top_den, full,
                                         force_set=sets[r], int_softmax=isoft)
        err = np.max(np.abs(out[b, h] - ref["out"]))
        assert err <= OUT_TOL, (b, h, err)
        if full:
            assert int(st["n_sel"][r]) + int(st["n_comp"][r]) == n_b
    return out, ndiff


def _random_case(seed, B, Hq, Hkv, N, d, n, lens=None, outliers=0):
    g = workloads.make_gen(seed)
    DK = workloads.gaussian_dictionary(n, d, g)
    DV = workloads.gaussian_dictionary(n, d, g)
    kw = workloads.random_codes((B, Hkv, N), n, g)
    vw = workloads.random_codes((B, Hkv, N), n, g)
    q = _unit(workloads.queries(B, Hq, d, g, n_outlier=outliers))
    lens = [N] * B if lens is None else lens
    return q, DK, DV, kw, vw, lens


def test_tiny_workload_oracle_encoded_codes():
    """Workload 'tiny': codes from the oracle's own greedy pursuit."""
    w = workloads.tiny()
    d, N = w["d"], w["n_tokens"]
    DK = w["DK"].float().double().numpy()
    DV = w["DV"].float().double().numpy()
    rk = oracle.encode_ref(w["xk"].reshape(N, d).double().numpy(), DK)
    rv = oracle.encode_ref(w["xv"].reshape(N, d).double().numpy(), DV)
    kw = oracle.pack_words(rk["idx"], oracle.store_coef_fp16(rk["coef"]))
    vw = oracle.pack_words(rv["idx"], oracle.store_coef_fp16(rv["coef"]))
    kw = torch.from_numpy(kw.view(np.int32)).view(1, 1, N, 16)
    vw = torch.from_numpy(vw.view(np.int32)).view(1, 1, N, 16)
    q = _unit(w["q"])
    for full in (False, True):
        _compare(q, w["DK"], w["DV"], kw, vw, [N], full=full)


@pytest.mark.parametrize("full,select", [(False, "radix"), (False, "bracket"), (True, None)])
def test_layer4k_shape_random_codes(full, select):
    """Workload 'layer4k' shape: 32 q / 8 KV heads, d=128, 32768 atoms,
    4096 tokens (random codes from the input generator), both selections."""
    q, DK, DV, kw, vw, lens = _random_case(77, 1, 32, 8, 4096, 128, 32768)
    _compare(q, DK, DV, kw, vw, lens, full=full, select=select)


def test_ragged_batch_small_and_odd_sizes():
    """B=3 with lengths 1, 5 and 333 (k = 1, 1, 34), GQA 6/2, d=64, 1000
    atoms (not a multiple of any tile)."""
    q, DK, DV, kw, vw, _ = _random_case(5, 3, 6, 2, 333, 64, 1000)
    lens = [1, 5, 333]
    for full in (False, True):
        _compare(q, DK, DV, kw, vw, lens, full=full)


@pytest.mark.parametrize("full,select", [(False, "radix"), (False, "bracket"), (True, None)])
def test_ragged_batch_many_ctas(full, select):
    """B=4 with lengths 9000, 40000, 2500 and 23000 (GQA 8/2, d=128, 4096
    atoms): the Klow scan and pass 2 split these unequal heads over many
    CTAs (the work split charges every head a start-up cost, so CTA bounds
    fall at arbitrary tokens of heads of different lengths).  Every head's
    keys, set and output are checked, so a token range that no CTA scanned,
    or that two did, fails."""
    q, DK, DV, kw, vw, _ = _random_case(91, 4, 8, 2, 40000, 128, 4096)
    lens = [9000, 40000, 2500, 23000]
    _compare(q, DK, DV, kw, vw, lens, full=full, select=select)


@pytest.mark.parametrize("full", [False, True])
def test_atom_count_not_a_multiple_of_eight(full):
    """1001 atoms (not a multiple of 4 or 8): the dictionary tensor maps
    read past n as zero, the weight parts of the last atoms take the scalar
    stores, and w D_V runs on the CUDA-core kernel (the tensor-core one needs
    16-byte rows of w)."""
    q, DK, DV, kw, vw, lens = _random_case(93, 2, 8, 2, 900, 128, 1001)
    _compare(q, DK, DV, kw, vw, lens, full=full)


def test_dense_special_case_matches_sdpa():
    """Klow=Khigh=16, top 100%: dense attention over the decoded keys and
    values, checked against torch SDPA in fp64 on the CPU."""
    q, DK, DV, kw, vw, lens = _random_case(9, 1, 4, 2, 300, 128, 2048)
    out, _ = _compare(q, DK, DV, kw, vw, lens, klow=16, khigh=16, top_num=1,
                      top_den=1)
    DKn, DVn = DK.double(), DV.double()
    kwn, vwn = words_np(kw), words_np(vw)
    for h in range(4):
        K = torch.from_numpy(oracle.decode_vectors(kwn[0, h // 2], DKn.numpy(), 16))
        V = torch.from_numpy(oracle.decode_vectors(vwn[0, h // 2], DVn.numpy(), 16))
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[0, h].double().view(1, 1, 1, -1), K.view(1, 1, 300, -1),
            V.view(1, 1, 300, -1)).view(-1).numpy()
        assert np.max(np.abs(out[0, h] - ref)) <= 2e-3


@pytest.mark.parametrize("full", [False, True])
def test_all_tokens_tie(full):
    """Every token carries the same key code: all s_lo tie, the selected
    set is the k lowest token indices (tie rule), p is uniform over it."""
    g = workloads.make_gen(3)
    n, d, N = 512, 64, 1000
    DK = workloads.gaussian_dictionary(n, d, g)
    DV = workloads.gaussian_dictionary(n, d, g)
    one = workloads.random_codes((1, 1, 1), n, g)
    kw = one.expand(1, 1, N, 16).contiguous()
    vw = workloads.random_codes((1, 1, N), n, g)
    q = _unit(workloads.queries(1, 2, d, g))
    store = _store(kw, vw)
    for select in ("radix", "bracket"):
        out, ws, lay, rc = _run(q, DK, DV, store, full_softmax=full, select=select)
        assert rc == 0
        sets = _gpu_sets(ws, lay, 2, N, [100, 100])
        for r in range(2):
            assert sorted(sets[r].tolist()) == list(range(100))
        _compare(q, DK, DV, kw, vw, [N], full=full, select=None if full else select)


def test_partial_ties_at_threshold():
    """Half the tokens share one code (ties across the k-th score), the rest
    random: the tie rule takes the lowest indices among the tied tokens."""
    g = workloads.make_gen(4)
    n, d, N = 512, 64, 2000
    DK = workloads.gaussian_dictionary(n, d, g)
    DV = workloads.gaussian_dictionary(n, d, g)
    kw = workloads.random_codes((1, 1, N), n, g)
    kw[0, 0, 1::2] = kw[0, 0, 7]
    vw = workloads.random_codes((1, 1, N), n, g)
    q = _unit(workloads.queries(1, 4, d, g))
    _compare(q, DK, DV, kw, vw, [N], select="radix")
    _compare(q, DK, DV, kw, vw, [N], select="bracket")
    _compare(q, DK, DV, kw, vw, [N], full=True)


def _lowbias32(x):
    """Chris Wellons' lowbias32 integer hash on uint32 numpy arrays."""
    x = np.asarray(x, dtype=np.uint64) & 0xFFFFFFFF
    x ^= x >> 16
    x = (x * 0x7FEB352D) & 0xFFFFFFFF
    x ^= x >> 15
    x = (x * 0x846CA68B) & 0xFFFFFFFF
    x ^= x >> 16
    return x


def _sampled_tokens(N, b, Hkv, kvh):
    """The tokens the decode's selection samples for KV head (b, kvh), by
    the rule include/sdk.h states for the sampled bracket: every token when
    N <= 8192, else runs of 8 tokens, one per block of blk = 8 ceil(ceil(N /
    1024) / 8) tokens, starting 8 (lowbias32(seed ^ block) mod (len / 8))
    into the block (the whole block when it holds fewer than 8 tokens)."""
    if N <= 8192:
        return np.arange(N)
    blk = 8 * ((-(-N // 1024) + 7) // 8)
    nb = -(-N // blk)
    seed = int(_lowbias32((0x9E3779B9 * (b * Hkv + kvh + 1)) & 0xFFFFFFFF))
    out = []
    for i in range(nb):
        ln = min(blk, N - i * blk)
        if ln < 8:
            out.extend(range(i * blk, i * blk + ln))
        else:
            off = 8 * int(_lowbias32(seed ^ i) % (ln // 8))
            out.extend(range(i * blk + off, i * blk + off + 8))
    return np.asarray(out, dtype=np.int64)


def test_sampled_bracket_misses_on_both_sides():
    """Planted Klow scores that make the sample unrepresentative, so that
    the k-th key falls outside the sampled bracket: KV head 0 gives its
    sampled tokens the highest scores (the bracket sits above the k-th key),
    KV head 1 the lowest (the bracket sits below it), KV head 2 draws
    scores at random (the bracket holds).  The selection must stay exact:
    heads 0 and 1 take the exact re-scan (path 2), head 2 the bracket
    (path 1); sets and outputs against the oracle.  Scores are planted
    through a dictionary whose atom a has first component x_a (increasing
    in a) and a query along the first axis, with one nonzero Klow word per
    key."""
    N, n, d, Hkv = 40000, 4096, 64, 3
    g = workloads.make_gen(21)
    x = torch.linspace(-0.95, 0.95, n, dtype=torch.float64)
    D = torch.zeros(n, d, dtype=torch.float64)
    D[:, 0] = x
    D[:, 1] = torch.sqrt(1.0 - x * x)
    DK = D.to(torch.bfloat16)
    DV = workloads.gaussian_dictionary(n, d, g)
    rng = np.random.default_rng(21)
    atoms = np.zeros((Hkv, N), dtype=np.int64)
    for kvh, kind in enumerate(("high", "low", "random")):
        smp = _sampled_tokens(N, 0, Hkv, kvh)
        rest = np.setdiff1d(np.arange(N), smp)
        if kind == "high":          # sampled: atoms 3600..4095, others 0..3500
            atoms[kvh, smp] = rng.integers(3600, n, smp.size)
            atoms[kvh, rest] = rng.integers(0, 3500, rest.size)
        elif kind == "low":         # sampled: atoms 0..499, others 600..4095
            atoms[kvh, smp] = rng.integers(0, 500, smp.size)
            atoms[kvh, rest] = rng.integers(600, n, rest.size)
        else:
            atoms[kvh] = rng.integers(0, n, N)
    one = np.uint32(oracle.pack_words(np.zeros(1, np.int64), np.ones(1))[0]) & 0xFFFF0000
    kwn = np.zeros((1, Hkv, N, 16), dtype=np.uint32)
    kwn[0, :, :, 0] = one | atoms.astype(np.uint32)
    # words 1.. carry coefficient 0 (fp16 zero bits) and random atoms
    kwn[0, :, :, 1:] = rng.integers(0, n, (Hkv, N, 15)).astype(np.uint32)
    kw = torch.from_numpy(kwn.view(np.int32))
    vw = workloads.random_codes((1, Hkv, N), n, g)
    q = torch.zeros(1, Hkv, d)
    q[0, :, 0] = 1.0
    store = _store(kw, vw)
    out, ws, lay, rc = _run(q, DK, DV, store, select="bracket")
    assert rc == 0
    st = sdk.read_select_state(ws, lay, Hkv)
    assert [int(v) for v in st["select_path"]] == [2, 2, 1]
    k = oracle.topk_count(N, 1, 10)
    assert int(st["n_above"][0]) + int(st["n_cand"][0]) < k     # bracket above the k-th key
    assert int(st["n_above"][1]) >= k                           # bracket below it
    sets = _gpu_sets(ws, lay, Hkv, N, [k] * Hkv)
    keys = _gpu_keys(ws, lay, Hkv, N)
    DKn, DVn = DK.float().double().numpy(), DV.float().double().numpy()
    for h in range(Hkv):
        ref = oracle.decode_head_ref(q[0, h].double().numpy(), kwn[0, h],
                                     words_np(vw)[0, h], DKn, DVn)
        s_gpu = _key_to_float(keys[h, :N]).astype(np.float64)
        assert np.max(np.abs(s_gpu - ref["s_lo"])) <= 1e-5 * np.max(np.abs(ref["s_lo"]))
        if check_selection(sets[h], ref["s_lo"], k):
            ref = oracle.decode_head_ref(q[0, h].double().numpy(), kwn[0, h],
                                         words_np(vw)[0, h], DKn, DVn, force_set=sets[h])
        assert np.max(np.abs(out[0, h] - ref["out"])) <= OUT_TOL


@pytest.mark.parametrize("full", [False, True])
def test_interleaved_layout(full):
    """k_full and v_full as views of one [B, Hkv, cap, 2, 16] array (a
    token's key and value records in one 128-byte line): the library
    detects the layout from v_full = k_full + 16 words; sets and outputs
    against the oracle (ragged batch of 9000 / 40000 / 2500 tokens, so the
    sampled bracket runs, and klow = 5 reads k_full words past the
    planes)."""
    q, DK, DV, kw, vw, _ = _random_case(94, 3, 8, 2, 40000, 128, 4096)
    lens = [9000, 40000, 2500]
    k_lo, k_full, v_full = workloads.layout(kw, vw, interleaved=True)
    assert v_full.data_ptr() - k_full.data_ptr() == 64
    store = sdk.CodeStore.from_tensors(k_lo.cuda(), k_full.cuda(), v_full.cuda(), lens)
    out, ws, lay, rc = _run(q, DK, DV, store, full_softmax=full)
    assert rc == 0
    ref_store = _store(kw, vw, lens)
    out_ref, _, _, rc = _run(q, DK, DV, ref_store, full_softmax=full)
    assert rc == 0
    assert np.max(np.abs(out - out_ref)) <= 1e-5
    heads = [(0, 0), (1, 7), (2, 3)]
    for klow in (3, 5):
        _compare_store(q, DK, DV, kw, vw, lens, store, klow=klow, full=full, heads=heads)


def _compare_store(q, DK, DV, kw, vw, lens, store, klow=3, full=False, heads=None):
    """_compare on a given (possibly interleaved) code store."""
    B, Hq, d = q.shape
    out, ws, lay, rc = _run(q, DK, DV, store, klow=klow, full_softmax=full)
    assert rc == 0
    R = B * Hq
    ks = [oracle.topk_count(lens[r // Hq], 1, 10) for r in range(R)]
    sets = _gpu_sets(ws, lay, R, max(lens), ks)
    qn = q.double().numpy()
    kwn, vwn = words_np(kw), words_np(vw)
    DKn, DVn = DK.float().double().numpy(), DV.float().double().numpy()
    g = Hq // kw.shape[1]
    for (b, h) in heads:
        r = b * Hq + h
        n_b = lens[b]
        ref = oracle.decode_head_ref(qn[b, h], kwn[b, h // g, :n_b], vwn[b, h // g, :n_b],
                                     DKn, DVn, klow, 16, 1, 10, full)
        if check_selection(sets[r], ref["s_lo"], ks[r]):
            ref = oracle.decode_head_ref(qn[b, h], kwn[b, h // g, :n_b], vwn[b, h // g, :n_b],
                                         DKn, DVn, klow, 16, 1, 10, full, force_set=sets[r])
        assert np.max(np.abs(out[b, h] - ref["out"])) <= OUT_TOL


def test_klow_and_khigh_variants():
    q, DK, DV, kw, vw, lens = _random_case(12, 2, 8, 4, 700, 128, 4096)
    _compare(q, DK, DV, kw, vw, lens, klow=1, khigh=8, top_num=1, top_den=4)
    _compare(q, DK, DV, kw, vw, lens, klow=5, khigh=16, top_num=3, top_den=10)


@pytest.mark.parametrize("full", [False, True])
def test_integer_softmax(full):
    """SDK_DECODE_INT_SOFTMAX: token-wise INT16 logits, I-BERT's integer
    exponential with the overflow guard, fixed-point reciprocal.  Outputs
    against the oracle's integer softmax; the kernel's integer sum and
    guard shift equal the oracle's on the kernel's own fp32 logits.  Cases:
    the tiny workload's oracle-encoded codes, the layer4k shape, a ragged
    batch, and all tokens tied."""
    w = workloads.tiny()
    d, N = w["d"], w["n_tokens"]
    DKn, DVn = w["DK"].float().double().numpy(), w["DV"].float().double().numpy()
    rk = oracle.encode_ref(w["xk"].reshape(N, d).double().numpy(), DKn)
    rv = oracle.encode_ref(w["xv"].reshape(N, d).double().numpy(), DVn)
    kw = torch.from_numpy(oracle.pack_words(rk["idx"], oracle.store_coef_fp16(rk["coef"]))
                          .view(np.int32)).view(1, 1, N, 16)
    vw = torch.from_numpy(oracle.pack_words(rv["idx"], oracle.store_coef_fp16(rv["coef"]))
                          .view(np.int32)).view(1, 1, N, 16)
    _compare(_unit(w["q"]), w["DK"], w["DV"], kw, vw, [N], full=full, isoft=True)
    q, DK, DV, kw, vw, lens = _random_case(78, 1, 32, 8, 4096, 128, 32768)
    _compare(q, DK, DV, kw, vw, lens, full=full, isoft=True,
             heads=[(0, h) for h in range(0, 32, 5)])
    q, DK, DV, kw, vw, _ = _random_case(15, 3, 6, 2, 333, 64, 1000)
    _compare(q, DK, DV, kw, vw, [1, 5, 333], full=full, isoft=True)
    g = workloads.make_gen(16)
    DK = workloads.gaussian_dictionary(512, 64, g)
    DV = workloads.gaussian_dictionary(512, 64, g)
    kw = workloads.random_codes((1, 1, 1), 512, g).expand(1, 1, 500, 16).contiguous()
    vw = workloads.random_codes((1, 1, 500), 512, g)
    _compare(_unit(workloads.queries(1, 2, 64, g)), DK, DV, kw, vw, [500], full=full,
             isoft=True)


def test_decode_flags_are_checked():
    """Flag bits other than the defined ones, and a query array that is
    not 16-byte aligned, are rejected before any launch."""
    q, DK, DV, kw, vw, lens = _random_case(17, 1, 2, 1, 64, 64, 1000)
    store = _store(kw, vw)
    lib = sdk.load()
    import ctypes
    ws = sdk.new_workspace(sdk.sdk_decode_workspace_bytes(1, 2, 64, 1000, 64))
    out = torch.empty(1, 2, 64, device="cuda")
    qd, DKd, DVd = q.cuda(), DK.cuda(), DV.cuda()
    lens_c = (ctypes.c_int32 * 1)(64)
    rc = lib.sdk_decode_attn(qd.data_ptr(), 1, 2, 1, 64, DKd.data_ptr(), DVd.data_ptr(), 1000,
                             store.k_lo.data_ptr(), store.k_full.data_ptr(),
                             store.v_full.data_ptr(), store.cap, lens_c, 3, 16, 1, 10, 32,
                             0.125, out.data_ptr(), ws.data_ptr(), ws.numel(), None)
    assert rc == 1
    qbuf = torch.zeros(1 + q.numel(), device="cuda")
    qbuf[1:] = qd.reshape(-1)
    rc = lib.sdk_decode_attn(qbuf.data_ptr() + 4, 1, 2, 1, 64, DKd.data_ptr(), DVd.data_ptr(),
                             1000, store.k_lo.data_ptr(), store.k_full.data_ptr(),
                             store.v_full.data_ptr(), store.cap, lens_c, 3, 16, 1, 10, 0,
                             0.125, out.data_ptr(), ws.data_ptr(), ws.numel(), None)
    assert rc == 1


def test_attention_kernel_timing():
    """sdk_timing_enable brackets every attention-kernel launch with CUDA
    events: two decode calls give two positive durations; once disabled,
    further calls record nothing; enabling again restarts at slot 0; two
    calls captured in a CUDA graph give two durations at every replay."""
    q, DK, DV, kw, vw, lens = _random_case(19, 1, 8, 2, 2000, 128, 4096)
    store = _store(kw, vw)
    sdk.sdk_timing_enable(True)
    try:
        for _ in range(2):
            _run(q, DK, DV, store)
        ms = sdk.sdk_timing_read(8)
        assert len(ms) == 2 and all(0.0 < t < 1000.0 for t in ms), ms
        sdk.sdk_timing_enable(False)
        _run(q, DK, DV, store)
        assert len(sdk.sdk_timing_read(8)) == 2
        sdk.sdk_timing_enable(True)
        assert sdk.sdk_timing_read(8) == []
        # calls captured in a CUDA graph keep their slots; every replay
        # records them again
        B, Hq, d = q.shape
        ws = sdk.new_workspace(sdk.sdk_decode_workspace_bytes(B, Hq, d, DK.shape[0], 2000))
        qd, DKd, DVd = q.cuda(), DK.cuda(), DV.cuda()
        out = torch.empty(B, Hq, d, device="cuda")
        sdk.sdk_decode_attn(qd, DKd, DVd, store, out=out, workspace=ws)
        torch.cuda.synchronize()
        sdk.sdk_timing_enable(True)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            sdk.sdk_decode_attn(qd, DKd, DVd, store, out=out, workspace=ws)
            sdk.sdk_decode_attn(qd, DKd, DVd, store, out=out, workspace=ws)
        sdk.sdk_timing_enable(False)
        for _ in range(2):
            g.replay()
            torch.cuda.synchronize()
            ms = sdk.sdk_timing_read(8)
            assert len(ms) == 2 and all(0.0 < t < 1000.0 for t in ms), ms
        assert sdk.sdk_check_status(ws)[0] == 0
    finally:
        sdk.sdk_timing_enable(False)


def test_bad_atom_index_is_reported_not_trapped():
    """Codes naming atom 1500 of a 1000-atom dictionary: the kernels skip
    the term and record SDK_ERR_DEVICE_CHECK with the index."""
    q, DK, DV, kw, vw, lens = _random_case(13, 1, 2, 1, 64, 64, 1000)
    kw[0, 0, 10, 0] = (kw[0, 0, 10, 0] & ~0x7FFF) | 1500
    store = _store(kw, vw)
    _, ws, _, rc = _run(q, DK, DV, store)
    assert rc == 6
    rc2, _ = sdk.sdk_check_status(ws)
    assert rc2 == 0                      # cleared by the first read


def _full_size_layer(name):
    lay = workloads.decode_layer(name, 0, device="cuda")
    k_lo, k_full, v_full = workloads.layout(lay["kwords"], lay["vwords"])
    store = sdk.CodeStore.from_tensors(k_lo, k_full, v_full, [lay["n_tokens"]] * lay["B"])
    return lay, store


@pytest.mark.parametrize("name,select", [("decode32k_b4", "bracket"), ("decode256k", "bracket"),
                                         ("decode256k", "radix")])
def test_full_size_layer_every_head(name, select):
    """One layer of the full-size decode workloads (256K tokens: 32 heads;
    32K tokens at batch 4: 128 heads) in the bench's launch configuration:
    for EVERY query head the selected set against the oracle's exact top k
    (ties only inside the band) and the output within 2e-3; then the same
    call keeping the keys, with every token's s_lo of every head within
    1e-5 of the oracle's largest score and the same sets."""
    lay, store = _full_size_layer(name)
    B, Hq, Hkv, N = lay["B"], lay["Hq"], lay["Hkv"], lay["n_tokens"]
    R, g = B * Hq, Hq // Hkv
    q = _unit(lay["q"])
    ws = sdk.new_workspace(sdk.sdk_decode_workspace_bytes(B, Hq, 128, 32768, N))
    out = sdk.sdk_decode_attn(q, lay["DK"], lay["DV"], store, workspace=ws, select=select)
    torch.cuda.synchronize()
    assert sdk.sdk_check_status(ws)[0] == 0
    layd = sdk.sdk_decode_layout_of(B, Hq, 128, 32768, N)
    k = oracle.topk_count(N, 1, 10)
    st = sdk.read_select_state(ws, layd, R)
    assert torch.all(st["n_sel"] == k)
    assert torch.all(st["select_path"] == (1 if select == "bracket" else 0))
    sets = _gpu_sets(ws, layd, R, N, [k] * R)
    outn = out.cpu().double().numpy()
    out2 = sdk.sdk_decode_attn(q, lay["DK"], lay["DV"], store, workspace=ws, keep_keys=True,
                               select=select)
    torch.cuda.synchronize()
    assert sdk.sdk_check_status(ws)[0] == 0
    sets2 = _gpu_sets(ws, layd, R, N, [k] * R)
    keys = _gpu_keys(ws, layd, R, N)
    assert np.max(np.abs(out2.cpu().double().numpy() - outn)) <= 1e-5
    qn = q.cpu().double().numpy()
    DKn = lay["DK"].cpu().float().double().numpy()
    DVn = lay["DV"].cpu().float().double().numpy()
    worst = 0.0
    for r in range(R):
        b, h = divmod(r, Hq)
        kvh = h // g
        kwn = words_np(lay["kwords"][b, kvh])
        vwn = words_np(lay["vwords"][b, kvh])
        ref = oracle.decode_head_ref(qn[b, h], kwn, vwn, DKn, DVn)
        assert set(sets[r].tolist()) == set(sets2[r].tolist())
        s_gpu = _key_to_float(keys[r, :N]).astype(np.float64)
        assert np.max(np.abs(s_gpu - ref["s_lo"])) <= 1e-5 * np.max(np.abs(ref["s_lo"]))
        if check_selection(sets[r], ref["s_lo"], k):
            ref = oracle.decode_head_ref(qn[b, h], kwn, vwn, DKn, DVn, force_set=sets[r])
        err = np.max(np.abs(outn[b, h] - ref["out"]))
        worst = max(worst, err)
        assert err <= OUT_TOL, (r, err)
    print("%s: %d heads, worst output error %.3g" % (name, R, worst))


def test_full_size_layer_integer_softmax_sampled_heads():
    """The 256K layer with the integer softmax: two sampled heads against
    the oracle's integer softmax, every head's set size and softmax mass."""
    lay, store = _full_size_layer("decode256k")
    B, Hq, N = lay["B"], lay["Hq"], lay["n_tokens"]
    q = _unit(lay["q"])
    ws = sdk.new_workspace(sdk.sdk_decode_workspace_bytes(B, Hq, 128, 32768, N))
    out = sdk.sdk_decode_attn(q, lay["DK"], lay["DV"], store, workspace=ws, int_softmax=True)
    torch.cuda.synchronize()
    assert sdk.sdk_check_status(ws)[0] == 0
    layd = sdk.sdk_decode_layout_of(B, Hq, 128, 32768, N)
    st = sdk.read_select_state(ws, layd, B * Hq)
    k = oracle.topk_count(N, 1, 10)
    assert torch.all(st["n_sel"] == k)
    assert torch.all(st["z"] >= 1.0)          # the max term's INT16 exponential
    assert torch.isfinite(out).all()
    R = B * Hq
    sets = _gpu_sets(ws, layd, R, N, [k] * R)
    qn = q.cpu().double().numpy()
    DKn = lay["DK"].cpu().float().double().numpy()
    DVn = lay["DV"].cpu().float().double().numpy()
    outn = out.cpu().double().numpy()
    for (b, h) in [(0, 0), (B - 1, Hq - 1)]:
        kvh = h // (Hq // lay["Hkv"])
        kwn = words_np(lay["kwords"][b, kvh])
        vwn = words_np(lay["vwords"][b, kvh])
        ref = oracle.decode_head_ref(qn[b, h], kwn, vwn, DKn, DVn, int_softmax=True)
        r = b * Hq + h
        if check_selection(sets[r], ref["s_lo"], k):
            ref = oracle.decode_head_ref(qn[b, h], kwn, vwn, DKn, DVn,
                                         force_set=sets[r], int_softmax=True)
        assert np.max(np.abs(outn[b, h] - ref["out"])) <= OUT_TOL


_QD_PATH_CASES = (("b1", (81, 1, 32, 8, 2000, 128, 32768)),
                  ("b2", (83, 2, 32, 8, 900, 64, 2048)),
                  ("b4", (82, 4, 32, 8, 600, 128, 4096)),
                  ("b2-640", (84, 2, 32, 8, 700, 128, 640)),
                  ("b1-d64", (86, 1, 32, 8, 1500, 64, 4096)),
                  ("b2-128", (85, 2, 32, 8, 300, 128, 128)),
                  ("b8", (87, 8, 32, 8, 200, 128, 2048)),
                  ("b3-h12", (88, 3, 12, 4, 400, 128, 1024)))
_QD_PATH_CASE = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
sys.path.insert(0, sys.argv[1] + "/tests")
import workloads, sparse_dictionary_coded_b200 as sdk
from test_gpu_decode import _random_case, _store, _QD_PATH_CASES
for name, args in _QD_PATH_CASES:
    q, DK, DV, kw, vw, lens = _random_case(*args)
    B, Hq, d = q.shape
    store = _store(kw, vw, lens)
    n = DK.shape[0]
    ws = sdk.new_workspace(sdk.sdk_decode_workspace_bytes(B, Hq, d, n, max(lens)))
    out = sdk.sdk_decode_attn(q.cuda(), DK.cuda(), DV.cuda(), store, workspace=ws)
    torch.cuda.synchronize()
    assert sdk.sdk_check_status(ws)[0] == 0
    lay = sdk.sdk_decode_layout_of(B, Hq, d, n, max(lens))
    qd = ws[lay["qd"]:lay["qd"] + B * Hq * n * 4].view(torch.float32).cpu().numpy()
    row = lay["row"]
    lst = ws[lay["list"]:lay["list"] + B * Hq * row * 4].view(torch.int32)
    np.save(sys.argv[2] + "/qd_" + name + ".npy", qd)
    np.save(sys.argv[2] + "/out_" + name + ".npy", out.cpu().numpy())
    np.save(sys.argv[2] + "/list_" + name + ".npy", lst.view(B * Hq, row).cpu().numpy())
print("saved")
"""


def test_gemvs_on_cuda_cores_match_tensor_cores(tmp_path):
    """D1 and D6 run on the tensor cores (q and w split into three bf16
    parts) unless SDK_DECODE_QD_TC=0 / SDK_DECODE_OUT_TC=0 select the fp32
    CUDA-core kernels (read once per process, hence child processes): both
    give QD within fp32 rounding of each other and the same outputs, and
    both paths' outputs match the oracle (first and last head of every
    case).  The w D_V cases cover 32, 64 and 128 query rows (row tiles of
    32, 64, 128), 256 rows (two row tiles of 128), 36 rows (a tile of 64
    with 28 empty rows), head_dim 64 at 32 and 64 rows (the zero upper half
    of the operand), 640 atoms (ten chunks over eight CTAs) and 128 atoms
    (two chunks: two of the cluster's four CTAs have no atoms)."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = {}
    for mode in ("1", "0"):
        d = tmp_path / mode
        d.mkdir()
        env = dict(os.environ, SDK_DECODE_QD_TC=mode, SDK_DECODE_OUT_TC=mode)
        r = subprocess.run([sys.executable, "-c", _QD_PATH_CASE, root, str(d)],
                           env=env, capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stdout + r.stderr
        res[mode] = d
    for name, args in _QD_PATH_CASES:
        qa = np.load(res["1"] / ("qd_" + name + ".npy"))
        qb = np.load(res["0"] / ("qd_" + name + ".npy"))
        assert np.max(np.abs(qa - qb)) <= 2e-6 * np.max(np.abs(qb))
        oa = np.load(res["1"] / ("out_" + name + ".npy"))
        ob = np.load(res["0"] / ("out_" + name + ".npy"))
        assert np.max(np.abs(oa - ob)) <= 1e-5, name
        q, DK, DV, kw, vw, lens = _random_case(*args)
        B, Hq, d = q.shape
        Hkv = kw.shape[1]
        qn = q.double().numpy()
        kwn, vwn = words_np(kw), words_np(vw)
        DKn, DVn = DK.float().double().numpy(), DV.float().double().numpy()
        for mode in ("1", "0"):
            out = np.load(res[mode] / ("out_" + name + ".npy"))
            lst = np.load(res[mode] / ("list_" + name + ".npy"))
            for b, h in ((0, 0), (B - 1, Hq - 1)):
                kvh = h // (Hq // Hkv)
                n_b = lens[b]
                k = oracle.topk_count(n_b, 1, 10)
                ref = oracle.decode_head_ref(qn[b, h], kwn[b, kvh, :n_b],
                                             vwn[b, kvh, :n_b], DKn, DVn)
                sel = lst[b * Hq + h, :k]
                if check_selection(sel, ref["s_lo"], k):
                    ref = oracle.decode_head_ref(qn[b, h], kwn[b, kvh, :n_b],
                                                 vwn[b, kvh, :n_b], DKn, DVn,
                                                 force_set=sel)
                err = np.max(np.abs(out[b, h] - ref["out"]))
                assert err <= OUT_TOL, (name, mode, b, h, err)
