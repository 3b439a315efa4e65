"""GPU parity of the greedy-pursuit encoder (sdk_encode / sdk_encode_simt
through the C ABI) and of sdk_append against the fp64 oracle."""

import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import workloads
import sparse_dictionary_coded_b200 as sdk
from parity import check_encode, words_np

pytestmark = pytest.mark.gpu

ENCODERS = ["sdk_encode", "sdk_encode_simt"]


def _enc(fn, x, D, k=16, rsq=False):
    ws = sdk.new_workspace(sdk.sdk_encode_workspace_bytes(
        x.reshape(-1, D.shape[1]).shape[0], D.shape[1], D.shape[0]))
    res = getattr(sdk, fn)(x.cuda(), D.cuda(), k_atoms=k, resid_sqnorm=rsq,
                           workspace=ws)
    torch.cuda.synchronize()
    rc, hdr = sdk.sdk_check_status(ws)
    assert rc == 0, (rc, [hex(h) for h in hdr])
    return res, hdr


def _oracle(x, D, k=16):
    return oracle.encode_ref(x.reshape(-1, D.shape[1]).double().numpy(),
                             D.float().double().numpy(), k)


@pytest.mark.parametrize("fn", ENCODERS)
def test_tiny_workload_all_vectors(fn):
    """Workload 'tiny': all 256 K and 256 V vectors, d=64, 1024 atoms."""
    w = workloads.tiny()
    for x, D in ((w["xk"], w["DK"]), (w["xv"], w["DV"])):
        (codes, rsq), _ = _enc(fn, x, D, rsq=True)
        ref = _oracle(x, D)
        stopped = []
        compared, div = check_encode(words_np(codes), ref, stopped=stopped)
        assert compared >= 0.9 * 256 * 16
        # residual energy of the GPU encode vs the oracle's final residual,
        # for every vector whose walk ran all 16 steps (the others took a
        # different but equally valid path at a near tie)
        r_or = np.sum(ref["resid"] ** 2, axis=1)
        ok = np.abs(rsq.cpu().double().numpy() - r_or) <= 1e-3 * (r_or + 1e-6)
        full = np.setdiff1d(np.arange(256), stopped)
        assert full.size >= 0.9 * 256
        assert ok[full].all(), np.flatnonzero(~ok)[:10]


@pytest.mark.parametrize("fn", ENCODERS)
def test_layer4k_sampled_vectors(fn):
    """Workload 'layer4k' (d=128, 32768 atoms): all 32768 K vectors encoded
    on the GPU, a sample of 96 checked step by step against the oracle."""
    w = workloads.layer4k()
    x = w["xk"].reshape(-1, 128)
    codes, _ = _enc(fn, x, w["DK"])
    sample = torch.randperm(x.shape[0], generator=workloads.make_gen(1))[:96]
    ref = _oracle(x[sample], w["DK"])
    compared, div = check_encode(words_np(codes.cpu()[sample]), ref)
    assert compared >= 0.8 * 96 * 16


@pytest.mark.parametrize("fn", ENCODERS)
def test_prefill_sampled_vectors_and_certificate(fn):
    """Workload 'prefill256k_vec' at full size (262144 dense Student-t K and
    V vectors, correlated dictionaries): a sample is checked against the
    oracle's own encode and replayed by the fp64 certificate."""
    w = workloads.prefill(device="cuda")
    for x, D in ((w["xk"], w["DK"]), (w["xv"], w["DV"])):
        xf = x.reshape(-1, 128)
        codes, hdr = _enc(fn, xf, D)
        g = workloads.make_gen(2)
        sample = torch.randperm(xf.shape[0], generator=g)[:48]
        xs = xf.cpu()[sample]
        ws = words_np(codes.cpu()[sample])
        ref = _oracle(xs, D.cpu())
        check_encode(ws, ref)
        cert = oracle.certify_codes(xs.double().numpy(),
                                    D.cpu().float().double().numpy(), ws)
        assert cert["ok_pick"].all()
        assert cert["ok_coef"].all()


def _certify_many(x, D, codes, n, seed):
    """fp64 replay certificate of n sampled vectors' GPU codes: every pick
    within 1e-4 relative of its step's largest |<r, d>|, every stored
    coefficient within 1e-3 of the exact projection."""
    g = workloads.make_gen(seed)
    sample = torch.randperm(x.shape[0], generator=g)[:n]
    cert = oracle.certify_codes_batched(x.cpu()[sample].double().numpy(),
                                        D.cpu().float().double().numpy(),
                                        words_np(codes.cpu()[sample]))
    bad = np.argwhere(~(cert["ok_pick"] & cert["ok_coef"]))
    assert bad.size == 0, (bad[:5], cert["pick_ratio"][tuple(bad[0])] if bad.size else None)


def test_certificate_4096_vectors_per_stream():
    """The tensor-core encoder at full size: 4096 sampled vectors of each
    stream of the prefill workload (262144 dense Student-t vectors,
    correlated dictionaries) and 4096 of the layer4k keys, every pick and
    coefficient certified by the fp64 replay (no oracle path of its own is
    needed, so paths that diverged at a near tie are checked too)."""
    w = workloads.prefill(device="cuda")
    for s, (x, D) in enumerate(((w["xk"], w["DK"]), (w["xv"], w["DV"]))):
        xf = x.reshape(-1, 128)
        codes, _ = _enc("sdk_encode", xf, D)
        _certify_many(xf, D, codes, 4096, 30 + s)
    del w
    w = workloads.layer4k()
    x = w["xk"].reshape(-1, 128)
    codes, _ = _enc("sdk_encode", x, w["DK"])
    _certify_many(x, w["DK"], codes, 4096, 32)


@pytest.mark.parametrize("fn", ENCODERS)
def test_edge_cases(fn):
    """Ragged vector count, a zero vector (atom 0, coefficient 0 at every
    step), a scaled atom (exact first pick; the residual then shrinks by
    about 2^-10 per step towards the fp32 subnormal range, which the
    operand scaling must survive), bf16 input, fewer picks, and a
    dictionary size that fills no tile."""
    g = workloads.make_gen(21)
    n, d = 1000, 128
    D = workloads.gaussian_dictionary(n, d, g)
    x = torch.randn(77, d, generator=g)
    x[3] = 0.0
    x[5] = 2.5 * D[417].float()
    codes = _enc(fn, x, D)[0]
    ref = _oracle(x, D)
    check_encode(words_np(codes), ref)
    w = words_np(codes)
    idx, coef = oracle.unpack_words(w)
    assert np.all(idx[3] == 0) and np.all(coef[3] == 0.0)
    assert idx[5, 0] == 417 and abs(coef[5, 0] - 2.5) < 2e-3
    # bf16 input and k=5
    xb = x.to(torch.bfloat16)
    codes_b = _enc(fn, xb, D, k=5)[0]
    assert codes_b.shape == (77, 5)
    ref_b = _oracle(xb.float(), D, 5)
    check_encode(words_np(codes_b), ref_b)


def test_tensor_core_and_simt_agree_exactly():
    """Both GPU encoders pick the exact fp32 argmax and share the fp32
    arithmetic of the coefficient and residual update, so their words and
    residual energies are bit-identical (planted and dense workloads)."""
    w = workloads.layer4k()
    p = workloads.prefill(n_tokens=256)
    for x, D in ((w["xv"].reshape(-1, 128)[:4096], w["DV"]),
                 (p["xk"].reshape(-1, 128), p["DK"])):
        (a, ra), ha = _enc("sdk_encode", x, D, rsq=True)
        (b, rb), hb = _enc("sdk_encode_simt", x, D, rsq=True)
        assert torch.equal(a.cpu(), b.cpu())
        assert torch.equal(ra.cpu(), rb.cpu())


def test_candidate_overflow_falls_back_to_exact_scan():
    """Twelve identical atoms tie for the first pick: the tensor-core
    encoder's candidate list overflows, the row is re-scanned exactly, and
    the pick is the lowest of the tied indices (counted in the header).
    80 vectors: more than the small-batch encoder takes."""
    g = workloads.make_gen(41)
    n, d = 512, 64
    D = workloads.gaussian_dictionary(n, d, g)
    D[20:32] = D[300]
    x = 3.0 * D[300].float()[None, :].repeat(80, 1)
    x += 0.01 * torch.randn(80, d, generator=g)
    (codes, _), hdr = _enc("sdk_encode", x, D, rsq=True)
    idx, _ = oracle.unpack_words(words_np(codes))
    assert np.all(idx[:, 0] == 20)
    assert hdr[2] >= 80                 # rows re-scanned exactly
    ref = _oracle(x, D)
    check_encode(words_np(codes), ref)
    b = _enc("sdk_encode_simt", x, D)[0]
    assert torch.equal(codes.cpu(), b.cpu())


@pytest.mark.parametrize("interleaved", [False, True], ids=["separate", "interleaved"])
def test_append_writes_the_layout(interleaved):
    """sdk_append encodes K and V and writes k_lo planes, k_full and v_full
    records at positions lens[b]..lens[b]+n_new-1, leaving the rest (also
    with the key and value records interleaved in one array)."""
    g = workloads.make_gen(31)
    n, d, B, Hkv, cap = 2048, 128, 2, 4, 64
    DK = workloads.gaussian_dictionary(n, d, g).cuda()
    DV = workloads.gaussian_dictionary(n, d, g).cuda()
    store = sdk.CodeStore(B, Hkv, cap, interleaved=interleaved)
    store.lens = [3, 17]
    store.k_full.fill_(0x12345)
    store.v_full.fill_(0x12345)
    xk = torch.randn(B, Hkv, 5, d, generator=g).cuda()
    xv = torch.randn(B, Hkv, 5, d, generator=g).cuda()
    ws = sdk.sdk_append(store, xk, xv, DK, DV)
    torch.cuda.synchronize()
    assert sdk.sdk_check_status(ws)[0] == 0
    assert store.lens == [8, 22]
    ck = sdk.sdk_encode(xk, DK).view(B, Hkv, 5, 16)
    cv = sdk.sdk_encode(xv, DV).view(B, Hkv, 5, 16)
    for b, l0 in enumerate([3, 17]):
        assert torch.equal(store.k_full[b, :, l0:l0 + 5], ck[b])
        assert torch.equal(store.v_full[b, :, l0:l0 + 5], cv[b])
        assert torch.equal(store.k_lo[b, :, :, l0:l0 + 5],
                           ck[b, :, :, :3].transpose(-1, -2))
        for t in (store.k_full, store.v_full):
            assert torch.all(t[b, :, :l0] == 0x12345)
            assert torch.all(t[b, :, l0 + 5:] == 0x12345)
    # capacity check: 22 + 50 > 64
    with pytest.raises(sdk.SdkError):
        sdk.sdk_append(store, torch.randn(B, Hkv, 50, d).cuda(),
                       torch.randn(B, Hkv, 50, d).cuda(), DK, DV)


_BF16_OPERANDS = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
import workloads, sparse_dictionary_coded_b200 as sdk
w = workloads.layer4k()
p = workloads.prefill(n_tokens=256)
for x, D in ((w["xv"].reshape(-1, 128)[:4096], w["DV"]),
             (p["xk"].reshape(-1, 128), p["DK"])):
    x, D = x.cuda(), D.cuda()
    out = []
    for fn in (sdk.sdk_encode, sdk.sdk_encode_simt):
        ws = sdk.new_workspace(sdk.sdk_encode_workspace_bytes(x.shape[0], 128, D.shape[0]))
        c, r = fn(x, D, resid_sqnorm=True, workspace=ws)
        torch.cuda.synchronize()
        assert sdk.sdk_check_status(ws)[0] == 0
        out.append((c.cpu(), r.cpu()))
    assert torch.equal(out[0][0], out[1][0]) and torch.equal(out[0][1], out[1][1])
print("bf16 operands: identical")
"""


def test_bf16_operands_agree_exactly():
    """The tensor-core encoder with bf16 operands (SDK_ENCODE_OPERANDS=bf16,
    read once per process, hence a child process) gives the same words and
    residual energies as the CUDA-core encoder."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SDK_ENCODE_OPERANDS="bf16")
    r = subprocess.run([sys.executable, "-c", _BF16_OPERANDS, root], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "identical" in r.stdout


SMALL_CASES = [
    # (n_vec, head_dim, n_atoms, x dtype, k_atoms)
    (1, 128, 32768, torch.float32, 16),
    (7, 64, 1000, torch.bfloat16, 16),
    (33, 128, 4097, torch.float32, 5),
    (64, 128, 32768, torch.float32, 16),
    (64, 64, 3, torch.float32, 16),
    (2, 128, 1, torch.float32, 4),
]


@pytest.mark.parametrize("case", SMALL_CASES, ids=lambda c: "m%d_d%d_n%d" % c[:3])
def test_small_batch_encoder_matches_simt_exactly(case):
    """At most 64 vectors go to the atom-parallel encoder (the dictionary
    spread over all SMs, one grid barrier per greedy step).  It keeps the
    CUDA-core encoder's fp32 arithmetic, so words and residual energies are
    bit-identical to sdk_encode_simt; the picks also pass the oracle walk.
    Cases: one vector, ragged counts, a full 64-row call, dictionaries of
    1 and 3 atoms (an atom picked again and again), bf16 input, k < 16."""
    m, d, n, dt, k = case
    g = workloads.make_gen(61 + m + n)
    D = workloads.gaussian_dictionary(n, d, g)
    if n >= 16:
        x, _, _ = workloads.planted_vectors(D, m, g, noise_rel=0.05)
    else:
        x = torch.randn(m, d, generator=g)
    x = x.to(dt)
    (a, ra), _ = _enc("sdk_encode", x, D, k=k, rsq=True)
    (b, rb), _ = _enc("sdk_encode_simt", x, D, k=k, rsq=True)
    assert torch.equal(a.cpu(), b.cpu())
    assert torch.equal(ra.cpu(), rb.cpu())
    # with fewer atoms than picks the greedy coefficients shrink
    # geometrically once every atom has been taken, down to the rounding
    # noise of an fp32 dot product on either side; the oracle walk covers
    # the first min(n, k) steps there
    k_or = min(k, n)
    ref = _oracle(x.float(), D, k_or)
    check_encode(words_np(a)[:, :k_or], ref)


def test_small_batch_encoder_edge_vectors():
    """Zero vector (atom 0 with coefficient 0 at every step, as the
    CUDA-core scan leaves it), a scaled atom (exact first pick), and
    identical atoms tied for the pick (the lowest index wins) in one call."""
    g = workloads.make_gen(71)
    n, d = 32768, 128
    D = workloads.gaussian_dictionary(n, d, g)
    D[20000:20012] = D[31000]
    x = torch.randn(5, d, generator=g)
    x[0] = 0.0
    x[1] = 2.5 * D[417].float()
    x[2] = 3.0 * D[31000].float() + 0.01 * torch.randn(d, generator=g)
    (a, ra), _ = _enc("sdk_encode", x, D, rsq=True)
    (b, rb), _ = _enc("sdk_encode_simt", x, D, rsq=True)
    assert torch.equal(a.cpu(), b.cpu()) and torch.equal(ra.cpu(), rb.cpu())
    idx, coef = oracle.unpack_words(words_np(a))
    assert np.all(idx[0] == 0) and np.all(coef[0] == 0.0)
    assert idx[1, 0] == 417 and abs(coef[1, 0] - 2.5) < 2e-3
    assert idx[2, 0] == 20000


APPEND_CASES = [
    # (B, Hkv, n_new, x dtype): K and V in one launch up to 32 vectors each,
    # two launches up to 64, the tensor-core encoder beyond
    (1, 8, 1, torch.float32),
    (4, 8, 1, torch.bfloat16),
    (3, 3, 3, torch.float32),
    (5, 8, 1, torch.float32),
    (2, 8, 5, torch.float32),
]


@pytest.mark.parametrize("interleaved", [False, True], ids=["separate", "interleaved"])
@pytest.mark.parametrize("case", APPEND_CASES, ids=lambda c: "B%d_H%d_n%d" % c[:3])
def test_token_append_writes_exact_codes(case, interleaved):
    """Per-token append (the decode loop's shape): the encoder writes the
    words straight into the code store at lens[b]..lens[b]+n_new-1, the
    first 3 key words also into the k_lo planes; every word equals the
    CUDA-core encoder's and nothing else in the store changes."""
    B, Hkv, n_new, dt = case
    g = workloads.make_gen(81 + B * Hkv * n_new)
    n, d, cap = 32768, 128, 40
    DK = workloads.gaussian_dictionary(n, d, g).cuda()
    DV = workloads.gaussian_dictionary(n, d, g).cuda()
    store = sdk.CodeStore(B, Hkv, cap, interleaved=interleaved)
    lens0 = [int(v) for v in torch.randint(0, cap - n_new + 1, (B,), generator=g)]
    store.lens = list(lens0)
    for t in (store.k_lo, store.k_full, store.v_full):
        t.fill_(0x12345)
    xk = torch.randn(B, Hkv, n_new, d, generator=g).to(dt).cuda()
    xv = torch.randn(B, Hkv, n_new, d, generator=g).to(dt).cuda()
    ws = sdk.sdk_append(store, xk, xv, DK, DV)
    torch.cuda.synchronize()
    assert sdk.sdk_check_status(ws)[0] == 0
    assert store.lens == [l + n_new for l in lens0]
    ck = sdk.sdk_encode_simt(xk, DK).view(B, Hkv, n_new, 16)
    cv = sdk.sdk_encode_simt(xv, DV).view(B, Hkv, n_new, 16)
    for b, l0 in enumerate(lens0):
        assert torch.equal(store.k_full[b, :, l0:l0 + n_new], ck[b])
        assert torch.equal(store.v_full[b, :, l0:l0 + n_new], cv[b])
        assert torch.equal(store.k_lo[b, :, :, l0:l0 + n_new],
                           ck[b, :, :, :3].transpose(-1, -2))
        for t in (store.k_full, store.v_full):
            assert torch.all(t[b, :, :l0] == 0x12345)
            assert torch.all(t[b, :, l0 + n_new:] == 0x12345)
        assert torch.all(store.k_lo[b, :, :, :l0] == 0x12345)
        assert torch.all(store.k_lo[b, :, :, l0 + n_new:] == 0x12345)
    ref = _oracle(xk.float().cpu(), DK.cpu())
    check_encode(words_np(ck.reshape(-1, 16)), ref)


_SMALL_OFF = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
import workloads, sparse_dictionary_coded_b200 as sdk
g = workloads.make_gen(91)
D = workloads.gaussian_dictionary(32768, 128, g).cuda()
x = torch.randn(24, 128, generator=g).cuda()
out = []
for fn in (sdk.sdk_encode, sdk.sdk_encode_simt):
    ws = sdk.new_workspace(sdk.sdk_encode_workspace_bytes(24, 128, 32768))
    c, r = fn(x, D, resid_sqnorm=True, workspace=ws)
    torch.cuda.synchronize()
    assert sdk.sdk_check_status(ws)[0] == 0
    out.append((c.cpu(), r.cpu()))
assert torch.equal(out[0][0], out[1][0]) and torch.equal(out[0][1], out[1][1])
print("small encoder off: identical")
"""


def test_small_batch_switch_off_uses_tensor_core_encoder():
    """With SDK_ENCODE_SMALL=0 (read once per process, hence a child
    process) a 24-vector call runs the tensor-core encoder; its words still
    equal the CUDA-core encoder's."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SDK_ENCODE_SMALL="0")
    r = subprocess.run([sys.executable, "-c", _SMALL_OFF, root], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "identical" in r.stdout


def test_exchange_wait_runs_out_cleanly():
    """The small-batch encoder's per-step exchange of slice winners is the
    one device wait on other CTAs' results.  With its limit at 0 (the
    first word not there yet gives up) a 16-vector encode records
    SDK_ERR_TIMEOUT with the exchange's detail code, and the call returns.
    With the default limit back, the next calls on the same device succeed
    and their codes equal the CUDA-core encoder's bit for bit (the kernel
    that gave up left its loop, freed its tensor memory and returned; no
    copy or MMA was in flight at that wait)."""
    g = workloads.make_gen(41)
    D = workloads.gaussian_dictionary(32768, 128, g).cuda()
    x = torch.randn(16, 128, generator=g).cuda()
    prev = sdk.sdk_set_exchange_timeout_ns(0)
    try:
        seen = None
        for _ in range(5):
            ws = sdk.new_workspace(sdk.sdk_encode_workspace_bytes(16, 128, 32768))
            sdk.sdk_encode(x, D, workspace=ws)
            rc, hdr = sdk.sdk_check_status(ws)
            assert rc in (0, 5), rc
            if rc == 5:
                seen = hdr
                break
        assert seen is not None, "no exchange wait ran out in 5 calls"
        assert (seen[1] >> 24) == 0x63, hex(seen[1])
    finally:
        assert sdk.sdk_set_exchange_timeout_ns(prev) == 0
    assert prev == 1000000000
    for _ in range(2):
        codes, _ = _enc("sdk_encode", x, D)
        ref, _ = _enc("sdk_encode_simt", x, D)
        assert torch.equal(codes.cpu(), ref.cpu())


@pytest.mark.parametrize("interleaved", [False, True], ids=["separate", "interleaved"])
def test_append_both_streams_in_one_launch(interleaved):
    """An append of 600 tokens x 8 KV heads (4800 key and 4800 value
    vectors: 19 row tiles each, one tensor-core launch over all 38, the
    value tiles after the key tiles, each with its own dictionary): every
    word in the store equals the CUDA-core encoder's for its own stream,
    bf16 and fp32 inputs."""
    g = workloads.make_gen(57)
    n, d, B, Hkv, n_new, cap = 32768, 128, 1, 8, 600, 640
    DK = workloads.correlated_dictionary(n, d, g).cuda()
    DV = workloads.gaussian_dictionary(n, d, g).cuda()
    for dt in (torch.float32, torch.bfloat16):
        store = sdk.CodeStore(B, Hkv, cap, interleaved=interleaved)
        store.lens = [13]
        xk = torch.randn(B, Hkv, n_new, d, generator=g).to(dt).cuda()
        xv = torch.randn(B, Hkv, n_new, d, generator=g).to(dt).cuda()
        ws = sdk.sdk_append(store, xk, xv, DK, DV)
        torch.cuda.synchronize()
        assert sdk.sdk_check_status(ws)[0] == 0
        ck = sdk.sdk_encode_simt(xk, DK).view(B, Hkv, n_new, 16)
        cv = sdk.sdk_encode_simt(xv, DV).view(B, Hkv, n_new, 16)
        assert torch.equal(store.k_full[:, :, 13:13 + n_new], ck)
        assert torch.equal(store.v_full[:, :, 13:13 + n_new], cv)
        assert torch.equal(store.k_lo[:, :, :, 13:13 + n_new], ck[..., :3].transpose(-1, -2))
