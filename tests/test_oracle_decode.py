"""Pins for the decode-attention oracle (CPU only).

Method source: "LLM Inference in a Flash!", evolve.pub review, Summary and
the FAQ on the 15x KV compression: score all tokens with Klow=3 atoms,
refine the top 10% with Khigh=16.  The pins: dense attention (a library
routine) as the special case Klow=Khigh=16 over all tokens, brute-force
top-k by counting, the q*D^T gather formulation and the per-atom scatter
formulation (an independent derivation of the same numbers), ragged
lengths, the GQA head mapping and the k count of the first workload.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import workloads


def _codes(rng, N, n, nterms=16):
    idx = rng.integers(0, n, (N, nterms))
    c = rng.standard_normal((N, nterms))
    c = np.take_along_axis(c, np.argsort(-np.abs(c), axis=1), axis=1)
    return oracle.pack_words(idx, oracle.store_coef_fp16(c))


def _dict(rng, n, d):
    a = rng.standard_normal((n, d))
    return a / np.linalg.norm(a, axis=1, keepdims=True)


def test_k_count_of_the_workloads():
    # the first workload's text fixes "top 10% = 26 tokens" at N=256
    assert oracle.topk_count(256, 1, 10) == 26
    assert oracle.topk_count(4096, 1, 10) == 410
    assert oracle.topk_count(32768, 1, 10) == 3277
    assert oracle.topk_count(262144, 1, 10) == 26215
    assert oracle.topk_count(5, 1, 10) == 1
    assert oracle.topk_count(7, 1, 1) == 7


def _bruteforce_top(s, k):
    """Token t is selected iff fewer than k tokens beat it, where u beats t
    when s_u > s_t, or s_u == s_t and u < t."""
    N = len(s)
    sel = []
    for t in range(N):
        better = 0
        for u in range(N):
            if s[u] > s[t] or (s[u] == s[t] and u < t):
                better += 1
        if better < k:
            sel.append(t)
    return sel


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_select_top_bruteforce_with_ties(seed):
    rng = np.random.default_rng(seed)
    s = rng.integers(-3, 4, 60).astype(np.float64)   # many exact ties
    for k in (1, 5, 6, 17, 60):
        got = sorted(oracle.select_top(s, k).tolist())
        assert got == _bruteforce_top(s.tolist(), k)


def test_dense_special_case_equals_sdpa():
    """Klow=Khigh=16 and top 100%: attention over the decoded K^, V^ with
    scale 1/sqrt(d) -- torch's scaled_dot_product_attention in fp64."""
    rng = np.random.default_rng(1)
    n, d, N = 300, 32, 97
    DK, DV = _dict(rng, n, d), _dict(rng, n, d)
    kw, vw = _codes(rng, N, n), _codes(rng, N, n)
    q = rng.standard_normal(d)
    r = oracle.decode_head_ref(q, kw, vw, DK, DV, klow=16, khigh=16,
                               top_num=1, top_den=1)
    K = torch.from_numpy(oracle.decode_vectors(kw, DK, 16))
    V = torch.from_numpy(oracle.decode_vectors(vw, DV, 16))
    qt = torch.from_numpy(q)
    ref = torch.nn.functional.scaled_dot_product_attention(
        qt.view(1, 1, 1, d), K.view(1, 1, N, d), V.view(1, 1, N, d))
    assert np.allclose(r["out"], ref.view(d).numpy(), rtol=0, atol=1e-13)


def test_full_softmax_with_klow_equal_khigh_is_dense():
    """With the full-softmax flag and Klow=Khigh=16 every token's logit is
    its 16-atom score, so any top fraction gives dense attention."""
    rng = np.random.default_rng(2)
    n, d, N = 200, 16, 50
    DK, DV = _dict(rng, n, d), _dict(rng, n, d)
    kw, vw = _codes(rng, N, n), _codes(rng, N, n)
    q = rng.standard_normal(d)
    dense = oracle.decode_head_ref(q, kw, vw, DK, DV, 16, 16, 1, 1)["out"]
    flag = oracle.decode_head_ref(q, kw, vw, DK, DV, 16, 16, 1, 10,
                                  full_softmax=True)["out"]
    assert np.allclose(dense, flag, rtol=0, atol=1e-13)


def test_gather_and_scatter_formulations_agree():
    """The GPU formulation: QD = D_K q, s_lo_t = sum_j c_tj QD[idx_tj];
    s_t from 16 terms; w[a] = sum_t p_t sum_j c^V_tj [idx^V_tj == a];
    out = w D_V.  Derived independently here from the codes, it must give
    the oracle's numbers (which decode the vectors first)."""
    rng = np.random.default_rng(3)
    n, d, N = 512, 64, 400
    DK, DV = _dict(rng, n, d), _dict(rng, n, d)
    kw, vw = _codes(rng, N, n), _codes(rng, N, n)
    q = rng.standard_normal(d)
    r = oracle.decode_head_ref(q, kw, vw, DK, DV)
    qd = DK @ q
    ik, ck = oracle.unpack_words(kw)
    s_lo = np.sum(ck[:, :3] * qd[ik[:, :3]], axis=1)
    assert np.allclose(s_lo, r["s_lo"], rtol=1e-12, atol=1e-12)
    sel = r["sel"]
    s = np.sum(ck[sel] * qd[ik[sel]], axis=1) / math.sqrt(d)
    p = np.exp(s - s.max())
    p /= p.sum()
    assert np.allclose(p, r["p"], rtol=1e-12, atol=1e-15)
    assert r["p"].sum() == pytest.approx(1.0, abs=1e-12)
    iv, cv = oracle.unpack_words(vw)
    w = np.zeros(n)
    for pi, t in zip(p, sel):
        for j in range(16):
            w[iv[t, j]] += pi * cv[t, j]
    assert np.allclose(w @ DV, r["out"], rtol=0, atol=1e-12)


def test_selection_uses_klow_terms_only():
    """Changing atoms 3..15 of a key code must not change s_lo or the set;
    changing atom 0 must change s_lo."""
    rng = np.random.default_rng(4)
    n, d, N = 128, 16, 40
    DK, DV = _dict(rng, n, d), _dict(rng, n, d)
    kw, vw = _codes(rng, N, n), _codes(rng, N, n)
    q = rng.standard_normal(d)
    a = oracle.decode_head_ref(q, kw, vw, DK, DV)
    kw2 = kw.copy()
    kw2[:, 3:] = _codes(rng, N, n)[:, 3:]
    b = oracle.decode_head_ref(q, kw2, vw, DK, DV)
    assert np.array_equal(a["s_lo"], b["s_lo"])
    assert np.array_equal(a["sel"], b["sel"])
    kw3 = kw.copy()
    kw3[:, 0] = _codes(rng, N, n)[:, 0]
    c = oracle.decode_head_ref(q, kw3, vw, DK, DV)
    assert not np.allclose(a["s_lo"], c["s_lo"])


def test_gqa_mapping_and_ragged_lengths():
    rng = np.random.default_rng(6)
    n, d, N = 256, 16, 64
    Hq, Hkv = 4, 2
    DK, DV = _dict(rng, n, d), _dict(rng, n, d)
    kw = np.stack([np.stack([_codes(rng, N, n) for _ in range(Hkv)])
                   for _ in range(2)])
    vw = np.stack([np.stack([_codes(rng, N, n) for _ in range(Hkv)])
                   for _ in range(2)])
    q = rng.standard_normal((2, Hq, d))
    lens = [N, 23]
    out, _ = oracle.decode_attn_ref(q, kw, vw, DK, DV, lens=lens)
    for b in range(2):
        for h in range(Hq):
            kvh = h // (Hq // Hkv)
            one = oracle.decode_head_ref(q[b, h], kw[b, kvh, :lens[b]],
                                         vw[b, kvh, :lens[b]], DK, DV)
            assert np.array_equal(one["out"], out[b, h])
    # head 2 reads KV head 1, not KV head 0
    wrong = oracle.decode_head_ref(q[0, 2], kw[0, 0], vw[0, 0], DK, DV)
    assert not np.allclose(wrong["out"], out[0, 2])


def test_identical_tokens_tie_to_lowest_index():
    """All tokens carry the same key code: every score ties and the set is
    the k lowest token indices."""
    rng = np.random.default_rng(8)
    n, d, N = 64, 16, 50
    DK, DV = _dict(rng, n, d), _dict(rng, n, d)
    one = _codes(rng, 1, n)
    kw = np.repeat(one, N, axis=0)
    vw = _codes(rng, N, n)
    q = rng.standard_normal(d)
    r = oracle.decode_head_ref(q, kw, vw, DK, DV)
    assert r["sel"].tolist() == list(range(5))
    assert np.allclose(r["p"], 0.2)


def test_tiny_workload_runs():
    w = workloads.tiny()
    assert w["xk"].shape == (1, 1, 256, 64)
    assert w["DK"].dtype == torch.bfloat16
    norms = w["DK"].float().norm(dim=1)
    assert torch.all((norms - 1).abs() < 1e-2)


# ---------------------------------------------------------------- integer softmax
# Pins of oracle.integer_softmax (token-wise INT16 logits, I-BERT's integer
# exponential, fixed-point reciprocal): against the fp64 softmax, closed
# forms and the integer invariants.

def _softmax64(x):
    x = np.asarray(x, dtype=np.float64)
    e = np.exp(x - x.max())
    return e / e.sum()


def test_integer_softmax_uniform_and_single():
    for n in (1, 2, 7, 300):
        for v in (0.0, 3.5, -2.0):
            P, E, sh = oracle.integer_softmax(np.full(n, v, dtype=np.float32))
            assert np.all(P == P[0])
            # each floor loses < 1, the reciprocal's floor < E / 2^31 < n
            assert (1 << 30) - 2 * n <= int(P.sum()) <= (1 << 30)
    P, _, _ = oracle.integer_softmax(np.array([1.25], dtype=np.float32))
    assert (1 << 30) - 1 <= int(P[0]) <= (1 << 30)


def test_integer_softmax_close_to_softmax():
    """The second-order polynomial is within 0.7 % of exp on (-ln 2, 0], so
    every probability is within about 1.5 % of the fp64 softmax (plus the
    INT16 rounding of the logits)."""
    rng = np.random.default_rng(11)
    for sigma in (0.05, 0.5, 2.0, 8.0):
        for n in (3, 50, 2000):
            x = (sigma * rng.standard_normal(n)).astype(np.float32)
            P, E, sh = oracle.integer_softmax(x)
            p = P / float(1 << 30)
            ref = _softmax64(x.astype(np.float64))
            assert np.all(np.abs(p - ref) <= 0.015 * ref + 2.0 ** -28 + 2e-5 * ref.max())
            assert abs(p.sum() - 1.0) <= 2 * n * 2.0 ** -30 + 1e-12


def test_integer_softmax_two_tokens_ratio():
    for t in (0.05, 0.3, 1.0, 2.5, 5.0):
        P, _, _ = oracle.integer_softmax(np.array([0.0, -t], dtype=np.float32))
        assert abs(P[1] / P[0] / np.exp(-t) - 1.0) <= 0.012


def test_integer_softmax_monotone_and_guard():
    rng = np.random.default_rng(12)
    x = np.sort(rng.standard_normal(500)).astype(np.float32)
    P, _, sh = oracle.integer_softmax(x)
    assert np.all(np.diff(P) >= 0)
    # small logit ranges engage the bit-shift guard (S = max|l| / 32767 too
    # fine for INT32 squares); large ones do not
    assert oracle.integer_softmax(np.array([1e-4, -2e-4], dtype=np.float32))[2] > 0
    assert oracle.integer_softmax(np.array([3.0, -20.0], dtype=np.float32))[2] == 0


def test_integer_softmax_nan_is_lowest():
    P, _, _ = oracle.integer_softmax(np.array([0.5, np.nan, -0.5], dtype=np.float32))
    Q, _, _ = oracle.integer_softmax(np.array([0.5, -0.5, -0.5], dtype=np.float32))
    assert P[1] <= P[2]
    assert abs(int(P[0]) - int(Q[0])) <= int(Q[0]) // 50
