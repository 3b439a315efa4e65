"""Pins for the encode oracle (CPU only).

Every check here is tied to something other than the oracle's own code: a
hand-derived worked example, brute force in plain Python loops, exact
recovery of planted codes, the energy identity of greedy pursuit over
unit-norm atoms, and special cases with a closed form.  Method source: "LLM
Inference in a Flash!", evolve.pub review, Summary (projection-based greedy
pursuit, K=16 atoms, no least-squares refit).
"""

import json
import math
import os

import numpy as np
import pytest

import oracle
import workloads

HERE = os.path.dirname(os.path.abspath(__file__))


def _unit_rows(rng, n, d):
    a = rng.standard_normal((n, d))
    return a / np.linalg.norm(a, axis=1, keepdims=True)


def test_hand_worked_example():
    g = json.load(open(os.path.join(HERE, "golden", "hand_example.json")))
    for case in g["cases"]:
        idx, coef, gap, r = oracle.greedy_pursuit(
            np.array(case["x"]), np.array(case["D"]), g["k_atoms"])
        for j, (ei, ec) in enumerate(zip(case["idx"], case["coef"])):
            if ei < 0:
                assert abs(coef[j]) < 1e-12
            else:
                assert idx[j] == ei, (case, j, idx)
                assert coef[j] == pytest.approx(ec, abs=1e-12)


def _bruteforce_pick(r, D):
    """Plain Python: the index of the largest |<r, d_i>| (lowest i on ties)
    and that inner product."""
    best_i, best_a, best_c = 0, -1.0, 0.0
    for i in range(len(D)):
        c = 0.0
        for k in range(len(r)):
            c += r[k] * D[i][k]
        if abs(c) > best_a:
            best_i, best_a, best_c = i, abs(c), c
    return best_i, best_c


def test_bruteforce_certificate_tiny_workload():
    """Recompute every greedy pick of a few 'tiny' vectors with plain loops
    from x and the emitted codes (no numpy arithmetic on the check side)."""
    w = workloads.tiny()
    D = w["DK"].float().double().numpy()
    X = w["xk"].reshape(-1, w["d"]).double().numpy()[:3]
    ref = oracle.encode_ref(X, D)
    Dl = D.tolist()
    for v in range(X.shape[0]):
        r = X[v].tolist()
        for j in range(16):
            i, c = _bruteforce_pick(r, Dl)
            if ref["gap"][v, j] > 1e-9:
                assert i == ref["idx"][v, j]
            assert c == pytest.approx(ref["coef"][v, j], rel=1e-9, abs=1e-12)
            ii = ref["idx"][v, j]
            cc = ref["coef"][v, j]
            r = [r[k] - cc * Dl[ii][k] for k in range(len(r))]
        assert np.allclose(r, ref["resid"][v], atol=1e-12)


@pytest.mark.parametrize("n,d", [(64, 64), (4096, 32), (1024, 64)])
def test_energy_identity_unit_atoms(n, d):
    """For exactly unit atoms, ||r_{j+1}||^2 = ||r_j||^2 - coef_j^2, hence
    ||x||^2 = ||r_16||^2 + sum coef^2 (orthonormal or not)."""
    rng = np.random.default_rng(7)
    if n == d:
        D, _ = np.linalg.qr(rng.standard_normal((d, d)))
        D = D.T.copy()
    else:
        D = _unit_rows(rng, n, d)
    X = rng.standard_normal((20, d))
    ref = oracle.encode_ref(X, D)
    lhs = np.sum(X * X, axis=1)
    rhs = np.sum(ref["resid"] ** 2, axis=1) + np.sum(ref["coef"] ** 2, axis=1)
    assert np.allclose(lhs, rhs, rtol=1e-12, atol=0)
    # the residual decreases monotonically
    assert np.all(np.sum(ref["resid"] ** 2, axis=1) <= lhs)


def test_exact_recovery_orthonormal():
    """Planted 16-sparse x over an orthonormal basis with distinct |coef|:
    greedy returns the support in order of decreasing |coef|, coefficients
    exact, residual zero."""
    rng = np.random.default_rng(11)
    d = 64
    Q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    D = Q.T.copy()       # rows orthonormal; Q is not symmetric
    for trial in range(10):
        supp = rng.choice(d, 16, replace=False)
        mags = np.sort(rng.uniform(0.5, 4.0, 16))[::-1]
        mags = mags + np.arange(16)[::-1] * 1e-3   # keep them distinct
        signs = rng.choice([-1.0, 1.0], 16)
        a = mags * signs
        x = a @ D[supp]
        idx, coef, gap, r = oracle.greedy_pursuit(x, D)
        assert list(idx) == list(supp)
        assert np.allclose(coef, a, atol=1e-12, rtol=0)
        assert np.linalg.norm(r) < 1e-12


def _hadamard(d):
    H = np.array([[1.0]])
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])
    return H


def test_near_orthogonal_recovery_identity_union_hadamard():
    """D = I u H/sqrt(d): mutual coherence mu = 1/sqrt(d).

    * K <= 6 < (1 + 1/mu)/2 planted atoms satisfy Tropp's exact recovery
      condition, under which matching pursuit only ever picks atoms of the
      planted support (until the residual is exactly zero, after which the
      zero-residual reading gives coefficient 0).
    * With K=4 and magnitudes decaying x0.5, the first four picks are the
      planted atoms in order, each coefficient within the coherence bound
      mu * sum_l |a_l| of its planted value.
    """
    d = 128
    D = np.vstack([np.eye(d), _hadamard(d) / math.sqrt(d)])
    mu = 1.0 / math.sqrt(d)
    rng = np.random.default_rng(5)
    for trial in range(40):
        K = 6
        supp = rng.choice(D.shape[0], K, replace=False)
        a = rng.uniform(0.5, 2.0, K) * rng.choice([-1.0, 1.0], K)
        x = a @ D[supp]
        idx, coef, gap, r = oracle.greedy_pursuit(x, D)
        for j in range(16):
            assert idx[j] in supp or abs(coef[j]) <= 1e-12 * np.linalg.norm(x)
        assert np.linalg.norm(r) < np.linalg.norm(x)
    for trial in range(40):
        K = 4
        supp = rng.choice(D.shape[0], K, replace=False)
        a = (0.5 ** np.arange(K)) * rng.choice([-1.0, 1.0], K) * 3.0
        x = a @ D[supp]
        idx, coef, gap, r = oracle.greedy_pursuit(x, D)
        assert list(idx[:K]) == list(supp)
        bound = mu * np.sum(np.abs(a))
        assert np.all(np.abs(coef[:K] - a) <= bound)


def test_first_pick_and_zero_residual():
    """x = 3 d_5 over unit atoms: atom 5 with coefficient 3, then the zero
    residual gives atom 0 with coefficient 0 at every later step."""
    rng = np.random.default_rng(3)
    D = _unit_rows(rng, 50, 16)
    x = 3.0 * D[5]
    idx, coef, gap, r = oracle.greedy_pursuit(x, D)
    assert idx[0] == 5 and coef[0] == pytest.approx(3.0, abs=1e-12)
    assert np.linalg.norm(r) < 1e-12
    assert np.all(np.abs(coef[1:]) < 1e-12)


def test_negative_dominant_projection_uses_magnitude():
    """The pick maximises |<r,d>|, not <r,d>: a negative dominant projection
    must win and keep its sign."""
    d = 8
    D = np.eye(d)
    x = np.zeros(d)
    x[7] = -2.0
    x[3] = 0.5
    idx, coef, _, r = oracle.greedy_pursuit(x, D, k_atoms=2)
    assert list(idx) == [7, 3]
    assert coef[0] == -2.0 and coef[1] == 0.5


def test_ties_go_to_lowest_index():
    d = 4
    D = np.eye(d)[[0, 1, 2, 1]]          # atom 3 duplicates atom 1
    x = np.array([0.0, 2.0, 0.0, 0.0])
    idx, coef, gap, _ = oracle.greedy_pursuit(x, D, k_atoms=1)
    assert idx[0] == 1 and gap[0] == 0.0
    D2 = np.vstack([np.eye(d), -np.eye(d)[0:1]])    # atom 4 = -atom 0
    x2 = np.array([-1.5, 0.0, 0.0, 0.0])
    idx, coef, gap, _ = oracle.greedy_pursuit(x2, D2, k_atoms=1)
    assert idx[0] == 0 and coef[0] == -1.5


def test_gap_definition():
    D = np.eye(3)
    x = np.array([1.0, -0.9, 0.1])
    _, _, gap, _ = oracle.greedy_pursuit(x, D, k_atoms=1)
    assert gap[0] == pytest.approx(0.1)


def test_fp16_storage_rounding_and_saturation():
    c = np.array([1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 70000.0, -1e6,
                  65504.0, 2.0 ** -26, -0.0])
    h = oracle.store_coef_fp16(c)
    assert h[0] == np.float16(1.0)                    # tie -> even
    assert h[1] == np.float16(1.0 + 2.0 ** -9)        # tie -> even (up)
    assert h[2] == np.float16(65504.0) and h[3] == np.float16(-65504.0)
    assert h[4] == np.float16(65504.0)
    assert np.isfinite(h).all()


def test_word_format_bits():
    w = oracle.pack_words(np.array([5, 32767, 0]),
                          np.array([1.0, -2.0, 0.0], dtype=np.float16))
    assert w.dtype == np.uint32
    assert int(w[0]) == 0x3C000005
    assert int(w[1]) == 0xC0007FFF
    assert int(w[2]) == 0
    idx, coef = oracle.unpack_words(w)
    assert idx.tolist() == [5, 32767, 0]
    assert coef.tolist() == [1.0, -2.0, 0.0]
    with pytest.raises(ValueError):
        oracle.pack_words(np.array([32768]), np.array([1.0], np.float16))


def test_generator_word_format_matches_oracle_unpack():
    """The input generator's word packing and the oracle's unpacking agree
    on the storage format (bit 15 of every word is zero)."""
    import torch
    g = workloads.make_gen(1)
    w = workloads.random_codes((3, 5), 32768, g)
    wn = w.numpy().view(np.uint32)
    assert np.all((wn & 0x8000) == 0)
    idx, coef = oracle.unpack_words(wn)
    assert idx.max() < 32768
    assert np.all(np.diff(np.abs(coef), axis=-1) <= 0)   # |coef| descending
    assert torch.equal(torch.from_numpy(wn.view(np.int32)), w)
