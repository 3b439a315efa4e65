"""Pins of the OMP oracle (the least-squares-refit encoder that the pages'
projection-based greedy pursuit replaces; evolve.pub review of "LLM
Inference in a Flash!", Summary and Strengths)."""

import numpy as np

import oracle
from oracle.omp import omp, omp_ref


def _orthonormal(n, seed):
    q, _ = np.linalg.qr(np.random.default_rng(seed).standard_normal((n, n)))
    return q.T          # rows orthonormal


def _hadamard(d):
    h = np.array([[1.0]])
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h / np.sqrt(d)


def test_orthonormal_dictionary_omp_equals_greedy():
    """With orthonormal atoms the projection of r on d_i is the least-squares
    coefficient, so the refit changes nothing: same picks, same
    coefficients, same residual as the greedy pursuit."""
    D = _orthonormal(32, 1)
    x = np.random.default_rng(2).standard_normal(32)
    i_o, c_o, r_o = omp(x, D, 8)
    i_g, c_g, _, r_g = oracle.greedy_pursuit(x, D, 8)
    assert np.array_equal(i_o, i_g)
    np.testing.assert_allclose(c_o, c_g, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r_o, r_g, rtol=0, atol=1e-12)


def test_residual_orthogonal_to_every_picked_atom():
    """After every step r is orthogonal to the span of the picked atoms (the
    normal equations of the refit), and no atom is picked twice."""
    rng = np.random.default_rng(3)
    D = rng.standard_normal((200, 32))
    D /= np.linalg.norm(D, axis=1, keepdims=True)
    x = rng.standard_normal(32)
    for k in (1, 4, 10, 20):
        idx, coef, r = omp(x, D, k)
        assert np.max(np.abs(D[idx] @ r)) <= 1e-10 * np.linalg.norm(x)
        assert len(set(idx.tolist())) == k
        np.testing.assert_allclose(x - D[idx].T @ coef, r, rtol=0, atol=1e-12)


def test_exact_recovery_where_greedy_pursuit_is_inexact():
    """Identity + Hadamard atoms in d=64 have coherence 1/8; OMP recovers
    every 4-sparse combination exactly in 4 steps (4 < (1 + 8) / 2, Tropp's
    exact-recovery condition).  The greedy pursuit picks the same atoms here
    but, without the refit, keeps a residual after 4 steps whenever the
    planted atoms are not orthogonal."""
    d = 64
    D = np.vstack([np.eye(d), _hadamard(d)])
    rng = np.random.default_rng(4)
    for trial in range(20):
        sup = np.concatenate([rng.choice(d, 2, replace=False),
                              d + rng.choice(d, 2, replace=False)])
        a = rng.standard_normal(4) + np.sign(rng.standard_normal(4))
        x = D[sup].T @ a
        idx, coef, r = omp(x, D, 4)
        assert set(idx.tolist()) == set(sup.tolist())
        got = dict(zip(idx.tolist(), coef.tolist()))
        for s, v in zip(sup.tolist(), a.tolist()):
            assert abs(got[s] - v) <= 1e-10
        assert np.linalg.norm(r) <= 1e-12 * np.linalg.norm(x)
        _, _, _, r_g = oracle.greedy_pursuit(x, D, 4)
        assert np.linalg.norm(r_g) > 1e-6 * np.linalg.norm(x)


def test_first_step_refit_divides_by_the_atom_norm():
    """Hand-sized case with atoms that are not unit norm: OMP's first
    coefficient is <x, d>/||d||^2 (the least-squares fit), the greedy
    pursuit's is <x, d>; the second step's refit equals the 2x2
    normal-equations solution written out by hand."""
    D = np.array([[2.0, 0.0, 0.0],
                  [0.0, 1.0, 1.0],
                  [1.0, 1.0, 0.0]])
    x = np.array([3.0, 1.0, 0.5])
    idx, coef, r = omp(x, D, 1)
    c = D @ x                      # [6, 1.5, 4]
    assert idx[0] == 0
    assert abs(coef[0] - 6.0 / 4.0) <= 1e-15
    _, c_g, _, _ = oracle.greedy_pursuit(x, D, 1)
    assert abs(c_g[0] - 6.0) <= 1e-15
    # step 2: r1 = x - 1.5 d0 = (0, 1, 0.5); D r1 = (0, 1.5, 1) -> atom 1
    idx, coef, r = omp(x, D, 2)
    assert idx.tolist() == [0, 1]
    A = D[[0, 1]]
    G = A @ A.T                    # [[4, 0], [0, 2]]
    sol = np.linalg.solve(G, A @ x)
    assert abs(sol[0] - 1.5) <= 1e-15 and abs(sol[1] - 0.75) <= 1e-15
    np.testing.assert_allclose(coef, sol, rtol=0, atol=1e-14)
    np.testing.assert_allclose(r, x - A.T @ sol, rtol=0, atol=1e-14)
    assert c[0] == 6.0


def test_refit_is_the_least_squares_minimum_over_its_support():
    """Perturbing any refitted coefficient never lowers ||r|| (the refit is
    the minimum over the picked support), and on the greedy pursuit's own
    support the least-squares residual is never above the greedy one."""
    rng = np.random.default_rng(5)
    D = rng.standard_normal((300, 24))
    D /= np.linalg.norm(D, axis=1, keepdims=True)
    X = rng.standard_normal((10, 24))
    ref = omp_ref(X, D, 6)
    for v in range(10):
        idx, coef = ref["idx"][v], ref["coef"][v]
        base = np.linalg.norm(ref["resid"][v])
        for j in range(6):
            for eps in (1e-3, -1e-3):
                c2 = coef.copy()
                c2[j] += eps
                assert np.linalg.norm(X[v] - D[idx].T @ c2) >= base
        i_g, _, _, r_g = oracle.greedy_pursuit(X[v], D, 6)
        a, *_ = np.linalg.lstsq(D[i_g].T, X[v], rcond=None)
        assert np.linalg.norm(X[v] - D[i_g].T @ a) <= np.linalg.norm(r_g) + 1e-12
