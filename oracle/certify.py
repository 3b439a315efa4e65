"""Oracle: fp64 replay certificate for codes produced elsewhere.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Given x, the dictionary and someone else's 16 picks, replay the greedy
pursuit of "LLM Inference in a Flash!" (evolve.pub review, Summary) in fp64
along THOSE picks: at each step recompute every |<r, d_i>|, check that the
picked atom is within ``rel_tol`` of that step's maximum, and continue with
the exact fp64 projection of the picked atom.  This checks a code path that
legitimately diverged from the oracle's own picks at a near tie, and it needs
no oracle encode of its own.
"""

import numpy as np

from .encode import unpack_words


def certify_codes(X, D, words, rel_tol=1e-4, coef_rel_tol=1e-3):
    """Replay ``words`` ([m, k] uint32) for rows of ``X`` ([m, d]).

    Returns a dict of arrays, one entry per (vector, step):
      pick_ratio  |c_pick| / max_i |c_i|   (1.0 when the pick is the argmax)
      coef_err    |stored coef - exact projection| / |exact projection|
    and booleans ``ok_pick`` (ratio >= 1 - rel_tol, or a zero residual) and
    ``ok_coef`` (coef_err <= coef_rel_tol, or both coefficients tiny
    relative to ||x||).
    """
    X = np.asarray(X, dtype=np.float64)
    D = np.asarray(D, dtype=np.float64)
    idx, coef_st = unpack_words(words)
    m, k = idx.shape
    ratio = np.ones((m, k))
    cerr = np.zeros((m, k))
    ok_pick = np.ones((m, k), dtype=bool)
    ok_coef = np.ones((m, k), dtype=bool)
    for v in range(m):
        r = X[v].copy()
        xnorm = np.linalg.norm(X[v])
        for j in range(k):
            c = D @ r
            a = np.abs(c)
            top = a.max()
            i = idx[v, j]
            if top > 0.0:
                ratio[v, j] = a[i] / top
                ok_pick[v, j] = ratio[v, j] >= 1.0 - rel_tol
            exact = c[i]
            if abs(exact) > 1e-12 * max(xnorm, 1e-300):
                cerr[v, j] = abs(coef_st[v, j] - exact) / abs(exact)
                ok_coef[v, j] = cerr[v, j] <= coef_rel_tol
            else:
                ok_coef[v, j] = abs(coef_st[v, j]) <= 1e-6 * max(xnorm, 1.0)
            r = r - exact * D[i]
    return {"pick_ratio": ratio, "coef_err": cerr, "ok_pick": ok_pick,
            "ok_coef": ok_coef}


def certify_codes_batched(X, D, words, rel_tol=1e-4, coef_rel_tol=1e-3,
                          batch=256):
    """certify_codes for many vectors: the same replay, step for step, for a
    batch of vectors at a time (each step's inner products of the batch's
    residuals with all atoms as one matrix product).  Same return value."""
    X = np.asarray(X, dtype=np.float64)
    D = np.asarray(D, dtype=np.float64)
    idx, coef_st = unpack_words(words)
    m, k = idx.shape
    ratio = np.ones((m, k))
    cerr = np.zeros((m, k))
    ok_pick = np.ones((m, k), dtype=bool)
    ok_coef = np.ones((m, k), dtype=bool)
    Dt = np.ascontiguousarray(D.T)
    for v0 in range(0, m, batch):
        sl = slice(v0, min(m, v0 + batch))
        R = X[sl].copy()
        rows = np.arange(R.shape[0])
        xnorm = np.linalg.norm(R, axis=1)
        for j in range(k):
            C = R @ Dt                          # [b, n] all <r, d_i>
            top = np.abs(C).max(axis=1)
            i = idx[sl, j]
            exact = C[rows, i]
            nz = top > 0.0
            ratio[sl, j] = np.where(nz, np.abs(exact) / np.where(nz, top, 1.0), 1.0)
            ok_pick[sl, j] = np.where(nz, ratio[sl, j] >= 1.0 - rel_tol, True)
            big = np.abs(exact) > 1e-12 * np.maximum(xnorm, 1e-300)
            ce = np.abs(coef_st[sl, j] - exact) / np.where(big, np.abs(exact), 1.0)
            cerr[sl, j] = np.where(big, ce, 0.0)
            ok_coef[sl, j] = np.where(big, ce <= coef_rel_tol,
                                      np.abs(coef_st[sl, j]) <= 1e-6 * np.maximum(xnorm, 1.0))
            R = R - exact[:, None] * D[i]
    return {"pick_ratio": ratio, "coef_err": cerr, "ok_pick": ok_pick,
            "ok_coef": ok_coef}
