"""Tolerance protocols shared by the GPU parity tests.

Encode (greedy pursuit, "LLM Inference in a Flash!" review, Summary): walk
the 16 steps of each vector; atom indices must match unless the oracle's
relative gap between the two largest |<r, d>| is <= 1e-4 at that step (then
both picks are correct and the rest of the vector legitimately diverges, so
the walk stops); coefficients (fp16 as stored) must be within 1e-3
relative of the oracle's.

A step whose oracle residual has fallen below 1e-5 ||x|| (the fp32
rounding floor of a residual kept in fp32 on the GPU) ends the walk: the
picks there are decided by rounding noise on both sides; the GPU's
remaining coefficients must then be below 1e-4 ||x|| in magnitude.

Decode: selected sets may differ only in tokens whose s_lo is within 1e-5
relative of the k-th largest s_lo; outputs must agree within 2e-3 max-abs
for unit-norm q (when the sets differ inside the tie band the oracle output
is recomputed on the GPU's set).
"""

import numpy as np

import oracle

GAP_TOL = 1e-4
RESID_FLOOR = 1e-5
COEF_TOL = 1e-3
SET_TOL = 1e-5
OUT_TOL = 2e-3


def words_np(t):
    """int32 torch tensor of code words -> uint32 numpy."""
    return t.detach().cpu().numpy().view(np.uint32)


def check_encode(words_gpu, ref, coef_tol=COEF_TOL, gap_tol=GAP_TOL,
                 stopped=None):
    """Returns (steps_compared, vectors_that_diverged_at_a_near_tie).
    Raises AssertionError on a violation.  `stopped`, if a list, receives
    the vectors whose walk ended early (a near tie or the residual floor)."""
    idx_g, coef_g = oracle.unpack_words(words_gpu)
    m, k = idx_g.shape
    compared = 0
    diverged = 0
    for v in range(m):
        for j in range(k):
            if ref["rnorm"][v, j] <= RESID_FLOOR * ref["xnorm"][v]:
                assert np.all(np.abs(coef_g[v, j:]) <= 1e-4 * ref["xnorm"][v])
                if stopped is not None:
                    stopped.append(v)
                break
            if idx_g[v, j] != ref["idx"][v, j]:
                assert ref["gap"][v, j] <= gap_tol, (
                    "vector %d step %d: gpu atom %d, oracle atom %d, oracle "
                    "gap %.3g" % (v, j, idx_g[v, j], ref["idx"][v, j],
                                  ref["gap"][v, j]))
                diverged += 1
                if stopped is not None:
                    stopped.append(v)
                break
            c_or = ref["coef"][v, j]
            err = abs(coef_g[v, j] - c_or)
            assert err <= coef_tol * abs(c_or) + 1e-7, (
                "vector %d step %d: coef %.8g vs oracle %.8g" % (
                    v, j, coef_g[v, j], c_or))
            compared += 1
    return compared, diverged


def check_selection(sel_gpu, s_lo_oracle, k, set_tol=SET_TOL):
    """sel_gpu: GPU-selected token indices (any order).  Checks size,
    uniqueness and that every difference to the oracle's exact top-k lies in
    the tie band.  Returns the number of differing tokens."""
    sel_gpu = np.asarray(sel_gpu, dtype=np.int64)
    assert sel_gpu.shape[0] == k
    assert np.unique(sel_gpu).shape[0] == k, "duplicate tokens selected"
    assert sel_gpu.min() >= 0 and sel_gpu.max() < s_lo_oracle.shape[0]
    sel_or = oracle.select_top(s_lo_oracle, k)
    sk = np.sort(s_lo_oracle)[::-1][k - 1]
    diff = np.setxor1d(sel_gpu, sel_or)
    band = set_tol * max(abs(sk), 1e-30)
    bad = diff[np.abs(s_lo_oracle[diff] - sk) > band]
    assert bad.size == 0, "tokens outside the tie band differ: %s (s_k=%g)" % (
        bad[:10], sk)
    return diff.size
