"""Oracle: orthogonal matching pursuit (OMP), the encoder the pages replace.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Nothing on the GPU
path implements OMP; it is here to measure what the projection-based greedy
pursuit gives up.

The evolve.pub review of "LLM Inference in a Flash!" (Summary; Strengths,
"hardware-aware replacement of OMP") says the paper swaps OMP for a
projection-based greedy pursuit so that no least-squares refit is needed.
OMP, written out in its textbook order (fp64):
  r <- x, S <- ()
  repeat k_atoms times:
    c   = D r                        (all n inner products)
    i*  = argmax_i |c_i|             (lowest i on ties, as in the greedy
                                      pursuit of encode.py)
    S   <- S + (i*,)
    a_S = argmin_a ||x - sum_{j in S} a_j D[j]||^2   (the least-squares refit
                                      over every atom picked so far)
    r   <- x - sum_{j in S} a_j D[j]
The coefficients of all picked atoms change at every step (the refit); r
stays orthogonal to the span of the picked atoms, so an atom is picked at
most once while the picked atoms are linearly independent.

Readings where the pages are silent: the selection rule is the greedy
pursuit's own (largest |<r, d_i>|, ties to the lowest index) so the two
encoders differ only in the refit; a dependent or repeated pick (possible
only once r is zero or at rounding level) keeps the minimum-norm
least-squares solution that numpy's lstsq returns.
"""

import numpy as np


def omp(x, D, k_atoms=16):
    """OMP of one vector ``x`` ([d]) over ``D`` ([n, d]), fp64.

    Returns (idx[int64, k], coef[fp64, k], r_final[fp64, d]); coef holds the
    refitted coefficients after the last step (coef[j] belongs to idx[j]).
    ``omp.last_rnorm`` holds ||r|| before every step.
    """
    D = np.asarray(D, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    r = x.copy()
    idx = np.zeros(k_atoms, dtype=np.int64)
    coef = np.zeros(k_atoms, dtype=np.float64)
    rnorm = np.zeros(k_atoms, dtype=np.float64)
    for j in range(k_atoms):
        rnorm[j] = np.sqrt(np.sum(r * r))
        c = D @ r
        idx[j] = int(np.argmax(np.abs(c)))
        A = D[idx[:j + 1]].T                       # [d, j+1]: picked atoms as columns
        a, *_ = np.linalg.lstsq(A, x, rcond=None)  # the least-squares refit
        coef[:j + 1] = a
        r = x - A @ a
    omp.last_rnorm = rnorm
    return idx, coef, r


def omp_ref(X, D, k_atoms=16):
    """OMP of every row of ``X`` ([m, d]).  Returns dict with idx [m,k],
    coef [m,k], resid [m,d], rnorm [m,k] and xnorm [m]."""
    X = np.asarray(X, dtype=np.float64)
    m = X.shape[0]
    out_idx = np.zeros((m, k_atoms), dtype=np.int64)
    out_coef = np.zeros((m, k_atoms), dtype=np.float64)
    out_r = np.zeros_like(X)
    out_rn = np.zeros((m, k_atoms), dtype=np.float64)
    Dd = np.asarray(D, dtype=np.float64)
    for v in range(m):
        i, c, r = omp(X[v], Dd, k_atoms)
        out_idx[v], out_coef[v], out_r[v] = i, c, r
        out_rn[v] = omp.last_rnorm
    return {"idx": out_idx, "coef": out_coef, "resid": out_r, "rnorm": out_rn,
            "xnorm": np.sqrt(np.sum(X * X, axis=1))}
