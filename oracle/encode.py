"""Oracle: sparse dictionary encoding by projection-based greedy pursuit (fp64).

TEST INFRASTRUCTURE ONLY (see the package docstring).

What the pages fix ("LLM Inference in a Flash!", evolve.pub review, Summary;
FAQ "What is the 15x KV cache compression ..."; authors' abstract):
  * every key and every value vector is represented as a linear combination
    of K=16 atoms of a static, per-layer, per-stream (key or value)
    overcomplete dictionary of 32,768 atoms;
  * what is stored per vector is the index and the coefficient of each of
    the 16 atoms;
  * the encoder is a projection-based greedy pursuit that replaces OMP so
    that no least-squares refit is done.

Readings where the pages are silent:
  * a step picks the atom that maximises |<r, d_i>|; ties go to the lowest
    atom index (np.argmax returns the first occurrence);
  * the coefficient is the projection <r, d_i*> itself, unrounded, and the
    residual update is r <- r - coef * d_i*; atoms are used exactly as given
    (no renormalisation by ||d||^2);
  * atoms may repeat (plain matching pursuit keeps no exclusion list);
  * a zero residual makes every |c| zero, so the pick is atom 0 with
    coefficient 0;
  * storage rounds the coefficient to fp16 (round to nearest even) with
    saturation to +-65504, and packs one (index, coefficient) pair into a
    32-bit word: fp16 bits in the high half, the 15-bit index in the low 15
    bits, bit 15 zero.
"""

import numpy as np

FP16_MAX = 65504.0


def greedy_pursuit(x, D, k_atoms=16):
    """Encode one vector ``x`` (shape [d]) over dictionary ``D`` ([n, d]).

    Follows the greedy pursuit of the review's Summary step by step, in fp64:
      r <- x
      repeat k_atoms times:
        c   = D r                     (all n inner products)
        i*  = argmax_i |c_i|          (lowest i on ties)
        coef = c_i*
        gap = (|c|_(1) - |c|_(2)) / |c|_(1)   (0 when |c|_(1) == 0)
        r  <- r - coef * D[i*]
    Returns (idx[int64, k], coef[fp64, k], gap[fp64, k], r_final[fp64, d]).
    ``greedy_pursuit.last_rnorm`` holds ||r|| before every step (a
    diagnostic for the parity tests).
    """
    D = np.asarray(D, dtype=np.float64)
    r = np.array(x, dtype=np.float64, copy=True)
    n = D.shape[0]
    idx = np.zeros(k_atoms, dtype=np.int64)
    coef = np.zeros(k_atoms, dtype=np.float64)
    gap = np.zeros(k_atoms, dtype=np.float64)
    rnorm = np.zeros(k_atoms, dtype=np.float64)
    for j in range(k_atoms):
        rnorm[j] = np.sqrt(np.sum(r * r))
        c = D @ r
        a = np.abs(c)
        i = int(np.argmax(a))
        top = a[i]
        if top > 0.0 and n > 1:
            second = np.max(np.delete(a, i))
            gap[j] = (top - second) / top
        else:
            gap[j] = 0.0
        idx[j] = i
        coef[j] = c[i]
        r = r - c[i] * D[i]
    greedy_pursuit.last_rnorm = rnorm
    return idx, coef, gap, r


def encode_ref(X, D, k_atoms=16):
    """Greedy pursuit of every row of ``X`` ([m, d]); one vector at a time.

    Returns dict with idx [m,k] int64, coef [m,k] fp64, gap [m,k] fp64,
    resid [m,d] fp64 (the final residuals), rnorm [m,k] (||r|| before each
    step) and xnorm [m].
    """
    X = np.asarray(X, dtype=np.float64)
    m = X.shape[0]
    out_idx = np.zeros((m, k_atoms), dtype=np.int64)
    out_coef = np.zeros((m, k_atoms), dtype=np.float64)
    out_gap = np.zeros((m, k_atoms), dtype=np.float64)
    out_r = np.zeros_like(X)
    out_rn = np.zeros((m, k_atoms), dtype=np.float64)
    Dd = np.asarray(D, dtype=np.float64)
    for v in range(m):
        i, c, g, r = greedy_pursuit(X[v], Dd, k_atoms)
        out_idx[v], out_coef[v], out_gap[v], out_r[v] = i, c, g, r
        out_rn[v] = greedy_pursuit.last_rnorm
    return {"idx": out_idx, "coef": out_coef, "gap": out_gap, "resid": out_r,
            "rnorm": out_rn, "xnorm": np.sqrt(np.sum(X * X, axis=1))}


def store_coef_fp16(coef):
    """fp16 storage of coefficients: round to nearest even, saturate to +-65504.

    Clipping first is the same as saturating after rounding because 65504 is
    the largest finite fp16 value and is exactly representable.
    """
    c = np.clip(np.asarray(coef, dtype=np.float64), -FP16_MAX, FP16_MAX)
    return c.astype(np.float16)


def pack_words(idx, coef16):
    """32-bit code words: (fp16 bits << 16) | (idx & 0x7fff)."""
    idx = np.asarray(idx, dtype=np.int64)
    if np.any(idx < 0) or np.any(idx > 0x7FFF):
        raise ValueError("atom index does not fit in 15 bits")
    hi = np.asarray(coef16, dtype=np.float16).view(np.uint16).astype(np.uint32)
    return (hi << np.uint32(16)) | idx.astype(np.uint32)


def unpack_words(words):
    """Inverse of the word format: (idx int64, coef fp64 from the fp16 bits)."""
    w = np.asarray(words, dtype=np.uint32)
    idx = (w & np.uint32(0x7FFF)).astype(np.int64)
    coef = (w >> np.uint32(16)).astype(np.uint16).view(np.float16)
    return idx, coef.astype(np.float64)
