"""Oracle: decode attention over dictionary codes with query-aware
hierarchical sparsity (fp64, plain definition over decoded vectors).

TEST INFRASTRUCTURE ONLY (see the package docstring).

What the pages fix ("LLM Inference in a Flash!", evolve.pub review, Summary
and FAQ "What is the 15x KV cache compression ..."): decoding scores all
tokens using Klow=3 atoms, keeps the top 10% and refines those with
Khigh=16 atoms.  The dictionary is per layer and per key/value stream.

This oracle does NOT use the q*D_K^T trick of the GPU path; it decodes the
key and value vectors first and then applies textbook attention:
  1. K^lo_t = sum_{j<klow}  c_tj D_K[idx_tj];  s_lo_t = <q, K^lo_t>
  2. S      = the first k tokens of the order (-s_lo_t, t), where
              k = ceil(top_num * N / top_den) in integer arithmetic (>= 1)
  3. K^_t   = sum_{j<khigh} c_tj D_K[idx_tj];  s_t = scale * <q, K^_t>, t in S
  4. p      = softmax over S of s   (full_softmax: softmax over all t, with
              scale * s_lo_t standing in for the tokens outside S)
  5. V^_t   = sum_{j<16} c^V_tj D_V[idx^V_tj];  out = sum_t p_t V^_t
Query head h reads KV head h // (Hq / Hkv).

Readings where the pages are silent: "first Klow
atoms" are the first three in greedy pick order; k uses ceil; ties in the
selection go to the lower token index; the logit scale is 1/sqrt(d) unless
given; selection is per query head; the full-softmax flag only widens the
softmax domain.

Integer softmax (optional, ``int_softmax=True``; ``integer_softmax``).  The review's Summary
says the paper runs Softmax as an integer polynomial approximation on
inputs requantised to token-wise INT16, with bit-shift guards against INT32
overflow and fixed-point reciprocals for the divisions; the polynomial is
not given.  Reading: I-BERT's integer exponential (Kim et al., 2021,
"I-BERT: Integer-only BERT Quantization"), the published second-order
polynomial exp(p) ~ 0.3585 (p + 1.353)^2 + 0.344 on p in (-ln 2, 0] with
exp(x) = 2^-z exp(p), x = p - z ln 2.  Steps for the logits l of one query
head (fp32, the precision the kernel holds them in):
  a. S = fp32(max |l|) / 32767 in fp32 (S = 1 if every l is 0);
     q_t = rint(l_t / S) in fp64, clipped to [-32767, 32767] (a NaN logit
     maps to -32767): token-wise INT16;
  b. x_t = (q_t - max q) >> sh (arithmetic shift), sh the smallest shift
     with q_b^2 + q_c < 2^31 at the scale Sw = S 2^sh (the overflow guard),
     where q_ln2 = floor(ln 2 / Sw) (at least 1), q_b = floor(1.353 / Sw),
     q_c = floor(0.344 / (0.3585 Sw^2)), all in fp64;
  c. z_t = floor(-x_t / q_ln2), p_t = x_t + z_t q_ln2,
     e_t = ((p_t + q_b)^2 + q_c) >> z_t   (0 when z_t >= 31);
  d. E = sum_t e_t (int64), recip = floor(2^61 / E),
     P_t = (e_t recip) >> 31: probabilities in Q30 (P_t / 2^30).
"""

import math

import numpy as np

from .encode import unpack_words

ISOFT_A, ISOFT_B, ISOFT_C = 0.3585, 1.353, 0.344
LN2 = math.log(2.0)


def integer_softmax(logits):
    """The integer softmax above for one query head's logits (any float
    array; taken as fp32).  Returns (P int64 Q30 probabilities, E int, sh
    int)."""
    l32 = np.asarray(logits, dtype=np.float32)
    if l32.size == 0:
        return np.zeros(0, dtype=np.int64), 0, 0
    finite = l32[np.isfinite(l32)]
    lmax = np.float32(np.max(np.abs(finite))) if finite.size else np.float32(0.0)
    S = np.float32(lmax / np.float32(32767.0)) if lmax > 0 else np.float32(1.0)
    q = np.empty(l32.shape, dtype=np.int64)
    for t, v in enumerate(l32.tolist()):
        if v != v:
            q[t] = -32767
        else:
            q[t] = int(min(max(np.rint(float(v) / float(S)), -32767.0), 32767.0))
    qmax = int(q.max())
    sh = 0
    while True:
        Sw = float(S) * 2.0 ** sh
        q_ln2 = max(1, int(math.floor(LN2 / Sw)))
        q_b = int(math.floor(ISOFT_B / Sw))
        q_c = int(math.floor(ISOFT_C / (ISOFT_A * Sw * Sw)))
        if q_b * q_b + q_c < 2 ** 31:
            break
        sh += 1
    e = np.zeros(q.shape, dtype=np.int64)
    for t in range(q.size):
        x = (int(q[t]) - qmax) >> sh          # Python >> floors, as an arithmetic shift
        z = (-x) // q_ln2
        pp = x + z * q_ln2
        L = (pp + q_b) * (pp + q_b) + q_c
        assert 0 <= L < 2 ** 31
        e[t] = L >> z if z < 31 else 0
    E = int(e.sum())
    recip = (1 << 61) // E
    P = np.array([(int(v) * recip) >> 31 for v in e.tolist()], dtype=np.int64)
    return P, E, sh


def topk_count(n_tokens, top_num, top_den):
    """k = ceil(top_num * N / top_den), at least 1, in integer arithmetic."""
    k = (top_num * n_tokens + top_den - 1) // top_den
    return max(1, min(int(k), int(n_tokens)))


def select_top(scores, k):
    """The first k tokens of the order (score descending, token ascending).

    np.lexsort sorts by its LAST key first: primary -score, secondary t.
    """
    s = np.asarray(scores, dtype=np.float64)
    t = np.arange(s.shape[0])
    order = np.lexsort((t, -s))
    return order[:k]


def decode_vectors(words, D, nterms, chunk=8192):
    """Decoded vectors sum_{j<nterms} coef_j D[idx_j] for each row of words.

    ``words`` is [N, >=nterms] uint32.  Rows are independent; the chunking
    over rows only bounds memory and changes no arithmetic.
    """
    D = np.asarray(D, dtype=np.float64)
    words = np.asarray(words)
    N = words.shape[0]
    out = np.zeros((N, D.shape[1]), dtype=np.float64)
    for s in range(0, N, chunk):
        idx, coef = unpack_words(words[s:s + chunk, :nterms])
        acc = np.zeros((idx.shape[0], D.shape[1]), dtype=np.float64)
        for j in range(nterms):
            acc += coef[:, j:j + 1] * D[idx[:, j]]
        out[s:s + chunk] = acc
    return out


def _softmax(z):
    z = np.asarray(z, dtype=np.float64)
    m = np.max(z)
    e = np.exp(z - m)
    return e / np.sum(e)


def decode_head_ref(q, kwords, vwords, DK, DV, klow=3, khigh=16,
                    top_num=1, top_den=10, full_softmax=False, scale=None,
                    force_set=None, int_softmax=False):
    """One query head over one sequence.

    q [d]; kwords, vwords [N, 16] uint32 words; DK, DV [n, d].
    ``force_set`` (optional) replaces step 2's set S by the given token
    indices; parity tests use it when two correct implementations picked
    different members among near-tied scores.
    Returns a dict: out [d], s_lo [N], sel (sorted indices of S), p (over the
    softmax domain, aligned with ``domain``), domain (token indices).
    """
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[0]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    N = kwords.shape[0]
    k_lo = decode_vectors(kwords, DK, klow)
    # row-wise products and sums (not a BLAS gemv, whose summation order can
    # differ between rows): identical codes get bit-identical scores
    s_lo = np.sum(k_lo * q[None, :], axis=1)
    k = topk_count(N, top_num, top_den)
    if force_set is None:
        sel = select_top(s_lo, k)
    else:
        sel = np.asarray(force_set, dtype=np.int64)
    sel = np.sort(sel)
    k_hi = decode_vectors(kwords[sel], DK, khigh)
    s_sel = scale * np.sum(k_hi * q[None, :], axis=1)
    if full_softmax:
        logits = scale * s_lo
        logits[sel] = s_sel
        domain = np.arange(N)
    else:
        logits = s_sel
        domain = sel
    if int_softmax:
        P, E, _ = integer_softmax(logits)
        p = P.astype(np.float64) / float(1 << 30)
    else:
        p = _softmax(logits)
    v_hat = decode_vectors(vwords[domain], DV, 16)
    out = p @ v_hat
    return {"out": out, "s_lo": s_lo, "sel": sel, "p": p, "domain": domain,
            "k": k}


def decode_attn_ref(q, kwords, vwords, DK, DV, lens=None, klow=3, khigh=16,
                    top_num=1, top_den=10, full_softmax=False, scale=None,
                    int_softmax=False):
    """One layer of decode attention for B sequences.

    q [B, Hq, d]; kwords, vwords [B, Hkv, N_max, 16] uint32 (only the first
    lens[b] tokens of sequence b are used); DK, DV [n, d].
    Returns out [B, Hq, d] fp64 and the per-head details.
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv = kwords.shape[1]
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    g = Hq // Hkv
    if lens is None:
        lens = [kwords.shape[2]] * B
    out = np.zeros((B, Hq, d), dtype=np.float64)
    details = {}
    for b in range(B):
        n_b = int(lens[b])
        for h in range(Hq):
            kvh = h // g
            r = decode_head_ref(q[b, h], kwords[b, kvh, :n_b],
                                vwords[b, kvh, :n_b], DK, DV, klow, khigh,
                                top_num, top_den, full_softmax, scale,
                                int_softmax=int_softmax)
            out[b, h] = r["out"]
            details[(b, h)] = r
    return out, details
