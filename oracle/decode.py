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
"""

import numpy as np

from .encode import unpack_words


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
                    force_set=None):
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
    p = _softmax(logits)
    v_hat = decode_vectors(vwords[domain], DV, 16)
    out = p @ v_hat
    return {"out": out, "s_lo": s_lo, "sel": sel, "p": p, "domain": domain,
            "k": k}


def decode_attn_ref(q, kwords, vwords, DK, DV, lens=None, klow=3, khigh=16,
                    top_num=1, top_den=10, full_softmax=False, scale=None):
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
                                top_num, top_den, full_softmax, scale)
            out[b, h] = r["out"]
            details[(b, h)] = r
    return out, details
