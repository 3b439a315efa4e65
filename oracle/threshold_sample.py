"""How well a sample of Klow scores brackets the k-th score (fp64).

TEST INFRASTRUCTURE ONLY: an oracle-side measurement, run on the CPU.

    python -m oracle.threshold_sample [--heads-every 3] [--samples 8192]

The exact top-10 % selection ("LLM Inference in a Flash!", evolve.pub
review, Summary) needs the k-th largest Klow score of every query head.  An
implementation can bracket it from a sample of the scores first: with m
sampled scores, the k-th score of all N lies, with high probability, between
the sample's order statistics of rank p m -+ z sqrt(m p (1 - p)) (p = k / N),
so that only the tokens between those two scores need an exact look.  This
script takes the oracle's fp64 Klow scores on the synthetic decode workloads
and reports, per sampling rule, how often the k-th score falls outside the
bracket and what share of the tokens lies inside it.  Sampling rules: every
(N / m)-th token, and a pseudo-random set of about m tokens per head (a hash
of token and head).
"""

import argparse
import math
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import workloads                        # noqa: E402  (seeded inputs only)
from oracle.encode import unpack_words  # noqa: E402


def klow_scores(q, kwords, DK):
    """s_lo of every token: sum over the first 3 words of c * <q, d_idx>."""
    idx, coef = unpack_words(kwords[:, :3])
    return (coef * (DK @ q)[idx]).sum(axis=1)


def hashed_mask(N, head, m):
    """About m of N tokens, chosen by a hash of (token, head): the golden-ratio
    increment and mixing steps of the SplitMix64 generator (Steele, Lea and
    Flood, OOPSLA 2014), taken modulo N / m."""
    t = np.arange(N, dtype=np.uint64)
    with np.errstate(over="ignore"):      # arithmetic modulo 2^64 is intended
        h = t * np.uint64(0x9E3779B97F4A7C15) + np.uint64(head) * np.uint64(0xBF58476D1CE4E5B9)
        h ^= h >> np.uint64(31)
        h *= np.uint64(0x94D049BB133111EB)
        h ^= h >> np.uint64(29)
    return (h % np.uint64(max(1, N // m))) == 0


def bracket(sample, p, z):
    """(low, high) scores of the bracket around the p-quantile from the top."""
    ss = np.sort(sample)[::-1]
    m = ss.size
    r = p * m
    sd = math.sqrt(m * p * (1 - p))
    hi_r = max(1, int(math.floor(r - z * sd)))
    lo_r = min(m, int(math.ceil(r + z * sd)))
    return ss[lo_r - 1], ss[hi_r - 1]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--heads-every", type=int, default=3)
    ap.add_argument("--samples", type=int, default=8192)
    ap.add_argument("--z", type=float, default=4.0)
    args = ap.parse_args()
    rows = {}
    for name in ("decode256k", "decode32k_b4"):
        lay = workloads.decode_layer(name, 0)
        B, Hq, Hkv, N = lay["B"], lay["Hq"], lay["Hkv"], lay["n_tokens"]
        DK = lay["DK"].float().double().numpy()
        q = lay["q"].double().numpy()
        q = q / np.linalg.norm(q, axis=-1, keepdims=True)
        kwords = lay["kwords"].numpy().view(np.uint32)
        g = Hq // Hkv
        k = (N + 9) // 10
        p = k / N
        m = min(args.samples, N)
        for b in range(B):
            for h in range(0, Hq, args.heads_every):
                s = klow_scores(q[b, h], kwords[b, h // g], DK)
                kth = np.sort(s)[::-1][k - 1]
                for rule, sample in (("strided", s[::max(1, N // m)]),
                                     ("hashed", s[hashed_mask(N, b * Hq + h, m)])):
                    lo, hi = bracket(sample, p, args.z)
                    r = rows.setdefault((name, rule), [0, 0, []])
                    r[0] += 1
                    r[1] += not (lo <= kth <= hi)
                    r[2].append(float(((s >= lo) & (s <= hi)).mean()))
    print("| workload | sample | heads | k-th score outside | tokens inside (mean, max) |")
    print("|---|---|---|---|---|")
    for (name, rule), (n, miss, share) in sorted(rows.items()):
        print("| %s | %s, about %d per head | %d | %d | %.2f %%, %.2f %% |"
              % (name, rule, args.samples, n, miss, 100 * np.mean(share), 100 * np.max(share)))


if __name__ == "__main__":
    main()
