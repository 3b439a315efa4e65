"""What the projection-based greedy pursuit gives up against OMP (fp64).

TEST INFRASTRUCTURE ONLY: an oracle-side measurement, run on the CPU.

    python -m oracle.compare_omp [--vectors 32]

For seeded samples of three workloads it encodes the same vectors with the
greedy pursuit (encode.py) and with OMP (omp.py) and prints, per number of
picks k, the mean residual energy ||r_k||^2 / ||x||^2 and, where vectors are
planted sparse combinations, the fraction of planted atoms among the first
16 picks.  On the small 'tiny' workload it also decodes one query head over
the coded keys and values (full softmax over all 256 tokens, every atom of
every code) and reports the largest deviation of the attention output from
dense attention over the uncoded vectors.
"""

import argparse
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import workloads                       # noqa: E402  (seeded inputs only)
from oracle.encode import encode_ref, store_coef_fp16, pack_words   # noqa: E402
from oracle.decode import decode_head_ref                            # noqa: E402
from oracle.omp import omp_ref                                       # noqa: E402

KS = (4, 8, 12, 16)


def energy_curve(X, D, k_max=16):
    """Mean ||r_k||^2 / ||x||^2 after k picks, for greedy and OMP."""
    g = encode_ref(X, D, k_max)
    o = omp_ref(X, D, k_max)
    x2 = g["xnorm"] ** 2
    out = {}
    for k in KS:
        # rnorm[:, j] is ||r|| before step j; after the last step use resid
        if k < k_max:
            rg, ro = g["rnorm"][:, k] ** 2, o["rnorm"][:, k] ** 2
        else:
            rg = np.sum(g["resid"] ** 2, axis=1)
            ro = np.sum(o["resid"] ** 2, axis=1)
        out[k] = (float(np.mean(rg / x2)), float(np.mean(ro / x2)))
    return out, g, o


def planted_hits(idx, planted):
    return float(np.mean([len(set(a.tolist()) & set(b.tolist())) / len(b)
                          for a, b in zip(idx, planted)]))


def words_of(idx, coef):
    return pack_words(idx, store_coef_fp16(coef))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--vectors", type=int, default=32)
    args = ap.parse_args()
    m = args.vectors
    rows = []

    # tiny: d=64, 1024 atoms, planted 16-sparse + N(0, 0.01^2)
    w = workloads.tiny()
    gen = workloads.make_gen(777)
    x, planted, _ = workloads.planted_vectors(w["DK"], m, gen, noise_abs=0.01)
    curve, g, o = energy_curve(x.double().numpy(), w["DK"].float().double().numpy())
    rows.append(("tiny (d=64, 1024 atoms, planted + 0.01 noise)", curve,
                 planted_hits(g["idx"], planted.numpy()), planted_hits(o["idx"], planted.numpy())))

    # layer4k-shaped: d=128, 32768 atoms, planted + noise of norm 0.05||x||
    gen = workloads.make_gen(778)
    D = workloads.gaussian_dictionary(32768, 128, gen)
    x, planted, _ = workloads.planted_vectors(D, m, gen, noise_rel=0.05)
    curve, g, o = energy_curve(x.double().numpy(), D.float().double().numpy())
    rows.append(("layer4k-shaped (d=128, 32768 atoms, planted + 5% noise)", curve,
                 planted_hits(g["idx"], planted.numpy()), planted_hits(o["idx"], planted.numpy())))

    # prefill-shaped: dense Student-t vectors, correlated dictionary
    p = workloads.prefill(n_tokens=max(1, m // 8))
    xs = p["xk"].reshape(-1, 128)[:m]
    curve, g, o = energy_curve(xs.double().numpy(), p["DK"].float().double().numpy())
    rows.append(("prefill-shaped (dense Student-t, correlated atoms)", curve, None, None))

    print("| workload | k | greedy ||r||^2/||x||^2 | OMP ||r||^2/||x||^2 |")
    print("|---|---|---|---|")
    for name, curve, hg, ho in rows:
        for k in KS:
            print("| %s | %d | %.4g | %.4g |" % (name, k, curve[k][0], curve[k][1]))
    print()
    for name, _, hg, ho in rows:
        if hg is not None:
            print("planted atoms among the 16 picks, %s: greedy %.3f, OMP %.3f" % (name, hg, ho))

    # attention over coded K/V on the tiny workload: one query head, full
    # softmax over the 256 tokens, all 16 atoms of every code
    N = w["n_tokens"]
    XK = w["xk"].reshape(N, -1).double().numpy()
    XV = w["xv"].reshape(N, -1).double().numpy()
    DK = w["DK"].float().double().numpy()
    DV = w["DV"].float().double().numpy()
    q = w["q"][0, 0].double().numpy()
    q = q / np.linalg.norm(q)
    scale = 1.0 / np.sqrt(q.shape[0])
    z = scale * (XK @ q)
    pz = np.exp(z - z.max())
    dense = (pz / pz.sum()) @ XV
    errs = {}
    for name, fn in (("greedy", encode_ref), ("OMP", omp_ref)):
        ek, ev = fn(XK, DK, 16), fn(XV, DV, 16)
        kw, vw = words_of(ek["idx"], ek["coef"]), words_of(ev["idx"], ev["coef"])
        res = decode_head_ref(q, kw, vw, DK, DV, klow=16, khigh=16, top_num=1, top_den=1,
                              full_softmax=True, scale=scale)
        errs[name] = float(np.max(np.abs(res["out"] - dense)))
    print("tiny, one query head, full softmax over 256 coded tokens: max |out - dense| "
          "greedy %.3g, OMP %.3g" % (errs["greedy"], errs["OMP"]))


if __name__ == "__main__":
    main()
