"""Pins for the replay certificate (CPU only): it accepts correct greedy
codes and rejects planted mistakes (a wrong pick, a wrong coefficient)."""

import numpy as np

import oracle


def _setup(seed=0, n=256, d=32, m=6):
    rng = np.random.default_rng(seed)
    D = rng.standard_normal((n, d))
    D /= np.linalg.norm(D, axis=1, keepdims=True)
    X = rng.standard_normal((m, d))
    return D, X


def _words(ref):
    return oracle.pack_words(ref["idx"], oracle.store_coef_fp16(ref["coef"]))


def test_certificate_accepts_oracle_codes():
    D, X = _setup()
    ref = oracle.encode_ref(X, D)
    c = oracle.certify_codes(X, D, _words(ref))
    assert c["ok_pick"].all() and c["ok_coef"].all()
    assert np.allclose(c["pick_ratio"], 1.0)


def test_certificate_rejects_wrong_pick():
    D, X = _setup(1)
    ref = oracle.encode_ref(X, D)
    bad = ref["idx"].copy()
    # swap the pick of vector 2 at step 4 for a clearly worse atom
    bad[2, 4] = (bad[2, 4] + 17) % D.shape[0]
    words = oracle.pack_words(bad, oracle.store_coef_fp16(ref["coef"]))
    c = oracle.certify_codes(X, D, words)
    assert not c["ok_pick"][2, 4]


def test_certificate_rejects_wrong_coefficient():
    D, X = _setup(2)
    ref = oracle.encode_ref(X, D)
    coef = ref["coef"].copy()
    coef[1, 3] *= 1.01
    words = oracle.pack_words(ref["idx"], oracle.store_coef_fp16(coef))
    c = oracle.certify_codes(X, D, words)
    assert not c["ok_coef"][1, 3]
    assert c["ok_pick"].all()


def test_batched_certificate_equals_the_loop():
    """The batched replay gives the per-vector replay's verdicts and ratios
    (to rounding of the matrix product) on correct codes, a planted wrong
    pick and a planted wrong coefficient, across a batch boundary."""
    D, X = _setup(3, m=37)
    ref = oracle.encode_ref(X, D)
    bad = ref["idx"].copy()
    bad[20, 5] = (bad[20, 5] + 11) % D.shape[0]
    coef = ref["coef"].copy()
    coef[33, 2] *= 1.01
    for words in (_words(ref), oracle.pack_words(bad, oracle.store_coef_fp16(ref["coef"])),
                  oracle.pack_words(ref["idx"], oracle.store_coef_fp16(coef))):
        a = oracle.certify_codes(X, D, words)
        b = oracle.certify_codes_batched(X, D, words, batch=8)
        assert np.array_equal(a["ok_pick"], b["ok_pick"])
        assert np.array_equal(a["ok_coef"], b["ok_coef"])
        assert np.allclose(a["pick_ratio"], b["pick_ratio"], rtol=1e-12, atol=0)
        assert np.allclose(a["coef_err"], b["coef_err"], rtol=1e-9, atol=1e-15)
    assert not b["ok_coef"][33, 2]
    assert not oracle.certify_codes_batched(
        X, D, oracle.pack_words(bad, oracle.store_coef_fp16(ref["coef"])))["ok_pick"][20, 5]
