"""Seeded synthetic inputs shaped like the Llama-3.1-8B KV workloads of
"LLM Inference in a Flash!" (evolve.pub review, Summary: per-layer,
per-stream dictionaries of 32,768 atoms; K=16 atoms per vector; Klow=3,
top 10%, Khigh=16).

This module holds NO arithmetic of the method: it only draws dictionaries,
vectors, queries and (for the decode-only workloads) random codes, and lays
the code words out in the storage format.  Both the CUDA path (through the
tests and the bench) and the fp64 oracle consume what it makes; neither of
them is imported here.  Random numbers come from ``torch.Generator`` seeded
per workload (CPU generator for the small cases, CUDA generator for the big
ones), so the same call always yields the same tensors on the same device.

Word format of a code (a storage format, fixed once for both sides):
  word = (fp16 bits of the coefficient << 16) | (atom index & 0x7fff).
Words are kept in int32 tensors holding those exact bits.

Layout of a code store for one layer (all int32 bit patterns):
  k_lo   [B, Hkv, 3, cap]   words 0..2 of each key code, one plane per word
  k_full [B, Hkv, cap, 16]  all 16 words of each key code (64-byte records)
  v_full [B, Hkv, cap, 16]  all 16 words of each value code
"""

import math

import torch

N_ATOMS = 32768
K_ATOMS = 16
KLOW_PLANES = 3

# The five workloads.
WORKLOADS = {
    "tiny": dict(
        index=0, d=64, n_atoms=1024, n_tokens=256, B=1, Hq=4, Hkv=1, L=1,
        desc="1 layer, 1 KV head / 4 query heads, d=64, 1024-atom Gaussian "
             "dictionaries, 256 tokens planted 16-sparse + N(0,0.01^2) noise, "
             "q~N(0,1/64)"),
    "layer4k": dict(
        index=1, d=128, n_atoms=32768, n_tokens=4096, B=1, Hq=32, Hkv=8, L=1,
        desc="1 Llama-3.1-8B layer, batch 1, 32 q / 8 KV heads, d=128, "
             "32768-atom bf16 dictionaries shared by the 8 KV heads, 4096 "
             "tokens planted 16-sparse + noise of norm 0.05||x||"),
    "decode32k_b4": dict(
        index=2, d=128, n_atoms=32768, n_tokens=32768, B=4, Hq=32, Hkv=8,
        L=32,
        desc="32-layer decode step, batch 4, 32768 tokens, random 16-atom "
             "codes, q~N(0,1/128) with 3 outlier channels x8"),
    "decode256k": dict(
        index=3, d=128, n_atoms=32768, n_tokens=262144, B=1, Hq=32, Hkv=8,
        L=32,
        desc="32-layer decode step, batch 1, 262144 tokens, random 16-atom "
             "codes, q~N(0,1/128)"),
    "prefill256k_vec": dict(
        index=4, d=128, n_atoms=32768, n_tokens=16384, B=1, Hq=32, Hkv=8,
        L=1,
        desc="encode 16384 tokens x 8 KV heads x 2 streams = 262144 dense "
             "Student-t(4) vectors with 4 outlier channels x10 against "
             "correlated dictionaries"),
}


def seed_of(name):
    return 1000 + WORKLOADS[name]["index"]


def make_gen(seed, device="cpu"):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _unit_rows(x):
    return x / x.norm(dim=1, keepdim=True)


def gaussian_dictionary(n, d, gen, device="cpu"):
    """n atoms ~ N(0, I_d), L2-normalised in fp32, then rounded to bf16."""
    g = torch.randn(n, d, generator=gen, device=device, dtype=torch.float32)
    return _unit_rows(g).to(torch.bfloat16)


def correlated_dictionary(n, d, gen, device="cpu"):
    """atom_i = normalise(g_i + 0.3 z_i s): g_i ~ N(0,I), z_i ~ N(0,1) and one
    shared direction s ~ N(0,I) drawn once (not normalised), then bf16."""
    s = torch.randn(d, generator=gen, device=device, dtype=torch.float32)
    g = torch.randn(n, d, generator=gen, device=device, dtype=torch.float32)
    z = torch.randn(n, 1, generator=gen, device=device, dtype=torch.float32)
    return _unit_rows(g + 0.3 * z * s[None, :]).to(torch.bfloat16)


def distinct_atoms(m, k, n, gen, device="cpu"):
    """[m, k] int64 atom indices, distinct within each row, uniform over n.

    Rows with a repeated index are redrawn until none is left.
    """
    idx = torch.randint(0, n, (m, k), generator=gen, device=device)
    while True:
        srt, _ = idx.sort(dim=1)
        bad = (srt[:, 1:] == srt[:, :-1]).any(dim=1)
        nbad = int(bad.sum())
        if nbad == 0:
            return idx
        idx[bad] = torch.randint(0, n, (nbad, k), generator=gen,
                                 device=device)


def planted_vectors(D, m, gen, noise_abs=None, noise_rel=None, k=K_ATOMS):
    """m vectors x = sum_{j<k} a_j D[i_j] + e with distinct uniform atoms,
    a_j ~ N(0,1), computed in fp32 from the (bf16) dictionary values.

    noise_abs: e ~ N(0, noise_abs^2) per component.
    noise_rel: e has norm noise_rel * ||x_clean|| (per-component sigma
               noise_rel * ||x_clean|| / sqrt(d)).
    Returns (x fp32 [m,d], planted idx [m,k], planted coef [m,k]).
    """
    device = D.device
    n, d = D.shape
    idx = distinct_atoms(m, k, n, gen, device)
    a = torch.randn(m, k, generator=gen, device=device, dtype=torch.float32)
    Df = D.float()
    x = torch.zeros(m, d, device=device, dtype=torch.float32)
    for j in range(k):
        x += a[:, j:j + 1] * Df[idx[:, j]]
    e = torch.randn(m, d, generator=gen, device=device, dtype=torch.float32)
    if noise_abs is not None:
        x = x + noise_abs * e
    elif noise_rel is not None:
        x = x + e * (noise_rel * x.norm(dim=1, keepdim=True) / math.sqrt(d))
    return x, idx, a


def student_t_vectors(m, d, gen, channels, nu=4, outlier_scale=10.0,
                      device="cpu"):
    """Dense Student-t(nu) vectors; the given fixed channels scaled up."""
    ch = channels
    z = torch.randn(m, d, generator=gen, device=device, dtype=torch.float32)
    chi2 = torch.zeros(m, d, device=device, dtype=torch.float32)
    for _ in range(nu):
        u = torch.randn(m, d, generator=gen, device=device,
                        dtype=torch.float32)
        chi2 += u * u
    x = z / torch.sqrt(chi2 / nu)
    x[:, ch] *= outlier_scale
    return x


def queries(B, Hq, d, gen, n_outlier=0, outlier_scale=8.0, device="cpu"):
    """q ~ N(0, 1/d) per component; n_outlier fixed channels (shared by all
    heads) scaled by outlier_scale."""
    q = torch.randn(B, Hq, d, generator=gen, device=device,
                    dtype=torch.float32) / math.sqrt(d)
    if n_outlier:
        ch = torch.randperm(d, generator=gen, device=device)[:n_outlier]
        q[..., ch] *= outlier_scale
    return q


def words_from(idx, coef):
    """Pack int64 indices and float coefficients (rounded to fp16 here, the
    values are within fp16 range) into int32 bit patterns of the word
    format."""
    hi = coef.to(torch.float16).view(torch.int16).to(torch.int32)
    return (hi << 16) | (idx.to(torch.int32) & 0x7FFF)


def random_codes(shape, n_atoms, gen, device="cpu"):
    """Random 16-atom codes: indices uniform over n_atoms (repeats allowed),
    coefficients N(0,1) ordered by decreasing magnitude (as a greedy pursuit
    emits them), rounded to fp16.  Returns int32 words [*shape, 16]."""
    idx = torch.randint(0, n_atoms, (*shape, K_ATOMS), generator=gen,
                        device=device)
    c = torch.randn(*shape, K_ATOMS, generator=gen, device=device,
                    dtype=torch.float32)
    order = c.abs().argsort(dim=-1, descending=True)
    c = torch.gather(c, -1, order)
    return words_from(idx, c)


def layout(kwords, vwords, cap=None, interleaved=False):
    """Code-store layout from [B, Hkv, N, 16] word tensors (pure copies).
    interleaved: k_full and v_full are views of one [B, Hkv, cap, 2, 16]
    array (a token's key and value records adjacent)."""
    B, Hkv, N, _ = kwords.shape
    cap = N if cap is None else cap
    dev = kwords.device
    if interleaved:
        kv = torch.zeros(B, Hkv, cap, 2, K_ATOMS, dtype=torch.int32, device=dev)
        k_full, v_full = kv[:, :, :, 0], kv[:, :, :, 1]
    else:
        k_full = torch.zeros(B, Hkv, cap, K_ATOMS, dtype=torch.int32, device=dev)
        v_full = torch.zeros(B, Hkv, cap, K_ATOMS, dtype=torch.int32, device=dev)
    k_lo = torch.zeros(B, Hkv, KLOW_PLANES, cap, dtype=torch.int32,
                       device=dev)
    k_full[:, :, :N] = kwords
    v_full[:, :, :N] = vwords
    k_lo[:, :, :, :N] = kwords[..., :KLOW_PLANES].transpose(-1, -2)
    return k_lo, k_full, v_full


# ---------------------------------------------------------------- workloads

def tiny(device="cpu"):
    """Workload 'tiny': everything the oracle finishes in seconds."""
    w = WORKLOADS["tiny"]
    gen = make_gen(seed_of("tiny"), device)
    d, n, N = w["d"], w["n_atoms"], w["n_tokens"]
    DK = gaussian_dictionary(n, d, gen, device)
    DV = gaussian_dictionary(n, d, gen, device)
    xk, _, _ = planted_vectors(DK, N, gen, noise_abs=0.01)
    xv, _, _ = planted_vectors(DV, N, gen, noise_abs=0.01)
    q = queries(1, w["Hq"], d, gen, device=device)
    return dict(DK=DK, DV=DV, xk=xk.view(1, 1, N, d), xv=xv.view(1, 1, N, d),
                q=q, **w)


def layer4k(device="cpu"):
    """Workload 'layer4k': one layer of planted K/V vectors for 8 KV heads."""
    w = WORKLOADS["layer4k"]
    gen = make_gen(seed_of("layer4k"), device)
    d, n, N, Hkv = w["d"], w["n_atoms"], w["n_tokens"], w["Hkv"]
    DK = gaussian_dictionary(n, d, gen, device)
    DV = gaussian_dictionary(n, d, gen, device)
    xk, _, _ = planted_vectors(DK, Hkv * N, gen, noise_rel=0.05)
    xv, _, _ = planted_vectors(DV, Hkv * N, gen, noise_rel=0.05)
    q = queries(1, w["Hq"], d, gen, device=device)
    return dict(DK=DK, DV=DV, xk=xk.view(1, Hkv, N, d),
                xv=xv.view(1, Hkv, N, d), q=q, **w)


def decode_layer(name, layer, device="cpu", n_tokens=None, B=None):
    """One layer of a decode-only workload ('decode32k_b4', 'decode256k'):
    own dictionaries, random codes, queries.  Layer l uses its own seed
    stream so layers can be made one at a time."""
    w = WORKLOADS[name]
    gen = make_gen(seed_of(name) * 1000 + layer, device)
    d, n, Hkv, Hq = w["d"], w["n_atoms"], w["Hkv"], w["Hq"]
    N = w["n_tokens"] if n_tokens is None else n_tokens
    Bn = w["B"] if B is None else B
    DK = gaussian_dictionary(n, d, gen, device)
    DV = gaussian_dictionary(n, d, gen, device)
    kw = random_codes((Bn, Hkv, N), n, gen, device)
    vw = random_codes((Bn, Hkv, N), n, gen, device)
    n_out = 3 if name == "decode32k_b4" else 0
    q = queries(Bn, Hq, d, gen, n_outlier=n_out, device=device)
    return dict(DK=DK, DV=DV, kwords=kw, vwords=vw, q=q, L=w["L"], B=Bn,
                Hq=Hq, Hkv=Hkv, d=d, n_atoms=n, n_tokens=N)


def append_token(name, layer, device="cpu"):
    """One generated token of a 32-layer decode workload ('decode32k_b4',
    'decode256k'): the new K and V vectors of every KV head of its B
    sequences in one layer ([B, Hkv, 1, d], planted 16-sparse + noise of
    norm 0.05||x||) and that layer's own dictionaries.  Seed stream apart
    from decode_layer's, so no context codes are drawn."""
    w = WORKLOADS[name]
    gen = make_gen(seed_of(name) * 1000 + 500 + layer, device)
    d, n, Hkv, B = w["d"], w["n_atoms"], w["Hkv"], w["B"]
    DK = gaussian_dictionary(n, d, gen, device)
    DV = gaussian_dictionary(n, d, gen, device)
    xk, _, _ = planted_vectors(DK, B * Hkv, gen, noise_rel=0.05)
    xv, _, _ = planted_vectors(DV, B * Hkv, gen, noise_rel=0.05)
    return dict(DK=DK, DV=DV, xk=xk.view(B, Hkv, 1, d),
                xv=xv.view(B, Hkv, 1, d), L=w["L"], B=B, Hkv=Hkv, d=d,
                n_atoms=n)


def prefill(device="cpu", n_tokens=None):
    """Workload 'prefill256k_vec': dense Student-t K and V vectors and the
    correlated K and V dictionaries of one layer."""
    w = WORKLOADS["prefill256k_vec"]
    gen = make_gen(seed_of("prefill256k_vec"), device)
    d, n, Hkv = w["d"], w["n_atoms"], w["Hkv"]
    N = w["n_tokens"] if n_tokens is None else n_tokens
    DK = correlated_dictionary(n, d, gen, device)
    DV = correlated_dictionary(n, d, gen, device)
    ch = torch.randperm(d, generator=gen, device=device)[:4]
    xk = student_t_vectors(Hkv * N, d, gen, ch, device=device)
    xv = student_t_vectors(Hkv * N, d, gen, ch, device=device)
    return dict(DK=DK, DV=DV, xk=xk.view(1, Hkv, N, d),
                xv=xv.view(1, Hkv, N, d), d=d, n_atoms=n, Hkv=Hkv,
                n_tokens=N)
