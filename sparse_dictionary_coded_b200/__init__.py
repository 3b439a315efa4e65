"""Dictionary-coded KV cache for B200: Python binding of libsdk.so.

"LLM Inference in a Flash!" (evolve.pub review, Summary) stores every key
and value vector as 16 (atom index, coefficient) pairs over static
per-layer, per-stream dictionaries of 32,768 atoms, encodes with a
projection-based greedy pursuit and decodes with query-aware hierarchical
sparsity (Klow=3 scores every token, the top 10% are refined with
Khigh=16).  The computation runs in the CUDA kernels of libsdk.so; this
module only marshals torch tensors (device memory) and the current CUDA
stream into the C ABI declared in include/sdk.h, under the same names.
"""

import ctypes
import math

import torch

from . import _capi
from ._capi import (SDK_OK, SDK_F32, SDK_BF16, MAX_ATOMS, K_ATOMS,
                    KLOW_PLANES, MAX_BATCH, SDK_DECODE_FULL_SOFTMAX,
                    SDK_DECODE_INT_SOFTMAX, SDK_DECODE_KEEP_KEYS,
                    SDK_DECODE_SELECT_RADIX, SDK_DECODE_SELECT_BRACKET, DecodeLayout,
                    load)

__all__ = [
    "SdkError", "load", "sdk_encode", "sdk_encode_simt", "sdk_append",
    "sdk_decode_attn", "sdk_encode_workspace_bytes",
    "sdk_append_workspace_bytes", "sdk_decode_workspace_bytes",
    "sdk_decode_layout_of", "sdk_workspace_init", "sdk_check_status",
    "new_workspace", "CodeStore", "read_select_state", "sdk_timing_enable",
    "sdk_set_exchange_timeout_ns", "decode_flags",
    "sdk_timing_read",
]


class SdkError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s returned %s" % (where, _capi.STATUS_NAMES.get(
            status, str(status))))


def _check(rc, where):
    if rc != SDK_OK:
        raise SdkError(rc, where)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _cuda_contig(t, name, dtypes):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if t.dtype not in dtypes:
        raise ValueError("%s has dtype %s, expected one of %s" %
                         (name, t.dtype, dtypes))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t


def _x_dtype(t):
    return SDK_F32 if t.dtype == torch.float32 else SDK_BF16


# ------------------------------------------------------------- workspaces

def new_workspace(nbytes, device=None):
    """A zero-header workspace of at least nbytes (uint8 CUDA tensor)."""
    nbytes = max(int(nbytes), 256)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device or "cuda")
    sdk_workspace_init(ws)
    return ws


def sdk_workspace_init(ws, stream=None):
    _check(load().sdk_workspace_init(_ptr(ws), ws.numel(), _stream(stream)),
           "sdk_workspace_init")


def sdk_check_status(ws, stream=None):
    """(status, [err, info, enc_fallback_rows, enc_candidates]); clears the
    recorded status."""
    buf = (ctypes.c_uint32 * 4)()
    rc = load().sdk_check_status(_ptr(ws), _stream(stream), buf)
    return rc, list(buf)


def sdk_set_exchange_timeout_ns(ns):
    """Limit (ns) of the device waits for other CTAs' results; returns the
    previous limit (include/sdk.h, sdk_set_exchange_timeout_ns)."""
    return int(load().sdk_set_exchange_timeout_ns(int(ns)))


def sdk_timing_enable(on):
    """Brackets every decode attention-kernel launch with CUDA events
    (include/sdk.h, sdk_timing_enable); turning it on restarts at slot 0."""
    _check(load().sdk_timing_enable(1 if on else 0), "sdk_timing_enable")


def sdk_timing_read(max_n=_capi.SDK_TIMING_SLOTS):
    """Durations (ms) of the attention-kernel launches recorded in slots
    0 .. n-1 since the last enable (waits for them)."""
    buf = (ctypes.c_float * max(1, max_n))()
    n = load().sdk_timing_read(buf, max_n)
    if n < 0:
        raise SdkError(4, "sdk_timing_read")      # SDK_ERR_CUDA
    return [float(buf[i]) for i in range(n)]


def sdk_encode_workspace_bytes(n_vec, head_dim, n_atoms):
    return load().sdk_encode_workspace_bytes(n_vec, head_dim, n_atoms)


def sdk_append_workspace_bytes(B, Hkv, n_new, head_dim, n_atoms):
    return load().sdk_append_workspace_bytes(B, Hkv, n_new, head_dim, n_atoms)


def sdk_decode_workspace_bytes(B, Hq, head_dim, n_atoms, max_len):
    return load().sdk_decode_workspace_bytes(B, Hq, head_dim, n_atoms,
                                             max_len)


def sdk_decode_layout_of(B, Hq, head_dim, n_atoms, max_len):
    lay = DecodeLayout()
    _check(load().sdk_decode_layout_of(B, Hq, head_dim, n_atoms, max_len,
                                       ctypes.byref(lay)),
           "sdk_decode_layout_of")
    return {f: getattr(lay, f) for f, _ in DecodeLayout._fields_}


def read_select_state(ws, layout, R):
    """The per-head selection state of the last decode call as a dict of
    int64 tensors (z as float32)."""
    o = layout["state"]
    raw = ws[o:o + R * 4 * _capi.SELECT_STATE_WORDS].view(torch.int32)
    raw = raw.view(R, _capi.SELECT_STATE_WORDS).cpu()
    out = {}
    for i, f in enumerate(_capi.SELECT_STATE_FIELDS):
        col = raw[:, i].clone()
        out[f] = col.view(torch.float32) if f == "z" else (
            col.to(torch.int64) & 0xFFFFFFFF)
    # integer softmax: the sum of the integer exponentials (int64)
    out["isoft_sum"] = out["isoft_sum_lo"] | (out["isoft_sum_hi"] << 32)
    return out


# ------------------------------------------------------------------ encode

def _encode(fn_name, x, dictionary, k_atoms, codes, resid_sqnorm, workspace,
            stream):
    lib = load()
    x = _cuda_contig(x, "x", (torch.float32, torch.bfloat16))
    D = _cuda_contig(dictionary, "dictionary", (torch.bfloat16,))
    n_atoms, d = D.shape
    xv = x.reshape(-1, d)
    n_vec = xv.shape[0]
    if codes is None:
        codes = torch.empty(n_vec, k_atoms, dtype=torch.int32, device=x.device)
    if workspace is None:
        workspace = new_workspace(
            lib.sdk_encode_workspace_bytes(n_vec, d, n_atoms), x.device)
    rsq = None
    if resid_sqnorm:
        rsq = torch.empty(n_vec, dtype=torch.float32, device=x.device)
    rc = getattr(lib, fn_name)(_ptr(xv), _x_dtype(x), n_vec, d, _ptr(D),
                               n_atoms, k_atoms, _ptr(codes), _ptr(rsq),
                               _ptr(workspace), workspace.numel(),
                               _stream(stream))
    _check(rc, fn_name)
    return (codes, rsq) if resid_sqnorm else codes


def sdk_encode(x, dictionary, k_atoms=K_ATOMS, codes=None, resid_sqnorm=False,
               workspace=None, stream=None):
    """Greedy-pursuit codes of every row of x (last dim = head_dim) over the
    bf16 dictionary [n_atoms, head_dim].  Returns int32 words [n_vec,
    k_atoms] (uint32 bit patterns) and, if asked, ||r_final||^2."""
    return _encode("sdk_encode", x, dictionary, k_atoms, codes, resid_sqnorm,
                   workspace, stream)


def sdk_encode_simt(x, dictionary, k_atoms=K_ATOMS, codes=None,
                    resid_sqnorm=False, workspace=None, stream=None):
    """As sdk_encode, on the exact CUDA-core kernel."""
    return _encode("sdk_encode_simt", x, dictionary, k_atoms, codes,
                   resid_sqnorm, workspace, stream)


# ------------------------------------------------------------- code store

class CodeStore:
    """Device buffers of one layer's code store (layout of include/sdk.h).
    interleaved: k_full and v_full are views of one [B, Hkv, cap, 2, 16]
    array, so a token's key and value records form one 128-byte line."""

    def __init__(self, B, Hkv, cap, device="cuda", interleaved=False):
        self.B, self.Hkv, self.cap = B, Hkv, cap
        self.k_lo = torch.zeros(B, Hkv, KLOW_PLANES, cap, dtype=torch.int32,
                                device=device)
        if interleaved:
            kv = torch.zeros(B, Hkv, cap, 2, K_ATOMS, dtype=torch.int32,
                             device=device)
            self.k_full, self.v_full = kv[:, :, :, 0], kv[:, :, :, 1]
        else:
            self.k_full = torch.zeros(B, Hkv, cap, K_ATOMS, dtype=torch.int32,
                                      device=device)
            self.v_full = torch.zeros(B, Hkv, cap, K_ATOMS, dtype=torch.int32,
                                      device=device)
        self.lens = [0] * B

    @classmethod
    def from_tensors(cls, k_lo, k_full, v_full, lens):
        self = cls.__new__(cls)
        self.B, self.Hkv, _, self.cap = k_lo.shape
        self.k_lo, self.k_full, self.v_full = k_lo, k_full, v_full
        self.lens = [int(v) for v in lens]
        return self


def sdk_append(store, xk, xv, dict_k, dict_v, workspace=None, stream=None):
    """Encode xk, xv [B, Hkv, n_new, head_dim] and append them to `store` at
    positions lens[b]..lens[b]+n_new-1; then advances store.lens."""
    lib = load()
    xk = _cuda_contig(xk, "xk", (torch.float32, torch.bfloat16))
    xv = _cuda_contig(xv, "xv", (xk.dtype,))
    dk = _cuda_contig(dict_k, "dict_k", (torch.bfloat16,))
    dv = _cuda_contig(dict_v, "dict_v", (torch.bfloat16,))
    B, Hkv, n_new, d = xk.shape
    n_atoms = dk.shape[0]
    lens = (ctypes.c_int32 * B)(*store.lens)
    if workspace is None:
        workspace = new_workspace(
            lib.sdk_append_workspace_bytes(B, Hkv, n_new, d, n_atoms),
            xk.device)
    rc = lib.sdk_append(_ptr(xk), _ptr(xv), _x_dtype(xk), B, Hkv, n_new, d,
                        _ptr(dk), _ptr(dv), n_atoms, _ptr(store.k_lo),
                        _ptr(store.k_full), _ptr(store.v_full), store.cap,
                        lens, _ptr(workspace), workspace.numel(),
                        _stream(stream))
    _check(rc, "sdk_append")
    store.lens = [v + n_new for v in store.lens]
    return workspace


# ------------------------------------------------------------------ decode

def decode_flags(full_softmax=False, int_softmax=False, keep_keys=False, select=None):
    """The flags word of sdk_decode_attn; select: None (the library's
    default), "radix" or "bracket"."""
    if select not in (None, "radix", "bracket"):
        raise ValueError("select must be None, 'radix' or 'bracket'")
    return ((SDK_DECODE_FULL_SOFTMAX if full_softmax else 0) |
            (SDK_DECODE_INT_SOFTMAX if int_softmax else 0) |
            (SDK_DECODE_KEEP_KEYS if keep_keys else 0) |
            (SDK_DECODE_SELECT_RADIX if select == "radix" else 0) |
            (SDK_DECODE_SELECT_BRACKET if select == "bracket" else 0))


def sdk_decode_attn(q, dict_k, dict_v, store, klow=3, khigh=16, top_num=1,
                    top_den=10, full_softmax=False, scale=None, out=None,
                    workspace=None, stream=None, int_softmax=False,
                    keep_keys=False, select=None):
    """One layer of decode attention.  q [B, Hq, head_dim] fp32.  Returns
    out [B, Hq, head_dim] fp32 (and leaves the intermediate results in the
    workspace).  full_softmax / int_softmax / keep_keys set
    SDK_DECODE_FULL_SOFTMAX / SDK_DECODE_INT_SOFTMAX / SDK_DECODE_KEEP_KEYS."""
    lib = load()
    q = _cuda_contig(q, "q", (torch.float32,))
    dk = _cuda_contig(dict_k, "dict_k", (torch.bfloat16,))
    dv = _cuda_contig(dict_v, "dict_v", (torch.bfloat16,))
    B, Hq, d = q.shape
    n_atoms = dk.shape[0]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
    max_len = max(store.lens)
    if workspace is None:
        workspace = new_workspace(
            lib.sdk_decode_workspace_bytes(B, Hq, d, n_atoms, max_len),
            q.device)
    lens = (ctypes.c_int32 * B)(*store.lens)
    rc = lib.sdk_decode_attn(_ptr(q), B, Hq, store.Hkv, d, _ptr(dk), _ptr(dv),
                             n_atoms, _ptr(store.k_lo), _ptr(store.k_full),
                             _ptr(store.v_full), store.cap, lens, klow, khigh,
                             top_num, top_den,
                             decode_flags(full_softmax, int_softmax, keep_keys, select),
                             float(scale), _ptr(out), _ptr(workspace),
                             workspace.numel(), _stream(stream))
    _check(rc, "sdk_decode_attn")
    return out
