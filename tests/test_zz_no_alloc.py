"""sdk_decode_attn_static (decode attention with the library's own fixed
device workspace) against sdk_decode_attn with a caller workspace, through
the C ABI.  Collected last on purpose: it must also pass after every other
GPU test has run in the same process."""

import ctypes

import pytest
import torch

import workloads
import sparse_dictionary_coded_b200 as sdk
from sparse_dictionary_coded_b200 import _capi

pytestmark = pytest.mark.gpu

TOL = 1e-5      # out is summed with fp32 atomics: the order may differ


def _case(seed, B, Hq, Hkv, N, d, n, cap=None):
    g = workloads.make_gen(seed)
    DK = workloads.gaussian_dictionary(n, d, g).cuda()
    DV = workloads.gaussian_dictionary(n, d, g).cuda()
    kw = workloads.random_codes((B, Hkv, N), n, g)
    vw = workloads.random_codes((B, Hkv, N), n, g)
    q = workloads.queries(B, Hq, d, g)
    q = (q / q.norm(dim=-1, keepdim=True)).cuda()
    return q, DK, DV, kw, vw, cap


def _store(kw, vw, lens, cap=None):
    k_lo, k_full, v_full = workloads.layout(kw, vw, cap)
    return sdk.CodeStore.from_tensors(k_lo.cuda(), k_full.cuda(),
                                      v_full.cuda(), lens)


def _static(q, DK, DV, store, out, status=None, full=False):
    """One call of the new entry point through ctypes."""
    lib = sdk.load()
    B, Hq, d = q.shape
    lens = (ctypes.c_int32 * B)(*store.lens)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return lib.sdk_decode_attn_static(
        p(q), B, Hq, store.Hkv, d, p(DK), p(DV), DK.shape[0], p(store.k_lo),
        p(store.k_full), p(store.v_full), store.cap, lens, 3, 16, 1, 10,
        1 if full else 0, 1.0 / d ** 0.5, p(out),
        None if status is None else p(status), None)


def _reference(q, DK, DV, store, full=False):
    B, Hq, d = q.shape
    ws = sdk.new_workspace(sdk.sdk_decode_workspace_bytes(
        B, Hq, d, DK.shape[0], max(store.lens)))
    out = sdk.sdk_decode_attn(q, DK, DV, store, full_softmax=full,
                              workspace=ws)
    torch.cuda.synchronize()
    assert sdk.sdk_check_status(ws)[0] == 0
    return out


@pytest.mark.parametrize("full", [False, True])
def test_layer_of_4096_tokens_twice_in_a_row(full):
    """B=1, 32 query heads over 8 KV heads, 4096 tokens, 32768 atoms, d=128
    (a decode workspace that fits the fixed array): two consecutive calls
    both match the call with a caller-owned workspace, and report no
    device-side failure."""
    assert sdk.sdk_decode_workspace_bytes(1, 32, 128, 32768, 4096) <= \
        _capi.DECODE_STATIC_WS_BYTES
    q, DK, DV, kw, vw, _ = _case(71, 1, 32, 8, 4096, 128, 32768)
    store = _store(kw, vw, [4096])
    ref = _reference(q, DK, DV, store, full)
    status = torch.full((2,), 77, dtype=torch.int32, device="cuda")
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        assert _static(q, DK, DV, store, out, status, full) == 0
        torch.cuda.synchronize()
        assert status.tolist() == [0, 0]
        assert torch.allclose(out, ref, rtol=0.0, atol=TOL)


def test_ragged_batch_and_no_status_words():
    """Three sequences of 1, 5 and 333 tokens (d=64, 1000 atoms), first
    without status words, then with them."""
    q, DK, DV, kw, vw, _ = _case(72, 3, 4, 2, 400, 64, 1000)
    store = _store(kw, vw, [1, 5, 333], cap=400)
    ref = _reference(q, DK, DV, store)
    out = torch.empty_like(ref)
    assert _static(q, DK, DV, store, out) == 0
    torch.cuda.synchronize()
    assert torch.allclose(out, ref, rtol=0.0, atol=TOL)
    status = torch.full((2,), 5, dtype=torch.int32, device="cuda")
    out2 = torch.empty_like(ref)
    assert _static(q, DK, DV, store, out2, status) == 0
    torch.cuda.synchronize()
    assert status.tolist() == [0, 0]
    assert torch.allclose(out2, ref, rtol=0.0, atol=TOL)


def test_beyond_the_fixed_size_is_rejected_before_launch():
    """A workspace need above SDK_DECODE_STATIC_WS_BYTES returns
    SDK_ERR_CAPACITY and leaves the output untouched."""
    B, Hq, d, n, N = 1, 32, 128, 32768, 16384
    assert sdk.sdk_decode_workspace_bytes(B, Hq, d, n, N) > \
        _capi.DECODE_STATIC_WS_BYTES
    g = workloads.make_gen(73)
    DK = workloads.gaussian_dictionary(n, d, g).cuda()
    store = sdk.CodeStore(B, 8, N)
    store.lens = [N]
    q = torch.randn(B, Hq, d, generator=g).cuda()
    out = torch.full((B, Hq, d), 3.0, device="cuda")
    assert _static(q, DK, DK, store, out) == 3
    torch.cuda.synchronize()
    assert torch.all(out == 3.0)


def test_device_check_is_reported_once():
    """An atom index beyond the dictionary is recorded on the device, copied
    to the status words of that call, and cleared for the next call."""
    q, DK, DV, kw, vw, _ = _case(74, 1, 2, 1, 64, 64, 1000)
    kw[0, 0, 10, 0] = (kw[0, 0, 10, 0] & ~0x7FFF) | 1500
    store = _store(kw, vw, [64])
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    out = torch.empty(1, 2, 64, device="cuda")
    assert _static(q, DK, DV, store, out, status) == 0
    torch.cuda.synchronize()
    assert status.tolist() == [6, 1500]
    kw[0, 0, 10, 0] = kw[0, 0, 10, 0] & ~0x7FFF
    store = _store(kw, vw, [64])
    assert _static(q, DK, DV, store, out, status) == 0
    torch.cuda.synchronize()
    assert status.tolist() == [0, 0]
