"""The C-ABI library loads, exports every symbol include/sdk.h declares and
rejects invalid arguments on the host (no GPU needed: every call here fails
validation before anything would be launched)."""

import ctypes
import os
import re

import pytest

import sparse_dictionary_coded_b200 as sdk
from sparse_dictionary_coded_b200 import _capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sdk.h")


def _declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"SDK_API\s+[\w\s\*]+?\b(sdk_\w+)\s*\(", txt)))


@pytest.fixture(scope="module")
def lib():
    return sdk.load()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "sdk_encode" in names and "sdk_append" in names
    assert "sdk_decode_attn" in names
    for n in names:
        assert hasattr(lib, n), n
        assert n in _capi.SIGNATURES, "binding misses " + n


def test_binding_covers_only_declared_symbols():
    assert sorted(_capi.SIGNATURES) == _declared()


def test_status_strings(lib):
    for code, name in _capi.STATUS_NAMES.items():
        assert lib.sdk_status_string(code).decode().startswith(name)
    assert lib.sdk_status_string(99) == b"SDK_ERR_UNKNOWN"
    assert lib.sdk_version() == 2


def test_workspace_sizes(lib):
    lay = sdk.sdk_decode_layout_of(1, 32, 128, 32768, 4096)
    offs = [lay[k] for k in ("header", "qd", "keys", "hist1", "hist2", "state",
                             "list", "cand_t", "cand_key", "sel_score", "w",
                             "part", "total")]
    assert offs == sorted(offs)
    assert all(o % 256 == 0 for o in offs)
    assert lay["keys"] - lay["qd"] >= 32 * 32768 * 4
    assert lib.sdk_decode_workspace_bytes(1, 32, 128, 32768, 4096) == lay["total"]
    # per-token regions: rows of max_len rounded up to a multiple of 4
    assert lay["row"] == 4096
    assert sdk.sdk_decode_layout_of(2, 8, 64, 1000, 4097)["row"] == 4100
    assert lay["list"] - lay["state"] >= 0 and lay["cand_t"] - lay["list"] >= 32 * 4096 * 4
    assert lib.sdk_decode_workspace_bytes(0, 32, 128, 32768, 4096) == 0
    assert lib.sdk_decode_workspace_bytes(1, 32, 96, 32768, 4096) == 0
    assert lib.sdk_encode_workspace_bytes(1000, 128, 32768) >= 256
    assert lib.sdk_append_workspace_bytes(1, 8, 4, 128, 32768) >= 256 + 32 * 64


FAKE = ctypes.c_void_p(256 * 1024)          # never dereferenced: checks fail first
MISALIGNED = ctypes.c_void_p(256 * 1024 + 8)


def _decode(lib, **kw):
    a = dict(q=FAKE, B=1, Hq=4, Hkv=1, d=64, dk=FAKE, dv=FAKE, n=1024,
             k_lo=FAKE, k_full=FAKE, v_full=FAKE, cap=256,
             lens=(ctypes.c_int32 * 1)(256), klow=3, khigh=16, top_num=1,
             top_den=10, full=0, scale=0.125, out=FAKE, ws=FAKE, ws_bytes=0)
    a.update(kw)
    return lib.sdk_decode_attn(a["q"], a["B"], a["Hq"], a["Hkv"], a["d"],
                               a["dk"], a["dv"], a["n"], a["k_lo"],
                               a["k_full"], a["v_full"], a["cap"], a["lens"],
                               a["klow"], a["khigh"], a["top_num"],
                               a["top_den"], a["full"], a["scale"], a["out"],
                               a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(B=0), 1), (dict(B=65), 1), (dict(Hq=6, Hkv=4), 1),
    (dict(d=96), 2), (dict(n=32769), 1), (dict(n=0), 1),
    (dict(klow=0), 1), (dict(klow=5, khigh=4), 1), (dict(khigh=17), 1),
    (dict(top_num=0), 1), (dict(top_num=11), 1), (dict(scale=0.0), 1),
    (dict(scale=float("nan")), 1), (dict(q=None), 1), (dict(ws=None), 1),
    (dict(ws=MISALIGNED), 1), (dict(lens=(ctypes.c_int32 * 1)(0)), 1),
    (dict(lens=(ctypes.c_int32 * 1)(257)), 1),
    (dict(ws_bytes=1024), 3),                 # workspace too small
    (dict(q=MISALIGNED), 1),                  # q must be 16-byte aligned
    (dict(full=32), 1),                       # unknown flag bit
    (dict(full=24), 1),                       # both selection flags
])
def test_decode_rejects_bad_arguments(lib, kw, status):
    assert _decode(lib, **kw) == status


def _encode(lib, fn="sdk_encode", **kw):
    a = dict(x=FAKE, dt=0, n_vec=10, d=128, dict_=FAKE, n=32768, k=16,
             codes=FAKE, rsq=None, ws=FAKE, ws_bytes=0)
    a.update(kw)
    return getattr(lib, fn)(a["x"], a["dt"], a["n_vec"], a["d"], a["dict_"],
                            a["n"], a["k"], a["codes"], a["rsq"], a["ws"],
                            a["ws_bytes"], None)


@pytest.mark.parametrize("fn", ["sdk_encode", "sdk_encode_simt"])
@pytest.mark.parametrize("kw,status", [
    (dict(n_vec=-1), 1), (dict(d=32), 2), (dict(n=0), 1), (dict(n=40000), 1),
    (dict(k=0), 1), (dict(k=17), 1), (dict(dt=7), 1), (dict(x=None), 1),
    (dict(codes=None), 1), (dict(dict_=MISALIGNED), 1), (dict(ws=None), 1),
    (dict(ws_bytes=16), 3),
])
def test_encode_rejects_bad_arguments(lib, fn, kw, status):
    assert _encode(lib, fn, **kw) == status


def test_encode_zero_vectors_is_a_no_op(lib):
    # n_vec == 0 returns before any launch
    assert _encode(lib, n_vec=0, ws_bytes=1 << 20) == 0


def test_append_capacity_and_arguments(lib):
    lens = (ctypes.c_int32 * 2)(10, 250)
    args = [FAKE, FAKE, 0, 2, 8, 8, 128, FAKE, FAKE, 32768, FAKE, FAKE, FAKE,
            256, lens, FAKE, 1 << 30, None]
    assert lib.sdk_append(*args) == 3          # 250 + 8 > 256
    args[3] = 0
    assert lib.sdk_append(*args) == 1          # B = 0
    args[3] = 2
    args[6] = 80
    assert lib.sdk_append(*args) == 2          # head_dim
    args[6] = 128
    args[14] = None
    assert lib.sdk_append(*args) == 1          # lens missing


def test_workspace_helpers_reject_bad_pointers(lib):
    assert lib.sdk_workspace_init(None, 1024, None) == 1
    assert lib.sdk_workspace_init(MISALIGNED, 1024, None) == 1
    assert lib.sdk_workspace_init(FAKE, 16, None) == 1
    assert lib.sdk_check_status(None, None, None) == 1
    assert lib.sdk_decode_layout_of(1, 4, 64, 1024, 256, None) == 1


def test_timing_calls_check_their_arguments(lib):
    # machine-independent: no device is queried for these
    assert lib.sdk_timing_read(None, 4) == -1
    buf = (ctypes.c_float * 4)()
    assert lib.sdk_timing_read(buf, -1) == -1
    assert lib.sdk_timing_enable(0) == 0
