"""ctypes declarations of libsdk.so (see include/sdk.h for the contracts).

Loading fails loudly when the library has not been built: there is no other
implementation of these operations in this package.
"""

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsdk.so")

SDK_OK = 0
STATUS_NAMES = {
    0: "SDK_OK", 1: "SDK_ERR_INVALID_ARG", 2: "SDK_ERR_UNSUPPORTED",
    3: "SDK_ERR_CAPACITY", 4: "SDK_ERR_CUDA", 5: "SDK_ERR_TIMEOUT",
    6: "SDK_ERR_DEVICE_CHECK",
}
SDK_F32, SDK_BF16 = 0, 1
SDK_DECODE_FULL_SOFTMAX, SDK_DECODE_INT_SOFTMAX, SDK_DECODE_KEEP_KEYS = 1, 2, 4
SDK_DECODE_SELECT_RADIX, SDK_DECODE_SELECT_BRACKET = 8, 16
MAX_ATOMS, K_ATOMS, KLOW_PLANES, MAX_BATCH, WS_ALIGN = 32768, 16, 3, 64, 256
DECODE_STATIC_WS_BYTES = 16 << 20

# every symbol include/sdk.h declares, with (restype, argtypes)
_vp, _i32, _i64, _sz, _f32 = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                              ctypes.c_size_t, ctypes.c_float)
SDK_TIMING_SLOTS = 256

SIGNATURES = {
    "sdk_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "sdk_version": (_i32, []),
    "sdk_set_exchange_timeout_ns": (ctypes.c_uint64, [ctypes.c_uint64]),
    "sdk_encode": (ctypes.c_int, [_vp, _i32, _i64, _i32, _vp, _i32, _i32, _vp,
                                  _vp, _vp, _sz, _vp]),
    "sdk_encode_simt": (ctypes.c_int, [_vp, _i32, _i64, _i32, _vp, _i32, _i32,
                                       _vp, _vp, _vp, _sz, _vp]),
    "sdk_encode_workspace_bytes": (_sz, [_i64, _i32, _i32]),
    "sdk_append": (ctypes.c_int, [_vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp,
                                  _vp, _i32, _vp, _vp, _vp, _i64, _vp, _vp,
                                  _sz, _vp]),
    "sdk_append_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i32]),
    "sdk_decode_attn": (ctypes.c_int, [_vp, _i32, _i32, _i32, _i32, _vp, _vp,
                                       _i32, _vp, _vp, _vp, _i64, _vp, _i32,
                                       _i32, _i32, _i32, _i32, _f32, _vp, _vp,
                                       _sz, _vp]),
    "sdk_decode_attn_static": (ctypes.c_int, [_vp, _i32, _i32, _i32, _i32,
                                              _vp, _vp, _i32, _vp, _vp, _vp,
                                              _i64, _vp, _i32, _i32, _i32,
                                              _i32, _i32, _f32, _vp, _vp,
                                              _vp]),
    "sdk_decode_attn_shard": (ctypes.c_int, [_i32, _i32, _i32, _vp, _vp, _i32,
                                             _i32, _i32, _i32, _vp, _vp, _i32,
                                             _vp, _vp, _vp, _i64, _vp, _vp,
                                             _i32, _i32, _i32, _i32, _i32, _f32,
                                             _vp, _vp, _sz, _vp]),
    "sdk_decode_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i64]),
    "sdk_decode_layout_of": (ctypes.c_int, [_i32, _i32, _i32, _i32, _i64,
                                            _vp]),
    "sdk_workspace_init": (ctypes.c_int, [_vp, _sz, _vp]),
    "sdk_check_status": (ctypes.c_int, [_vp, _vp, _vp]),
    "sdk_timing_enable": (ctypes.c_int, [_i32]),
    "sdk_timing_read": (_i32, [_vp, _i32]),
}


class DecodeLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "header", "qd", "keys", "hist1", "hist2", "state", "list", "cand_t",
        "cand_key", "sel_score", "w", "part", "total", "row")]


SELECT_STATE_FIELDS = ("kth_key", "k", "n_above", "n_cand", "n_sel", "n_comp",
                       "eq_total", "eq_taken", "max_score", "max_comp", "z",
                       "isoft_sum_lo", "isoft_sum_hi", "isoft_shift",
                       "bracket_lo", "bracket_hi", "select_path")
SELECT_STATE_WORDS = 20

_lib = None


def load():
    """The loaded library (ctypes.CDLL) with argument types declared."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            "libsdk.so is not built (expected at %s); run "
            "`python -m sparse_dictionary_coded_b200.build`" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
