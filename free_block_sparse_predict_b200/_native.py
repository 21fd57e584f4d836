"""ctypes declarations of libsparge's C ABI (include/sparge.h)."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libsparge.so")

SPARGE_F16, SPARGE_BF16, SPARGE_F32 = 0, 1, 2


class SpargeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"sparge status {code}: {msg}")
        self.code = code


class SpargeParams(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
        ("N", ctypes.c_int32), ("d", ctypes.c_int32), ("bq", ctypes.c_int32),
        ("bk", ctypes.c_int32), ("tau", ctypes.c_float), ("theta", ctypes.c_float),
        ("lam", ctypes.c_float), ("scale", ctypes.c_float), ("causal", ctypes.c_int32),
        ("qk_int8", ctypes.c_int32), ("io_dtype", ctypes.c_int32), ("o_dtype", ctypes.c_int32),
    ]


class SpargeStats(ctypes.Structure):
    _fields_ = [("tiles", ctypes.c_uint64), ("qk_blocks", ctypes.c_uint64),
                ("pv_blocks", ctypes.c_uint64), ("pv_slices", ctypes.c_uint64),
                ("skipped_slices", ctypes.c_uint64)]


_P = ctypes.POINTER(SpargeParams)
_V = ctypes.c_void_p
_I = ctypes.c_int32
_S = ctypes.c_size_t

SIGNATURES = {
    "sparge_workspace_bytes": (_S, [_P]),
    "sparge_hilbert_workspace_bytes": (_S, [_I, _I, _I]),
    "sparge_hilbert_index": (ctypes.c_int, [_I, _I, _I, _I, _I, _V, _V, _S, _V]),
    "sparge_hilbert_permute": (ctypes.c_int, [_V, _V, _I, _I, _I, _I, ctypes.c_int, _V, _V]),
    "sparge_inverse_permute": (ctypes.c_int, [_V, _V, _I, _I, _I, _I, ctypes.c_int, _V, _V]),
    "sparge_predict_mask": (ctypes.c_int, [_P, _V, _V, _V, _V, _V, _V, _V, _V, _S, _V]),
    "sparge_predict_mask_noalloc": (ctypes.c_int, [_P, _V, _V, _V, _V, _V, _V, _V, _V]),
    "sparge_predict_pool": (ctypes.c_int, [_P, _V, _V, _V, _S, _V]),
    "sparge_predict_select": (ctypes.c_int, [_P, _V, _V, _V, _V, _V, _V, _S, _V]),
    "sparge_mask_compact": (ctypes.c_int, [_P, _V, _V, _V, _V]),
    "sparge_attn_fwd": (ctypes.c_int, [_P, _V, _V, _V, _V, _V, _V, _V, _S, _V, _V]),
    "sparge_device_status": (ctypes.c_int, [_V, _V]),
    "sparge_selftest_wait_timeout": (ctypes.c_int, [_V, _V]),
    "sparge_status_string": (ctypes.c_char_p, [ctypes.c_int]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built (no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise ImportError(
                f"libsparge.so not found at {lib_path}; build it with "
                "`python -m free_block_sparse_predict_b200.build` (needs nvcc)")
        L = ctypes.CDLL(lib_path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib
