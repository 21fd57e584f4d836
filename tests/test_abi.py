"""The C-ABI library loads, exports every symbol its header declares, and
rejects bad arguments on the host before touching the GPU.  No GPU needed:
no call here reaches a CUDA runtime function."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sparge.h")


@pytest.fixture(scope="module")
def native():
    from free_block_sparse_predict_b200 import build
    build.build()
    from free_block_sparse_predict_b200 import _native
    return _native


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sparge_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(native):
    lib = ctypes.CDLL(native.lib_path)
    names = declared_symbols()
    assert len(names) >= 10
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(native.SIGNATURES)


def test_status_strings(native):
    L = native.lib()
    for code in range(7):
        assert L.sparge_status_string(code)
    assert L.sparge_status_string(99) == b"unknown status"


def _params(native, **kw):
    p = native.SpargeParams()
    base = dict(B=1, Hq=32, Hkv=8, N=131072, d=128, bq=128, bk=64, tau=0.95, theta=0.6,
                lam=-8.0, scale=128 ** -0.5, causal=1, qk_int8=1, io_dtype=1, o_dtype=1)
    base.update(kw)
    for k, v in base.items():
        setattr(p, k, v)
    return p


def test_workspace_bytes_covers_every_region(native):
    L = native.lib()
    p = _params(native)
    n = L.sparge_workspace_bytes(ctypes.byref(p))
    B, Hq, Hkv, N, d = 1, 32, 8, 131072, 128
    Tm, Tn = N // 128, N // 64
    floor = (B * Hq * Tm * d * 4 + B * Hkv * Tn * d * 4      # pooled means
             + B * Hkv * N * d * 2                           # fp16 V
             + B * (Hq + Hkv) * N * d                        # INT8 codes
             + B * Hkv * Tn * d * 8)                         # float64 K block sums (kbar)
    assert floor <= n <= floor + 16 * 1024 * 1024
    assert L.sparge_workspace_bytes(ctypes.byref(_params(native, qk_int8=0, io_dtype=0,
                                                          o_dtype=0))) < n


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=6, Hkv=4), 1), (dict(tau=0.0), 1), (dict(tau=float("nan")), 1),
    (dict(lam=0.5), 1), (dict(scale=-1.0), 1), (dict(io_dtype=2), 1), (dict(o_dtype=0), 1),
    (dict(d=96), 2), (dict(bq=64), 2), (dict(qk_int8=1, d=64), 2), (dict(N=400000), 2),
])
def test_invalid_parameters_rejected_before_launch(native, kw, code):
    L = native.lib()
    p = _params(native, **kw)
    assert L.sparge_workspace_bytes(ctypes.byref(p)) == 0
    fake = ctypes.c_void_p(0x10000)
    r = L.sparge_predict_mask(ctypes.byref(p), fake, fake, fake, fake, fake, None, None, fake,
                              1 << 40, None)
    assert r == code


def test_null_pointers_and_small_workspace(native):
    L = native.lib()
    p = _params(native)
    fake = ctypes.c_void_p(0x10000)
    assert L.sparge_predict_mask(None, fake, fake, fake, fake, fake, None, None, fake, 1 << 40,
                                 None) == 1
    assert L.sparge_predict_mask(ctypes.byref(p), None, fake, fake, fake, fake, None, None, fake,
                                 1 << 40, None) == 1
    # the two halves of the predictor check their own arguments
    assert L.sparge_predict_pool(ctypes.byref(p), None, fake, fake, 1 << 40, None) == 1
    assert L.sparge_predict_pool(ctypes.byref(p), fake, fake, None, 1 << 40, None) == 1
    assert L.sparge_predict_pool(ctypes.byref(p), fake, fake, fake, 1024, None) == 5
    assert L.sparge_predict_select(ctypes.byref(p), None, fake, fake, None, None, fake, 1 << 40,
                                   None) == 1
    assert L.sparge_predict_select(ctypes.byref(p), fake, fake, fake, None, None, fake, 1024,
                                   None) == 5
    assert L.sparge_attn_fwd(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, 1024,
                             None, None) == 5
    misaligned = ctypes.c_void_p(0x10008)
    assert L.sparge_attn_fwd(ctypes.byref(p), misaligned, fake, fake, fake, fake, fake, fake,
                             1 << 40, None, None) == 1
    # empty problems succeed without a launch
    assert L.sparge_attn_fwd(ctypes.byref(_params(native, N=0)), None, None, None, None, None,
                             None, None, 0, None, None) == 0
    assert L.sparge_hilbert_permute(fake, fake, 1, 2, 0, 64, 0, fake, None) == 0


def test_hilbert_validation(native):
    L = native.lib()
    assert L.sparge_hilbert_workspace_bytes(13, 30, 45) >= 4 * (64 ** 3 // 1024)
    assert L.sparge_hilbert_index(100, 10, 1, 10, 10, ctypes.c_void_p(0x10000),
                                  ctypes.c_void_p(0x20000), 1 << 20, None) == 1  # grid too big
    assert L.sparge_hilbert_index(4096, 0, 1, 64, 64, ctypes.c_void_p(0x10000),
                                  ctypes.c_void_p(0x20000), 4, None) == 5
    fake = ctypes.c_void_p(0x10000)
    assert L.sparge_hilbert_permute(fake, fake, 1, 2, 16, 64, 0, fake, None) == 1   # overlap
    assert L.sparge_hilbert_permute(fake, ctypes.c_void_p(0x90000), 1, 2, 16, 4, 0, fake,
                                    None) == 2                                        # 8-byte rows
