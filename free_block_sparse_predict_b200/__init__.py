"""Python binding of libsparge, the sm_100a SpargeAttn sparse-attention library.

Every function here has the name of the C entry point it wraps (include/sparge.h)
and only marshals arguments: tensors become device pointers, the current torch
stream becomes the launch stream, and a non-zero status raises SpargeError.  All
computation happens in the library's CUDA kernels; there is no fallback.

PyTorch supplies device memory and streams.  Helpers at the end
(``workspace``, ``predict_outputs``, ``sparge_forward``) only allocate buffers
with torch and chain the entry points.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

from ._native import (SPARGE_BF16, SPARGE_F16, SPARGE_F32, SpargeError, SpargeParams,
                      SpargeStats, lib, lib_path)

__all__ = [
    "SpargeError", "SpargeParams", "SpargeStats", "make_params", "lib_path",
    "sparge_workspace_bytes", "sparge_hilbert_workspace_bytes", "sparge_hilbert_index",
    "sparge_hilbert_permute", "sparge_inverse_permute", "sparge_predict_mask",
    "sparge_predict_pool", "sparge_predict_select", "sparge_predict_mask_noalloc",
    "sparge_mask_compact", "sparge_attn_fwd", "sparge_device_status",
    "sparge_selftest_wait_timeout", "sparge_status_string",
    "workspace", "predict_outputs", "sparge_forward",
]

_DT = {torch.float16: SPARGE_F16, torch.bfloat16: SPARGE_BF16, torch.float32: SPARGE_F32}


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    if not t.is_cuda:
        raise SpargeError(1, "expected a CUDA tensor")
    if not t.is_contiguous():
        raise SpargeError(1, "expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _check(code: int) -> None:
    if code != 0:
        raise SpargeError(code, sparge_status_string(code))


_TD = {SPARGE_F16: torch.float16, SPARGE_BF16: torch.bfloat16, SPARGE_F32: torch.float32}


def _need(t, name: str, numel: int, dtype, device) -> None:
    """The C ABI takes bare pointers and trusts the sizes that the parameters
    imply; a tensor that is smaller, of another element type or on another
    device would be read or written out of bounds, so it is refused here."""
    if t is None:
        return
    if not t.is_cuda or t.device != device:
        raise SpargeError(1, f"{name}: expected a tensor on {device}, got {t.device}")
    if numel == 0:
        return                      # an empty problem touches no memory
    if dtype is not None and t.dtype != dtype:
        raise SpargeError(1, f"{name}: expected {dtype}, got {t.dtype}")
    if t.numel() < numel:
        raise SpargeError(1, f"{name}: needs {numel} elements, has {t.numel()}")


def _tiles(params):
    B, Hq, Hkv = params.B, params.Hq, params.Hkv
    Tm = -(-params.N // params.bq) if params.bq > 0 else 0
    Tn = -(-params.N // params.bk) if params.bk > 0 else 0
    return B, Hq, Hkv, Tm, Tn


def _need_qk(params, q, k, v=None) -> None:
    io = _TD.get(params.io_dtype)
    dev = q.device
    _need(q, "q", params.B * params.Hq * params.N * params.d, io, dev)
    _need(k, "k", params.B * params.Hkv * params.N * params.d, io, dev)
    _need(v, "v", params.B * params.Hkv * params.N * params.d, io, dev)


def _need_mask(params, dev, mask=None, kv_idx=None, kv_cnt=None, s_q=None, s_k=None) -> None:
    B, Hq, Hkv, Tm, Tn = _tiles(params)
    _need(mask, "mask", B * Hq * Tm * Tn, torch.uint8, dev)
    _need(kv_idx, "kv_idx", B * Hq * Tm * Tn, torch.int32, dev)
    _need(kv_cnt, "kv_cnt", B * Hq * Tm, torch.int32, dev)
    _need(s_q, "s_q", B * Hq * Tm, torch.float32, dev)
    _need(s_k, "s_k", B * Hkv * Tn, torch.float32, dev)


def make_params(B, Hq, Hkv, N, d, tau, theta, lam, causal=False, qk_int8=False,
                io_dtype=torch.float16, o_dtype=None, scale=None, bq=128, bk=64) -> SpargeParams:
    """Hyper-parameters of one call: shapes, b_q/b_k, tau, theta, lambda, causal, INT8."""
    p = SpargeParams()
    p.B, p.Hq, p.Hkv, p.N, p.d, p.bq, p.bk = B, Hq, Hkv, N, d, bq, bk
    p.tau, p.theta, p.lam = float(tau), float(theta), float(lam)
    p.scale = float(scale) if scale is not None else 1.0 / math.sqrt(d)
    p.causal, p.qk_int8 = int(bool(causal)), int(bool(qk_int8))
    p.io_dtype = _DT[io_dtype]
    p.o_dtype = _DT[o_dtype if o_dtype is not None else io_dtype]
    return p


def sparge_workspace_bytes(params: SpargeParams) -> int:
    return int(lib().sparge_workspace_bytes(ctypes.byref(params)))


def sparge_hilbert_workspace_bytes(T: int, Hg: int, Wg: int) -> int:
    return int(lib().sparge_hilbert_workspace_bytes(T, Hg, Wg))


def sparge_hilbert_index(N, prefix_len, T, Hg, Wg, perm, ws, stream=None) -> None:
    _need(perm, "perm", max(int(N), 0), torch.int32, perm.device)
    _need(ws, "ws", 0, None, perm.device)
    _check(lib().sparge_hilbert_index(N, prefix_len, T, Hg, Wg, _ptr(perm), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream)))


def _perm_call(fn, src, dst, perm, stream):
    if src.dim() != 4 or src.shape != dst.shape or src.dtype != dst.dtype:
        raise SpargeError(1, "expected two [B, H, N, d] tensors of one shape and dtype")
    B, H, N, d = src.shape
    _need(dst, "destination", 0, None, src.device)
    _need(perm, "perm", N, torch.int32, src.device)
    _check(fn(_ptr(src), _ptr(dst), B, H, N, d, _DT[src.dtype], _ptr(perm), _stream(stream)))


def sparge_hilbert_permute(x, y, perm, stream=None) -> None:
    """y[b, h, p] = x[b, h, perm[p]]"""
    _perm_call(lib().sparge_hilbert_permute, x, y, perm, stream)


def sparge_inverse_permute(y, x, perm, stream=None) -> None:
    """x[b, h, perm[p]] = y[b, h, p]"""
    _perm_call(lib().sparge_inverse_permute, y, x, perm, stream)


def sparge_predict_mask(params, q, k, mask, kv_idx, kv_cnt, s_q, s_k, ws, stream=None) -> None:
    _need_qk(params, q, k)
    _need_mask(params, q.device, mask, kv_idx, kv_cnt, s_q, s_k)
    _need(ws, "ws", 0, None, q.device)
    _check(lib().sparge_predict_mask(ctypes.byref(params), _ptr(q), _ptr(k), _ptr(mask),
                                     _ptr(kv_idx), _ptr(kv_cnt), _ptr(s_q), _ptr(s_k), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)))


def sparge_predict_pool(params, q, k, ws, stream=None) -> None:
    """First half of sparge_predict_mask: block means, self-similarities and
    (qk_int8) the INT8 codes, written into ws."""
    _need_qk(params, q, k)
    _need(ws, "ws", 0, None, q.device)
    _check(lib().sparge_predict_pool(ctypes.byref(params), _ptr(q), _ptr(k), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)))


def sparge_predict_select(params, mask, kv_idx, kv_cnt, s_q, s_k, ws, stream=None) -> None:
    """Second half: the block mask and skip list from what sparge_predict_pool
    left in the same ws."""
    _need(ws, "ws", 0, None, ws.device)
    _need_mask(params, ws.device, mask, kv_idx, kv_cnt, s_q, s_k)
    _check(lib().sparge_predict_select(ctypes.byref(params), _ptr(mask), _ptr(kv_idx),
                                       _ptr(kv_cnt), _ptr(s_q), _ptr(s_k), _ptr(ws),
                                       ws.numel() * ws.element_size(), _stream(stream)))


def sparge_predict_mask_noalloc(params, q, k, mask, kv_idx, kv_cnt, s_q=None, s_k=None,
                                stream=None) -> None:
    """sparge_predict_mask without a workspace: for callers that cannot
    allocate device memory when they call it.  The library's own static
    device scratch (32 MiB per GPU) holds the intermediates; calls that run
    concurrently on the GPU share it and race."""
    _need_qk(params, q, k)
    _need_mask(params, q.device, mask, kv_idx, kv_cnt, s_q, s_k)
    _check(lib().sparge_predict_mask_noalloc(ctypes.byref(params), _ptr(q), _ptr(k), _ptr(mask),
                                             _ptr(kv_idx), _ptr(kv_cnt), _ptr(s_q), _ptr(s_k),
                                             _stream(stream)))


def sparge_mask_compact(params, mask, kv_idx, kv_cnt, stream=None) -> None:
    _need_mask(params, mask.device, mask, kv_idx, kv_cnt)
    _check(lib().sparge_mask_compact(ctypes.byref(params), _ptr(mask), _ptr(kv_idx),
                                     _ptr(kv_cnt), _stream(stream)))


def sparge_attn_fwd(params, q, k, v, kv_idx, kv_cnt, o, ws, stats=None, stream=None) -> None:
    _need_qk(params, q, k, v)
    _need_mask(params, q.device, kv_idx=kv_idx, kv_cnt=kv_cnt)
    _need(o, "o", params.B * params.Hq * params.N * params.d, _TD.get(params.o_dtype), q.device)
    _need(ws, "ws", 0, None, q.device)
    if stats is not None:
        _need(stats, "stats", 0, None, q.device)
        if stats.numel() * stats.element_size() < ctypes.sizeof(SpargeStats):
            raise SpargeError(1, f"stats: needs {ctypes.sizeof(SpargeStats)} bytes")
    _check(lib().sparge_attn_fwd(ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v), _ptr(kv_idx),
                                 _ptr(kv_cnt), _ptr(o), _ptr(ws), ws.numel() * ws.element_size(),
                                 _ptr(stats), _stream(stream)))


def sparge_device_status(ws, stream=None) -> int:
    return int(lib().sparge_device_status(_ptr(ws), _stream(stream)))


def sparge_selftest_wait_timeout(ws, stream=None) -> None:
    """Runs the unsatisfiable bounded wait; sparge_device_status then reports
    SPARGE_ETIMEOUT (4)."""
    _check(lib().sparge_selftest_wait_timeout(_ptr(ws), _stream(stream)))


def sparge_status_string(code: int) -> str:
    return lib().sparge_status_string(int(code)).decode()


# ----------------------------------------------------------------------------
# allocation helpers (torch memory only)
# ----------------------------------------------------------------------------

def workspace(params: SpargeParams, device="cuda") -> torch.Tensor:
    n = sparge_workspace_bytes(params)
    if n == 0:
        raise SpargeError(1, "invalid parameters")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def predict_outputs(params: SpargeParams, device="cuda"):
    """mask [B,Hq,Tm,Tn] u8, kv_idx [B,Hq,Tm,Tn] i32, kv_cnt [B,Hq,Tm] i32,
    s_q [B,Hq,Tm] f32, s_k [B,Hkv,Tn] f32."""
    Tm, Tn = -(-params.N // params.bq), -(-params.N // params.bk)
    B, Hq, Hkv = params.B, params.Hq, params.Hkv
    return (torch.empty((B, Hq, Tm, Tn), dtype=torch.uint8, device=device),
            torch.empty((B, Hq, Tm, Tn), dtype=torch.int32, device=device),
            torch.empty((B, Hq, Tm), dtype=torch.int32, device=device),
            torch.empty((B, Hq, Tm), dtype=torch.float32, device=device),
            torch.empty((B, Hkv, Tn), dtype=torch.float32, device=device))


def sparge_forward(params, q, k, v, perm=None, ws=None, stats=None, stream=None):
    """permute (optional) -> predict -> attention -> inverse permute.

    Returns (o, mask, kv_idx, kv_cnt).  ``perm`` is a device table from
    sparge_hilbert_index; ``ws`` a workspace of sparge_workspace_bytes."""
    dev = q.device
    if ws is None:
        ws = workspace(params, dev)
    if perm is not None:
        qp, kp, vp = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        sparge_hilbert_permute(q, qp, perm, stream)
        sparge_hilbert_permute(k, kp, perm, stream)
        sparge_hilbert_permute(v, vp, perm, stream)
        q, k, v = qp, kp, vp
    mask, kv_idx, kv_cnt, s_q, s_k = predict_outputs(params, dev)
    sparge_predict_mask(params, q, k, mask, kv_idx, kv_cnt, None, None, ws, stream)
    odt = {SPARGE_F16: torch.float16, SPARGE_BF16: torch.bfloat16, SPARGE_F32: torch.float32}
    o = torch.empty(q.shape, dtype=odt[params.o_dtype], device=dev)
    sparge_attn_fwd(params, q, k, v, kv_idx, kv_cnt, o, ws, stats, stream)
    if perm is not None:
        out = torch.empty_like(o)
        sparge_inverse_permute(o, out, perm, stream)
        o = out
    return o, mask, kv_idx, kv_cnt
