"""Seeded synthetic workloads for the sparse-attention hot path.

This module is shared by the CPU oracle, the tests and the benchmark.  It holds
no step of the attention method itself: it only draws Q, K, V tensors with the
shapes, dtypes and structure of the five workloads below, and converts the
stored 16-bit values to float for whoever consumes them.

The structures stand in for the pages' model tensors (Llama3.1, CogVideoX,
Mochi, Flux; "SpargeAttn" paper review, section 六 experiments), which are not
available here:

  tiny         B1 H1 N1024 d64 fp16: 16 segments of 64 tokens, each a centroid
               N(0,1)^d plus per-token N(0,0.3^2); 4 random segments iid N(0,1).
  image_dit    B1 H24 N4608 d128 bf16: 512 iid text tokens, then a 64x64 grid
               from a stationary Gaussian random field (covariance
               exp(-r^2 / (2*4^2))) with N(0,0.1^2) noise.
  video_dit    B1 H24 N17776 d64 fp16: 226 iid text tokens, then a 13x30x45 grid
               from a 3D field (covariance exp(-dt^2/(2*2^2) - (dy^2+dx^2)/(2*4^2)))
               with N(0,0.1^2) noise.
  llm_32k      B1 Hq32 Hkv8 N32768 d128 bf16 causal: AR(1) tokens
               x_t = 0.95 x_{t-1} + N(0,0.3^2), a x8 sink key at position 0 and
               16 needle key blocks copied from causally later query blocks.
  llm_128k     as llm_32k at N=131072, with the INT8 QK path.

All randomness is NumPy PCG64; Q, K and V use independent streams spawned from
SeedSequence(seed).  Values are drawn in float32/float64 and rounded once
(round-to-nearest-even) to the workload dtype; bf16 is carried as uint16 bit
patterns because NumPy has no bf16 type.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "get_workload", "make_qkv", "bf16_bits_from_f32",
    "to_f64", "to_f32", "grid_of",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    dtype: str            # "f16" or "bf16"
    causal: bool
    tau: float
    theta: float
    lam: float
    bq: int = 128
    bk: int = 64
    qk_int8: bool = False
    prefix_len: int = 0   # text tokens kept in front of the grid
    grid: tuple = ()      # (T, H, W) of the visual-token grid, () if none
    kind: str = "segments"

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 1, 1024, 64, "f16", False, 0.9, 0.5, -5.0,
                     kind="segments"),
    "image_dit": Workload("image_dit", 1, 24, 24, 4608, 128, "bf16", False, 0.9, 0.6, -6.0,
                          prefix_len=512, grid=(1, 64, 64), kind="grf"),
    "video_dit": Workload("video_dit", 1, 24, 24, 17776, 64, "f16", False, 0.92, 0.6, -6.0,
                          prefix_len=226, grid=(13, 30, 45), kind="grf"),
    "llm_32k": Workload("llm_32k", 1, 32, 8, 32768, 128, "bf16", True, 0.95, 0.6, -8.0,
                        kind="ar1"),
    "llm_128k": Workload("llm_128k", 1, 32, 8, 131072, 128, "bf16", True, 0.95, 0.6, -8.0,
                         qk_int8=True, kind="ar1"),
}


def get_workload(name: str, **overrides) -> Workload:
    return WORKLOADS[name].replace(**overrides) if overrides else WORKLOADS[name]


def grid_of(w: Workload):
    """(prefix_len, T, H, W) of the token grid, or None without one."""
    if not w.grid:
        return None
    T, H, W = w.grid
    return (w.prefix_len, T, H, W)


# ----------------------------------------------------------------------------
# 16-bit storage helpers
# ----------------------------------------------------------------------------

def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even) and return the uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> 16) & np.uint32(1)
    r = (u + (np.uint32(0x7FFF) + lsb)) >> 16
    return r.astype(np.uint16)


def to_f32(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float32 value of stored 16-bit data."""
    if dtype == "f16":
        return a.astype(np.float32)
    if dtype == "bf16":
        return (a.astype(np.uint32) << 16).view(np.float32)
    if dtype == "f32":
        return a.astype(np.float32)
    raise ValueError(dtype)


def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    return to_f32(a, dtype).astype(np.float64)


def _store(x32: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f16":
        return x32.astype(np.float16)
    if dtype == "bf16":
        return bf16_bits_from_f32(x32)
    raise ValueError(dtype)


# ----------------------------------------------------------------------------
# generators
# ----------------------------------------------------------------------------

def _segments(rng: np.random.Generator, H: int, N: int, d: int, seg: int = 64,
              n_random: int = 4) -> np.ndarray:
    nseg = N // seg
    out = np.empty((H, N, d), dtype=np.float32)
    for h in range(H):
        centroids = rng.standard_normal((nseg, d))
        noise = 0.3 * rng.standard_normal((nseg, seg, d))
        x = centroids[:, None, :] + noise
        rand_ids = rng.choice(nseg, size=n_random, replace=False)
        x[rand_ids] = rng.standard_normal((n_random, seg, d))
        out[h] = x.reshape(N, d)
    return out


def _grf_spectrum(shape, corr):
    """Square root of the spectral density of a Gaussian covariance on a torus."""
    axes = []
    for n, c in zip(shape, corr):
        r = np.minimum(np.arange(n), n - np.arange(n)).astype(np.float64)
        axes.append(np.exp(-r * r / (2.0 * c * c)))
    cov = axes[0]
    for a in axes[1:]:
        cov = np.multiply.outer(cov, a)
    spec = np.fft.rfftn(cov).real
    return np.sqrt(np.maximum(spec, 0.0))


def _grf_fields(rng, n_fields, grid, corr, pad):
    """n_fields independent unit-variance stationary fields cropped to grid."""
    padded = tuple(g + p for g, p in zip(grid, pad))
    sq = _grf_spectrum(padded, corr)
    white = rng.standard_normal((n_fields,) + padded)
    axes = tuple(range(1, 1 + len(padded)))
    f = np.fft.irfftn(np.fft.rfftn(white, axes=axes) * sq, s=padded, axes=axes)
    sl = (slice(None),) + tuple(slice(0, g) for g in grid)
    f = f[sl]
    f = f.reshape(n_fields, -1)
    f = (f - f.mean(axis=1, keepdims=True)) / f.std(axis=1, keepdims=True)
    return f  # [n_fields, prod(grid)]


def _grf_tokens(rng, H, d, prefix_len, grid, corr, pad, noise=0.1):
    T, Hg, Wg = grid
    dims = tuple(g for g in (T, Hg, Wg) if g > 1)
    cr = tuple(c for g, c in zip((T, Hg, Wg), corr) if g > 1)
    pd = tuple(p for g, p in zip((T, Hg, Wg), pad) if g > 1)
    L = T * Hg * Wg
    out = np.empty((H, prefix_len + L, d), dtype=np.float32)
    for h in range(H):
        out[h, :prefix_len] = rng.standard_normal((prefix_len, d))
        fields = _grf_fields(rng, d, dims, cr, pd)          # [d, L]
        out[h, prefix_len:] = fields.T + noise * rng.standard_normal((L, d))
    return out


def _ar1_head(rng, N, d, phi=0.95, sigma=0.3, chunk=256):
    """One head of x_t = phi x_{t-1} + N(0, sigma^2) per channel, x_0 drawn
    from the stationary law.  The recurrence runs in chunks (vectorised over
    chunks and channels) and the chunk carries are added afterwards."""
    e = rng.standard_normal((N, d), dtype=np.float32)
    e *= np.float32(sigma)
    e[0] *= np.float32(1.0 / math.sqrt(1.0 - phi * phi))
    nc = -(-N // chunk)
    E = np.zeros((nc * chunk, d), dtype=np.float32)
    E[:N] = e
    Y = E.reshape(nc, chunk, d)
    ph = np.float32(phi)
    for t in range(1, chunk):
        Y[:, t] += ph * Y[:, t - 1]
    carry = np.empty((nc, d), dtype=np.float32)
    carry[0] = Y[0, -1]
    phc = np.float32(phi ** chunk)
    for c in range(1, nc):
        carry[c] = Y[c, -1] + phc * carry[c - 1]
    pw = (phi ** np.arange(1, chunk + 1)).astype(np.float32)
    Y[1:] += pw[None, :, None] * carry[:-1, None, :]
    return Y.reshape(nc * chunk, d)[:N]


def _head(kind, w, seed_seq):
    rng = np.random.Generator(np.random.PCG64(seed_seq))
    if kind == "segments":
        x = _segments(rng, 1, w.N, w.d)[0]
    elif kind == "grf":
        L = int(np.prod(w.grid))
        if w.prefix_len + L != w.N:
            raise ValueError("grid workload needs N == prefix_len + T*H*W")
        corr, pad = ((2.0, 4.0, 4.0), (0, 32, 32)) if w.grid[0] == 1 else \
            ((2.0, 4.0, 4.0), (11, 18, 19))
        x = _grf_tokens(rng, 1, w.d, w.prefix_len, w.grid, corr, pad)[0]
    elif kind == "ar1":
        x = _ar1_head(rng, w.N, w.d)
    else:
        raise ValueError(kind)
    return _store(x, w.dtype)


def make_qkv(w: Workload, seed: int = 0):
    """Q [B,Hq,N,d], K, V [B,Hkv,N,d] in the workload's storage dtype.

    Every (tensor, batch, head) slab draws from its own PCG64 stream spawned
    from SeedSequence(seed), so slabs are generated in parallel.  Returns a
    dict with 'q', 'k', 'v' (np.float16, or uint16 bf16 bits), the workload,
    and for the AR(1) workloads the needle records (kv_head, k_block, q_block).
    """
    import concurrent.futures as cf
    import os
    root = np.random.SeedSequence(seed)
    sq, sk, sv, sn = root.spawn(4)
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    sdt = np.float16 if w.dtype == "f16" else np.uint16
    tensors = {}
    jobs = []
    with cf.ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
        for name, ss, H in (("q", sq, Hq), ("k", sk, Hkv), ("v", sv, Hkv)):
            arr = np.empty((B, H, N, d), dtype=sdt)
            tensors[name] = arr
            for idx, child in enumerate(ss.spawn(B * H)):
                b, h = divmod(idx, H)
                jobs.append((arr, b, h, ex.submit(_head, w.kind, w, child)))
        for arr, b, h, fut in jobs:
            arr[b, h] = fut.result()
    needles = []
    if w.kind == "ar1":
        rn = np.random.Generator(np.random.PCG64(sn))
        g = Hq // Hkv
        Tm = -(-N // w.bq)
        Tn = -(-N // w.bk)
        q, k = tensors["q"], tensors["k"]
        for _ in range(16 if Tn > 2 else 0):
            hk = int(rn.integers(0, Hkv))
            j = int(rn.integers(0, Tn - 2))
            i_lo = -(-((j + 1) * w.bk) // w.bq)
            if i_lo >= Tm:
                continue
            i = int(rn.integers(i_lo, Tm))
            rows = min(w.bk, N - i * w.bq)
            for b in range(B):
                k[b, hk, j * w.bk: j * w.bk + rows] = q[b, g * hk, i * w.bq: i * w.bq + rows]
            needles.append((hk, j, i))
        # sink: the first key of every KV head scaled by 8 (exact in binary)
        if w.dtype == "f16":
            k[:, :, 0] = (k[:, :, 0].astype(np.float32) * 8).astype(np.float16)
        else:
            k[:, :, 0] = bf16_bits_from_f32(to_f32(k[:, :, 0], "bf16") * 8)
    return {"q": tensors["q"], "k": tensors["k"], "v": tensors["v"],
            "workload": w, "needles": needles}
