"""Helpers shared by the GPU parity tests: moving synthetic inputs to the
device, running the library's entry points, and comparing with the oracle."""
import functools

import numpy as np
import torch

import free_block_sparse_predict_b200 as fb
from oracle import sparge_oracle as orc
from synth import get_workload, make_qkv, to_f64

TD = {"f16": torch.float16, "bf16": torch.bfloat16}

# Output tolerance on the float32 output mode (max |dO|, mean relative L1)
MAX_ABS = 2e-3
MEAN_REL_L1 = 1e-3
# INT8 Q K^T bars against exact scores
INT8_REL_L1 = 1e-2
INT8_COS = 0.999


def dev():
    return torch.device("cuda:0")


def to_dev(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype == "bf16":
        t = t.view(torch.bfloat16)
    return t.to(dev())


@functools.lru_cache(maxsize=8)
def workload(name, **over):
    w = get_workload(name, **over)
    t = make_qkv(w, seed=0)
    return w, t


def oracle_inputs(w, t):
    return tuple(to_f64(t[x], w.dtype) for x in ("q", "k", "v"))


def params_for(w, **kw):
    args = dict(causal=w.causal, qk_int8=w.qk_int8, io_dtype=TD[w.dtype],
                o_dtype=torch.float32)
    args.update(kw)
    tau = args.pop("tau", w.tau)
    theta = args.pop("theta", w.theta)
    lam = args.pop("lam", w.lam)
    return fb.make_params(w.B, w.Hq, w.Hkv, w.N, w.d, tau, theta, lam, **args)


def gpu_predict(p, q, k):
    ws = fb.workspace(p, dev())
    mask, idx, cnt, sq, sk = fb.predict_outputs(p, dev())
    fb.sparge_predict_mask(p, q, k, mask, idx, cnt, sq, sk, ws)
    torch.cuda.synchronize()
    return ws, mask, idx, cnt, sq, sk


def gpu_compact(p, M):
    m = torch.from_numpy(M.astype(np.uint8)).to(dev())
    Tm, Tn = M.shape[-2], M.shape[-1]
    idx = torch.empty(M.shape, dtype=torch.int32, device=dev())
    cnt = torch.empty(M.shape[:-1], dtype=torch.int32, device=dev())
    fb.sparge_mask_compact(p, m, idx, cnt)
    return idx, cnt


def gpu_attention(p, q, k, v, idx, cnt, ws=None, out_dtype=torch.float32):
    if ws is None:
        ws = fb.workspace(p, dev())
    o = torch.empty(q.shape, dtype=out_dtype, device=dev())
    st = torch.zeros(5, dtype=torch.int64, device=dev())
    fb.sparge_attn_fwd(p, q, k, v, idx, cnt, o, ws, st)
    torch.cuda.synchronize()
    assert fb.sparge_device_status(ws) == 0
    return o, st.cpu().numpy()


def compare_rows(o_gpu, O, rows_mask=None, exclude=None):
    """max |d| and mean relative L1 over the selected rows ([B,H,N] masks)."""
    g = o_gpu.astype(np.float64)
    sel = np.ones(O.shape[:-1], dtype=bool) if rows_mask is None else rows_mask.copy()
    if exclude is not None:
        sel &= ~exclude
    d = np.abs(g - O)[sel]
    ref = np.abs(O)[sel]
    return float(d.max()) if d.size else 0.0, float(d.sum() / max(ref.sum(), 1e-30))


def torch_dense_attention(q, k, v, scale, causal):
    """Plain PyTorch float32 softmax attention (the textbook op)."""
    g = q.shape[1] // k.shape[1]
    kf = k.float().repeat_interleave(g, 1)
    vf = v.float().repeat_interleave(g, 1)
    out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    N = q.shape[2]
    for h in range(q.shape[1]):
        s = (q[:, h].float() @ kf[:, h].transpose(-1, -2)) * scale
        if causal:
            m = torch.ones(N, N, dtype=torch.bool, device=q.device).tril()
            s = s.masked_fill(~m, float("-inf"))
        out[:, h] = torch.softmax(s, -1) @ vf[:, h]
    return out


def ws_regions(p):
    """Byte offsets of the workspace regions, mirroring the documented carving
    (256-byte aligned, in declaration order)."""
    al = lambda x: (x + 255) // 256 * 256
    Tm, Tn = -(-p.N // p.bq), -(-p.N // p.bk)
    off, out = 0, {}
    for name, nbytes in (("status", 256), ("q_mean", p.B * p.Hq * Tm * p.d * 4),
                         ("k_mean", p.B * p.Hkv * Tn * p.d * 4), ("s_q", p.B * p.Hq * Tm * 4),
                         ("s_k", p.B * p.Hkv * Tn * 4)):
        out[name] = off
        off += al(nbytes)
    if p.io_dtype == 1:
        out["v16"] = off
        off += al(p.B * p.Hkv * p.N * p.d * 2)
    if p.qk_int8:
        for name, nbytes in (("q_codes", p.B * p.Hq * p.N * p.d),
                             ("k_codes", p.B * p.Hkv * p.N * p.d), ("dq", p.B * p.Hq * Tm * 4),
                             ("dk", p.B * p.Hkv * Tn * 4), ("kbar", p.B * p.Hkv * p.d * 4),
                             ("k_sum64", p.B * p.Hkv * Tn * p.d * 8)):
            out[name] = off
            off += al(nbytes)
    return out


def sample_tiles(w, per_head=3, heads=None, seed=7, needles=()):
    """Seeded tile sample: first and last tile of each chosen head, random
    tiles, and the query tiles of needle blocks."""
    rng = np.random.default_rng(seed)
    Tm = -(-w.N // w.bq)
    heads = list(range(w.Hq)) if heads is None else heads
    tiles = set()
    for h in heads:
        tiles.add((0, h, 0))
        tiles.add((0, h, Tm - 1))
        for i in rng.choice(Tm, size=min(per_head, Tm), replace=False):
            tiles.add((0, h, int(i)))
    g = w.Hq // w.Hkv
    for (hk, j, i) in needles:
        tiles.add((0, g * hk, int(i)))
    return sorted(tiles)


def tile_rows(w, tiles):
    sel = np.zeros((w.B, w.Hq, w.N), dtype=bool)
    for (b, h, i) in tiles:
        sel[b, h, i * w.bq:min(w.N, (i + 1) * w.bq)] = True
    return sel


# Bounds on the mask comparison.  The ambiguity bands (1e-4 of cumulative
# mass around tau, 1e-4 around theta) flag about 2e-4 of the visible blocks
# on the sparse settings; a band too wide to be honest would flag far more.
# Small masks get a few entries of slack (a row of near-equal weights).
AMB_CUT_MAX_FRAC, AMB_CUT_MIN = 1e-3, 16   # entries flagged near the TopCdf cut
DIFF_MAX_FRAC, DIFF_MIN = 1e-4, 2          # entries where the GPU and the oracle differ


def check_mask(M, pr, label):
    """GPU mask M [B,Hq,Tm,Tn] bool against the oracle's prediction: equal
    outside the ambiguous entries, with the counts printed and bounded."""
    B, Hq = M.shape[:2]
    vis = int(pr["visible"].sum()) * B * Hq
    diff = M != pr["M"]
    bad = diff & ~pr["amb"]
    n_cut, n_th = int(pr["amb_cut"].sum()), int(pr["amb_theta"].sum())
    d_cut, d_th = int((diff & pr["amb_cut"]).sum()), int((diff & pr["amb_theta"]).sum())
    print(f"[mask {label}] visible {vis}, kept {int(M.sum())}: ambiguous near the cut "
          f"{n_cut}, in rows/columns near theta {n_th}; differing {int(diff.sum())} "
          f"(near the cut {d_cut}, near theta {d_th})")
    assert not bad.any(), f"{int(bad.sum())} mismatches outside the ambiguous entries, " \
                          f"first {np.argwhere(bad)[:3]}"
    assert n_cut <= max(AMB_CUT_MAX_FRAC * vis, AMB_CUT_MIN), (n_cut, vis)
    assert d_cut <= max(DIFF_MAX_FRAC * vis, DIFF_MIN), (d_cut, vis)
    return {"visible": vis, "amb_cut": n_cut, "amb_theta": n_th, "diff": int(diff.sum())}


def report_lambda(ost, label, rows=None):
    """Prints the lambda decisions within 1e-3 of the threshold and the rows
    they exclude from the comparison.  Bounded to 1e-3 of all (slice, block)
    decisions the oracle took, and to half of the compared rows (a long tile
    takes tens of thousands of decisions, each of which excludes 32 rows)."""
    near = ost["near_rows"] if rows is None else ost["near_rows"] & rows
    n_rows = int(near.sum())
    total = int(near.size if rows is None else rows.sum())
    decisions = 4 * int(ost["qk_blocks"])
    print(f"[lambda {label}] near-threshold decisions {ost['near_lambda']} of {decisions}, "
          f"rows excluded {n_rows} of {total}")
    assert ost["near_lambda"] <= 1e-3 * max(decisions, 1), (ost["near_lambda"], decisions)
    assert n_rows <= 0.5 * max(total, 1), (n_rows, total)
    return n_rows
