"""Every configuration the ablation sweeps visit (bench.py --sweep; the
paper review's Table 6 split, sparsity against length, speed against
sparsity by tau, and Table 4's token orders), at reduced sizes, against the
CPU oracle: the GPU mask bit for bit outside the ambiguous entries, and the
attention output at sampled tiles within the stated bars (the INT8 bars for
the INT8 workload).  The points come from bench.sweep_points, so the test
checks the same hyper-parameters and orders that the sweeps time."""
import numpy as np
import pytest
import torch

import bench
import free_block_sparse_predict_b200 as fb
from oracle import sparge_oracle as orc
from synth import get_workload, make_qkv

from gpu_common import (INT8_COS, INT8_REL_L1, MAX_ABS, MEAN_REL_L1, TD, check_mask,
                        compare_rows, dev, gpu_attention, gpu_predict, oracle_inputs, params_for,
                        report_lambda, sample_tiles, tile_rows, to_dev)

pytestmark = pytest.mark.gpu


def _check_point(label, w, t, perm=None, tiles_per_head=2):
    Q, K, V = oracle_inputs(w, t)
    q, k, v = (to_dev(t[x], w.dtype) for x in ("q", "k", "v"))
    if perm is not None:
        Q, K, V = (orc.permute_tokens(x, perm) for x in (Q, K, V))
        pt = torch.from_numpy(perm.astype(np.int32)).to(dev())
        out = []
        for x in (q, k, v):
            y = torch.empty_like(x)
            fb.sparge_hilbert_permute(x, y, pt)
            out.append(y)
        q, k, v = out
    p = params_for(w)
    ws, mask, idx, cnt, sq, sk = gpu_predict(p, q, k)
    pr = orc.predict_mask(Q, K, w.bq, w.bk, w.tau, w.theta, w.causal, w.scale)
    M = mask.cpu().numpy().astype(bool)
    check_mask(M, pr, label)
    tiles = sample_tiles(w, tiles_per_head, heads=list(range(w.Hq)), needles=t["needles"])
    rows = tile_rows(w, tiles)
    o, st = gpu_attention(p, q, k, v, idx, cnt, ws)
    io, co = orc.mask_compact(M)
    O, ost = orc.sparse_attention(Q, K, V, io, co, w.bq, w.bk, w.lam, w.causal, w.scale,
                                  tiles=tiles)
    on = o.cpu().numpy()
    if w.qk_int8:
        a, b = on[rows].astype(np.float64), O[rows]
        l1 = np.abs(a - b).sum() / np.abs(b).sum()
        cos = (a * b).sum() / np.linalg.norm(a) / np.linalg.norm(b)
        print(f"[sweep {label}] INT8 rel L1 {l1:.2e} cos {cos:.6f}")
        assert l1 <= INT8_REL_L1 and cos >= INT8_COS, (label, l1, cos)
    else:
        report_lambda(ost, label, rows)
        mx, l1 = compare_rows(on, O, rows, exclude=ost["near_rows"])
        assert mx <= MAX_ABS and l1 <= MEAN_REL_L1, (label, mx, l1)


@pytest.mark.parametrize("kind", ["table6", "tau"])
def test_hyperparameter_sweeps(kind):
    base = get_workload("llm_128k", N=2048 + 64, Hq=4, Hkv=1)
    t = make_qkv(base, seed=0)
    for label, w, _ in bench.sweep_points(kind, base):
        _check_point(f"{kind} {label}", w, t)


def test_length_sweep():
    # the sweep's lengths, scaled down 32 times (256 .. 4096 tokens)
    base = get_workload("llm_128k", Hq=2, Hkv=1)
    for label, w, _ in bench.sweep_points("length", base):
        ws = w.replace(N=w.N // 32)
        _check_point(f"length {label} / 32", ws, make_qkv(ws, seed=0))


def test_permutation_sweep():
    base = get_workload("video_dit", Hq=2, Hkv=2)
    t = make_qkv(base, seed=0)
    perms = bench.permutation_tables(base)
    perms["hilbert"] = orc.hilbert_permutation(base.N, base.prefix_len, *base.grid)
    for label, w, pname in bench.sweep_points("permutation", base):
        _check_point(f"permutation {label}", w, t, perm=perms[pname], tiles_per_head=1)
