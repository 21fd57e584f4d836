"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: closed forms,
brute force on tiny inputs, invariants the pages state, the authors' worked
example, or hand-worked rows.  No GPU.
"""
import itertools
import math
import os

import numpy as np
import pytest

from oracle import sparge_oracle as orc
from synth import get_workload, make_qkv, to_f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


# ----------------------------------------------------------------------------
# brute-force references written directly from the textbook definitions
# ----------------------------------------------------------------------------

def dense_attention(Q, K, V, scale, causal=False, allowed=None):
    """softmax(scale * Q K^T) V per head with an optional boolean key mask."""
    B, Hq, N, d = Q.shape
    g = Hq // K.shape[1]
    O = np.zeros_like(Q)
    for b in range(B):
        for h in range(Hq):
            S = scale * Q[b, h] @ K[b, h // g].T
            ok = np.ones_like(S, dtype=bool)
            if causal:
                ok &= np.tril(np.ones((N, N), dtype=bool))
            if allowed is not None:
                ok &= allowed[b, h]
            S = np.where(ok, S, -np.inf)
            for r in range(N):
                if not ok[r].any():
                    continue
                e = np.exp(S[r] - S[r][ok[r]].max())
                O[b, h, r] = (e / e.sum()) @ V[b, h // g]
    return O


def rand_qkv(B, Hq, Hkv, N, d, scale=1.0):
    Q = RNG.standard_normal((B, Hq, N, d)) * scale
    K = RNG.standard_normal((B, Hkv, N, d)) * scale
    V = RNG.standard_normal((B, Hkv, N, d))
    return Q, K, V


# ----------------------------------------------------------------------------
# Hilbert curve
# ----------------------------------------------------------------------------

def _curve_points(ndim, bits):
    side = 1 << bits
    pts = list(itertools.product(range(side), repeat=ndim))
    idx = [orc.hilbert_index(p, bits) for p in pts]
    order = np.argsort(idx)
    return np.array(pts)[order], np.array(sorted(idx))


@pytest.mark.parametrize("ndim,bits", [(2, 1), (2, 2), (2, 3), (2, 4), (3, 1), (3, 2), (3, 3)])
def test_hilbert_is_a_continuous_bijection(ndim, bits):
    pts, idx = _curve_points(ndim, bits)
    n = 1 << (ndim * bits)
    assert np.array_equal(idx, np.arange(n))                      # bijection onto [0, 2^(nb))
    steps = np.abs(np.diff(pts, axis=0)).sum(axis=1)
    assert np.all(steps == 1)                                     # each step moves to a grid neighbour
    assert np.all(pts[0] == 0)                                    # starts at the origin corner
    end = pts[-1]
    side = (1 << bits) - 1
    assert set(np.unique(end)) <= {0, side} and (end == side).sum() == 1  # ends on an adjacent corner


@pytest.mark.parametrize("ndim,bits", [(2, 4), (3, 3)])
def test_hilbert_visits_aligned_subcubes_contiguously(ndim, bits):
    pts, _ = _curve_points(ndim, bits)
    for level in range(1, bits):
        run = 1 << (ndim * level)
        for start in range(0, len(pts), run):
            chunk = pts[start:start + run]
            corner = chunk.min(axis=0)
            assert np.all(corner % (1 << level) == 0)
            assert np.all(chunk.max(axis=0) - corner == (1 << level) - 1)


@pytest.mark.parametrize("grid", [(1, 5, 7), (3, 4, 6), (13, 30, 45), (1, 64, 64), (2, 1, 9)])
def test_hilbert_permutation_bijection_and_prefix(grid):
    T, H, W = grid
    P = 7
    N = P + T * H * W + 3
    perm = orc.hilbert_permutation(N, P, T, H, W)
    assert sorted(perm.tolist()) == list(range(N))
    assert np.array_equal(perm[:P], np.arange(P))
    assert np.array_equal(perm[N - 3:], np.arange(N - 3, N))
    x = RNG.standard_normal((1, 2, N, 3))
    y = orc.permute_tokens(x, perm)
    assert np.array_equal(orc.inverse_permute_tokens(y, perm), x)
    # consecutive grid tokens in curve order are never far apart in the grid
    lin = perm[P:P + T * H * W] - P
    t, r = np.divmod(lin, H * W)
    yy, xx = np.divmod(r, W)
    pos = np.stack([t, yy, xx], 1)
    jumps = np.abs(np.diff(pos, axis=0)).sum(1)
    assert np.median(jumps) == 1


def test_dense_attention_invariant_under_permutation():
    # standard attention is permutation invariant (rebuttal page, reply to Weakness 3.2)
    N, P, grid = 40, 4, (1, 6, 6)
    perm = orc.hilbert_permutation(N, P, *grid)
    Q, K, V = rand_qkv(1, 2, 2, N, 8)
    O = dense_attention(Q, K, V, 8 ** -0.5)
    Qp, Kp, Vp = (orc.permute_tokens(x, perm) for x in (Q, K, V))
    Op = orc.inverse_permute_tokens(dense_attention(Qp, Kp, Vp, 8 ** -0.5), perm)
    assert np.allclose(O, Op, atol=1e-12)


def test_hilbert_raises_block_similarity_over_rowmajor_and_random():
    # Table 4 of the paper review: HilbertCurve > Rowmajor > Random on Sim-q / Sim-k
    w = get_workload("image_dit", Hq=1, Hkv=1)
    x = to_f64(make_qkv(w, seed=3)["k"], "bf16")[0, 0]
    N = w.N
    perm_h = orc.hilbert_permutation(N, w.prefix_len, *w.grid)
    perm_r = np.arange(N)
    perm_x = np.concatenate([np.arange(w.prefix_len),
                             w.prefix_len + RNG.permutation(N - w.prefix_len)])
    P0 = w.prefix_len // 64
    sims = {}
    for name, perm in (("hilbert", perm_h), ("row", perm_r), ("random", perm_x)):
        s = orc.block_cossim(x[perm], 64)[P0:]
        sims[name] = s.mean()
    assert sims["hilbert"] > sims["row"] > sims["random"]


# ----------------------------------------------------------------------------
# pooling and CosSim (Eq. 4-6)
# ----------------------------------------------------------------------------

def test_block_mean_tail_uses_valid_tokens_only():
    X = np.arange(10, dtype=np.float64)[:, None] * np.array([[1.0, -2.0]])
    m = orc.block_mean(X, 4)
    assert m.shape == (3, 2)
    assert np.allclose(m[0], [1.5, -3.0])
    assert np.allclose(m[2], [8.5, -17.0])                    # rows 8, 9 only


def test_cossim_identical_tokens_is_one():
    x = RNG.standard_normal(16)
    assert math.isclose(orc.cossim(np.tile(x, (64, 1))), 1.0, rel_tol=1e-12)


def test_cossim_orthogonal_tokens_is_one_over_n():
    n = 12
    X = np.eye(n) * RNG.uniform(0.5, 3.0, size=(n, 1))
    assert math.isclose(orc.cossim(X), 1.0 / n, rel_tol=1e-12)


def test_cossim_antipodal_pair_is_zero_and_scale_invariant():
    x = RNG.standard_normal(8)
    assert abs(orc.cossim(np.stack([x, -3 * x]))) < 1e-12
    X = RNG.standard_normal((20, 8))
    c = RNG.uniform(0.1, 10, size=(20, 1))
    assert math.isclose(orc.cossim(X), orc.cossim(X * c), rel_tol=1e-10)


def test_cossim_equals_norm_of_unit_sum_closed_form():
    # mean_{a,b} xhat_a.xhat_b = |sum_a xhat_a|^2 / n^2 (expand the double sum)
    for n in (1, 5, 64, 128):
        X = RNG.standard_normal((n, 32))
        Xh = X / np.linalg.norm(X, axis=1, keepdims=True)
        closed = np.sum(Xh.sum(0) ** 2) / n ** 2
        assert math.isclose(orc.cossim(X), closed, rel_tol=1e-10, abs_tol=1e-14)
        assert 0.0 <= orc.cossim(X) <= 1.0 + 1e-12


# ----------------------------------------------------------------------------
# TopCdf (Eq. 8), fix rule (Eq. 9), worked example
# ----------------------------------------------------------------------------

def _golden_rows():
    rows = []
    with open(os.path.join(GOLDEN, "topcdf_rows.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            tau, p, keep = (s.strip() for s in line.split("|"))
            rows.append((float(tau), np.array([float(v) for v in p.split()]),
                         sorted(int(v) for v in keep.split())))
    return rows


@pytest.mark.parametrize("tau,p,keep", _golden_rows())
def test_topcdf_hand_worked_rows(tau, p, keep):
    k, _, _ = orc.topcdf(p, tau)
    assert sorted(np.flatnonzero(k).tolist()) == keep


def test_topcdf_matches_subset_brute_force():
    # the kept set holds every value >= the k-th largest, where k is the least
    # size of ANY subset whose mass reaches tau * total (enumerated, no sorting)
    for _ in range(300):
        n = int(RNG.integers(1, 8))
        p = RNG.integers(0, 6, size=n).astype(np.float64)   # small ints: exact sums, ties
        if p.sum() == 0:
            p[0] = 1.0
        tau = float(RNG.choice([0.1, 0.33, 0.5, 0.66, 0.9, 0.99]))
        target = tau * p.sum()
        best = None
        for size in range(1, n + 1):
            for sub in itertools.combinations(range(n), size):
                if sum(p[list(sub)]) >= target:
                    thr = min(p[list(sub)])
                    best = thr if best is None else max(best, thr)
            if best is not None:
                break
        keep, _, _ = orc.topcdf(p, tau)
        assert np.array_equal(keep, p >= best)


def test_topcdf_tau_one_keeps_every_finite_entry():
    S = np.array([0.0, -900.0, np.inf * -1, 3.0])          # exp underflows for -900
    P = orc.row_softmax(S)
    assert P[1] == 0.0
    fin = np.isfinite(S)
    keep, _, _ = orc.topcdf(P[fin], 1.0)
    assert keep.all()


def test_fix_rule_theta_above_one_gives_dense_mask():
    Q, K, _ = rand_qkv(1, 2, 1, 300, 16)
    for causal in (False, True):
        pr = orc.predict_mask(Q, K, 128, 64, 0.5, 1.01, causal, 0.25)
        assert np.array_equal(pr["M"][0, 0], pr["visible"])
        assert np.array_equal(pr["M"][0, 1], pr["visible"])


def test_fix_rule_theta_below_minus_one_is_pure_topcdf():
    Q, K, _ = rand_qkv(1, 1, 1, 512, 16)
    pr = orc.predict_mask(Q, K, 128, 64, 0.4, -1.01, False, 0.25)
    for i in range(4):
        P = orc.row_softmax(pr["S_hat"][0, 0, i])
        keep, _, _ = orc.topcdf(P, 0.4)
        assert np.array_equal(pr["M"][0, 0, i], keep)
    assert pr["M"].sum() < pr["M"].size


def test_theta_comparisons_are_strict():
    """Eq. 7 and Eq. 9 compare with a strict "<": a K block whose
    self-similarity equals theta keeps a finite S_hat column and is not forced
    on; blocks below theta are -inf in S_hat and forced on in M."""
    rng = np.random.default_rng(77)
    K = rng.standard_normal((1, 1, 512, 16))
    # self-similar query blocks (s_q near 1), so no row is a fix row
    Q = (np.repeat(rng.standard_normal((4, 16)), 128, axis=0)
         + 0.01 * rng.standard_normal((512, 16)))[None, None]
    sk = orc.predict_mask(Q, K, 128, 64, 0.3, -2.0, False, 0.25)["s_k"][0, 0]
    j0 = int(np.argsort(sk)[len(sk) // 2])
    theta = float(sk[j0])
    pr = orc.predict_mask(Q, K, 128, 64, 0.3, theta, False, 0.25)
    S, M = pr["S_hat"][0, 0], pr["M"][0, 0]
    below = sk < theta
    assert not below[j0] and below.any() and (~below).sum() >= 2
    assert np.isfinite(S[:, ~below]).all() and np.isneginf(S[:, below]).all()
    assert (pr["s_q"][0, 0] >= theta).all()
    for i in range(S.shape[0]):
        keep, _, _ = orc.topcdf(orc.row_softmax(S[i]), 0.3)
        assert np.array_equal(M[i], keep | below)
    assert not M[:, j0].all()          # the data tell a forced column from a kept one


def test_fix_rule_rows_and_columns():
    vis = np.ones((3, 4), dtype=bool)
    M = np.zeros((3, 4), dtype=bool)
    out = orc.apply_fix_rule(M, np.array([0.9, 0.1, 0.9]), np.array([0.9, 0.9, 0.2, 0.9]), 0.5, vis)
    exp = np.zeros((3, 4), dtype=bool)
    exp[1, :] = True
    exp[:, 2] = True
    assert np.array_equal(out, exp)


def _worked_rows():
    rows = []
    with open(os.path.join(GOLDEN, "worked_block_arithmetic.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, f_, s_, comp, spars = line.split()
            rows.append((name, float(f_), float(s_), float(comp), float(spars)))
    return rows


@pytest.mark.parametrize("name,f,s,computed,sparsity", _worked_rows())
def test_worked_block_arithmetic_reproduced_from_mask_statistics(name, f, s, computed, sparsity):
    # 10 query blocks x 10 key blocks; a fraction (1-f) of query blocks are fix
    # rows; TopCdf drops a fraction s of every selective row.
    Tm = Tn = 10
    theta = 0.5
    n_fix = round((1 - f) * Tm)
    s_q = np.where(np.arange(Tm) < n_fix, 0.1, 0.9)
    s_k = np.full(Tn, 0.9)
    vis = np.ones((Tm, Tn), dtype=bool)
    top = np.ones((Tm, Tn), dtype=bool)
    n_drop = round(s * Tn)
    for i in range(Tm):
        top[i, RNG.choice(Tn, n_drop, replace=False)] = False
    M = orc.apply_fix_rule(top, s_q, s_k, theta, vis)
    f_, s_, comp, spars = orc.mask_statistics(M, s_q, s_k, theta, vis)
    assert math.isclose(f_, f) and math.isclose(s_, s)
    assert math.isclose(comp, computed, abs_tol=1e-12)
    assert math.isclose(spars, sparsity, abs_tol=1e-12)
    assert math.isclose(comp, (1 - s) * f + (1 - f), abs_tol=1e-12)


def test_causal_visibility_and_future_blocks_zero():
    vis = orc.visible(300, 128, 64, True)
    assert vis.shape == (3, 5)
    assert vis[0].tolist() == [True, True, False, False, False]
    assert vis[1].tolist() == [True, True, True, True, False]
    assert vis[2].tolist() == [True, True, True, True, True]     # rows 256..299 see block 4 (256..299)
    Q, K, _ = rand_qkv(1, 1, 1, 300, 16)
    pr = orc.predict_mask(Q, K, 128, 64, 0.9, 0.0, True, 0.25)
    assert not (pr["M"][0, 0] & ~vis).any()


def test_mask_compact_roundtrip():
    M = RNG.random((2, 3, 5, 9)) < 0.4
    idx, cnt = orc.mask_compact(M)
    for pos in np.ndindex(2, 3, 5):
        js = idx[pos][:cnt[pos]]
        assert np.all(np.diff(js) > 0)
        back = np.zeros(9, dtype=bool)
        back[js] = True
        assert np.array_equal(back, M[pos])
        assert np.all(idx[pos][cnt[pos]:] == -1)


# ----------------------------------------------------------------------------
# attention (Eq. 1-3)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,Hq,Hkv", [(256, 1, 1), (300, 4, 2), (77, 2, 1)])
def test_full_mask_no_lambda_equals_dense_softmax(causal, N, Hq, Hkv):
    d = 16
    Q, K, V = rand_qkv(1, Hq, Hkv, N, d)
    pr = orc.predict_mask(Q, K, 128, 64, 0.9, 1.5, causal, d ** -0.5)   # theta > 1: all fixed
    idx, cnt = orc.mask_compact(pr["M"])
    O, st = orc.sparse_attention(Q, K, V, idx, cnt, 128, 64, -np.inf, causal, d ** -0.5)
    assert np.allclose(O, dense_attention(Q, K, V, d ** -0.5, causal), atol=1e-12)
    assert st["skipped_slices"] == 0


def test_block_mask_equals_key_masked_dense_attention():
    N, d = 320, 16
    Q, K, V = rand_qkv(1, 2, 1, N, d)
    Tm, Tn = 3, 5
    M = RNG.random((1, 2, Tm, Tn)) < 0.5
    M[..., 0] = True
    idx, cnt = orc.mask_compact(M)
    O, _ = orc.sparse_attention(Q, K, V, idx, cnt, 128, 64, -np.inf, False, d ** -0.5)
    allowed = np.zeros((1, 2, N, N), dtype=bool)
    for h in range(2):
        for i in range(Tm):
            for j in range(Tn):
                if M[0, h, i, j]:
                    allowed[0, h, i * 128:(i + 1) * 128, j * 64:(j + 1) * 64] = True
    assert np.allclose(O, dense_attention(Q, K, V, d ** -0.5, allowed=allowed), atol=1e-12)


def test_lambda_skip_drops_pv_but_keeps_rowsum():
    # key block 1 has scores far below block 0 for every row: with lambda
    # between the gap and 0 its P~V is skipped for every warp slice while its
    # probabilities still enter l (Eq. 1 and Eq. 3).
    N, d = 128, 8
    Q = np.zeros((1, 1, N, d))
    Q[..., 0] = 1.0
    K = np.zeros((1, 1, N, d))
    K[0, 0, :64, 0] = 5.0
    K[0, 0, 64:, 0] = -5.0 + 0.01 * RNG.standard_normal(64)
    V = RNG.standard_normal((1, 1, N, d))
    idx, cnt = orc.mask_compact(np.ones((1, 1, 1, 2), dtype=bool))
    scale = 1.0
    O, st = orc.sparse_attention(Q, K, V, idx, cnt, 128, 64, -3.0, False, scale)
    s = scale * Q[0, 0] @ K[0, 0].T
    p = np.exp(s - s.max(axis=1, keepdims=True))
    expect = (p[:, :64] @ V[0, 0, :64]) / p.sum(axis=1, keepdims=True)
    assert np.allclose(O[0, 0], expect, atol=1e-12)
    assert st["skipped_slices"] == 4 and st["pv_slices"] == 4
    # with lambda below the gap nothing is skipped and O is the dense result
    O2, st2 = orc.sparse_attention(Q, K, V, idx, cnt, 128, 64, -20.0, False, scale)
    assert np.allclose(O2, dense_attention(Q, K, V, scale), atol=1e-12)
    assert st2["skipped_slices"] == 0


def test_lambda_decision_is_per_warp_slice_and_order_dependent():
    N, d = 128, 4
    Q = np.zeros((1, 1, N, d))
    Q[0, 0, :, 0] = 1.0
    Q[0, 0, 32:64, 0] = -1.0             # warp 1 prefers the second block
    K = np.zeros((1, 1, N, d))
    K[0, 0, :64, 0] = 4.0
    K[0, 0, 64:, 0] = -4.0
    V = RNG.standard_normal((1, 1, N, d))
    idx, cnt = orc.mask_compact(np.ones((1, 1, 1, 2), dtype=bool))
    _, st = orc.sparse_attention(Q, K, V, idx, cnt, 128, 64, -1.0, False, 1.0)
    # block 0 is first: never skipped (m_local = m_new somewhere).  Block 1:
    # warps 0, 2, 3 see scores 8 below their max -> skip; warp 1 sees its max.
    assert st["skipped_slices"] == 3 and st["pv_slices"] == 5
    # processing order matters: a reversed list processes block 1 first
    idx_r = idx.copy()
    idx_r[0, 0, 0, :2] = [1, 0]
    _, st_r = orc.sparse_attention(Q, K, V, idx_r, cnt, 128, 64, -1.0, False, 1.0)
    assert st_r["skipped_slices"] == 1 and st_r["pv_slices"] == 7
    # Eq. 3's test is strict: slices exactly lambda = -8 below their max are kept
    _, st_eq = orc.sparse_attention(Q, K, V, idx, cnt, 128, 64, -8.0, False, 1.0)
    assert st_eq["skipped_slices"] == 0 and st_eq["pv_slices"] == 8
    _, st_lt = orc.sparse_attention(Q, K, V, idx, cnt, 128, 64, -7.999, False, 1.0)
    assert st_lt["skipped_slices"] == 3


def test_row_with_no_visible_key_outputs_zero():
    N, d = 128, 8
    Q, K, V = rand_qkv(1, 1, 1, N, d)
    M = np.zeros((1, 1, 1, 2), dtype=bool)
    M[..., 1] = True                     # only keys 64..127, causal: rows 0..63 see none
    idx, cnt = orc.mask_compact(M)
    O, st = orc.sparse_attention(Q, K, V, idx, cnt, 128, 64, -np.inf, True, d ** -0.5)
    assert np.all(O[0, 0, :64] == 0.0) and st["zero_l_rows"] == 64
    allowed = np.zeros((1, 1, N, N), dtype=bool)
    allowed[..., 64:] = True
    assert np.allclose(O[0, 0, 64:], dense_attention(Q, K, V, d ** -0.5, True, allowed)[0, 0, 64:],
                       atol=1e-12)


# ----------------------------------------------------------------------------
# INT8 per-block quantisation with K smoothing
# ----------------------------------------------------------------------------

def test_quantize_blocks_reconstruction_bound_and_extremes():
    X = (RNG.standard_normal((200, 32)) * 3).astype(np.float32)
    X[5, 3] = 0.0
    codes, delta = orc.quantize_blocks(X, 64)
    for i in range(4):
        blk = X[i * 64:(i + 1) * 64]
        c = codes[i * 64:(i + 1) * 64].astype(np.float64)
        assert np.abs(c).max() == 127                         # absmax maps to +-127
        err = np.abs(c * delta[i] - blk)
        assert err.max() <= delta[i] * (0.5 + 1e-5)
    z, dz = orc.quantize_blocks(np.zeros((64, 4), np.float32), 64)
    assert dz[0] == 0 and not z.any()


def test_quantize_blocks_rounds_ties_to_even():
    """With absmax 127 the multiplier 127/absmax is exactly 1, so x * inv is
    x itself: halves must go to the even neighbour (2.5 -> 2, 3.5 -> 4,
    -2.5 -> -2, 126.5 -> 126), which a round-half-away or floor(x + 0.5)
    reading would get wrong."""
    X = np.zeros((64, 8), np.float32)
    X[0, :8] = [127.0, 2.5, 3.5, -2.5, -3.5, 126.5, 0.5, -0.5]
    codes, delta = orc.quantize_blocks(X, 64)
    assert delta[0] == np.float32(1.0)
    assert codes[0].tolist() == [127, 2, 4, -2, -4, 126, 0, 0]


def test_k_smoothing_leaves_exact_attention_unchanged():
    # subtracting kbar shifts every score row by q.kbar: softmax is invariant
    N, d = 200, 16
    Q, K, V = rand_qkv(1, 2, 1, N, d)
    K = K + 3.0
    kbar = K.mean(axis=2, keepdims=True)
    O1 = dense_attention(Q, K, V, d ** -0.5)
    O2 = dense_attention(Q, K - kbar, V, d ** -0.5)
    assert np.allclose(O1, O2, atol=1e-12)


def test_int8_scores_track_exact_scores():
    w = get_workload("llm_32k", N=512, Hq=2, Hkv=1)
    t = make_qkv(w, seed=5)
    Q = to_f64(t["q"], "bf16")
    K = to_f64(t["k"], "bf16")
    V = to_f64(t["v"], "bf16")
    qt = orc.quantize_qk(Q.astype(np.float32), K.astype(np.float32), 128, 64)
    full = np.ones((1, 2, 4, 8), dtype=bool)
    idx, cnt = orc.mask_compact(full & orc.visible(512, 128, 64, True))
    OA, _ = orc.sparse_attention(Q, K, V, idx, cnt, 128, 64, -np.inf, True, w.scale)
    OB, _ = orc.sparse_attention(Q, K, V, idx, cnt, 128, 64, -np.inf, True, w.scale, quant=qt)
    l1 = np.abs(OA - OB).sum() / np.abs(OA).sum()
    cos = (OA * OB).sum() / np.linalg.norm(OA) / np.linalg.norm(OB)
    assert l1 < 1e-2 and cos > 0.999


# ----------------------------------------------------------------------------
# generators
# ----------------------------------------------------------------------------

def test_generators_shapes_and_determinism():
    for name, over in (("tiny", {}), ("image_dit", {"Hq": 2, "Hkv": 2}),
                       ("video_dit", {"Hq": 1, "Hkv": 1}), ("llm_32k", {"N": 2048})):
        w = get_workload(name, **over)
        a = make_qkv(w, seed=0)
        b = make_qkv(w, seed=0)
        assert a["q"].shape == (w.B, w.Hq, w.N, w.d)
        assert a["k"].shape == (w.B, w.Hkv, w.N, w.d)
        assert np.array_equal(a["q"], b["q"]) and np.array_equal(a["v"], b["v"])
        assert a["q"].dtype == (np.float16 if w.dtype == "f16" else np.uint16)


def test_tiny_segments_are_self_similar_except_random_ones():
    w = get_workload("tiny")
    K = to_f64(make_qkv(w)["k"], "f16")[0, 0]
    s = orc.block_cossim(K, 64)
    assert (s > 0.8).sum() == 12 and (s < 0.2).sum() == 4


def test_compressed_scores_equal_token_scores_for_constant_blocks():
    # when every token of a block is the same vector, the block mean is that
    # token, so S_hat[i, j] must equal Eq. 1's score between any query of
    # block i and any key of block j (this pins the 1/sqrt(d) scale too)
    N, d = 384, 16
    Q = np.repeat(RNG.standard_normal((1, 1, 3, d)), 128, axis=2)
    K = np.repeat(RNG.standard_normal((1, 1, 6, d)), 64, axis=2)
    pr = orc.predict_mask(Q, K, 128, 64, 0.9, -2.0, False, d ** -0.5)
    S = d ** -0.5 * Q[0, 0] @ K[0, 0].T
    assert np.allclose(pr["S_hat"][0, 0], S[::128, ::64], atol=1e-12)
    assert np.allclose(pr["s_q"], 1.0) and np.allclose(pr["s_k"], 1.0)


# ----------------------------------------------------------------------------
# pins added for steps a plausible slip could break without any pin above
# noticing: the softmax of Algorithm 1 step 5, Eq. 9's strict row test, the K
# smoothing of Algorithm 1 step 2, the INT8 quotient, and the ambiguity map
# ----------------------------------------------------------------------------

def _constant_block_inputs(shat_row, n_q=192, d=4):
    """Q and K whose blocks are constant tokens, so that S_hat[i, j] equals
    the given values for every query block i (Eq. 4-7 with identical tokens:
    the block mean is the token itself and its self-similarity is 1).
    With d = 4 the scale is 1/2; q = (2, 0, 0, 0) and k_j = (v_j, 0, 0, 0)
    give scale * q . k_j = v_j."""
    Tn = len(shat_row)
    N = max(n_q, 64 * Tn)
    Q = np.zeros((1, 1, N, d))
    Q[..., 0] = 2.0
    K = np.zeros((1, 1, N, d))
    K[..., 1] = 1.0                         # keys past the listed blocks: some token
    for j, v in enumerate(shat_row):
        K[0, 0, 64 * j:64 * (j + 1), 0] = v
        K[0, 0, 64 * j:64 * (j + 1), 1] = 0.0
    return Q, K, N


def test_row_softmax_hand_worked():
    # S_hat = (ln 5, ln 3, ln 2) + c: the softmax is (5, 3, 2) / 10 whatever c
    for c in (0.0, 7.25, -40.0):
        P = orc.row_softmax(np.log([5.0, 3.0, 2.0]) + c)
        assert np.allclose(P, [0.5, 0.3, 0.2], rtol=0, atol=1e-14)
    # -inf entries get weight 0 and leave the others' ratio alone
    P = orc.row_softmax(np.array([np.log(3.0), -np.inf, 0.0, -np.inf]))
    assert np.allclose(P, [0.75, 0.0, 0.25, 0.0], rtol=0, atol=1e-14)
    assert np.all(orc.row_softmax(np.full(3, -np.inf)) == 0)


@pytest.mark.parametrize("tau,keep", [(0.45, [0]), (0.6, [0, 1]), (0.85, [0, 1, 2])])
def test_predicted_row_from_hand_worked_shat(tau, keep):
    """Constant blocks give S_hat = (ln 5, ln 3, ln 2) + 1.5 on every query
    row, so P_hat = (0.5, 0.3, 0.2) and TopCdf(tau) keeps {0} at tau = 0.45,
    {0, 1} at 0.6 and all three at 0.85 (Eq. 7, 8).  A softmax at another
    temperature (e.g. exp(2 S)) gives (0.66, 0.24, 0.11) and keeps {0} at 0.6."""
    row = np.log([5.0, 3.0, 2.0]) + 1.5
    Q, K, N = _constant_block_inputs(row)
    pr = orc.predict_mask(Q, K, 128, 64, tau, 0.5, False, 0.5)
    assert np.allclose(pr["S_hat"][0, 0, :, :3], row, atol=1e-12)
    assert np.allclose(pr["s_q"], 1.0) and np.allclose(pr["s_k"][0, 0, :3], 1.0)
    for i in range(pr["M"].shape[2]):
        assert np.flatnonzero(pr["M"][0, 0, i, :3]).tolist() == keep
        assert not pr["amb"][0, 0, i].any()


def test_fix_rule_row_test_is_strict():
    """Eq. 9 forces the rows of query blocks with s_q < theta: a row whose
    self-similarity is exactly theta is not a fix row, one just below is."""
    theta = 0.5
    vis = np.ones((3, 4), dtype=bool)
    s_q = np.array([theta, np.nextafter(theta, -1.0), theta + 0.25])
    out = orc.apply_fix_rule(np.zeros((3, 4), dtype=bool), s_q, np.full(4, 0.9), theta, vis)
    assert out.sum(axis=1).tolist() == [0, 4, 0]
    # and through the whole predictor: a query block with s_q exactly theta
    rng = np.random.default_rng(11)
    Q = rng.standard_normal((1, 1, 512, 16))
    K = (np.repeat(rng.standard_normal((8, 16)), 64, axis=0)
         + 0.01 * rng.standard_normal((512, 16)))[None, None]       # s_k near 1
    sq = orc.predict_mask(Q, K, 128, 64, 0.3, -2.0, False, 0.25)["s_q"][0, 0]
    i0 = int(np.argmax(sq))
    pr = orc.predict_mask(Q, K, 128, 64, 0.3, float(sq[i0]), False, 0.25)
    M = pr["M"][0, 0]
    assert (pr["s_k"] >= sq[i0]).all()                               # no fix column
    keep, _, _ = orc.topcdf(orc.row_softmax(pr["S_hat"][0, 0, i0]), 0.3)
    assert np.array_equal(M[i0], keep) and not M[i0].all()
    below = sq < sq[i0]
    assert below.any() and M[below].all()


def test_k_smoothing_mean_hand_value_and_offset_invariance():
    """Algorithm 1 step 2 subtracts the per-head mean of K over all tokens
    before the per-block INT8 of K.  On dyadic inputs every step is exact, so
    kbar equals the rational mean and adding any per-channel constant c to K
    leaves K - kbar, and therefore every code and scale, unchanged."""
    from fractions import Fraction
    rng = np.random.default_rng(5)
    N, d = 256, 8
    K = (rng.integers(-40, 41, size=(1, 1, N, d)) / 8.0).astype(np.float32)
    K[0, 0, :, 3] += 5.0
    want = [Fraction(0)] * d
    for n in range(N):
        for c in range(d):
            want[c] += Fraction(float(K[0, 0, n, c]))
    want = [w / N for w in want]
    Q = rng.standard_normal((1, 2, N, d)).astype(np.float32)
    qt = orc.quantize_qk(Q, K, 128, 64)
    assert [Fraction(float(v)) for v in qt["kbar"][0, 0]] == want
    off = (64.0 * (1 + np.arange(d))).astype(np.float32)
    qt2 = orc.quantize_qk(Q, K + off, 128, 64)
    assert np.array_equal(qt2["kbar"][0, 0], qt["kbar"][0, 0] + off)
    assert np.array_equal(qt2["k_codes"], qt["k_codes"])
    assert np.array_equal(qt2["dk"], qt["dk"])
    assert (qt["k_codes"] != 0).any()


def _f32_round(q):
    """Round a rational to the nearest float32, ties to even (IEEE 754),
    by exact integer arithmetic on the significand."""
    from fractions import Fraction
    if q == 0:
        return Fraction(0)
    sgn = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -126)                      # subnormals keep the bottom exponent
    ulp = Fraction(2) ** (e - 23)
    m = round(a / ulp)                    # Python rounds Fractions half to even
    return sgn * m * ulp


def _exact_int8_code(x, delta):
    """rint of the correctly rounded float32 quotient x / delta, clamped."""
    from fractions import Fraction
    if delta == 0:
        return 0
    v = round(_f32_round(Fraction(float(x)) / Fraction(float(delta))))
    return max(-127, min(127, v))


# (absmax, x) float32 pairs whose float32 quotient x / (absmax / 127) rounds to
# one integer while x * (127 / absmax) rounds to the next: they tell the
# division of reading R9 from a multiply by the reciprocal
_QUOTIENT_CASES = [(2.408083438873291, -2.28483510017395),
                   (7.719466686248779, -6.534193992614746),
                   (7.485044002532959, -5.5106425285339355),
                   (7.883794784545898, 5.617980003356934),
                   (3.9020028114318848, 2.842010021209717),
                   (3.9020028114318848, 3.149254322052002)]


def test_int8_codes_are_rint_of_the_float32_quotient():
    """Reading R9: delta = fl32(absmax / 127) and code = rint(fl32(x / delta)).
    Checked against exact rational arithmetic: on crafted blocks where the
    quotient and the product with the reciprocal round to different integers,
    and on random blocks."""
    from fractions import Fraction
    for amax, x in _QUOTIENT_CASES:
        blk = np.zeros((64, 4), np.float32)
        blk[0, 0] = np.float32(amax)
        blk[1, 1] = np.float32(x)
        codes, delta = orc.quantize_blocks(blk, 64)
        assert Fraction(float(delta[0])) == _f32_round(Fraction(float(np.float32(amax))) / 127)
        assert int(codes[1, 1]) == _exact_int8_code(np.float32(x), delta[0])
        assert int(codes[0, 0]) == 127
    X = (RNG.standard_normal((128, 16)) * 2.5).astype(np.float32)
    codes, delta = orc.quantize_blocks(X, 64)
    for i in range(2):
        for r in range(64):
            for c in range(16):
                assert int(codes[64 * i + r, c]) == _exact_int8_code(X[64 * i + r, c], delta[i])


def test_ambiguity_map_flags_only_decisions_near_the_cut():
    """Entries are ambiguous when the normalised mass before them is within
    1e-4 of tau, or when near-equal weights sit on both sides of the cut.
    P_hat = (0.5, 0.3, 0.2): at tau = 0.5 + 5e-5 the second entry (mass 0.5
    before it) is flagged; at tau = 0.5 + 1e-3 nothing is."""
    row = np.log([5.0, 3.0, 2.0]) + 1.5
    Q, K, N = _constant_block_inputs(row)
    pr = orc.predict_mask(Q, K, 128, 64, 0.5 + 5e-5, 0.5, False, 0.5)
    assert pr["amb"][0, 0, :, :3].tolist() == [[False, True, False]] * 2
    pr = orc.predict_mask(Q, K, 128, 64, 0.5 + 1e-3, 0.5, False, 0.5)
    assert not pr["amb"].any()
    assert pr["M"][0, 0, :, :3].tolist() == [[True, True, False]] * 2
    # weights 4 : 3 : 3(1 - 5e-6) : 1 at tau = 0.5: the cut falls between the
    # two near-equal weights, so both are flagged and nothing else
    row = np.log([4.0, 3.0, 3.0 * (1 - 5e-6), 1.0]) + 1.5     # no zero key token
    Q, K, N = _constant_block_inputs(row)
    pr = orc.predict_mask(Q, K, 128, 64, 0.5, 0.5, False, 0.5)
    assert pr["amb"][0, 0, 0, :4].tolist() == [False, True, True, False]
    assert pr["M"][0, 0, 0, :4].tolist() == [True, True, False, False]
    # a weight alone at the cut is not ambiguous
    row = np.log([4.0, 3.0, 2.0, 1.0]) + 1.5
    Q, K, N = _constant_block_inputs(row)
    pr = orc.predict_mask(Q, K, 128, 64, 0.5, 0.5, False, 0.5)
    assert not pr["amb"].any()


def test_whole_forward_dense_limit_with_permutation_equals_softmax_attention():
    """sparge_forward chains permute -> predict -> attention -> inverse.  With
    theta > 1 (every block a fix block) and lambda = -inf, and with or without
    the Hilbert permutation (dense attention is permutation invariant, rebuttal
    page, reply to Weakness 3.2), it is plain softmax attention."""
    N, P, grid, d = 300, 12, (2, 8, 9), 16
    perm = orc.hilbert_permutation(N, P, *grid)
    Q, K, V = rand_qkv(1, 4, 2, N, d)
    ref = dense_attention(Q, K, V, d ** -0.5)
    for pm in (None, perm):
        O, pred, st = orc.sparge_forward(Q, K, V, 128, 64, 0.9, 1.5, -np.inf, False, d ** -0.5,
                                         perm=pm)
        assert np.allclose(O, ref, atol=1e-12)
        assert pred["M"].all() and st["skipped_slices"] == 0
