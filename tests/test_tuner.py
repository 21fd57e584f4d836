"""The L1-rule hyper-parameter search (paper review page, section 三,
hyper-parameter determination): CPU checks of the band logic on monotone
error curves, for tau alone and for the tau -> lambda -> theta order, and a
GPU check that a tuned layer's L1, recomputed from the float64 oracle at the
chosen hyper-parameters, agrees with the library's and lies in the band."""
import math

import numpy as np
import pytest

from free_block_sparse_predict_b200.tuner import RANGES, search_params, search_tau


def curve(scale):
    # a monotone stand-in for L1(tau): falls as tau keeps more mass
    return lambda tau: (scale * (1.0 - tau) ** 2, 1.0 - tau)


def test_lands_in_band_when_possible():
    r = search_tau(curve(0.5), band=(0.05, 0.06))
    assert r.in_band and 0.05 <= r.l1 <= 0.06
    # the band corresponds to tau in [1 - sqrt(0.12), 1 - sqrt(0.10)]
    assert 1 - math.sqrt(0.12) - 1e-9 <= r.tau <= 1 - math.sqrt(0.10) + 1e-9


def test_error_above_band_even_at_tau_one_returns_tau_one():
    r = search_tau(lambda tau: (0.2, 0.0), band=(0.05, 0.06))
    assert r.tau == 1.0 and not r.in_band


def test_band_unreachable_returns_sparsest_admissible():
    # the error jumps over the band: keep the smallest tau with L1 <= l2
    f = lambda tau: ((0.0, 1 - tau) if tau > 0.5 else (0.5, 1 - tau))
    r = search_tau(f, band=(0.05, 0.06), iters=20)
    assert not r.in_band and r.l1 <= 0.06 and 0.5 < r.tau < 0.5 + 1e-3


def test_never_returns_an_inadmissible_tau():
    rng = np.random.default_rng(0)
    for _ in range(50):
        a, b = sorted(rng.uniform(0.01, 0.2, size=2))
        s = rng.uniform(0.05, 2.0)
        r = search_tau(curve(s), band=(a, b))
        assert r.l1 <= b or r.tau == 1.0


def _model(a, b, c):
    # a monotone stand-in for L1(tau, lambda, theta): each term grows toward
    # the parameter's sparse end (tau 1 -> 0.05, lambda -50 -> -0.5, theta 1 -> -1)
    def f(hp):
        e = a * (1 - hp["tau"]) ** 2 + b * math.exp(hp["lambda"]) + c * (1 - hp["theta"]) / 2
        return e, e
    return f


def test_tau_alone_reaches_the_band_and_the_rest_stay():
    r = search_params(_model(0.2, 0.0, 0.0), {"tau": 0.9, "lambda": -8.0, "theta": 0.6},
                      band=(0.05, 0.06))
    assert r.in_band and 0.05 <= r.l1 <= 0.06
    assert r.lam == -8.0 and r.theta == 0.6
    assert {t[0] for t in r.trace} == {"tau"}


def test_lambda_searched_when_tau_cannot_reach_the_band():
    # tau's whole range gives at most 0.02 (< l1 = 0.05): lambda takes over
    r = search_params(_model(0.02, 0.2, 0.0), {"tau": 0.9, "lambda": -50.0, "theta": 2.0},
                      band=(0.05, 0.06), iters=30)
    assert r.in_band and 0.05 <= r.l1 <= 0.06
    assert r.tau == pytest.approx(RANGES["tau"][1], abs=1e-6)     # tau went all the way
    assert RANGES["lambda"][0] < r.lam < RANGES["lambda"][1]
    assert [t[0] for t in r.trace][0] == "tau" and r.trace[-1][0] == "lambda"
    assert r.theta == 2.0


def test_theta_searched_last():
    r = search_params(_model(0.01, 0.01, 0.2), {"tau": 0.9, "lambda": -8.0, "theta": 1.0},
                      band=(0.05, 0.06), iters=30)
    assert r.in_band and r.trace[-1][0] == "theta"
    assert -1.0 < r.theta < 1.0


def test_error_above_band_at_the_dense_end_stops():
    # the caller's lambda alone exceeds l2: tau stays at its dense end, nothing else moves
    r = search_params(_model(0.1, 0.2, 0.0), {"tau": 0.9, "lambda": -1.0, "theta": 0.6},
                      band=(0.05, 0.06))
    assert not r.in_band and r.tau == 1.0 and r.lam == -1.0


@pytest.mark.gpu
def test_tuned_layer_l1_matches_the_oracle_and_lies_in_the_band():
    import torch
    from free_block_sparse_predict_b200 import make_params
    from free_block_sparse_predict_b200.tuner import tune_layer
    from gpu_common import oracle_inputs, to_dev, workload
    from oracle import sparge_oracle as orc
    w, t = workload("llm_32k", N=2048, Hq=2, Hkv=1)
    q, k, v = (to_dev(t[x], w.dtype) for x in ("q", "k", "v"))
    band = (0.02, 0.04)
    p = make_params(w.B, w.Hq, w.Hkv, w.N, w.d, 0.9, 0.6, w.lam, causal=True,
                    io_dtype=torch.bfloat16)
    r = tune_layer(p, q, k, v, band=band, iters=16)
    print(f"[tuner] tau {r.tau:.4f} lambda {r.lam:.4f} theta {r.theta:.4f} L1 {r.l1:.5f} "
          f"sparsity {r.sparsity:.4f} steps {len(r.trace)}")
    assert r.in_band and r.l1 <= band[1]
    # the same hyper-parameters through the float64 oracle
    Q, K, V = oracle_inputs(w, t)
    dense = orc.predict_mask(Q, K, w.bq, w.bk, 0.9, 2.0, True, w.scale)
    io, co = orc.mask_compact(dense["M"])
    O, _ = orc.sparse_attention(Q, K, V, io, co, w.bq, w.bk, -np.inf, True, w.scale)
    pr = orc.predict_mask(Q, K, w.bq, w.bk, r.tau, r.theta, True, w.scale)
    io, co = orc.mask_compact(pr["M"])
    O2, st = orc.sparse_attention(Q, K, V, io, co, w.bq, w.bk, r.lam, True, w.scale)
    l1 = np.abs(O - O2).sum() / np.abs(O).sum()
    print(f"[tuner] oracle L1 {l1:.5f}, near-threshold lambda decisions {st['near_lambda']}")
    assert abs(l1 - r.l1) <= 2e-3, (l1, r.l1)
    assert band[0] - 2e-3 <= l1 <= band[1] + 2e-3
