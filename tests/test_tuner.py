"""The L1-rule tau search (paper review page, section 三, hyper-parameter
determination): CPU checks of the band logic on monotone error curves, and a
GPU check that a tuned layer lands in its band."""
import math

import numpy as np
import pytest

from free_block_sparse_predict_b200.tuner import search_tau


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


@pytest.mark.gpu
def test_tuned_layer_meets_its_band():
    import torch
    from free_block_sparse_predict_b200 import make_params
    from free_block_sparse_predict_b200.tuner import tune_layer
    from gpu_common import to_dev, workload
    w, t = workload("llm_32k", N=4096, Hq=4, Hkv=1)
    q, k, v = (to_dev(t[x], w.dtype) for x in ("q", "k", "v"))
    p = make_params(w.B, w.Hq, w.Hkv, w.N, w.d, 0.9, -1.0, w.lam, causal=True,
                    io_dtype=torch.bfloat16)
    r = tune_layer(p, q, k, v, band=(0.02, 0.04))
    assert r.l1 <= 0.04 + 1e-6
    assert r.in_band and r.sparsity > 0.0
