"""Failure detection on the GPU without a fault: a device wait that can never
be satisfied ends by its time limit, the status word reports it, the host
reads and clears it, and the next calls run normally."""
import time

import numpy as np
import pytest
import torch

import free_block_sparse_predict_b200 as fb

from gpu_common import (MAX_ABS, dev, gpu_attention, gpu_predict, params_for, to_dev,
                        torch_dense_attention, workload)

pytestmark = pytest.mark.gpu


def test_unsatisfiable_wait_times_out_and_context_survives():
    ws = torch.zeros(4096, dtype=torch.uint8, device=dev())
    assert fb.sparge_device_status(ws) == 0
    t0 = time.time()
    fb.sparge_selftest_wait_timeout(ws)
    assert fb.sparge_device_status(ws) == 4          # SPARGE_ETIMEOUT, then cleared
    assert 0.5 < time.time() - t0 < 30
    assert fb.sparge_device_status(ws) == 0
    # the context is intact: a normal forward still runs and is correct
    w, t = workload("tiny")
    p = params_for(w, theta=2.0, lam=float("-inf"))
    q, k, v = (to_dev(t[x], w.dtype) for x in ("q", "k", "v"))
    ws2, mask, idx, cnt, _, _ = gpu_predict(p, q, k)
    o, _ = gpu_attention(p, q, k, v, idx, cnt, ws2)
    ref = torch_dense_attention(q, k, v, w.scale, w.causal)
    assert (o - ref).abs().max().item() <= MAX_ABS
