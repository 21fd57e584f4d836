"""The allocation-free predictor entry point against the workspace one.

sparge_predict_mask_noalloc serves callers that cannot allocate device memory
when they call (their host framework owns all device buffers, or allocation is
forbidden after start-up): its scratch is a static device array inside the
library.  Its outputs must equal sparge_predict_mask's on the same inputs, on
two calls in a row with different inputs (so stale scratch contents would
show).  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import free_block_sparse_predict_b200 as fb

from gpu_common import dev, params_for, to_dev, workload

pytestmark = pytest.mark.gpu


def _with_workspace(p, q, k):
    ws = fb.workspace(p, dev())
    outs = fb.predict_outputs(p, dev())
    fb.sparge_predict_mask(p, q, k, *outs, ws)
    return outs


def _without_workspace(p, q, k):
    outs = fb.predict_outputs(p, dev())
    fb.sparge_predict_mask_noalloc(p, q, k, *outs)
    return outs


def _same(a, b, p):
    mask_a, idx_a, cnt_a, sq_a, sk_a = (x.cpu().numpy() for x in a)
    mask_b, idx_b, cnt_b, sq_b, sk_b = (x.cpu().numpy() for x in b)
    assert np.array_equal(mask_a, mask_b)
    assert np.array_equal(cnt_a, cnt_b)
    for pos in np.ndindex(*cnt_a.shape):
        assert np.array_equal(idx_a[pos][:cnt_a[pos]], idx_b[pos][:cnt_b[pos]])
    assert np.array_equal(sq_a, sq_b) and np.array_equal(sk_a, sk_b)


def test_noalloc_predictor_matches_workspace_predictor_twice():
    cases = [("llm_32k", {"N": 8192, "Hq": 8, "Hkv": 2}), ("video_dit", {"Hq": 4, "Hkv": 4})]
    for name, over in cases:                       # two calls in a row, different inputs
        w, t = workload(name, **over)
        p = params_for(w)
        q, k = to_dev(t["q"], w.dtype), to_dev(t["k"], w.dtype)
        ref = _with_workspace(p, q, k)
        got = _without_workspace(p, q, k)
        torch.cuda.synchronize()
        _same(ref, got, p)


def test_noalloc_second_call_same_shape_new_inputs():
    """Two calls with the same parameters and different inputs: a scratch
    region the second call failed to rewrite would still hold the first
    call's values, which would be right for the first inputs only."""
    w, _ = workload("llm_32k", N=8192, Hq=8, Hkv=2)
    p = params_for(w)
    from synth import make_qkv
    for seed in (1, 2):
        t = make_qkv(w, seed=seed)
        q, k = to_dev(t["q"], w.dtype), to_dev(t["k"], w.dtype)
        got = _without_workspace(p, q, k)
        ref = _with_workspace(p, q, k)
        torch.cuda.synchronize()
        _same(ref, got, p)


def test_noalloc_leaves_the_current_device_alone():
    w, t = workload("tiny")
    p = params_for(w)
    q, k = to_dev(t["q"], w.dtype), to_dev(t["k"], w.dtype)
    before = torch.cuda.current_device()
    _without_workspace(p, q, k)
    torch.cuda.synchronize()
    assert torch.cuda.current_device() == before


def test_noalloc_rejects_what_it_cannot_hold():
    w, t = workload("llm_32k", N=4096, Hq=2, Hkv=1)
    q, k = to_dev(t["q"], w.dtype), to_dev(t["k"], w.dtype)
    big = params_for(w.replace(N=131072, Hq=64, Hkv=8))   # pooled means exceed 32 MiB
    outs = fb.predict_outputs(params_for(w), dev())
    # through the C entry point itself: the binding would refuse these
    # tensors (smaller than the parameters imply) before the library saw them
    P = lambda x: ctypes.c_void_p(x.data_ptr())
    code = fb._native.lib().sparge_predict_mask_noalloc(ctypes.byref(big), P(q), P(k),
                                                        *[P(x) for x in outs], None)
    assert code == 5
    with pytest.raises(fb.SpargeError) as e:
        fb.sparge_predict_mask_noalloc(big, q, k, *outs)
    assert e.value.code == 1
    with pytest.raises(fb.SpargeError) as e:
        fb.sparge_predict_mask_noalloc(params_for(w, qk_int8=True), q, k, *outs)
    assert e.value.code == 2
    # a parameter set the workspace predictor calls unsupported (d = 96) gets
    # the same status here
    odd = params_for(w)
    odd.d = 96
    code = fb._native.lib().sparge_predict_mask_noalloc(ctypes.byref(odd), P(q), P(k),
                                                        *[P(x) for x in outs], None)
    assert code == 2
