"""The attention softmax evaluates some exponentials with a cubic on the FMA
pipe.  These CPU checks pin that evaluation: the constants embedded in the
kernel are the ones the fitting script produces, and the float32 step sequence
the kernel runs (round-to-nearest split, Horner cubic, exponent add) stays
within its stated relative error of 2^y on the range the kernel uses."""
import os
import re

import numpy as np

from free_block_sparse_predict_b200 import exp2_poly

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "free_block_sparse_predict_b200", "csrc", "attn_sm100.cu")


def kernel_constants():
    text = open(SRC).read()
    vals = {k: float(v) for k, v in re.findall(r"(kC[0-3]) = ([0-9.e+-]+)f", text)}
    return np.array([vals["kC0"], vals["kC1"], vals["kC2"], vals["kC3"]], dtype=np.float32)


def emulate(y, c):
    """The kernel's float32 steps for 2^y."""
    f32 = np.float32
    y = np.maximum(y.astype(f32), f32(-125.0))
    magic = f32(12582912.0)
    t = (y + magic).astype(f32)
    n = (t - magic).astype(f32)
    f = (y - n).astype(f32)                       # exact (fma with -1 in the kernel)
    p = (c[3] * f + c[2]).astype(f32)
    p = (p * f + c[1]).astype(f32)
    p = (p * f + c[0]).astype(f32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(f32)


def test_kernel_constants_match_the_fit():
    c32, err = exp2_poly.float32_coefficients()
    assert np.array_equal(kernel_constants(), c32)
    assert err < 8e-5


def test_emulated_steps_meet_the_bound():
    c = kernel_constants()
    y = np.concatenate([np.linspace(-40.0, 8.0, 400001), -np.random.default_rng(0).random(10000) * 120])
    y = y.astype(np.float32)
    got = emulate(y, c).astype(np.float64)
    ref = np.exp2(y.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 8e-5
    # far below the range: a value that is 0 for every later use
    assert emulate(np.array([-1e6, -np.inf], np.float32), c).max() < 1e-37
