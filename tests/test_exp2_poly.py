"""The prefill kernel computes a quarter of its softmax exponentials without
the multi-function unit: x is rounded to the nearest integer n, f = x - n
lies in [-1/2, 1/2], 2^f comes from a degree-3 polynomial fitted for
minimax relative error, and n is added into the exponent field.  This test
replays those float32 steps in numpy (the coefficients are restated from the
kernel source) and checks the result against exact 2^x: the relative error
must stay below 1e-4, far under the 2^-9 rounding of the bf16 P it feeds."""
import re
import os

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "ragged_paged_attention_03_b200", "csrc", "prefill2_kernel.cu")


def coefficients():
    src = open(SRC).read()
    body = src[src.index("float exp2_fma(float x)"):]
    body = body[:body.index("}")]
    c = [float(v) for v in re.findall(r"([0-9]+\.[0-9]+)f", body) if float(v) < 2.0]
    # the polynomial's coefficients in Horner order: c3, c2, c1, c0
    assert len(c) == 4, c
    return tuple(np.float32(v) for v in c)


def emulate(x):
    c3, c2, c1, c0 = coefficients()
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-125.0))
    r = (x + f32(12582912.0)).astype(f32)
    n = (r - f32(12582912.0)).astype(f32)
    f = (x - n).astype(f32)
    p = (c3 * f + c2).astype(f32)
    p = (p * f + c1).astype(f32)
    p = (p * f + c0).astype(f32)
    ni = r.view(np.int32) - np.int32(0x4B400000)
    return (p.view(np.int32) + (ni << 23)).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-60.0, 8.0, 200001).astype(np.float32)
    got = emulate(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 1e-4, rel.max()


def test_clamped_tail_is_tiny_and_positive():
    x = np.array([-125.0, -200.0, -1e30, -np.inf], dtype=np.float32)
    got = emulate(x)
    assert np.all(got > 0) and np.all(got < 1e-37)
