"""The attention softmax evaluates a quarter of its exponentials with a cubic
on the FMA pipe instead of the special-function unit. This CPU test replays
that fp32 arithmetic (round-to-nearest split, cubic, exponent-field add) with
numpy, reading the coefficients from the kernel source, and bounds its error
against the exact 2^x: it has to stay well below the 2^-9 rounding of the
bf16 probabilities it produces."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "free_block_sparse_eigenbasis_b200", "csrc", "attn.cu")


def _kernel_poly():
    text = open(SRC).read()
    body = text[text.index("__device__ __forceinline__ float exp2_poly"):]
    body = body[:body.index("\n}\n")]
    coef = [float(v) for v in re.findall(r"(-?\d+\.\d+)f", body.split("const float q =")[1])]
    assert len(coef) == 4, coef
    c3, c2, c1, c0 = coef
    return np.float32(c0), np.float32(c1), np.float32(c2), np.float32(c3)


def _emulate(x):
    c0, c1, c2, c3 = _kernel_poly()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic)).astype(np.float32)
    q = np.float32(c3) * f + c2
    q = q.astype(np.float32) * f + c1
    q = q.astype(np.float32) * f + c0
    q = q.astype(np.float32)
    bits = q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    bits = ((bits + 2**31) % 2**32 - 2**31).astype(np.int32)
    return bits.view(np.float32)


def test_exp2_poly_relative_error():
    x = np.linspace(-125.9, 9.0, 2_000_001, dtype=np.float64).astype(np.float32)
    y = _emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 1e-4, rel.max()


def test_exp2_poly_integers_and_clamp():
    n = np.arange(-125, 9, dtype=np.float32)  # 2^-126 itself lands in the subnormal range
    y = _emulate(n).astype(np.float64)
    assert np.all(np.abs(y / np.exp2(n.astype(np.float64)) - 1.0) < 1e-4)
    # masked logits (-inf) and very negative ones clamp to 2^-126, not NaN
    z = _emulate(np.array([-np.inf, -1000.0, -127.5], dtype=np.float32)).astype(np.float64)
    assert np.all(np.isfinite(z)) and np.all(z >= 0) and np.all(z <= 2.0 ** -125)
