"""The FMA-pipe 2^x of the fused kernel (exp2_poly.h), re-evaluated on the
CPU in float32 with the same operations, against numpy's exp2."""

import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "partitioned_attention_state_b200", "csrc", "exp2_poly.h")


def coeffs():
    text = open(HDR).read()
    return [np.float32(float.fromhex(re.search(rf"#define DT_EXP2_C{k} (\S+)f", text).group(1)))
            for k in range(4)]


def exp2_like_kernel(x):
    c0, c1, c2, c3 = coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    j = (x + magic).astype(np.float32)
    n = (j - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    q = (np.float32(c3) * f + c2).astype(np.float32)      # fma rounding differs by <= 1 ulp
    q = (q * f + c1).astype(np.float32)
    q = (q * f + c0).astype(np.float32)
    bits = q.view(np.int32) + (j.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_polynomial_relative_error_bound():
    f = np.linspace(-0.5, 0.5, 200001, dtype=np.float32)
    c0, c1, c2, c3 = coeffs()
    q = ((c3 * f + c2) * f + c1) * f + c0
    rel = np.abs(q.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1)
    assert rel.max() < 8e-5


def test_range_reduction_and_reconstruction():
    rng = np.random.Generator(np.random.PCG64(0))
    x = np.concatenate([rng.uniform(-120, 8, 100000), np.arange(-120, 9, 0.5), [0.0, -0.5, 0.5, 7.999]])
    x = x.astype(np.float32)
    got = exp2_like_kernel(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1)
    assert rel.max() < 1.2e-4
    # clamp: very negative inputs give a negligible, non-negative value
    tiny = exp2_like_kernel(np.array([-1e4, -300.0], dtype=np.float32))
    assert np.all(tiny >= 0) and np.all(tiny < 1e-37)
