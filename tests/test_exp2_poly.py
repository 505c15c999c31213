"""Error bound of the FMA-pipe exp2 used for part of the softmax exponentials.

The kernel's polynomial (coefficients read from the CUDA source, so the test follows the
shipped constants) is replayed step by step in float32 and compared with exp2 in float64.
It must stay within 1e-4 relative error on [-125, 8] (the kernel only passes x <= 8), far
below the 2^-9 relative rounding of the bf16 probabilities it produces. CPU only."""
import os
import re

import numpy as np

from tests.conftest import ROOT


def _coeffs():
    src = open(os.path.join(ROOT, "block_sparse_attention_query_b200", "csrc", "attention.cuh")).read()
    val = {}
    for name in ("kExp2Clamp", "kExp2Magic", "kExp2C3", "kExp2C2", "kExp2C1", "kExp2C0"):
        m = re.search(r"constexpr float " + name + r" = (-?[0-9]+\.[0-9]+)f;", src)
        val[name] = np.float32(m.group(1))
    assert val["kExp2Clamp"] == np.float32(-125.0) and val["kExp2Magic"] == np.float32(12582912.0)
    return val["kExp2C3"], val["kExp2C2"], val["kExp2C1"], val["kExp2C0"]


def _exp2_fma(x):
    c3, c2, c1, c0 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0))).astype(np.float32)
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    return (p.view(np.int32) + (t.view(np.int32) << 23)).view(np.float32)


def test_exp2_fma_relative_error_bound():
    x = np.linspace(-125.0, 8.0, 2_000_001).astype(np.float32)
    ref = np.exp2(x.astype(np.float64))
    got = _exp2_fma(x).astype(np.float64)
    assert np.max(np.abs(got - ref) / ref) < 1e-4


def test_exp2_fma_integer_points_and_underflow():
    n = np.arange(-125, 9).astype(np.float32)
    got = _exp2_fma(n).astype(np.float64)
    assert np.max(np.abs(got / np.exp2(n.astype(np.float64)) - 1)) < 1e-4
    low = _exp2_fma(np.array([-126.0, -500.0, -np.inf], np.float32))
    assert np.all(low > 0) and np.all(low < 3e-38)
