"""The FMA-pipe 2^x of the E4M3 softmax (``ex2_fma2`` in csrc/sm100.cuh), checked
on the CPU against the exact 2^x.

The device function reduces x to n + f (n = round(x) from the low mantissa bits of
x + 1.5 * 2^23, f in [-1/2, 1/2]), evaluates a degree-4 polynomial for 2^f and adds
n to the exponent field. This test reads its five coefficients from the header,
repeats those steps in numpy float32 arithmetic (products and sums rounded
separately, so at least as inexact as the device's fused multiply-adds), and
bounds the relative error against 2^x in float64 over the range the softmax uses
(x <= 2 after the lazy rescale, results that are normal numbers).
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(__file__), "..", "chunk_routed_sparse_b200", "csrc", "sm100.cuh")


def _coefficients():
    src = open(HDR).read()
    body = src[src.index("ex2_fma2"):]
    vals = {m.group(1): float(m.group(2)) for m in re.finditer(r"\b(c[0-4]) = ([0-9.eE+-]+)f", body)}
    return [np.float32(vals[f"c{i}"]) for i in range(5)]


def _ex2_fma(x):
    c = _coefficients()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    n = (t - shift).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = c[4]
    for k in (3, 2, 1, 0):
        p = (p * f).astype(np.float32)
        p = (p + c[k]).astype(np.float32)
    e = (t.view(np.int32) - np.int32(0x4B400000)) << 23
    return (p.view(np.int32) + e).view(np.float32), n


def test_reduction_is_round_to_nearest():
    x = np.linspace(-125.5, 2.0, 100_001, dtype=np.float32)
    _, n = _ex2_fma(x)
    assert np.all(np.abs(x - n) <= 0.5)
    assert np.array_equal(n, np.round(n))


def test_relative_error_over_the_softmax_range():
    x = np.concatenate([np.linspace(-125.0, 2.0, 400_001), np.linspace(-1.0, 1.0, 200_001),
                        np.arange(-125, 3, dtype=np.float64)]).astype(np.float32)
    y, _ = _ex2_fma(x)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(y.astype(np.float64) / exact - 1.0)
    assert rel.max() < 4e-6, rel.max()


def test_polynomial_alone_on_the_reduced_interval():
    c = [float(v) for v in _coefficients()]
    f = np.linspace(-0.5, 0.5, 100_001)
    p = sum(c[k] * f ** k for k in range(5))
    assert np.max(np.abs(p / np.exp2(f) - 1.0)) < 3e-6


def test_masked_scores_give_a_negligible_weight():
    y, _ = _ex2_fma(np.array([-np.inf, -1e30, -126.0, -200.0], dtype=np.float32))
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y < 2.0 ** -125)
