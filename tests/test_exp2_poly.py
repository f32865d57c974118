"""Error bound of the attention kernel's FMA-pipe exp2 (used for a share of
the softmax exponentials instead of the MUFU unit): the shipped coefficients,
evaluated step by step in float32 as the kernel does (round-to-nearest by a
1.5 * 2^23 addition, degree-3 Horner on [-1/2, 1/2], exponent-field add),
must stay within 1e-4 relative error of 2^x over the clamped domain. P is
rounded to bf16 (relative 2^-9) right after, so 1e-4 is far inside it."""
import os
import re

import numpy as np

from conftest import ROOT


def _coeffs():
    src = open(os.path.join(ROOT, "chunk_routed_sparse_b200", "csrc", "sm100.cuh")).read()
    return [np.float32(float(re.search(rf"kExp2C{i} = ([0-9.eE+-]+)f;", src).group(1))) for i in range(4)]


def _poly_exp2(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = ((c3 * f + c2) * f + c1) * f + c0
    bits = p.astype(np.float32).view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_fma_pipe_exp2_error_bound():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001), np.arange(-125, 9) + 0.5,
                        np.arange(-125, 9).astype(np.float64)]).astype(np.float32)
    y = _poly_exp2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 1e-4, rel.max()
    assert np.all(np.isfinite(y)) and np.all(y > 0)


def test_fma_pipe_exp2_clamps_below_range():
    y = _poly_exp2(np.array([-1000.0, -126.0, -125.0], dtype=np.float32)).astype(np.float64)
    assert np.all(y > 0) and np.all(y < 2.0 ** -124)
