"""Context drop-off and drop-in on a routed selection - TEST INFRASTRUCTURE.

Only the tests may import this module. Plain Python loops, meant for a few
thousand query rows at a time; it shares nothing with the CUDA library.

What it computes ("Mixture of Contexts for Long Video Generation | Summary",
training details of the appendix; "【DL輪読会】Mixture of Contexts for Long Video
Generation", slide 14): during training each query's routed selection is
perturbed. Drop-off draws p_drop ~ Uniform(0, p_max) and removes
floor(p_drop * k) of the selected chunks at random; drop-in draws
m ~ Poisson(lambda) and adds m random chunks.

Readings where the pages leave a step open (each stated in the design notes):
- only routed chunks are dropped; the mandatory anchors stay (they are forced);
- at most the chunks actually selected are dropped (queries with fewer than k
  candidates have fewer than k selections);
- added chunks are drawn uniformly without replacement from the query's routing
  candidates (causal, not mandatory) that were not in its original selection,
  so drop-in never re-adds a chunk drop-off just removed;
- m is capped at m_max, the extra width of the output selection (the
  truncated mass P(m >= m_max) goes to m_max);
- caption queries keep their dense attention (no selection, nothing added).

The random draws are inputs: per query 2 + k + m_max uint32 words w -
w[0] -> p_drop = (w[0] / 2^32) * p_max, w[1] -> m by inversion of the Poisson
distribution function, w[2 + j] -> the drop priority of selected entry j (the
n_drop entries with the smallest (priority, j) are dropped: a uniform subset),
w[2 + k + a] -> the a-th added chunk, index floor(w * n_left / 2^32) into the
remaining candidates in ascending chunk order.

Output per query: the surviving selections in their original order, then the
added chunks in draw order, padded with -1 to k + m_max entries.
"""
from __future__ import annotations

import math
from typing import List

import numpy as np

ROLE_CAND = 2
VIDEO = 1


def poisson_thresholds(lam: float, m_max: int) -> List[int]:
    """thr[i] = floor(F(i) * 2^32) for the Poisson(lam) distribution function
    F(i) = sum_{j <= i} e^-lam lam^j / j!, accumulated in double from
    p_0 = exp(-lam), p_j = p_{j-1} * lam / j; m = #{i < m_max : thr[i] <= w}."""
    lam = float(np.float32(lam))  # the rates are single-precision arguments of the call
    thr = []
    p = math.exp(-lam)
    cdf = p
    for i in range(m_max):
        if i > 0:
            p = p * lam / float(i)
            cdf = cdf + p
        thr.append(min(int(math.floor(cdf * 4294967296.0)), 1 << 32))
    return thr


def n_drop(w0: int, p_max: float, k: int) -> int:
    """floor(p_drop * k) with p_drop = (w0 / 2^32) * p_max, in double, left to right."""
    return int(math.floor(float(w0) * (2.0 ** -32) * float(np.float32(p_max)) * float(k)))


def perturb_row(sel_row, cands, words, k: int, p_max: float, thr: List[int], m_max: int):
    """One query: sel_row (k ints, -1 padded), cands (ascending candidate chunk ids),
    words (2 + k + m_max uint32) -> k + m_max ints."""
    s = [int(x) for x in sel_row if x >= 0]
    n_sel = len(s)
    nd = min(n_drop(int(words[0]), p_max, k), n_sel)
    order = sorted(range(n_sel), key=lambda j: (int(words[2 + j]), j))
    dropped = set(order[:nd])
    kept = [s[j] for j in range(n_sel) if j not in dropped]
    w1 = int(words[1])
    m = sum(1 for i in range(m_max) if thr[i] <= w1)
    chosen = set(s)
    rem = [int(c) for c in cands if int(c) not in chosen]
    added: List[int] = []
    for a in range(min(m, len(rem))):
        n_left = len(rem) - a
        idx = (int(words[2 + k + a]) * n_left) >> 32
        left = [c for c in rem if c not in added]
        added.append(left[idx])
    out = kept + added
    return out + [-1] * (k + m_max - len(out))


def perturb(lay, sel: np.ndarray, rnd: np.ndarray, k: int, p_max: float, lam: float, m_max: int,
            rows=None) -> np.ndarray:
    """Perturb the selections of the given rows of every (b, h).

    lay: oracle.Layout (roles already carry the causal mask); sel: [B, H, n, k]
    selections of those rows; rnd: [B, H, n, 2 + k + m_max] uint32 words;
    rows: the query token of each of the n rows (default 0..L-1).
    Returns int32 [B, H, n, k + m_max]."""
    B, H, n = sel.shape[0], sel.shape[1], sel.shape[2]
    rows = np.arange(lay.L) if rows is None else np.asarray(rows)
    thr = poisson_thresholds(lam, m_max)
    out = np.full((B, H, n, k + m_max), -1, dtype=np.int32)
    cands_of = {}
    for i, t in enumerate(rows):
        qc = int(lay.chunk_of_token[int(t)])
        if lay.kind[qc] != VIDEO:
            continue
        if qc not in cands_of:
            cands_of[qc] = np.nonzero(lay.role[qc] == ROLE_CAND)[0]
        for b in range(B):
            for h in range(H):
                out[b, h, i] = perturb_row(sel[b, h, i], cands_of[qc], rnd[b, h, i], k, p_max, thr, m_max)
    return out
