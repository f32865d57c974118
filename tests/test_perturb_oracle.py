"""Pins of the drop-off / drop-in oracle (oracle/perturb.py) against the
distributions the pages name and against structural invariants, not against a
restatement of its own steps: floor(p_drop k) with p_drop ~ U(0, p_max) has a
closed-form law; m follows Poisson(lambda) truncated at m_max; a uniform random
subset drops every selected entry equally often; added chunks are uniform over
the remaining candidates; and on routed scenes the outputs keep the mask."""
import math

import numpy as np
import pytest
from scipy import stats

import moc_workloads as W
import oracle
from oracle import perturb as P

RNG = np.random.default_rng(20260)


def _words(n, width):
    return RNG.integers(0, 1 << 32, size=(n, width), dtype=np.uint64)


def test_identity_when_both_rates_are_zero():
    wl = W.tiny()
    Q, K, V = W.make_qkv(wl)
    orc = oracle.Layout(wl)
    kbar = oracle.pool(wl, K, orc)
    rt = oracle.route(wl, Q, kbar, lay=orc)
    m_max = 3
    rnd = _words(wl.B * wl.H * wl.L, 2 + wl.k + m_max).reshape(wl.B, wl.H, wl.L, -1)
    out = P.perturb(orc, rt["sel"], rnd, wl.k, 0.0, 0.0, m_max)
    assert np.array_equal(out[..., :wl.k], rt["sel"]) and (out[..., wl.k:] == -1).all()


@pytest.mark.parametrize("p_max,k", [(0.5, 3), (1.0, 8), (0.3, 5)])
def test_drop_count_law(p_max, k):
    """P(floor(U c) = j) = 1/c for j < floor(c), (c - floor(c))/c for j = floor(c), c = p_max k."""
    c = float(np.float32(p_max)) * k
    n = 200_000
    w0 = RNG.integers(0, 1 << 32, size=n, dtype=np.uint64)
    counts = np.bincount([P.n_drop(int(x), p_max, k) for x in w0], minlength=int(math.floor(c)) + 1)
    jmax = int(math.floor(c))
    probs = np.array([1.0 / c] * jmax + [(c - jmax) / c])
    keep = probs > 0
    obs, exp = counts[:jmax + 1][keep], n * probs[keep]
    assert counts[jmax + 1:].sum() == 0
    assert stats.chisquare(obs, exp * obs.sum() / exp.sum()).pvalue > 1e-4


@pytest.mark.parametrize("lam,m_max", [(0.5, 4), (2.0, 6), (1.0, 1)])
def test_added_count_is_truncated_poisson(lam, m_max):
    thr = P.poisson_thresholds(lam, m_max)
    n = 200_000
    w1 = RNG.integers(0, 1 << 32, size=n, dtype=np.uint64)
    m = np.array([sum(1 for t in thr if t <= int(x)) for x in w1])
    pmf = stats.poisson.pmf(np.arange(m_max), lam)
    probs = np.append(pmf, 1.0 - pmf.sum())
    obs = np.bincount(m, minlength=m_max + 1)
    assert stats.chisquare(obs, n * probs).pvalue > 1e-4


def test_dropped_subset_is_uniform():
    """Selection of 5 chunks, n_drop fixed at 2 (w0 chosen so): every entry is
    dropped with probability 2/5."""
    k, m_max, p_max = 5, 0, 0.5
    sel = [10, 11, 12, 13, 14]
    w0 = int(0.9 * 2 ** 32)  # floor(0.9 * 0.5 * 5) = 2
    n = 40_000
    words = _words(n, 2 + k + m_max)
    words[:, 0] = w0
    dropped = np.zeros(k)
    for w in words:
        out = P.perturb_row(sel, sel, w, k, p_max, [], m_max)
        kept = [x for x in out if x >= 0]
        assert len(kept) == 3 and kept == sorted(kept)  # original order survives
        for i, c in enumerate(sel):
            dropped[i] += c not in kept
    assert stats.chisquare(dropped, np.full(k, n * 2 / 5)).pvalue > 1e-4


def test_added_chunks_are_uniform_without_replacement():
    k, m_max = 2, 2
    cands = list(range(0, 12))
    sel = [3, 7]
    rem = [c for c in cands if c not in sel]
    thr = P.poisson_thresholds(50.0, m_max)  # lambda large: m = m_max almost surely
    n = 60_000
    words = _words(n, 2 + k + m_max)
    words[:, 0] = 0            # no drop
    words[:, 1] = (1 << 32) - 1
    first = np.zeros(len(rem))
    pairs = {}
    for w in words:
        out = P.perturb_row(sel, cands, w, k, 0.5, thr, m_max)
        a, b = out[2], out[3]
        assert a in rem and b in rem and a != b
        first[rem.index(a)] += 1
        pairs[(a, b)] = pairs.get((a, b), 0) + 1
    assert stats.chisquare(first, np.full(len(rem), n / len(rem))).pvalue > 1e-4
    npair = len(rem) * (len(rem) - 1)
    obs = np.array([pairs.get((a, b), 0) for a in rem for b in rem if a != b])
    assert len(obs) == npair and stats.chisquare(obs, np.full(npair, n / npair)).pvalue > 1e-4


@pytest.mark.parametrize("name,causal", [("tiny", True), ("ragged", True), ("ragged", False)])
def test_invariants_on_routed_scenes(name, causal):
    wl = getattr(W, name)().replace(causal=causal)
    wl = wl.replace(B=1, H=1)
    Q, K, V = W.make_qkv(wl)
    orc = oracle.Layout(wl)
    kbar = oracle.pool(wl, K, orc)
    rows = np.unique(np.concatenate([np.arange(0, wl.L, max(1, wl.L // 1500)), [wl.L - 1]]))
    rt = oracle.route(wl, Q, kbar, rows=rows, lay=orc)
    k, m_max, p_max, lam = wl.k, 3, 0.7, 1.5
    rnd = _words(len(rows), 2 + k + m_max).reshape(1, 1, len(rows), -1)
    out = P.perturb(orc, rt["sel"], rnd, k, p_max, lam, m_max, rows=rows)
    for i, t in enumerate(rows):
        qc = int(orc.chunk_of_token[t])
        s = [int(x) for x in rt["sel"][0, 0, i] if x >= 0]
        o = [int(x) for x in out[0, 0, i] if x >= 0]
        assert (out[0, 0, i][len(o):] == -1).all()           # -1 only as padding
        if orc.kind[qc] != P.VIDEO:
            assert not o
            continue
        cands = set(np.nonzero(orc.role[qc] == P.ROLE_CAND)[0].tolist())
        nd = min(P.n_drop(int(rnd[0, 0, i, 0]), p_max, k), len(s))
        kept = [x for x in o if x in s]
        added = [x for x in o if x not in s]
        assert kept == [x for x in s if x in kept] and len(kept) == len(s) - nd
        assert o[:len(kept)] == kept                          # survivors first, in order
        assert len(set(added)) == len(added) and set(added) <= cands - set(s)
        if causal:
            assert all(c < qc for c in o)
