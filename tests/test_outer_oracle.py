"""Pins of the outer-loop routing oracle (oracle/outer.py) against the plain
inner oracle and structural facts, not against a restatement of its own steps:
with M at least the number of candidate segments the masked routing is the
plain routing; with M = 0 in shot mode nothing is left to route; the segment
feature is the length-weighted mean of the pinned chunk means; kept segments
outscore the dropped ones, number min(M, candidates) and respect causality."""
import numpy as np
import pytest

import moc_workloads as W
import oracle
from oracle import outer as OU


def _scene(name, causal=True, H=1):
    wl = getattr(W, name)().replace(causal=causal, H=H, B=1)
    Q, K, V = W.make_qkv(wl)
    lay = oracle.Layout(wl)
    return wl, lay, Q, K


def _rows(lay, n=1200):
    return np.unique(np.concatenate([np.arange(0, lay.L, max(1, lay.L // n)), [lay.L - 1]]))


@pytest.mark.parametrize("name,causal", [("tiny", True), ("ragged", True), ("ragged", False)])
def test_large_M_equals_plain_routing(name, causal):
    wl, lay, Q, K = _scene(name, causal)
    kbar = oracle.pool(wl, K, lay)
    o = OU.outer(wl, lay, Q, K, M=64)
    rows = _rows(lay)
    sel, _ = OU.route_masked(wl, lay, Q, kbar, o["mask"], o["blocks"], o["seg"], rows, wl.k)
    rt = oracle.route(wl, Q, kbar, rows=rows, lay=lay)
    assert np.array_equal(sel, rt["sel"])


def test_zero_M_leaves_no_candidates_in_shot_mode():
    wl, lay, Q, K = _scene("ragged")
    kbar = oracle.pool(wl, K, lay)
    o = OU.outer(wl, lay, Q, K, M=0)
    sel, _ = OU.route_masked(wl, lay, Q, kbar, o["mask"], o["blocks"], o["seg"], _rows(lay), wl.k)
    assert (sel == -1).all()


def test_segment_feature_is_weighted_chunk_mean():
    wl, lay, Q, K = _scene("ragged")
    kbar = oracle.pool(wl, K, lay)[0, 0]
    seg = OU.segments(lay)
    n = np.diff(lay.off)
    Kf = K[0, 0].double().numpy()
    for s in range(int(seg.max()) + 1):
        cs = np.nonzero(seg == s)[0]
        toks = np.concatenate([np.arange(lay.off[c], lay.off[c + 1]) for c in cs])
        np.testing.assert_allclose(Kf[toks].mean(axis=0), (n[cs, None] * kbar[cs]).sum(0) / n[cs].sum(),
                                   rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal,M", [(True, 2), (False, 3), (True, 1)])
def test_kept_segments_outscore_the_rest(causal, M):
    wl, lay, Q, K = _scene("ragged", causal, H=2)
    o = OU.outer(wl, lay, Q, K, M=M)
    seg = o["seg"]
    for b in range(wl.B):
        for h in range(wl.H):
            for g, chunks in enumerate(o["blocks"]):
                m = int(o["mask"][b, h, g])
                if lay.kind[chunks[0]] != OU.VIDEO:
                    assert m == 0
                    continue
                own = int(seg[chunks[0]])
                sc = o["scores"][b, h, g]
                cands = [s for s in range(len(sc)) if not np.isnan(sc[s])]
                kept = [s for s in cands if (m >> s) & 1]
                dropped = [s for s in cands if not (m >> s) & 1]
                assert (m >> own) & 1 and len(kept) == min(M, len(cands))
                if kept and dropped:
                    assert min(sc[kept]) >= max(sc[dropped])
                if causal:
                    assert all(s < own for s in cands)


def test_scores_are_products_of_weighted_chunk_means():
    """Block feature from the queries, segment feature from the keys: both as
    length-weighted means of the pinned per-chunk pooling."""
    wl, lay, Q, K = _scene("ragged", H=1)
    o = OU.outer(wl, lay, Q, K, M=2)
    qbar = oracle.pool(wl, Q, lay)[0, 0]
    kbar = oracle.pool(wl, K, lay)[0, 0]
    n = np.diff(lay.off).astype(np.float64)
    seg = o["seg"]
    for g, chunks in enumerate(o["blocks"]):
        if lay.kind[chunks[0]] != OU.VIDEO:
            continue
        qf = (n[chunks, None] * qbar[chunks]).sum(0) / n[chunks].sum()
        for s in range(o["scores"].shape[-1]):
            if np.isnan(o["scores"][0, 0, g, s]):
                continue
            cs = np.nonzero(seg == s)[0]
            kf = (n[cs, None] * kbar[cs]).sum(0) / n[cs].sum()
            assert abs(o["scores"][0, 0, g, s] - qf @ kf) <= 1e-9 * (1 + abs(qf @ kf))


def test_ties_keep_the_lowest_segments():
    wl, lay, Q, K = _scene("ragged", causal=False)
    Q.zero_()
    o = OU.outer(wl, lay, Q, K, M=2)
    seg = o["seg"]
    for g, chunks in enumerate(o["blocks"]):
        if lay.kind[chunks[0]] != OU.VIDEO:
            continue
        own = int(seg[chunks[0]])
        want = [s for s in range(int(seg.max()) + 1) if s != own][:2] + [own]
        assert int(o["mask"][0, 0, g]) == sum(1 << s for s in set(want))
