"""The routing-validity check the GPU parity tests rely on
(``oracle.check_selection``), tested on the CPU with planted mistakes: a
selection that holds a mandatory chunk, a causally hidden chunk, a repeat, a
wrong count, or a reordering without a near tie must be rejected; a swap of
two exactly tied candidates must be accepted as a near-tie swap."""
import numpy as np
import torch

import moc_workloads as W
import oracle


def _routed():
    """Three shots of three 48-token frames after a caption: a query of the
    middle shot has the first shot's frames as candidates and the last shot's
    frames hidden by the causal mask."""
    segs = [W.Segment(16, W.CAPTION, -1, -1)]
    segs += [W.Segment(48, W.VIDEO, s, f) for s in range(3) for f in range(3)]
    wl = W.custom("three_shots", 1, 1, 64, segs, "shot", 0, True, 2, 41, "frame")
    Q, K, V = W.make_qkv(wl)
    lay = oracle.Layout(wl)
    kbar = oracle.pool(wl, K, lay)
    rt = oracle.route(wl, Q, kbar, lay=lay)
    return wl, Q, K, lay, kbar, rt


def _row_with_full_selection(rt):
    """A row whose selection holds k valid picks."""
    full = np.nonzero((rt["sel"][0, 0] >= 0).all(-1) & (rt["rows"] < 16 + 6 * 48))[0]
    assert len(full)
    return int(full[len(full) // 2])


def test_oracle_selection_is_exact():
    wl, Q, K, lay, kbar, rt = _routed()
    res = oracle.check_selection(wl, Q, kbar, rt["sel"].copy(), rt, lay)
    assert res["exact"] == res["rows"] and res["mismatch"] == 0 and not res["bad"]


def test_planted_mistakes_are_rejected():
    wl, Q, K, lay, kbar, rt = _routed()
    r = _row_with_full_selection(rt)
    t = int(rt["rows"][r])
    qc = int(lay.chunk_of_token[t])
    anchors = np.nonzero(lay.role[qc] == oracle.ROLE_ANCHOR)[0]
    hidden = np.nonzero(lay.role[qc] == oracle.ROLE_NONE)[0]
    assert len(hidden)
    plants = {
        "anchor chunk": lambda s: s.__setitem__(0, anchors[-1]),
        "causally hidden chunk": lambda s: s.__setitem__(0, hidden[0]),
        "repeat": lambda s: s.__setitem__(1, s[0]),
        "missing pick": lambda s: s.__setitem__(1, -1),
        "reorder without a tie": lambda s: s.__setitem__(slice(0, 2), s[[1, 0]]),
    }
    for name, plant in plants.items():
        sel = rt["sel"].copy()
        plant(sel[0, 0, r])
        res = oracle.check_selection(wl, Q, kbar, sel, rt, lay)
        assert res["mismatch"] == 1, name
        assert len(res["bad"]) == 1 and res["bad"][0]["row"] == t, (name, res["bad"])


def test_swap_of_exactly_tied_candidates_is_admissible():
    """Give two candidate chunks of a row identical pooled keys: their scores
    tie exactly, the oracle orders them by id, and the reversed order is a
    valid selection under the near-tie rule."""
    wl, Q, K, lay, kbar, rt = _routed()
    r = _row_with_full_selection(rt)
    a, b = (int(x) for x in rt["sel"][0, 0, r, :2])
    kbar2 = kbar.copy()
    kbar2[0, 0, b] = kbar2[0, 0, a]
    rt2 = oracle.route(wl, Q, kbar2, rows=rt["rows"], lay=lay)
    s = rt2["sel"][0, 0, r]
    assert set(s[:2].tolist()) == {a, b} and s[0] == min(a, b)
    sel = rt2["sel"].copy()
    sel[0, 0, r, :2] = sel[0, 0, r, [1, 0]]
    res = oracle.check_selection(wl, Q, kbar2, sel, rt2, lay)
    assert res["mismatch"] >= 1 and not res["bad"], res["bad"]
    assert res["near_tie_rows"] >= 1
