"""CPU oracle for the Mixture of Contexts (MoC) forward pass - TEST INFRASTRUCTURE.

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package. It wraps ``libmoc_oracle.so`` (plain C, fp64, built
from ``moc_oracle.c`` by ``oracle/build.py``) with ctypes and shares nothing
with the CUDA library. ``oracle.bruteforce`` holds an even plainer NumPy
restatement (dense L x L masks) used to pin this one on tiny inputs.

Pages followed (see the header of ``moc_oracle.c`` for the full statement):
"Mixture of Contexts for Long Video Generation | Summary" §3.1-§3.3 and the
jxzklqfsx.com MoC write-up, section "計算效率".
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import numpy as np
import torch

from . import build as _build

_ANCHOR = {"shot": 0, "local": 1, "chunk": 2}
ROLE_NONE, ROLE_ANCHOR, ROLE_CAND = 0, 1, 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i64, i32, vp, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_double
        L.moc_oracle_threads.restype = i32
        L.moc_oracle_roles.argtypes = [i32, vp, vp, vp, i32, i32, i32, vp]
        L.moc_oracle_roles.restype = i32
        L.moc_oracle_pool.argtypes = [i64, i64, i32, vp, i32, vp, vp]
        L.moc_oracle_route.argtypes = [i64, i64, i32, vp, i32, vp, vp, vp, i32, i64, vp, vp, vp,
                                       vp, vp, vp]
        L.moc_oracle_scores.argtypes = [i64, i64, i32, vp, i32, vp, i64, vp, vp, vp, vp, vp]
        L.moc_oracle_attend.argtypes = [i64, i64, i32, vp, vp, vp, i32, vp, vp, i32, vp, dbl, i64,
                                        vp, vp, vp, vp]
        L.moc_oracle_kept_pairs.argtypes = [i64, i32, vp, vp, i32, vp]
        L.moc_oracle_kept_pairs.restype = i64
        _lib = L
    return _lib


def threads() -> int:
    return lib().moc_oracle_threads()


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> contiguous uint16 NumPy view of its bit patterns."""
    assert t.dtype == torch.bfloat16 and t.device.type == "cpu"
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


class Layout:
    """The oracle's own view of a workload's chunking: offsets and roles."""

    def __init__(self, wl):
        ln, kind, shot, frame = wl.seg_arrays()
        self.C = len(ln)
        self.off = np.zeros(self.C + 1, dtype=np.int64)
        self.off[1:] = np.cumsum(np.asarray(ln, dtype=np.int64))
        self.L = int(self.off[-1])
        self.kind = np.asarray(kind, dtype=np.int32)
        self.shot = np.asarray(shot, dtype=np.int32)
        self.frame = np.asarray(frame, dtype=np.int32)
        self.role = np.zeros((self.C, self.C), dtype=np.uint8)
        rc = lib().moc_oracle_roles(self.C, _p(self.kind), _p(self.shot), _p(self.frame),
                                    _ANCHOR[wl.anchor], wl.radius, int(wl.causal), _p(self.role))
        if rc != 0:
            raise ValueError("bad anchor mode")
        self.chunk_of_token = np.repeat(np.arange(self.C), np.diff(self.off))


def pool(wl, K: torch.Tensor, lay: Optional[Layout] = None) -> np.ndarray:
    """Mean-pooled keys Kbar[B, H, C, d] (fp64)."""
    lay = lay or Layout(wl)
    Kb = _bits(K)
    BH = wl.B * wl.H
    out = np.zeros((wl.B, wl.H, lay.C, wl.d), dtype=np.float64)
    lib().moc_oracle_pool(BH, lay.L, wl.d, _p(Kb), lay.C, _p(lay.off), _p(out))
    return out


def _rows(lay: Layout, rows) -> np.ndarray:
    if rows is None:
        return np.arange(lay.L, dtype=np.int64)
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64))


def route(wl, Q: torch.Tensor, Kbar: np.ndarray, rows=None, k: Optional[int] = None,
          lay: Optional[Layout] = None) -> dict:
    """Top-k routing of the given query rows (all rows by default) of every head.

    Returns a dict of arrays shaped [B, H, nrows, ...]: sel (int32, -1 padded),
    ncand, top_s / top_a / top_j (the first k+1 entries of the sorted
    candidate list: score, |q|.|Kbar| magnitude, chunk id)."""
    lay = lay or Layout(wl)
    k = wl.k if k is None else k
    r = _rows(lay, rows)
    BH, n = wl.B * wl.H, len(r)
    Qb = _bits(Q)
    Kbar = np.ascontiguousarray(Kbar, dtype=np.float64)
    sel = np.zeros((BH, n, max(k, 1)), dtype=np.int32)[..., :k].copy()
    ncand = np.zeros((BH, n), dtype=np.int32)
    ts = np.zeros((BH, n, k + 1))
    ta = np.zeros((BH, n, k + 1))
    tj = np.zeros((BH, n, k + 1), dtype=np.int32)
    lib().moc_oracle_route(BH, lay.L, wl.d, _p(Qb), lay.C, _p(lay.off), _p(lay.role), _p(Kbar),
                           k, n, _p(r), _p(sel), _p(ncand), _p(ts), _p(ta), _p(tj))
    shp = (wl.B, wl.H, n)
    return {"sel": sel.reshape(shp + (k,)), "ncand": ncand.reshape(shp),
            "top_s": ts.reshape(shp + (k + 1,)), "top_a": ta.reshape(shp + (k + 1,)),
            "top_j": tj.reshape(shp + (k + 1,)), "rows": r}


def scores(wl, Q: torch.Tensor, Kbar: np.ndarray, bh, tok, chunk, lay: Optional[Layout] = None):
    """Router score and magnitude for arbitrary (b*H+h, token, chunk) triples."""
    lay = lay or Layout(wl)
    bh = np.ascontiguousarray(np.asarray(bh, dtype=np.int64))
    tok = np.ascontiguousarray(np.asarray(tok, dtype=np.int64))
    ch = np.ascontiguousarray(np.asarray(chunk, dtype=np.int32))
    s = np.zeros(len(bh))
    a = np.zeros(len(bh))
    lib().moc_oracle_scores(wl.B * wl.H, lay.L, wl.d, _p(_bits(Q)), lay.C,
                            _p(np.ascontiguousarray(Kbar, dtype=np.float64)), len(bh), _p(bh),
                            _p(tok), _p(ch), _p(s), _p(a))
    return s, a


def attend(wl, Q, K, V, sel: np.ndarray, rows=None, scale: Optional[float] = None,
           lay: Optional[Layout] = None):
    """Softmax attention over Omega(t) for the given rows; sel is [B, H, nrows, k].

    Returns (O [B,H,nrows,d] fp64, lse [B,H,nrows] fp64, nkeys [B,H,nrows])."""
    lay = lay or Layout(wl)
    r = _rows(lay, rows)
    BH, n = wl.B * wl.H, len(r)
    k = sel.shape[-1]
    scale = 1.0 / math.sqrt(wl.d) if scale is None else scale
    sel = np.ascontiguousarray(sel, dtype=np.int32).reshape(BH, n, k)
    O = np.zeros((BH, n, wl.d))
    lse = np.zeros((BH, n))
    nk = np.zeros((BH, n), dtype=np.int64)
    lib().moc_oracle_attend(BH, lay.L, wl.d, _p(_bits(Q)), _p(_bits(K)), _p(_bits(V)), lay.C,
                            _p(lay.off), _p(lay.role), k, _p(sel), float(scale), n, _p(r), _p(O),
                            _p(lse), _p(nk))
    return (O.reshape(wl.B, wl.H, n, wl.d), lse.reshape(wl.B, wl.H, n),
            nk.reshape(wl.B, wl.H, n))


def forward(wl, Q, K, V, rows=None, lay: Optional[Layout] = None) -> dict:
    """Pool -> route -> attend for the given rows of every head."""
    lay = lay or Layout(wl)
    kbar = pool(wl, K, lay)
    rt = route(wl, Q, kbar, rows=rows, lay=lay)
    O, lse, nk = attend(wl, Q, K, V, rt["sel"], rows=rt["rows"], lay=lay)
    rt.update({"kbar": kbar, "O": O, "lse": lse, "nkeys": nk})
    return rt


def kept_pairs(wl, sel_head: np.ndarray, lay: Optional[Layout] = None) -> int:
    """Kept (query, key) pairs of one head: sum over all tokens of |Omega(t)|.
    ``sel_head`` is that head's full selection [L, k]."""
    lay = lay or Layout(wl)
    s = np.ascontiguousarray(sel_head, dtype=np.int32)
    return int(lib().moc_oracle_kept_pairs(lay.L, lay.C, _p(lay.off), _p(lay.role), s.shape[-1],
                                           _p(s)))


# Near-tie rule for comparing a selection computed in lower precision with this
# fp64 one: the gap between two adjacent entries of the sorted candidate list
# is "near" when it is below 1e-4 of the larger magnitude of the two scores, or
# below 1e-5 of the larger |q|.|Kbar| magnitude sum (the latter guards scores
# that cancel to near zero, where a relative test on the score alone is
# meaningless for an fp32 computation).
REL_TIE = 1e-4
MAG_TIE = 1e-5


def is_near(s1, s2, a1, a2):
    gap = np.abs(np.asarray(s1) - np.asarray(s2))
    return (gap < REL_TIE * np.maximum(np.abs(s1), np.abs(s2))) | \
           (gap < MAG_TIE * np.maximum(a1, a2))


def check_selection(wl, Q: torch.Tensor, Kbar: np.ndarray, sel_other: np.ndarray, rt: dict,
                    lay: Optional[Layout] = None) -> dict:
    """Classify a selection computed elsewhere (in lower precision) against this
    oracle's routing ``rt`` of the same rows (``route``): sel_other is
    [B, H, nrows, k]. A row is exact when it equals the oracle's selection. A
    differing row is admissible only when all of these hold:
      - the oracle flags the row as near-tied (``near_tie_flags``);
      - every pick is a routing candidate of the query's chunk (role CAND in the
        oracle's own role table: never a mandatory or caption chunk, never a
        chunk the causal mask hides), with no repeats and the same number of
        -1 pads as the oracle;
      - position by position, the pick's fp64 score equals or is near the
        oracle's sorted score there, and the picks are in non-increasing score
        order up to near ties.
    Returns counts and the (b, h, r) indices of the mismatched and of the
    inadmissible rows, with a reason for each inadmissible one."""
    lay = lay or Layout(wl)
    sel_o = rt["sel"]
    k = sel_o.shape[-1]
    out = {"rows": int(np.prod(sel_o.shape[:3])), "exact": 0, "mismatch": 0, "near_tie_rows": 0,
           "mismatch_rows": [], "bad": []}
    if k == 0:
        out["exact"] = out["rows"]
        return out
    flags = near_tie_flags(rt)
    near = flags["boundary"] | flags["inner"]
    eq = np.all(sel_o == sel_other, axis=-1)
    out["exact"] = int(eq.sum())
    out["near_tie_rows"] = int(near.sum())
    mism = [tuple(int(x) for x in m) for m in np.argwhere(~eq)]
    out["mismatch"] = len(mism)
    out["mismatch_rows"] = mism
    for b, h, r in mism:
        t = int(rt["rows"][r])
        g, o = sel_other[b, h, r], sel_o[b, h, r]
        gv = g[g >= 0]
        why = None
        if not near[b, h, r]:
            why = "no near tie"
        elif (g < 0).sum() != (o < 0).sum():
            why = "different number of picks"
        elif len(set(gv.tolist())) != len(gv):
            why = "repeated pick"
        elif np.any(gv >= lay.C) or np.any(lay.role[lay.chunk_of_token[t], gv] != ROLE_CAND):
            why = "pick is not a routing candidate of the query"
        else:
            bh = b * wl.H + h
            s, a = scores(wl, Q, Kbar, [bh] * len(gv), [t] * len(gv), gv, lay)
            so, ao = rt["top_s"][b, h, r, :len(gv)], rt["top_a"][b, h, r, :len(gv)]
            for x in range(len(gv)):
                if not (s[x] == so[x] or is_near(s[x], so[x], a[x], ao[x])):
                    why = f"score at position {x} not near the oracle's"
                    break
                if x + 1 < len(gv) and not (s[x] >= s[x + 1] or is_near(s[x], s[x + 1], a[x], a[x + 1])):
                    why = f"positions {x}, {x + 1} out of order"
                    break
        if why is not None:
            out["bad"].append({"b": b, "h": h, "row": t, "why": why, "sel": g.tolist(),
                               "oracle": o.tolist()})
    return out


def near_tie_flags(rt: dict) -> dict:
    """Per row: 'boundary' = k-th and (k+1)-th candidates near-tied;
    'inner' = two adjacent selected entries near-tied (their order may swap)."""
    ts, ta = rt["top_s"], rt["top_a"]
    k = ts.shape[-1] - 1
    with np.errstate(invalid="ignore"):
        if k >= 1:
            b = is_near(ts[..., k - 1], ts[..., k], ta[..., k - 1], ta[..., k])
            b = b & ~np.isnan(ts[..., k])
        else:
            b = np.zeros(ts.shape[:-1], dtype=bool)
        inner = np.zeros(ts.shape[:-1], dtype=bool)
        for x in range(max(k - 1, 0)):
            nn = is_near(ts[..., x], ts[..., x + 1], ta[..., x], ta[..., x + 1])
            inner |= nn & ~np.isnan(ts[..., x + 1])
    return {"boundary": b, "inner": inner}
