"""Brute-force NumPy restatement of MoC attention for tiny inputs - TEST INFRASTRUCTURE.

A second, deliberately different restatement used to pin the C oracle: it
builds the full L x L boolean mask token by token from the definition, routes
with Python's ``sorted`` over every candidate, and runs dense masked softmax
attention with NumPy matrix products, all in fp64. Quadratic in L: tiny
inputs only. It calls nothing in ``moc_oracle.c``.

Definition followed ("Mixture of Contexts for Long Video Generation | Summary"
§3.1-§3.2; jxzklqfsx.com MoC write-up, "計算效率"): a caption query sees every
token; a video query sees every caption token, its mandatory video chunks
(own shot / frame window / own chunk) and the top-k of its candidate chunks,
ranked by q . mean(K over the chunk) with ties to the lower chunk index;
candidates are the non-mandatory video chunks, restricted to earlier chunks
when the causal mask is on.
"""
from __future__ import annotations

import math

import numpy as np
import torch


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


def segments_table(wl):
    """Per token: (chunk index, kind, shot, frame)."""
    rows = []
    for c, s in enumerate(wl.segments):
        rows += [(c, s.kind, s.shot, s.frame)] * s.length
    return rows


def mandatory(wl, qt, kt) -> bool:
    """Is key token ``kt`` mandatory for query token ``qt``? (tuples from segments_table)"""
    qc, qkind, qshot, qframe = qt
    kc, kkind, kshot, kframe = kt
    if qkind == 0 or kkind == 0:        # caption query, or caption key
        return True
    if wl.anchor == "shot":
        return kshot == qshot
    if wl.anchor == "local":
        return kshot == qshot and abs(kframe - qframe) <= wl.radius
    return kc == qc


def candidates(wl, qt):
    """Video chunks a video query may route to, in chunk-id order."""
    tab = {}
    for c, s in enumerate(wl.segments):
        tab[c] = (c, s.kind, s.shot, s.frame)
    out = []
    for c, kt in tab.items():
        if kt[1] == 0 or mandatory(wl, qt, kt):
            continue
        if wl.causal and not (c < qt[0]):
            continue
        out.append(c)
    return out


def forward(wl, Q, K, V, k=None, scale=None):
    """Return (O [B,H,L,d], lse [B,H,L], sel list-of-lists per (b,h,t), mask [L,L] of b=h=0)."""
    k = wl.k if k is None else k
    scale = 1.0 / math.sqrt(wl.d) if scale is None else scale
    toks = segments_table(wl)
    L = len(toks)
    starts = np.cumsum([0] + [s.length for s in wl.segments])
    Qf, Kf, Vf = _f64(Q), _f64(K), _f64(V)
    B, H, d = wl.B, wl.H, wl.d
    O = np.zeros((B, H, L, d))
    lse = np.zeros((B, H, L))
    sels = {}
    mask0 = None
    cand_of = {}
    for b in range(B):
        for h in range(H):
            kbar = [Kf[b, h, starts[c]:starts[c + 1]].mean(axis=0) for c in range(len(wl.segments))]
            mask = np.zeros((L, L), dtype=bool)
            # mandatory links depend only on the two tokens' segments: fill per block
            for qc in range(len(wl.segments)):
                for kc in range(len(wl.segments)):
                    if mandatory(wl, toks[starts[qc]], toks[starts[kc]]):
                        mask[starts[qc]:starts[qc + 1], starts[kc]:starts[kc + 1]] = True
            for t in range(L):
                qt = toks[t]
                if qt[1] == 0:
                    sel = []
                else:
                    key = (qt[0],)
                    if key not in cand_of:
                        cand_of[key] = candidates(wl, qt)
                    cand = cand_of[key]
                    scored = [(-float(Qf[b, h, t] @ kbar[c]), c) for c in cand]
                    sel = [c for _, c in sorted(scored)[:k]]
                    for c in sel:
                        mask[t, starts[c]:starts[c + 1]] = True
                sels[(b, h, t)] = sel
            s = (Qf[b, h] @ Kf[b, h].T) * scale
            s = np.where(mask, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            w = np.exp(s - m)
            z = w.sum(axis=1, keepdims=True)
            O[b, h] = (w / z) @ Vf[b, h]
            lse[b, h] = (m + np.log(z))[:, 0]
            if b == 0 and h == 0:
                mask0 = mask
    return O, lse, sels, mask0
