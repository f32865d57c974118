"""Backward pass of MoC attention (dQ, dK, dV) - TEST INFRASTRUCTURE (oracle).

Only the tests may import this module. NumPy, fp64, one query row at a time;
it shares nothing with the CUDA library.

What it computes ("Mixture of Contexts for Long Video Generation | Summary":
§3.1 attention over Omega(q_i) = the anchors and the selected chunks; the
training notes: the top-k choice is discrete and not differentiated, the model
adapts through the gradients of attention over the selected keys and values):
with the selection held fixed, each query row's output
    o_t = sum_{u in Omega(t)} p_u v_u,  p = softmax_u(scale * q_t . k_u)
is differentiated for an upstream gradient dO:
    dv_u += p_u dO_t,  dp_u = dO_t . v_u,  D_t = dO_t . o_t,
    ds_u = p_u (dp_u - D_t),  dq_t = scale * sum_u ds_u k_u,  dk_u += scale * ds_u q_t.
Readings (stated in the design notes): routing is constant (no gradient through
the top-k); the pooled keys feed only the routing, so no gradient flows
through the pooling; the loss depends on O only (no upstream gradient on lse).

``backward`` differentiates every row of every head; ``backward_rows`` gives
dQ of chosen query rows and ``backward_keys`` dK, dV of one chosen chunk's
keys (the sums over the queries whose Omega holds them), so that large scenes
can be checked on samples. ``backward_keys`` takes each attending query's o_t
and lse_t from the oracle's own forward (``oracle.attend``, fp64).
"""
from __future__ import annotations

import math

import numpy as np
import torch

ROLE_ANCHOR = 1


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


def _omega(lay, qc, sel_row, cache):
    """Token indices of Omega(t) for a query of chunk qc selecting sel_row."""
    if qc not in cache:
        chunks = np.nonzero(lay.role[qc] == ROLE_ANCHOR)[0]
        cache[qc] = np.concatenate([np.arange(lay.off[c], lay.off[c + 1]) for c in chunks])
    extra = [np.arange(lay.off[c], lay.off[c + 1]) for c in sel_row if c >= 0]
    return np.concatenate([cache[qc]] + extra) if extra else cache[qc]


def backward_rows(wl, lay, Q, K, V, sel: np.ndarray, dO, rows, scale=None):
    """dQ (fp64 [B, H, len(rows), d]) of the given query rows; sel is the
    full selection [B, H, L, k]."""
    scale = 1.0 / math.sqrt(wl.d) if scale is None else scale
    Qf, Kf, Vf, Gf = _f64(Q), _f64(K), _f64(V), _f64(dO) if isinstance(dO, torch.Tensor) else dO
    rows = np.asarray(rows, dtype=np.int64)
    dQ = np.zeros((wl.B, wl.H, len(rows), wl.d))
    cache = {}
    for b in range(wl.B):
        for h in range(wl.H):
            for i, t in enumerate(rows):
                om = _omega(lay, int(lay.chunk_of_token[t]), sel[b, h, t], cache)
                q, g = Qf[b, h, t], Gf[b, h, t]
                kk, vv = Kf[b, h, om], Vf[b, h, om]
                s = scale * (kk @ q)
                p = np.exp(s - s.max())
                p /= p.sum()
                o = p @ vv
                ds = p * (vv @ g - g @ o)
                dQ[b, h, i] = scale * (ds @ kk)
    return dQ


def backward_keys(wl, lay, Q, K, V, sel: np.ndarray, dO, b: int, h: int, chunk: int, scale=None):
    """dK, dV (fp64 [n_c, d]) of the keys of ``chunk`` in head (b, h): sums
    over every query t whose Omega(t) holds the chunk (as an anchor, or as a
    selected chunk), with p_tu = exp(scale q_t . k_u - lse_t) and
    D_t = dO_t . o_t from the oracle's forward of those rows."""
    from . import attend

    scale = 1.0 / math.sqrt(wl.d) if scale is None else scale
    anchored = lay.role[lay.chunk_of_token, chunk] == ROLE_ANCHOR
    chosen = np.any(sel[b, h] == chunk, axis=-1) if sel.shape[-1] else np.zeros(lay.L, dtype=bool)
    rows = np.nonzero(anchored | chosen)[0]
    w1 = wl.replace(B=1, H=1)
    q1, k1, v1 = (t[b:b + 1, h:h + 1].contiguous() for t in (Q, K, V))
    O, lse, _ = attend(w1, q1, k1, v1, np.ascontiguousarray(sel[b:b + 1, h:h + 1, rows]), rows=rows, lay=lay)
    O, lse = O[0, 0], lse[0, 0]
    Qa, Ga = _f64(Q)[b, h, rows], (_f64(dO) if isinstance(dO, torch.Tensor) else dO)[b, h, rows]
    u = np.arange(lay.off[chunk], lay.off[chunk + 1])
    Kc, Vc = _f64(K)[b, h, u], _f64(V)[b, h, u]
    P = np.exp(scale * (Qa @ Kc.T) - lse[:, None])
    D = np.sum(Ga * O, axis=1)
    dS = P * (Ga @ Vc.T - D[:, None])
    return scale * (dS.T @ Qa), P.T @ Ga


def backward(wl, lay, Q, K, V, sel: np.ndarray, dO, scale=None):
    """dQ, dK, dV (fp64 [B, H, L, d]) for selections sel [B, H, L, k] (-1 padded)
    on every row; lay is an oracle.Layout of wl."""
    scale = 1.0 / math.sqrt(wl.d) if scale is None else scale
    Qf, Kf, Vf, Gf = _f64(Q), _f64(K), _f64(V), _f64(dO) if isinstance(dO, torch.Tensor) else dO
    dQ = np.zeros_like(Qf)
    dK = np.zeros_like(Kf)
    dV = np.zeros_like(Vf)
    anchor_tok = {}
    for b in range(wl.B):
        for h in range(wl.H):
            for t in range(lay.L):
                qc = int(lay.chunk_of_token[t])
                if qc not in anchor_tok:
                    chunks = np.nonzero(lay.role[qc] == ROLE_ANCHOR)[0]
                    anchor_tok[qc] = np.concatenate([np.arange(lay.off[c], lay.off[c + 1]) for c in chunks])
                extra = [np.arange(lay.off[c], lay.off[c + 1]) for c in sel[b, h, t] if c >= 0]
                om = np.concatenate([anchor_tok[qc]] + extra) if extra else anchor_tok[qc]
                q, g = Qf[b, h, t], Gf[b, h, t]
                kk, vv = Kf[b, h, om], Vf[b, h, om]
                s = scale * (kk @ q)
                p = np.exp(s - s.max())
                p /= p.sum()
                o = p @ vv
                dV[b, h, om] += np.outer(p, g)
                dp = vv @ g
                ds = p * (dp - g @ o)
                dQ[b, h, t] = scale * (ds @ kk)
                dK[b, h, om] += scale * np.outer(ds, q)
    return dQ, dK, dV
