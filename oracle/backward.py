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
"""
from __future__ import annotations

import math

import numpy as np
import torch

ROLE_ANCHOR = 1


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


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
