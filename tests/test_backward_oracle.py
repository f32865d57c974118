"""Pins of the backward oracle (oracle/backward.py) against PyTorch autograd:
on the dense masked formulation whose mask the brute force builds token by
token (its own routing), and, with the causal mask off and every chunk
selected, against autograd through torch's scaled_dot_product_attention."""
import math

import numpy as np
import pytest
import torch

import moc_workloads as W
import oracle
from oracle import backward as BW
from oracle import bruteforce as BF


def _grad_case(wl, seed):
    Q, K, V = W.make_qkv(wl)
    g = torch.Generator().manual_seed(seed)
    dO = torch.randn(wl.B, wl.H, wl.L, wl.d, generator=g, dtype=torch.float64)
    return Q, K, V, dO


@pytest.mark.parametrize("anchor,causal,k", [("shot", True, 2), ("local", True, 1), ("chunk", False, 3),
                                             ("shot", False, 0)])
def test_matches_autograd_on_the_masked_dense_formulation(anchor, causal, k):
    wl = W.tiny().replace(anchor=anchor, radius=1, causal=causal, H=1).with_k(k)
    Q, K, V, dO = _grad_case(wl, 3)
    lay = oracle.Layout(wl)
    kbar = oracle.pool(wl, K, lay)
    sel = oracle.route(wl, Q, kbar, lay=lay)["sel"]
    dQ, dK, dV = BW.backward(wl, lay, Q, K, V, sel, dO)
    _, _, _, mask = BF.forward(wl, Q, K, V)        # the brute force's own routing and mask
    q, kk, v = (t[0, 0].double().requires_grad_(True) for t in (Q, K, V))
    s = (q @ kk.T) / math.sqrt(wl.d)
    s = s.masked_fill(~torch.from_numpy(mask), float("-inf"))
    o = torch.softmax(s, dim=-1) @ v
    o.backward(dO[0, 0])
    for mine, ref in ((dQ, q.grad), (dK, kk.grad), (dV, v.grad)):
        np.testing.assert_allclose(mine[0, 0], ref.numpy(), rtol=0, atol=1e-10)


def test_dense_case_matches_sdpa_autograd():
    """Causal off and k >= every candidate count: Omega is every token."""
    wl = W.tiny().replace(causal=False, H=2).with_k(30)
    Q, K, V, dO = _grad_case(wl, 4)
    lay = oracle.Layout(wl)
    kbar = oracle.pool(wl, K, lay)
    sel = oracle.route(wl, Q, kbar, lay=lay)["sel"]
    dQ, dK, dV = BW.backward(wl, lay, Q, K, V, sel, dO)
    q, kk, v = (t.double().requires_grad_(True) for t in (Q, K, V))
    o = torch.nn.functional.scaled_dot_product_attention(q, kk, v)
    o.backward(dO)
    for mine, ref in ((dQ, q.grad), (dK, kk.grad), (dV, v.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=0, atol=1e-10)


def test_value_gradient_sums_to_upstream():
    """Softmax weights sum to one, so the value gradients of a row's keys sum to
    its upstream gradient: sum over keys of dV equals sum over queries of dO."""
    wl = W.tiny().replace(H=1)
    Q, K, V, dO = _grad_case(wl, 5)
    lay = oracle.Layout(wl)
    sel = oracle.route(wl, Q, oracle.pool(wl, K, lay), lay=lay)["sel"]
    _, _, dV = BW.backward(wl, lay, Q, K, V, sel, dO)
    np.testing.assert_allclose(dV.sum(axis=2), dO.numpy().sum(axis=2), rtol=0, atol=1e-9)


@pytest.mark.parametrize("anchor,causal,k", [("shot", True, 2), ("local", True, 1), ("chunk", False, 3)])
def test_row_and_key_samples_match_the_full_backward(anchor, causal, k):
    """backward_rows and backward_keys (the sampled forms used on large scenes)
    equal the full backward on the rows / keys they cover, for every chunk
    kind: caption chunks (attended by every query), and video chunks attended
    as anchors and as selections."""
    wl = W.tiny().replace(anchor=anchor, radius=1, causal=causal, H=2).with_k(k)
    Q, K, V, dO = _grad_case(wl, 6)
    lay = oracle.Layout(wl)
    sel = oracle.route(wl, Q, oracle.pool(wl, K, lay), lay=lay)["sel"]
    dQ, dK, dV = BW.backward(wl, lay, Q, K, V, sel, dO)
    rows = np.array([0, 63, 64, 300, 1111, wl.L - 1])
    np.testing.assert_allclose(BW.backward_rows(wl, lay, Q, K, V, sel, dO, rows), dQ[:, :, rows],
                               rtol=0, atol=1e-10)
    for b, h, c in [(0, 0, 0), (0, 1, 2), (0, 0, 5), (0, 1, lay.C - 1)]:
        dk, dv = BW.backward_keys(wl, lay, Q, K, V, sel, dO, b, h, c)
        u = slice(lay.off[c], lay.off[c + 1])
        np.testing.assert_allclose(dk, dK[b, h, u], rtol=0, atol=1e-10)
        np.testing.assert_allclose(dv, dV[b, h, u], rtol=0, atol=1e-10)
