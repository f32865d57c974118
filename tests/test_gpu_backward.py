"""Parity of the backward pass (moc_attention_bwd, through the C ABI) with the
CPU oracle (oracle/backward.py, fp64, pinned against PyTorch autograd).

The selection is an input of the backward pass (routing is constant), so every
case feeds the oracle's own routing to both sides; O and lse come from the GPU
forward pass over that same selection, as in training.

Tolerances. The kernels round P and dS to bf16 (unit roundoff u = 2^-9) before
the dV / dQ / dK products, accumulate in fp32, and round the outputs to bf16
(u again). Rounding errors of independent terms add in quadrature, so the
relative error of a sum of many terms is about u when its terms do not
cancel, plus u from the output rounding: ~2u = 3.9e-3. dQ and dK sum
p (dp - D) terms whose weighted sum over a row is zero, so the relative error
there can be a few times larger. The bound per tensor is a relative Frobenius
error of REL_F = 2e-2 (about 5x the estimate) and a largest element error of
MAX_REL = 5e-2 of the tensor's largest reference magnitude.
"""
import numpy as np
import pytest
import torch

import chunk_routed_sparse_b200 as moc
import moc_workloads as W
import oracle
from oracle import backward as BW

pytestmark = pytest.mark.gpu

REL_F = 2e-2
MAX_REL = 5e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _close(name, got: np.ndarray, ref: np.ndarray):
    err = got - ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-30)
    mx = np.abs(err).max() / max(np.abs(ref).max(), 1e-30)
    assert rel <= REL_F and mx <= MAX_REL, f"{name}: relative Frobenius {rel:.3e}, max {mx:.3e}"
    return rel, mx


def _upstream(wl, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(wl.B, wl.H, wl.L, wl.d, generator=g).to(torch.bfloat16)


def _gpu_backward(wl, Q, K, V, dO, sel):
    lay = moc.Layout.from_workload(wl)
    Qd, Kd, Vd, Gd = (t.cuda() for t in (Q, K, V, dO))
    seld = torch.from_numpy(np.ascontiguousarray(sel, dtype=np.int32)).cuda()
    O, lse = moc.attention_fwd(lay, Qd, Kd, Vd, seld, wl.k)
    ws = torch.empty(int(moc.lib().moc_attention_bwd_workspace_bytes(lay.handle, wl.B, wl.H, wl.d, wl.k)),
                     dtype=torch.uint8, device="cuda")
    dQ, dK, dV = moc.attention_bwd(lay, Qd, Kd, Vd, O, lse, Gd, seld, wl.k, ws=ws)
    torch.cuda.synchronize()
    assert moc.check_device_error(ws) == 0
    return dQ.cpu().double().numpy(), dK.cpu().double().numpy(), dV.cpu().double().numpy(), ws


def _full_case(wl, seed=21):
    Q, K, V = W.make_qkv(wl)
    dO = _upstream(wl, seed)
    orc = oracle.Layout(wl)
    sel = oracle.route(wl, Q, oracle.pool(wl, K, orc), lay=orc)["sel"]
    gQ, gK, gV, _ = _gpu_backward(wl, Q, K, V, dO, sel)
    rQ, rK, rV = BW.backward(wl, orc, Q, K, V, sel, dO)
    return [_close(n, g, r) for n, g, r in (("dQ", gQ, rQ), ("dK", gK, rK), ("dV", gV, rV))]


def test_tiny_every_row_and_key():
    _full_case(W.tiny())


@pytest.mark.parametrize("anchor,radius,causal,k", [("chunk", 0, True, 1), ("local", 1, True, 3),
                                                    ("shot", 0, False, 2), ("shot", 0, True, 0)])
def test_tiny_anchor_modes(anchor, radius, causal, k):
    _full_case(W.tiny().replace(anchor=anchor, radius=radius, causal=causal).with_k(k))


def test_small_ragged_scene_d128():
    """Chunks shorter than a key tile and of every tail length, captions
    interleaved, d = 128: partial key tiles in both kernels, query lists
    shorter than a tile, a caption run as a key block."""
    segs = [W.Segment(37, W.CAPTION, 0, -1)]
    lens = [1, 64, 65, 127, 128, 129, 200, 3, 300, 17]
    for i, ln in enumerate(lens):
        segs.append(W.Segment(ln, W.VIDEO, i // 4, i % 4))
        if i == 3:
            segs.append(W.Segment(5, W.CAPTION, 1, -1))
    wl = W.custom("ragsmall", 2, 2, 128, segs, "shot", 0, True, 3, 31, "frame")
    _full_case(wl)


def test_largest_k_every_row_and_key():
    """k = 31 (the largest top-k): 32 partial dQ slots a row, 31 of them routed;
    three shots of 16 sub-chunks of 20-80 tokens, every row and key."""
    rng = np.random.default_rng(7)
    segs = []
    for s_ in range(3):
        segs.append(W.Segment(16, W.CAPTION, s_, -1))
        for f in range(16):
            segs.append(W.Segment(int(rng.integers(20, 81)), W.VIDEO, s_, f))
    _full_case(W.custom("manychunks", 1, 2, 128, segs, "shot", 0, True, 31, 33, "frame"))


def test_backward_is_deterministic():
    wl = W.tiny()
    Q, K, V = W.make_qkv(wl)
    dO = _upstream(wl, 3)
    orc = oracle.Layout(wl)
    sel = oracle.route(wl, Q, oracle.pool(wl, K, orc), lay=orc)["sel"]
    a = _gpu_backward(wl, Q, K, V, dO, sel)
    b = _gpu_backward(wl, Q, K, V, dO, sel)
    for x, y in zip(a[:3], b[:3]):
        assert np.array_equal(x, y)


def test_eight_shot_sampled_rows_and_chunks():
    """The full 180k-token eight-shot scene (24 heads computed): dQ on
    boundary + random rows of two heads, dK / dV of whole chunks - a video
    chunk of the first shot (selected by many later queries), one of the last
    shot, and the caption run (attended by every query) - against the oracle."""
    wl = W.eight()
    Q, K, V = W.make_qkv(wl)
    dO = _upstream(wl, 8)
    orc = oracle.Layout(wl)
    heads = [(0, 0), (0, 17)]
    sel = np.zeros((wl.B, wl.H, wl.L, wl.k), dtype=np.int32)
    for b, h in heads:
        w1 = wl.replace(B=1, H=1)
        q, kk = (t[b:b + 1, h:h + 1].contiguous() for t in (Q, K))
        sel[b, h] = oracle.route(w1, q, oracle.pool(w1, kk, orc), lay=orc)["sel"][0, 0]
    # the other heads route on the GPU (their inputs are seeded noise too)
    lay = moc.Layout.from_workload(wl)
    Qd, Kd = Q.cuda(), K.cuda()
    sel_gpu = moc.route(lay, Qd, moc.pool_keys(lay, Kd), wl.k).cpu().numpy()
    for b in range(wl.B):
        for h in range(wl.H):
            if (b, h) not in heads:
                sel[b, h] = sel_gpu[b, h]
    del Qd, Kd
    gQ, gK, gV, _ = _gpu_backward(wl, Q, K, V, dO, sel)
    rng = np.random.default_rng(4)
    rows = np.unique(np.concatenate([[0, 511, 512, 513, 1500 * 7 + 512, wl.L - 1],
                                     rng.integers(0, wl.L, size=48)]))
    for b, h in heads:
        w1 = wl.replace(B=1, H=1)
        q, kk, v, g = (t[b:b + 1, h:h + 1].contiguous() for t in (Q, K, V, dO))
        s1 = np.ascontiguousarray(sel[b:b + 1, h:h + 1])
        rq = BW.backward_rows(w1, orc, q, kk, v, s1, g, rows)
        _close(f"dQ rows head {h}", gQ[b:b + 1, h:h + 1, rows], rq)
    for b, h, c in [(0, 0, 8 + 3), (0, 17, 8 + 7 * 15 + 9), (0, 0, 0)]:
        w1 = wl.replace(B=1, H=1)
        q, kk, v, g = (t[b:b + 1, h:h + 1].contiguous() for t in (Q, K, V, dO))
        s1 = np.ascontiguousarray(sel[b:b + 1, h:h + 1])
        dk, dvv = BW.backward_keys(w1, orc, q, kk, v, s1, g, 0, 0, c)
        u = slice(orc.off[c], orc.off[c + 1])
        _close(f"dK chunk {c} head {h}", gK[b, h, u], dk)
        _close(f"dV chunk {c} head {h}", gV[b, h, u], dvv)
