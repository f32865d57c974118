"""The CTA-pair attention kernel (moc_set_attend_kernel(2): clusters of two
SMs sharing every MMA, items of 512 query rows) against the oracle, and its
schedule independence.

Same comparisons as test_gpu_parity.py (tolerances in tests/parity.py); the
kernel exists for bf16 with d = 128, so every scene here has d = 128.
"""
import contextlib

import numpy as np
import pytest
import torch

import chunk_routed_sparse_b200 as moc
import moc_workloads as W
import oracle
from parity import attend_reference, compare_attention, compare_routing, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


@contextlib.contextmanager
def attend_kernel(variant):
    moc.set_attend_kernel(variant)
    try:
        yield
    finally:
        moc.set_attend_kernel(0)


def _ragsmall(B=2, H=3, k=2, anchor="shot"):
    segs = [W.Segment(37, W.CAPTION, 0, -1)]
    for i, ln in enumerate([1, 64, 65, 127, 128, 129, 200, 3, 300, 17, 600, 513, 511]):
        segs.append(W.Segment(ln, W.VIDEO, i // 4, i % 4))
        if i == 3:
            segs.append(W.Segment(5, W.CAPTION, 1, -1))
    return W.custom("ragsmall", B, H, 128, segs, anchor, 0, True, k, 31, "frame")


def _check(wl, rows=None, n_random=0, seed=0, heads=None):
    Q, K, V = W.make_qkv(wl, heads=heads)
    orc = oracle.Layout(wl)
    if rows is None and n_random:
        rows = sample_rows(orc, n_random, seed)
    lay = moc.Layout.from_workload(wl)
    with attend_kernel(2):
        O, lse, sel, kbar = moc.forward(lay, Q.cuda(), K.cuda(), V.cuda(), wl.k, wl.causal)
        torch.cuda.synchronize()
    O, lse, sel, kbar = O.cpu(), lse.cpu(), sel.cpu().numpy(), kbar.cpu().numpy()
    heads = heads or [(b, h) for b in range(wl.B) for h in range(wl.H)]
    w1 = wl.replace(B=1, H=1)
    for b, h in heads:
        q, kk, v = (t[b:b + 1, h:h + 1].contiguous() for t in (Q, K, V))
        kbar_o = oracle.pool(w1, kk, orc)
        rt = oracle.route(w1, q, kbar_o, rows=rows, lay=orc)
        r = rt["rows"]
        sel_g = np.ascontiguousarray(sel[b:b + 1, h:h + 1][:, :, r, :])
        res = compare_routing(w1, q, kbar_o, sel_g, rt, orc)
        O_o, lse_o = attend_reference(w1, q, kk, v, rt["sel"], sel_g, r, orc, res)
        compare_attention(O[b:b + 1, h:h + 1][:, :, r], lse[b:b + 1, h:h + 1][:, :, r], O_o, lse_o)


def test_pair_kernel_rejects_other_head_dims():
    wl = W.tiny()  # d = 64
    Q, K, V = (t.cuda() for t in W.make_qkv(wl))
    lay = moc.Layout.from_workload(wl)
    with attend_kernel(2):
        with pytest.raises(RuntimeError):
            moc.forward(lay, Q, K, V, wl.k, wl.causal)
    torch.cuda.synchronize()


@pytest.mark.parametrize("k,anchor", [(0, "shot"), (2, "shot"), (5, "chunk"), (9, "shot")])
def test_small_ragged_scene_every_row(k, anchor):
    """Items of one row up to several 512-row items, pair tiles B present and
    absent, CTA 1 without rows, key ranges shorter than a tile."""
    _check(_ragsmall(k=k, anchor=anchor))


def test_largest_k_every_row():
    """k = 31: 32 partial slots a row; three shots of 16 sub-chunks of 20-140
    tokens (the last shot's queries pick 31 of 32 candidates)."""
    rng = np.random.default_rng(7)
    segs = []
    for s_ in range(3):
        segs.append(W.Segment(16, W.CAPTION, s_, -1))
        for f in range(16):
            segs.append(W.Segment(int(rng.integers(20, 141)), W.VIDEO, s_, f))
    _check(W.custom("manychunks", 1, 2, 128, segs, "shot", 0, True, 31, 33, "frame"))


def test_non_causal_scene_every_row():
    """Routing over earlier and later chunks: longer query lists per chunk."""
    wl = _ragsmall(k=4)
    _check(wl.replace(causal=False))


def test_odd_head_count_every_row():
    """B x H = 10 slices: items and clusters that do not divide evenly."""
    _check(_ragsmall(B=2, H=5, k=3))


def test_single_shot_clip_sampled():
    _check(W.single(), n_random=512, seed=3)


def test_eight_shot_scene_sampled_heads():
    wl = W.eight()
    _check(wl, n_random=384, seed=4, heads=[(0, 0), (0, 13), (0, 23)])


@pytest.mark.parametrize("k", [2, 16])
def test_ragged_scene_k(k):
    wl = W.ragged().with_k(k)
    _check(wl, n_random=256, seed=5, heads=[(0, 1), (0, 20)])


def test_stress_scene_two_heads():
    wl = W.stress()
    _check(wl, n_random=256, seed=6, heads=[(0, 2), (1, 17)])


def test_pair_kernel_is_bitwise_under_another_schedule_and_close_to_single_cta():
    """Full-size eight-shot forward on the pair kernel: 5 clusters taking the
    items in reversed order reproduce the default schedule bit for bit; the
    single-CTA kernel agrees within the parity tolerance."""
    wl = W.eight()
    g = torch.Generator(device="cuda").manual_seed(13)
    Q, K, V = (torch.randn(wl.B, wl.H, wl.L, wl.d, device="cuda", generator=g).to(torch.bfloat16)
               for _ in range(3))
    lay = moc.Layout.from_workload(wl)
    ws = moc.workspace(lay, wl.B, wl.H, wl.d, wl.k)
    with attend_kernel(2):
        O1, lse1, sel1, _ = moc.forward(lay, Q, K, V, wl.k, ws=ws)
        torch.cuda.synchronize()
        assert moc.check_device_error(ws) == 0
        try:
            moc.set_attend_schedule(10, reverse=True)
            ws.fill_(0x7F)
            O2, lse2, sel2, _ = moc.forward(lay, Q, K, V, wl.k, ws=ws)
            torch.cuda.synchronize()
        finally:
            moc.set_attend_schedule(0, reverse=False)
        assert moc.check_device_error(ws) == 0
    with attend_kernel(1):
        O3, lse3, sel3, _ = moc.forward(lay, Q, K, V, wl.k, ws=ws)
        torch.cuda.synchronize()
    assert torch.isfinite(O1.float()).all() and torch.isfinite(lse1).all()
    assert torch.equal(sel1, sel2) and torch.equal(sel1, sel3)
    assert torch.equal(O1.view(torch.int16), O2.view(torch.int16)) and torch.equal(lse1, lse2)
    d = (O1.float() - O3.float()).abs()
    assert d.max().item() <= 2e-2 and d.mean().item() <= 1e-4
    assert (lse1 - lse3).abs().max().item() <= 1e-3
