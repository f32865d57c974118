"""Parity of the CUDA path (called through the C ABI) with the CPU oracle.

Inputs are the seeded synthetic workloads of ``moc_workloads``; the same CPU
bytes feed the oracle and the GPU. Tolerances are in ``tests/parity.py``.
"""
import ctypes
import math
import time

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


def _run(wl, Q, K, V, k=None, causal=None):
    k = wl.k if k is None else k
    causal = wl.causal if causal is None else causal
    lay = moc.Layout.from_workload(wl)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    O, lse, sel, kbar = moc.forward(lay, Qd, Kd, Vd, k, causal)
    torch.cuda.synchronize()
    return lay, O.cpu(), lse.cpu(), sel.cpu().numpy(), kbar.cpu().numpy()


def _check_full(wl, rows=None, k=None, n_random=0, seed=0, heads=None):
    """Run the GPU forward on the whole problem, then check pool, routing and
    attention of every (b, h) in ``heads`` (default: all) against the oracle,
    on ``rows`` (None: every row; n_random > 0: boundary + random rows)."""
    k = wl.k if k is None else k
    wl = wl.with_k(k)
    Q, K, V = W.make_qkv(wl, heads=heads)
    orc = oracle.Layout(wl)
    if rows is None and n_random:
        rows = sample_rows(orc, n_random, seed)
    lay, O, lse, sel, kbar = _run(wl, Q, K, V)
    heads = heads or [(b, h) for b in range(wl.B) for h in range(wl.H)]
    w1 = wl.replace(B=1, H=1)
    tot = {"exact": 0, "mismatch": 0, "near": 0, "max_abs": 0.0, "mean_abs": 0.0}
    for b, h in heads:
        q, kk, v = (t[b:b + 1, h:h + 1].contiguous() for t in (Q, K, V))
        kbar_o = oracle.pool(w1, kk, orc)
        np.testing.assert_allclose(kbar[b:b + 1, h:h + 1], kbar_o, rtol=0, atol=2e-5)
        rt = oracle.route(w1, q, kbar_o, rows=rows, lay=orc)
        r = rt["rows"]
        sel_g = np.ascontiguousarray(sel[b:b + 1, h:h + 1][:, :, r, :])
        res = compare_routing(w1, q, kbar_o, sel_g, rt, orc)
        O_o, lse_o = attend_reference(w1, q, kk, v, rt["sel"], sel_g, r, orc, res)
        mx, mean = compare_attention(O[b:b + 1, h:h + 1][:, :, r], lse[b:b + 1, h:h + 1][:, :, r],
                                     O_o, lse_o)
        tot["exact"] += res["exact"]
        tot["mismatch"] += res["mismatch"]
        tot["near"] += res["near_tie_rows"]
        tot["max_abs"] = max(tot["max_abs"], mx)
        tot["mean_abs"] = max(tot["mean_abs"], mean)
    return tot


def test_tiny_all_rows():
    res = _check_full(W.tiny())
    assert res["mismatch"] == 0


def _many_chunk_scene(d: int, k: int):
    """Three shots of 16 sub-chunks (20-140 tokens each) with a 16-token caption
    before each shot: queries of the last shot have 32 routing candidates."""
    rng = np.random.default_rng(7)
    segs = []
    for s_ in range(3):
        segs.append(W.Segment(16, W.CAPTION, s_, -1))
        for f in range(16):
            segs.append(W.Segment(int(rng.integers(20, 141)), W.VIDEO, s_, f))
    return W.custom("manychunks", 1, 2, d, segs, "shot", 0, True, k, 33, "frame")


@pytest.mark.parametrize("d", [64, 128])
def test_largest_k_every_row(d):
    """k = 31, the largest top-k the library takes (1 + k partial slots a row fill
    one warp; query-list entries keep the slot in 5 bits): every row against the
    oracle, with lists of 32 candidates (31 picked), 16 (all picked, 15 pads) and
    none; then chunk anchors without the causal mask (47 candidates a query)."""
    wl = _many_chunk_scene(d, 31)
    _check_full(wl)
    _check_full(wl.replace(anchor="chunk", causal=False))


def test_largest_slice_count():
    """B * H = 65,535 (b, h) slices, the library's limit (slices index the second
    launch dimension of the pool and query-list kernels): an 80-token scene with
    every stage launched over all slices; the first two and the last slice are
    generated and checked against the oracle on every row (the rest are zero
    inputs). One slice more is rejected before any launch."""
    segs = [W.Segment(16, W.CAPTION, 0, -1)]
    for s_ in range(2):
        for f in range(2):
            segs.append(W.Segment(16, W.VIDEO, s_, f))
    wl = W.custom("manyslices", 1, 65535, 64, segs, "shot", 0, True, 1, 35, "frame")
    _check_full(wl, heads=[(0, 0), (0, 1), (0, 65534)])
    lay = moc.Layout.from_workload(wl)
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    lib = moc.lib()
    assert lib.moc_pool_keys(lay.handle, 1, 65536, 64, p, p, moc._stream()) == 1
    assert lib.moc_route(lay.handle, 2, 32768, 64, p, p, 1, 1, p, moc._stream()) == 1
    assert lib.moc_attention_fwd(lay.handle, 1, 65536, 64, p, p, p, p, 1, 0.125, p, None, p,
                                 1 << 30, moc._stream()) == 1


@pytest.mark.parametrize("k", [0, 1, 3, 8])
def test_tiny_k_edge_cases(k):
    """k = 0 (anchors only), k > |candidates| (shot 1 has 4): padding with -1."""
    _check_full(W.tiny(), k=k)


@pytest.mark.parametrize("anchor,radius,causal", [("chunk", 0, True), ("local", 1, True),
                                                  ("shot", 0, False), ("chunk", 0, False)])
def test_tiny_anchor_modes(anchor, radius, causal):
    _check_full(W.tiny().replace(anchor=anchor, radius=radius, causal=causal, H=3))


def test_small_ragged_scene_d128():
    """Chunks shorter than a key tile, tails of every size, captions interleaved."""
    segs = [W.Segment(37, W.CAPTION, 0, -1)]
    lens = [1, 64, 65, 127, 128, 129, 200, 3, 300, 17]
    for i, ln in enumerate(lens):
        segs.append(W.Segment(ln, W.VIDEO, i // 4, i % 4))
        if i == 3:
            segs.append(W.Segment(5, W.CAPTION, 1, -1))
    wl = W.custom("ragsmall", 2, 3, 128, segs, "shot", 0, True, 2, 31, "frame")
    _check_full(wl)
    _check_full(wl.replace(anchor="chunk"), k=5)


def test_single_shot_clip_sampled():
    _check_full(W.single(), n_random=512, seed=1)


def test_eight_shot_scene_sampled():
    """Full 180k-token eight-shot scene: routing of every row of every head,
    attention on boundary + random rows."""
    wl = W.eight()
    Q, K, V = W.make_qkv(wl)
    orc = oracle.Layout(wl)
    lay, O, lse, sel, kbar = _run(wl, Q, K, V)
    kbar_o = oracle.pool(wl, K, orc)
    np.testing.assert_allclose(kbar, kbar_o, rtol=0, atol=2e-5)
    rt = oracle.route(wl, Q, kbar_o, lay=orc)
    res = compare_routing(wl, Q, kbar_o, sel, rt, orc)
    # every mismatch is an admissible near-tie swap (asserted in compare_routing)
    assert res["exact"] + res["mismatch"] == wl.H * wl.L, (res["exact"], res["mismatch"])
    rows = sample_rows(orc, 256, seed=3)
    # attention of the sampled rows plus every mismatched (near-tie) row
    mis_rows = sorted({int(rt["rows"][r]) for _, _, r in res["mismatch_rows"]})
    rows = np.unique(np.concatenate([rows, np.asarray(mis_rows, dtype=np.int64)]))
    sub = {key: (v[:, :, rows] if key in ("sel", "top_s", "top_a", "top_j", "ncand") else v)
           for key, v in rt.items()}
    sub["rows"] = rows
    sel_sub = np.ascontiguousarray(sel[:, :, rows])
    res_sub = compare_routing(wl, Q, kbar_o, sel_sub, sub, orc)
    O_o, lse_o = attend_reference(wl, Q, K, V, sub["sel"], sel_sub, rows, orc, res_sub)
    compare_attention(O[:, :, rows], lse[:, :, rows], O_o, lse_o)
    # pruned fraction from the GPU routing equals the oracle's count
    kept = sum(oracle.kept_pairs(wl, sel[0, h], orc) for h in range(wl.H))
    assert kept == wl.H * 4_943_332_144


@pytest.mark.parametrize("k", [2, 4, 8, 16])
def test_ragged_scene_k_sweep(k):
    _check_full(W.ragged(), k=k, n_random=128, seed=k, heads=[(0, 0), (0, 7), (0, 23)])


def test_stress_scene_two_heads():
    """B=2, 361k tokens per sample, k=8: two heads carry data (the others are
    zero and still run); checked on boundary + random rows."""
    _check_full(W.stress(), n_random=64, seed=5, heads=[(0, 0), (1, 23)])


@pytest.mark.parametrize("name,k,pairs", [("eight", 2, 4_707_082_144), ("stress", 8, 12_888_328_576)])
def test_kept_pairs_match_closed_form(name, k, pairs):
    """The number of kept (query, key) pairs per (b, h) depends only on the
    layout and k (every query keeps min(k, |candidates|) chunks), so the GPU
    routing of every head - data-carrying or all-zero (ties to the lowest ids)
    - must give the closed-form count exactly; eight-shot k=2 and stress k=8."""
    wl = W.CONFIGS[name]().with_k(k)
    heads = [(0, 0), (wl.B - 1, wl.H - 1)]
    Q, K, V = W.make_qkv(wl, heads=heads)
    lay, O, lse, sel, kbar = _run(wl, Q, K, V)
    orc = oracle.Layout(wl)
    for b in range(wl.B):
        for h in (0, wl.H // 2, wl.H - 1):
            assert oracle.kept_pairs(wl, sel[b, h], orc) == pairs, (b, h)


def test_empty_batch_is_a_noop():
    wl = W.tiny()
    lay = moc.Layout.from_workload(wl)
    Q = torch.zeros(0, 2, wl.L, 64, dtype=torch.bfloat16, device="cuda")
    O, lse, sel, kbar = moc.forward(lay, Q, Q, Q, 2)
    assert O.shape[0] == 0


def test_single_chunk_scene_is_dense():
    """One video chunk: no candidates, attention = dense over the chunk."""
    wl = W.custom("one", 1, 2, 64, [W.Segment(300, W.VIDEO, 0, 0)], "chunk", 0, True, 3, 9, "none")
    Q, K, V = W.make_qkv(wl)
    lay, O, lse, sel, kbar = _run(wl, Q, K, V)
    assert (sel == -1).all()
    ref = torch.nn.functional.scaled_dot_product_attention(Q.double(), K.double(), V.double())
    assert (O.double() - ref).abs().max() < 2e-2


def test_argument_errors():
    wl = W.tiny()
    lay = moc.Layout.from_workload(wl)
    Q, K, V = (t.cuda() for t in W.make_qkv(wl))
    kbar = moc.pool_keys(lay, K)
    sel = moc.route(lay, Q, kbar, 2)
    ws = moc.workspace(lay, 1, 2, 64, 2)
    O = torch.empty_like(Q)
    lib = moc.lib()
    s = moc._stream()
    p = lambda t: moc._ptr(t)
    # misaligned pointer
    bad = torch.empty(Q.numel() * 2 + 16, dtype=torch.uint8, device="cuda")
    assert lib.moc_pool_keys(lay.handle, 1, 2, 64, bad.data_ptr() + 2, p(kbar), s) == 1
    # d not supported
    assert lib.moc_pool_keys(lay.handle, 1, 2, 96, p(K), p(kbar), s) == 1
    # k out of range
    assert lib.moc_route(lay.handle, 1, 2, 64, p(Q), p(kbar), 32, 1, p(sel), s) == 1
    # workspace too small
    assert lib.moc_attention_fwd(lay.handle, 1, 2, 64, p(Q), p(K), p(V), p(sel), 2, 0.125, p(O),
                                 None, p(ws), ws.numel() - 256, s) == 3
    # non-positive scale
    assert lib.moc_attention_fwd(lay.handle, 1, 2, 64, p(Q), p(K), p(V), p(sel), 2, 0.0, p(O),
                                 None, p(ws), ws.numel(), s) == 1
    # a good call after the rejected ones: it clears and leaves a clean device error word
    moc.attention_fwd(lay, Q, K, V, sel, 2, ws=ws, O=O)
    assert moc.check_device_error(ws) == 0


def test_qlists_invert_selection():
    """(3) round trip: every list entry points back at its chunk; lists are
    sorted by query and hold exactly the valid selections."""
    wl = W.ragged(k=4, n_shots=3, H=2, d=64)
    Q, K, V = W.make_qkv(wl)
    lay = moc.Layout.from_workload(wl)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    kbar = moc.pool_keys(lay, Kd)
    sel = moc.route(lay, Qd, kbar, 4)
    ws = moc.workspace(lay, 1, 2, 64, 4)
    moc.build_qlists(lay, sel, 1, 2, 4, ws)
    torch.cuda.synchronize()
    BH, C, L, k = 2, lay.C, lay.L, 4
    a = lambda x: (x + 255) // 256 * 256
    nblk = (L + 1023) // 1024
    off_qoff = a(256) + a(BH * nblk * C * 4)
    off_tile = off_qoff + a((BH * C + 1) * 4)
    off_tile2 = off_tile + a((BH * C + 1) * 4)
    off_list = off_tile2 + a((BH * C + 1) * 4)
    wsc = ws.cpu()
    qoff = wsc[off_qoff:off_qoff + (BH * C + 1) * 4].view(torch.int32).numpy()
    tile = wsc[off_tile:off_tile + (BH * C + 1) * 4].view(torch.int32).numpy()
    tile2 = wsc[off_tile2:off_tile2 + (BH * C + 1) * 4].view(torch.int32).numpy()
    n_valid = int((sel >= 0).sum())
    qlist = wsc[off_list:off_list + n_valid * 4].view(torch.int32).numpy()
    s = sel.cpu().numpy().reshape(BH, L, k)
    assert qoff[-1] == n_valid
    for bh in range(BH):
        for c in range(C):
            x = bh * C + c
            ent = qlist[qoff[x]:qoff[x + 1]]
            q, slot = ent >> 5, ent & 31
            assert np.all(np.diff(q) > 0)
            assert np.all(s[bh, q, slot] == c)
            want = np.nonzero((s[bh] == c).any(-1))[0]
            assert np.array_equal(q, want)
            assert tile[x + 1] - tile[x] == (len(ent) + 255) // 256
            assert tile2[x + 1] - tile2[x] == (len(ent) + 511) // 512


def test_deterministic_repeat():
    wl = W.tiny()
    Q, K, V = (t.cuda() for t in W.make_qkv(wl))
    lay = moc.Layout.from_workload(wl)
    a = moc.forward(lay, Q, K, V, 2)
    b = moc.forward(lay, Q, K, V, 2)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])


def test_eight_shot_repeat_is_bitwise_with_poisoned_workspace():
    """Full-size forward twice, the workspace filled with 0x7f bytes in
    between: every partial row and log-sum-exp the merge reads must be written
    again, and nothing may depend on timing (the attention kernel hands items
    out through an atomic counter), so both passes agree bit for bit."""
    wl = W.eight()
    g = torch.Generator(device="cuda").manual_seed(7)
    Q, K, V = (torch.randn(wl.B, wl.H, wl.L, wl.d, device="cuda", generator=g).to(torch.bfloat16)
               for _ in range(3))
    lay = moc.Layout.from_workload(wl)
    ws = moc.workspace(lay, wl.B, wl.H, wl.d, wl.k)
    O1, lse1, sel1, _ = moc.forward(lay, Q, K, V, wl.k, ws=ws)
    torch.cuda.synchronize()
    ws.fill_(0x7F)
    O2, lse2, sel2, _ = moc.forward(lay, Q, K, V, wl.k, ws=ws)
    torch.cuda.synchronize()
    assert moc.check_device_error(ws) == 0
    assert torch.isfinite(O1.float()).all() and torch.isfinite(lse1).all()
    assert torch.equal(sel1, sel2)
    assert torch.equal(O1.view(torch.int16), O2.view(torch.int16)) and torch.equal(lse1, lse2)


def test_eight_shot_is_bitwise_under_another_schedule():
    """The full-size forward with the attention kernel on 37 CTAs taking the
    work items in reversed order (routed items first, anchor items last,
    shortest first) equals the default schedule (one CTA per SM, natural
    order) bit for bit: every item's partial depends on its inputs only, not on
    which CTA computes it, when, or what ran on that SM before."""
    wl = W.eight()
    g = torch.Generator(device="cuda").manual_seed(11)
    Q, K, V = (torch.randn(wl.B, wl.H, wl.L, wl.d, device="cuda", generator=g).to(torch.bfloat16)
               for _ in range(3))
    lay = moc.Layout.from_workload(wl)
    ws = moc.workspace(lay, wl.B, wl.H, wl.d, wl.k)
    O1, lse1, sel1, _ = moc.forward(lay, Q, K, V, wl.k, ws=ws)
    torch.cuda.synchronize()
    try:
        moc.set_attend_schedule(37, reverse=True)
        ws.fill_(0x7F)
        O2, lse2, sel2, _ = moc.forward(lay, Q, K, V, wl.k, ws=ws)
        torch.cuda.synchronize()
    finally:
        moc.set_attend_schedule(0, reverse=False)
    assert moc.check_device_error(ws) == 0
    assert torch.equal(sel1, sel2)
    assert torch.equal(O1.view(torch.int16), O2.view(torch.int16)) and torch.equal(lse1, lse2)


def test_bounded_wait_reports_timeout_and_context_survives():
    """A device wait that can never complete gives up after its limit, the
    error reaches the host through the workspace error word, and the context
    keeps working (failure detection without a GPU fault or hang)."""
    wl = W.tiny()
    Q, K, V = (t.cuda() for t in W.make_qkv(wl))
    lay = moc.Layout.from_workload(wl)
    ws = moc.workspace(lay, 1, 2, 64, 2)
    O1, lse1, sel, _ = moc.forward(lay, Q, K, V, 2, ws=ws)
    assert moc.check_device_error(ws) == 0
    t0 = time.time()
    assert moc.lib().moc_selftest_bounded_wait(moc._ptr(ws), moc._stream()) == 0
    with pytest.raises(moc.MocError) as ei:
        moc.check_device_error(ws)
    assert ei.value.status == 5 and time.time() - t0 >= 1.5
    assert moc.check_device_error(ws) == 0          # cleared
    O2, lse2, _, _ = moc.forward(lay, Q, K, V, 2, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(O1, O2) and torch.equal(lse1, lse2)
    assert moc.check_layout_error(lay) == 0


@pytest.mark.parametrize("anchor,causal,k", [("chunk", True, 16), ("shot", False, 4)])
def test_ragged_scene_more_than_256_candidates(anchor, causal, k):
    """Up to 297 candidates per group: the router's multi-block path, with
    the own-chunk anchor and with the causal mask off."""
    _check_full(W.ragged().replace(anchor=anchor, causal=causal), k=k, n_random=96, seed=11,
                heads=[(0, 3), (0, 17)])


def test_selection_entry_that_is_not_a_chunk_is_reported():
    """The query-list builder ignores a selection entry >= C and records
    MOC_ERR_DEVICE_CHECK (detail 3) in the workspace's error word; the word is
    cleared by reading it and the next clean call reports nothing."""
    wl = W.tiny()
    Q, K, V = (t.cuda() for t in W.make_qkv(wl))
    lay = moc.Layout.from_workload(wl)
    sel = moc.route(lay, Q, moc.pool_keys(lay, K), 2)
    bad = sel.clone()
    bad[0, 0, 100, 1] = lay.C
    ws = moc.workspace(lay, 1, 2, 64, 2)
    moc.attention_fwd(lay, Q, K, V, bad, 2, ws=ws)
    with pytest.raises(moc.MocError) as ei:
        moc.check_device_error(ws)
    assert ei.value.status == 7
    moc.attention_fwd(lay, Q, K, V, sel, 2, ws=ws)
    assert moc.check_device_error(ws) == 0


@pytest.mark.parametrize("which", ["tiny", "ragsmall"])
def test_fused_attend_merge_matches_oracle(which):
    """moc_attend_merged ((4) with (5) in the anchor items' epilogue) against
    the oracle on every row, under the default and a reversed schedule."""
    if which == "tiny":
        wl = W.tiny()
    else:
        segs = [W.Segment(37, W.CAPTION, 0, -1)]
        for i, ln in enumerate([1, 64, 65, 127, 128, 129, 200, 3, 300, 17]):
            segs.append(W.Segment(ln, W.VIDEO, i // 4, i % 4))
        wl = W.custom("ragsmall", 2, 3, 128, segs, "shot", 0, True, 3, 31, "frame")
    Q, K, V = W.make_qkv(wl)
    orc = oracle.Layout(wl)
    ref = oracle.forward(wl, Q, K, V, lay=orc)
    lay = moc.Layout.from_workload(wl)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    sel = torch.from_numpy(np.ascontiguousarray(ref["sel"])).cuda()
    ws = moc.workspace(lay, wl.B, wl.H, wl.d, wl.k)
    outs = []
    try:
        for n_ctas, rev in [(0, False), (5, True)]:
            moc.set_attend_schedule(n_ctas, reverse=rev)
            O = torch.empty_like(Qd)
            lse = torch.empty(wl.B, wl.H, wl.L, dtype=torch.float32, device="cuda")
            moc.build_qlists(lay, sel, wl.B, wl.H, wl.k, ws)
            moc.attend_merged(lay, Qd, Kd, Vd, sel, wl.k, ws, O, lse)
            torch.cuda.synchronize()
            assert moc.check_device_error(ws) == 0
            compare_attention(O.cpu(), lse.cpu(), ref["O"], ref["lse"])
            outs.append((O.cpu(), lse.cpu()))
    finally:
        moc.set_attend_schedule(0, reverse=False)
    assert torch.equal(outs[0][0].view(torch.int16), outs[1][0].view(torch.int16))
    assert torch.equal(outs[0][1], outs[1][1])
