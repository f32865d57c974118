"""Pins of the CPU oracle against things other than itself (CPU only).

Each test fixes the oracle to an independent fact: a hand-worked example, a
textbook library routine (fp64 scaled-dot-product attention), a closed form, an
invariant of softmax attention, or the brute-force NumPy restatement.
"""
import math

import numpy as np
import pytest
import torch

import moc_workloads as W
import oracle
from oracle import bruteforce
from conftest import read_golden


def _small(anchor="shot", causal=True, k=2, radius=1, seed=11, H=2, d=16, offsets="frame",
           caption_first=True):
    segs = []
    if caption_first:
        segs.append(W.Segment(5, W.CAPTION, -1, -1))
    lens = [7, 9, 4, 8, 6, 5, 7, 3]
    for i, ln in enumerate(lens):
        shot, frame = divmod(i, 3)
        segs.append(W.Segment(ln, W.VIDEO, shot, frame))
    if not caption_first:
        segs.insert(4, W.Segment(3, W.CAPTION, 1, -1))
    return W.custom("small", 1, H, d, segs, anchor, radius, causal, k, seed, offsets)


def _golden_example(tie=False):
    g = read_golden("three_chunk_example.txt")
    d = int(g["d"])
    segs = [W.Segment(2, W.VIDEO, s, 0) for s in range(3)]
    wl = W.custom("three", 1, 1, d, segs, "shot", 0, True, int(g["k"]), 0, "none")

    def mat(prefix):
        return torch.tensor([g[f"{prefix}{i}"] for i in range(6)], dtype=torch.float64)

    Q, K, V = mat("Q"), mat("K"), mat("V")
    if tie:
        Q[4] = torch.tensor(g["tie_Q4"], dtype=torch.float64)
    cast = lambda x: x.to(torch.bfloat16).reshape(1, 1, 6, d)
    return g, wl, cast(Q), cast(K), cast(V)


def test_hand_worked_three_chunk_example():
    g, wl, Q, K, V = _golden_example()
    scale = math.log(3.0) / 2
    lay = oracle.Layout(wl)
    kbar = oracle.pool(wl, K, lay)
    assert np.array_equal(kbar[0, 0, 0], [1, 0, 0, 0])
    assert np.array_equal(kbar[0, 0, 1], [0, 1, 0, 0])
    assert np.array_equal(kbar[0, 0, 2], [0, 0, 0, 0])
    rt = oracle.route(wl, Q, kbar, lay=lay)
    assert rt["sel"][0, 0, :, 0].tolist() == [int(x) for x in g["sel"]]
    O, lse, nk = oracle.attend(wl, Q, K, V, rt["sel"], scale=scale, lay=lay)
    for t in range(6):
        np.testing.assert_allclose(O[0, 0, t], g[f"O{t}"], rtol=0, atol=1e-12)
    assert nk[0, 0].tolist() == [2, 2, 4, 4, 4, 4]
    # lse of a uniform row over n keys with score 0 is log n
    np.testing.assert_allclose(lse[0, 0, :4], [math.log(2)] * 2 + [math.log(4)] * 2, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0, 4], math.log(6.0), atol=1e-12)   # 3+1+1+1


def test_hand_worked_tie_goes_to_lower_chunk():
    g, wl, Q, K, V = _golden_example(tie=True)
    lay = oracle.Layout(wl)
    kbar = oracle.pool(wl, K, lay)
    rt = oracle.route(wl, Q, kbar, lay=lay)
    assert rt["sel"][0, 0, 4, 0] == int(g["tie_sel4"])
    O, _, _ = oracle.attend(wl, Q, K, V, rt["sel"], scale=math.log(3.0) / 2, lay=lay)
    np.testing.assert_allclose(O[0, 0, 4], g["tie_O4"], atol=1e-12)


def test_dense_flop_convention_matches_printed_eq5():
    g = read_golden("dense_flops_eq5.txt")
    L, d = int(g["L"]), int(g["d"])
    dense = 4 * L * L * d
    assert float(f"{dense:.{int(g['printed_digits']) - 1}e}") == g["dense_flops_printed"]
    assert float(f"{dense:.{int(g['table1_digits']) - 1}e}") == g["table1_dense_flops"]


@pytest.mark.parametrize("d", [16, 64])
def test_noncausal_all_selected_equals_library_dense_attention(d):
    """With the causal mask off and k >= C, every chunk is in Omega: MoC must
    reduce to plain dense softmax(QK^T/sqrt(d))V (torch SDPA in fp64)."""
    wl = _small(causal=False, k=20, d=d)
    Q, K, V = W.make_qkv(wl)
    res = oracle.forward(wl, Q, K, V)
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q.double(), K.double(), V.double())
    np.testing.assert_allclose(res["O"], ref.numpy(), rtol=0, atol=1e-12)
    s = (Q.double() @ K.double().transpose(-1, -2)) / math.sqrt(d)
    np.testing.assert_allclose(res["lse"], torch.logsumexp(s, -1).numpy(), atol=1e-10)


@pytest.mark.parametrize("anchor,radius", [("shot", 0), ("local", 1), ("chunk", 0)])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("k", [0, 1, 2, 3, 30])
def test_oracle_matches_bruteforce(anchor, radius, causal, k):
    wl = _small(anchor=anchor, radius=radius, causal=causal, k=k, caption_first=(k != 1))
    Q, K, V = W.make_qkv(wl)
    res = oracle.forward(wl, Q, K, V)
    Ob, lb, sels, _ = bruteforce.forward(wl, Q, K, V)
    for (b, h, t), s in sels.items():
        got = [int(x) for x in res["sel"][b, h, t] if x >= 0]
        assert got == s, (b, h, t)
    np.testing.assert_allclose(res["O"], Ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(res["lse"], lb, rtol=0, atol=1e-10)


def test_all_candidates_selected_equals_dense_masked_attention():
    """k >= #candidates: Omega is the full chunk-causal + anchor mask."""
    wl = _small(k=50)
    Q, K, V = W.make_qkv(wl)
    res = oracle.forward(wl, Q, K, V)
    lay = oracle.Layout(wl)
    _, _, _, mask = bruteforce.forward(wl, Q, K, V)
    allowed = lay.role[lay.chunk_of_token][:, lay.chunk_of_token] != oracle.ROLE_NONE
    assert np.array_equal(mask, allowed)
    s = (Q[0, 0].double() @ K[0, 0].double().T).numpy() / math.sqrt(wl.d)
    s = np.where(mask, s, -np.inf)
    w = np.exp(s - s.max(1, keepdims=True))
    w /= w.sum(1, keepdims=True)
    np.testing.assert_allclose(res["O"][0, 0], w @ V[0, 0].double().numpy(), atol=1e-12)


def test_convexity_and_ones_column():
    wl = _small(k=2)
    Q, K, V = W.make_qkv(wl)
    V = V.clone()
    V[..., 3] = 1.0
    res = oracle.forward(wl, Q, K, V)
    # weights sum to one: a constant-1 value column comes out as 1
    assert np.abs(res["O"][..., 3] - 1.0).max() < 1e-12
    # every output coordinate lies in [min, max] of V over Omega(t)
    lay = oracle.Layout(wl)
    for t in range(lay.L):
        i = lay.chunk_of_token[t]
        keys = [u for u in range(lay.L) if lay.role[i, lay.chunk_of_token[u]] == oracle.ROLE_ANCHOR
                or lay.chunk_of_token[u] in set(res["sel"][0, 0, t].tolist())]
        vv = V[0, 0, keys].double().numpy()
        assert len(keys) == res["nkeys"][0, 0, t]
        assert np.all(res["O"][0, 0, t] <= vv.max(0) + 1e-12)
        assert np.all(res["O"][0, 0, t] >= vv.min(0) - 1e-12)


def test_pool_closed_forms():
    wl = _small()
    Q, K, V = W.make_qkv(wl)
    lay = oracle.Layout(wl)
    K2 = K.clone()
    K2[0, 1, lay.off[2]:lay.off[3]] = K2[0, 1, lay.off[2]]  # a chunk of identical rows
    kbar = oracle.pool(wl, K2, lay)
    assert np.array_equal(kbar[0, 1, 2], K2[0, 1, lay.off[2]].double().numpy())
    # sum_c n_c Kbar_c = sum_t K_t
    n = np.diff(lay.off).astype(np.float64)
    tot = (kbar[0] * n[None, :, None]).sum(1)
    np.testing.assert_allclose(tot, K2[0].double().sum(1).numpy(), atol=1e-10)
    # library mean per segment
    for c in range(lay.C):
        ref = K2[0, :, lay.off[c]:lay.off[c + 1]].double().mean(1).numpy()
        np.testing.assert_allclose(kbar[0, :, c], ref, atol=1e-13)


def test_route_special_cases():
    wl = _small(k=3)
    Q, K, V = W.make_qkv(wl)
    lay = oracle.Layout(wl)
    kbar = oracle.pool(wl, K, lay)
    # k = 0 selects nothing
    rt0 = oracle.route(wl, Q, kbar, k=0, lay=lay)
    assert rt0["sel"].shape[-1] == 0
    # k >= |Cand| selects exactly the candidate set
    rt = oracle.route(wl, Q, kbar, k=40, lay=lay)
    for t in range(lay.L):
        cand = set(np.nonzero(lay.role[lay.chunk_of_token[t]] == oracle.ROLE_CAND)[0].tolist())
        got = [x for x in rt["sel"][0, 0, t].tolist() if x >= 0]
        assert set(got) == cand and len(got) == len(cand) == rt["ncand"][0, 0, t]
    # q = 0: every score ties at 0, so the lowest chunk ids win, in id order
    Qz = torch.zeros_like(Q)
    rtz = oracle.route(wl, Qz, kbar, k=2, lay=lay)
    for t in range(lay.L):
        cand = sorted(np.nonzero(lay.role[lay.chunk_of_token[t]] == oracle.ROLE_CAND)[0].tolist())
        want = (cand[:2] + [-1, -1])[:2]
        assert rtz["sel"][0, 0, t].tolist() == want


def test_route_matches_full_python_sort():
    wl = _small(k=3, anchor="chunk", causal=False)
    Q, K, V = W.make_qkv(wl)
    lay = oracle.Layout(wl)
    kbar = oracle.pool(wl, K, lay)
    rt = oracle.route(wl, Q, kbar, lay=lay)
    q = Q.double().numpy()
    for h in range(wl.H):
        for t in range(lay.L):
            i = lay.chunk_of_token[t]
            cand = np.nonzero(lay.role[i] == oracle.ROLE_CAND)[0]
            order = sorted(cand.tolist(), key=lambda j: (-float(q[0, h, t] @ kbar[0, h, j]), j))
            want = (order[:3] + [-1] * 3)[:3]
            assert rt["sel"][0, h, t].tolist() == want


def _first_candidates_sel(wl, lay, k):
    """A selection that takes the first min(k, |Cand|) candidates of each token."""
    sel = np.full((lay.L, k), -1, dtype=np.int32)
    for i in range(lay.C):
        cand = np.nonzero(lay.role[i] == oracle.ROLE_CAND)[0][:k]
        sel[lay.off[i]:lay.off[i + 1], :len(cand)] = cand
    return sel


def test_kept_pairs_closed_forms():
    """Closed-form kept-pair counts of the uniform-chunk scenes (every chunk of a
    scene has the same size, so only min(k, |Cand|) matters)."""
    # eight-shot: 8x64 captions, 8 shots x 15 frames x 1500, k = 3
    wl = W.eight()
    lay = oracle.Layout(wl)
    L = 512 + 8 * 15 * 1500
    assert lay.L == L == 180_512
    want = 512 * L + 180_000 * (512 + 22_500) + 7 * 22_500 * 3 * 1500
    assert want == 4_943_332_144
    assert oracle.kept_pairs(wl, _first_candidates_sel(wl, lay, 3), lay) == want
    # k = 2
    want2 = 512 * L + 180_000 * 23_012 + 7 * 22_500 * 2 * 1500
    assert oracle.kept_pairs(wl, _first_candidates_sel(wl, lay, 2), lay) == want2 == 4_707_082_144
    # stress (per sample): 16x64 captions + 16 shots, k = 8
    ws = W.stress()
    lay_s = oracle.Layout(ws)
    Ls = 1024 + 16 * 15 * 1500
    want_s = 1024 * Ls + 360_000 * (1024 + 22_500) + 15 * 22_500 * 8 * 1500
    assert oracle.kept_pairs(ws, _first_candidates_sel(ws, lay_s, 8), lay_s) == want_s
    assert want_s == 12_888_328_576
    # single-shot: frame window +-1, candidates are frames <= f-2, k = 4
    w1 = W.single()
    lay1 = oracle.Layout(w1)
    win = sum(min(20, f + 1) - max(0, f - 1) + 1 for f in range(21))
    sel = sum(min(4, max(0, f - 1)) for f in range(21))
    want1 = 512 * 33_272 + 1560 * (21 * 512 + 1560 * (win + sel))
    assert (win, sel) == (61, 70)
    assert oracle.kept_pairs(w1, _first_candidates_sel(w1, lay1, 4), lay1) == want1 == 352_609_984


def test_tiny_scene_routing_and_kept_pairs():
    wl = W.tiny()
    Q, K, V = W.make_qkv(wl)
    lay = oracle.Layout(wl)
    kbar = oracle.pool(wl, K, lay)
    rt = oracle.route(wl, Q, kbar, lay=lay)
    for h in range(wl.H):
        assert oracle.kept_pairs(wl, rt["sel"][0, h], lay) == \
            64 * 2112 + 2048 * (64 + 1024) + 1024 * 2 * 256 == 2_887_680
    # shot 0 has no candidates, shot 1 has the 4 frames of shot 0
    assert rt["ncand"][0, 0, lay.off[1]:lay.off[5]].max() == 0
    assert rt["ncand"][0, 0, lay.off[5]:].min() == 4


def test_near_tie_rule():
    s = np.array([1.0, 1.0 + 5e-5, 0.0, 1e-9])
    a = np.array([1.0, 1.0, 1.0, 1.0])
    assert oracle.is_near(s[0], s[1], a[0], a[1])
    assert not oracle.is_near(s[0], s[2], a[0], a[2])
    assert oracle.is_near(s[2], s[3], a[2], a[3])     # guarded by magnitude


def test_dense_comparison_layouts():
    """The benchmark's dense and FLOP-matched block-diagonal layouts (k = 0):
    the oracle's kept-pair counts are L^2 and the block sum of squares, and the
    block-diagonal one (``bench.flop_matched_blocks``) matches the eight-shot
    scene's MoC count within 0.02 %."""
    import bench
    wl = W.eight()
    L = wl.L
    n_cap = sum(s.length for s in wl.segments if s.kind == W.CAPTION)
    n_fr, rest = divmod(L - n_cap, 1500)
    dense = [W.Segment(n_cap, W.CAPTION, -1, -1)] + \
        [W.Segment(1500 + (rest if f == n_fr - 1 else 0), W.VIDEO, 0, f) for f in range(n_fr)]
    blk, n_blk, r_blk = bench.flop_matched_blocks(L, 4_943_332_144)
    blocks = [W.Segment(blk, W.VIDEO, s, 0) for s in range(n_blk)] + ([W.Segment(r_blk, W.VIDEO, n_blk, 0)] if r_blk else [])
    for segs, want in ((dense, L * L), (blocks, sum(s.length ** 2 for s in blocks))):
        w2 = W.custom("cmp", 1, 1, 128, segs, "shot", 0, True, 0, 1, "none")
        assert w2.L == L
        lay = oracle.Layout(w2)
        assert oracle.kept_pairs(w2, np.full((L, 0), -1, dtype=np.int32), lay) == want
    moc_pairs = 4_943_332_144
    assert abs(sum(s.length ** 2 for s in blocks) - moc_pairs) < 2e-4 * moc_pairs
