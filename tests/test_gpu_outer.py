"""Outer-loop routing on the GPU (moc_outer_route, moc_route_masked) against
the oracle in oracle/outer.py: segment masks exact except where the M-th and
(M+1)-th segment scores are near-tied; masked inner routing (fed the oracle's
masks) exact except near-tied swaps, judged on the oracle's fp64 scores."""
import numpy as np
import pytest
import torch

import chunk_routed_sparse_b200 as moc
import moc_workloads as W
import oracle
from oracle import outer as OU
from parity import sample_rows

pytestmark = pytest.mark.gpu

REL = 1e-4  # near tie: gap below this fraction of the largest score magnitude


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _setup(wl):
    Q, K, V = W.make_qkv(wl)
    lay = moc.Layout.from_workload(wl)
    Qd, Kd = Q.cuda(), K.cuda()
    qbar, kbar = moc.pool_keys(lay, Qd), moc.pool_keys(lay, Kd)
    return Q, K, lay, Qd, qbar, kbar


def _mask_mismatches_are_near_ties(gpu, ref, M):
    bad = 0
    for (b, h, g) in zip(*np.nonzero(gpu != ref["mask"])):
        sc = ref["scores"][b, h, g]
        s = np.sort(sc[~np.isnan(sc)])[::-1]
        assert len(s) > M, (b, h, g)
        if s[M - 1] - s[M] >= REL * max(1e-30, np.abs(s).max()):
            bad += 1
    return bad


@pytest.mark.parametrize("name,causal,M,H", [("eight", True, 2, 2), ("eight", True, 3, 2),
                                             ("ragged", True, 3, 2), ("ragged", False, 2, 2),
                                             ("stress", True, 4, 1)])
def test_segment_masks(name, causal, M, H):
    wl = getattr(W, name)().replace(causal=causal, H=H, B=1)
    Q, K, lay, Qd, qbar, kbar = _setup(wl)
    gpu = moc.outer_route(lay, qbar, kbar, M, causal=causal).cpu().numpy().view(np.uint64)
    ref = OU.outer(wl, oracle.Layout(wl), Q, K, M)
    assert gpu.shape == ref["mask"].shape
    assert _mask_mismatches_are_near_ties(gpu, ref, M) == 0
    print(f"{name} M={M}: {int((gpu != ref['mask']).sum())} near-tied mask differences of {gpu.size}")


@pytest.mark.parametrize("name,causal,M,k", [("eight", True, 2, 3), ("ragged", True, 3, 4),
                                             ("ragged", False, 2, 8)])
def test_masked_inner_routing(name, causal, M, k):
    wl = getattr(W, name)().replace(causal=causal, H=2, B=1)
    Q, K, lay, Qd, qbar, kbar = _setup(wl)
    olay = oracle.Layout(wl)
    ref = OU.outer(wl, olay, Q, K, M)
    seg_mask = torch.from_numpy(ref["mask"].view(np.int64)).cuda()
    sel = moc.route_masked(lay, Qd, kbar, k, seg_mask, causal=causal).cpu().numpy()
    rows = sample_rows(olay, 512, seed=11)
    kbar_o = oracle.pool(wl, K, olay)
    sel_o, lists = OU.route_masked(wl, olay, Q, kbar_o, ref["mask"], ref["blocks"], ref["seg"], rows, k)
    mism = 0
    for b in range(wl.B):
        for h in range(wl.H):
            for i, t in enumerate(rows):
                g_row, o_row = sel[b, h, t], sel_o[b, h, i]
                if np.array_equal(g_row, o_row):
                    continue
                mism += 1
                lst = lists[b][h][i]
                score = dict((c, s) for s, c in lst)
                top = max(abs(s) for s, _ in lst)
                gs = [c for c in g_row if c >= 0]
                assert len(gs) == len(set(gs)) == min(k, len(lst)) and all(c in score for c in gs)
                # the GPU's picks, ranked by the oracle, match the oracle's ranks up to near ties
                got = sorted((score[c] for c in gs), reverse=True)
                want = [s for s, _ in lst[:len(gs)]]
                assert all(abs(x - y) < REL * top for x, y in zip(got, want)), (b, h, t)
    print(f"{name}: {mism} near-tie row differences of {len(rows) * wl.H}")


def test_argument_checks():
    wl = W.tiny()
    lay = moc.Layout.from_workload(wl)
    q = torch.zeros(1, 2, lay.C, 64, device="cuda")
    lib = moc.lib()
    m = torch.zeros(1, 2, 8, dtype=torch.int64, device="cuda")
    assert lib.moc_outer_route(lay.handle, 1, 2, 64, moc._ptr(q), moc._ptr(q), -1, 1, moc._ptr(m),
                               moc._stream()) == 1
    # 65 one-chunk shots: more segments than one 64-bit mask holds
    segs = [W.Segment(16, W.VIDEO, s, 0) for s in range(65)]
    w2 = W.custom("many", 1, 1, 64, segs, "shot", 0, True, 2, 3, "none")
    lay2 = moc.Layout.from_workload(w2)
    q2 = torch.zeros(1, 1, 65, 64, device="cuda")
    m2 = torch.zeros(1, 1, 65, dtype=torch.int64, device="cuda")
    assert lib.moc_outer_route(lay2.handle, 1, 1, 64, moc._ptr(q2), moc._ptr(q2), 2, 1, moc._ptr(m2),
                               moc._stream()) == 6
