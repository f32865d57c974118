"""C-ABI library checks that need no GPU: it loads, exports every symbol the
header declares, builds host-only layouts whose tables agree with the oracle's
role table, and rejects bad arguments before touching a device."""
import ctypes
import os
import re

import numpy as np
import pytest

import chunk_routed_sparse_b200 as moc
import moc_workloads as W
import oracle
from conftest import ROOT


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "moc.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(moc_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    lib = moc.lib()
    declared = _declared_functions()
    assert len(declared) >= 12
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(moc.SIGNATURES)


def test_status_strings():
    lib = moc.lib()
    for s in range(8):
        assert lib.moc_status_string(s).decode() == moc.STATUS[s]


def _host_layout(wl):
    return moc.Layout.from_workload(wl, device=-1)


WORKLOADS = [W.tiny(), W.single(), W.eight(), W.ragged(), W.stress(),
             W.tiny().replace(anchor="chunk"), W.single().replace(anchor="shot"),
             W.ragged().replace(anchor="local", radius=2)]


def _random_workload(rng, i):
    """A random valid scene: 1-6 shots of 1-5 frames, each frame cut into 1-3
    sub-chunks of 1-50 tokens, caption segments of 1-30 tokens placed before
    shots at random (sometimes several in a row, sometimes none), any anchor
    mode, radius 0-2, causal on or off."""
    segs = []
    for s in range(rng.integers(1, 7)):
        for _ in range(rng.integers(0, 3)):
            segs.append(W.Segment(int(rng.integers(1, 31)), W.CAPTION, s, -1))
        for f in range(rng.integers(1, 6)):
            for _ in range(rng.integers(1, 4)):
                segs.append(W.Segment(int(rng.integers(1, 51)), W.VIDEO, s, f))
    anchor = ["shot", "local", "chunk"][int(rng.integers(0, 3))]
    return W.custom(f"rand{i}", 1, 1, 64, segs, anchor, int(rng.integers(0, 3)), bool(rng.integers(0, 2)),
                    2, 7, "none")


RANDOM = [_random_workload(np.random.default_rng(1000 + i), i) for i in range(120)]


@pytest.mark.parametrize("wl", WORKLOADS + RANDOM, ids=lambda w: f"{w.name}-{w.anchor}")
def test_layout_tables_agree_with_oracle_roles(wl):
    lay = _host_layout(wl)
    orc = oracle.Layout(wl)
    assert lay.L == orc.L and lay.C == orc.C
    assert lay.table(0) == orc.off.tolist()
    grp = np.array(lay.table(1)).reshape(-1, 2)
    ar = np.array(lay.table(2)).reshape(-1, 2)
    ar_off = lay.table(3)
    cand = lay.table(4)
    cand_off = lay.table(5)
    ncausal = lay.table(6)
    # groups tile the token stream in order
    assert grp[0, 0] == 0 and grp[-1, 1] == orc.L
    assert np.all(grp[1:, 0] == grp[:-1, 1])
    for g, (q0, q1) in enumerate(grp):
        chunks = sorted(set(orc.chunk_of_token[q0:q1].tolist()))
        # anchor key ranges cover exactly the tokens of the oracle's anchor chunks
        keys = np.zeros(orc.L, dtype=bool)
        for s, e in ar[ar_off[g]:ar_off[g + 1]]:
            assert not keys[s:e].any()
            keys[s:e] = True
        for i in chunks:
            want = (orc.role[i] == oracle.ROLE_ANCHOR)[orc.chunk_of_token]
            assert np.array_equal(keys, want), (g, i)
            cand_all = np.nonzero(orc.role[i] != oracle.ROLE_ANCHOR)[0]
            cand_all = [c for c in cand_all if orc.kind[c] == W.VIDEO]
            got = cand[cand_off[g]:cand_off[g + 1]]
            if wl.causal:
                assert sorted(got[:ncausal[g]]) == np.nonzero(orc.role[i] == oracle.ROLE_CAND)[0].tolist()
            assert sorted(got) == sorted(cand_all)


@pytest.mark.parametrize("bad", ["zero_len", "bad_kind", "split_shot", "frames_back", "anchor",
                                 "radius", "empty"])
def test_bad_layouts_rejected(bad):
    ln, kind, shot, frame = [4, 5, 6, 7], [0, 1, 1, 1], [0, 0, 0, 1], [-1, 0, 1, 0]
    anchor, radius = "shot", 0
    if bad == "zero_len":
        ln[2] = 0
    elif bad == "bad_kind":
        kind[1] = 3
    elif bad == "split_shot":
        shot = [0, 0, 1, 0]
    elif bad == "frames_back":
        frame = [-1, 1, 0, 0]
    elif bad == "anchor":
        anchor = 7
    elif bad == "radius":
        anchor, radius = "local", -1
    elif bad == "empty":
        ln, kind, shot, frame = [], [], [], []
    with pytest.raises(moc.MocError) as ei:
        moc.Layout(ln, kind, shot, frame, anchor, radius, device=-1)
    assert ei.value.status == 2


def test_compute_calls_reject_host_only_layout():
    lay = _host_layout(W.tiny())
    lib = moc.lib()
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    assert lib.moc_pool_keys(lay.handle, 1, 2, 64, p, p, None) == 1
    assert lib.moc_route(lay.handle, 1, 2, 64, p, p, 2, 1, p, None) == 1
    assert lib.moc_attention_fwd(lay.handle, 1, 2, 64, p, p, p, p, 2, 0.125, p, None, p,
                                 1 << 30, None) == 1
    assert lib.moc_forward_host(lay.handle, 1, 2, 64, 2, 1, 0.125, p, p, p, p, None, None, p,
                                1 << 30, 0, None) == 1


def test_host_pipeline_device_bytes():
    """Scratch of the host-buffer pipeline: two input stages (Q, K, V) and two
    output stages (O, lse, sel) of one chunk, its pooled keys and its attention
    workspace - it shrinks with the chunk and needs no GPU to size."""
    wl = W.eight()
    lay = _host_layout(wl)
    lib = moc.lib()
    per_head = wl.L * 128 * 2
    n0 = lib.moc_forward_host_device_bytes(lay.handle, 1, 24, 128, 3, 0)    # default: 12 chunks of 2
    n2 = lib.moc_forward_host_device_bytes(lay.handle, 1, 24, 128, 3, 2)
    n3 = lib.moc_forward_host_device_bytes(lay.handle, 1, 24, 128, 3, 3)
    n24 = lib.moc_forward_host_device_bytes(lay.handle, 1, 24, 128, 3, 24)
    assert n0 == n2 < n3
    ws3 = lay.workspace_bytes(1, 3, 128, 3)
    assert n3 >= 3 * (2 * 3 + 2) * per_head + ws3
    assert n3 < n24 and n24 >= lay.workspace_bytes(1, 24, 128, 3) + 8 * 24 * per_head
    assert lib.moc_forward_host_device_bytes(lay.handle, 1, 24, 128, 3, 100) == n24  # clamped to B*H
    assert lib.moc_forward_host_device_bytes(lay.handle, 1, 24, 96, 3, 0) == 0
    assert lib.moc_forward_host_device_bytes(None, 1, 24, 128, 3, 0) == 0


def test_workspace_size_query():
    wl = W.eight()
    lay = _host_layout(wl)
    n = lay.workspace_bytes(1, 24, 128, 3)
    partials = 24 * wl.L * 4 * 128 * 4
    assert partials < n < partials * 1.05
    assert lay.workspace_bytes(1, 24, 96, 3) == 0     # d must be 64 or 128
    assert lay.workspace_bytes(1, 24, 128, 40) == 0   # k limit
    assert moc.lib().moc_attention_workspace_bytes(None, 1, 1, 128, 1) == 0


def test_layout_info_counts_shots():
    lay = _host_layout(W.ragged())
    assert lay.n_shots == 8
    lay1 = _host_layout(W.single())
    assert lay1.n_shots == 1


@pytest.mark.parametrize("wl", [W.tiny(), W.ragged(), W.eight()] + RANDOM[:60],
                         ids=lambda w: f"{w.name}-{w.anchor}")
def test_segment_tables_agree_with_oracle(wl):
    """Segments (shots in stream order) as the outer router and the masked
    router see them, against the oracle's own segmentation and roles."""
    from oracle import outer as OU
    lay = _host_layout(wl)
    orc = oracle.Layout(wl)
    seg = OU.segments(orc)
    cand, cand_off = lay.table(4), lay.table(5)
    cand_seg, grp_seg = lay.table(7), lay.table(8)
    seg_voff, vid = lay.table(9), lay.table(10)
    assert len(seg_voff) == int(seg.max()) + 2 and vid == [c for c in range(orc.C) if orc.kind[c] == 1]
    for s_ in range(len(seg_voff) - 1):
        assert all(seg[c] == s_ for c in vid[seg_voff[s_]:seg_voff[s_ + 1]])
    assert cand_seg == [int(seg[c]) for c in cand]
    grp = lay.table(1)
    for g in range(len(grp) // 2):
        c0 = int(orc.chunk_of_token[grp[2 * g]])
        assert grp_seg[g] == (int(seg[c0]) if orc.kind[c0] == 1 else -1)
    # router tile cost prefixes: increasing, one entry per router tile plus one
    for which in (11, 12):
        pre = lay.table(which)
        assert pre[0] == 0 and all(b > a for a, b in zip(pre, pre[1:]))
        ntiles = sum((grp[2 * g + 1] - grp[2 * g] + 127) // 128 for g in range(len(grp) // 2))
        assert len(pre) == ntiles + 1


@pytest.mark.parametrize("wl", WORKLOADS + RANDOM[:80], ids=lambda w: f"{w.name}-{w.anchor}")
def test_backward_key_blocks_agree_with_oracle_roles(wl):
    """Key blocks of the backward pass: they tile the token stream in order;
    each is one video chunk or a run of caption chunks; its group list is
    exactly the groups whose queries hold every chunk of the block as an
    anchor (oracle role table); blocks are ordered by descending anchoring
    query rows and the tile prefix counts 128-key tiles in that order."""
    lay = _host_layout(wl)
    orc = oracle.Layout(wl)
    rng_ = np.array(lay.table(13)).reshape(-1, 2)
    kb_chunk, kb_goff, kb_grp = lay.table(14), lay.table(15), lay.table(16)
    kb_order, kt_off = lay.table(17), lay.table(18)
    grp = np.array(lay.table(1)).reshape(-1, 2)
    nkb = len(kb_chunk)
    assert rng_[0, 0] == 0 and rng_[-1, 1] == orc.L and np.all(rng_[1:, 0] == rng_[:-1, 1])
    rows = []
    for b in range(nkb):
        k0, k1 = rng_[b]
        chunks = sorted(set(orc.chunk_of_token[k0:k1].tolist()))
        assert orc.off[chunks[0]] == k0 and orc.off[chunks[-1] + 1] == k1
        if kb_chunk[b] >= 0:
            assert chunks == [kb_chunk[b]] and orc.kind[kb_chunk[b]] == W.VIDEO
        else:
            assert all(orc.kind[c] == W.CAPTION for c in chunks)
        want = set()
        for g, (q0, q1) in enumerate(grp):
            qc = int(orc.chunk_of_token[q0])
            hold = [orc.role[qc, c] == oracle.ROLE_ANCHOR for c in chunks]
            assert all(hold) or not any(hold), (b, g)
            if all(hold):
                want.add(g)
        got = kb_grp[kb_goff[b]:kb_goff[b + 1]]
        assert len(set(got)) == len(got) and set(got) == want, (b, got, want)
        rows.append(sum(grp[g, 1] - grp[g, 0] for g in got))
    assert sorted(kb_order) == list(range(nkb))
    assert all(rows[a] >= rows[b] for a, b in zip(kb_order, kb_order[1:]))
    assert kt_off[0] == 0 and len(kt_off) == nkb + 1
    for x, b in enumerate(kb_order):
        assert kt_off[x + 1] - kt_off[x] == (rng_[b, 1] - rng_[b, 0] + 127) // 128


@pytest.mark.parametrize("n_chunks,ok", [(16384, True), (16385, False)])
def test_chunk_count_limit(n_chunks, ok):
    """C = 16,384 chunks (the library's limit: the query-list counters of one
    (b, h) live in shared memory) builds; one more is rejected as a bad layout.
    One-token frames, 16 shots (the last shot takes the remainder)."""
    per = 1024
    ln = [1] * n_chunks
    kind = [1] * n_chunks
    shot = [min(i // per, 15) for i in range(n_chunks)]
    frame = [i - shot[i] * per for i in range(n_chunks)]
    if ok:
        lay = moc.Layout(ln, kind, shot, frame, "shot", 0, device=-1)
        assert lay.C == n_chunks and lay.L == n_chunks
    else:
        with pytest.raises(moc.MocError) as ei:
            moc.Layout(ln, kind, shot, frame, "shot", 0, device=-1)
        assert ei.value.status == 2
