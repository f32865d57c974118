"""Outer-loop context routing - TEST INFRASTRUCTURE (oracle).

Only the tests may import this module. NumPy, fp64, shares nothing with the
CUDA library.

What it computes ("Mixture of Contexts for Long Video Generation | Summary",
appendix I): before the inner MoC routing, a coarse router selects the top-M
large context segments by the similarity between the mean-pooled features of
the current query block and of the candidate segments; the inner routing then
chooses among those segments' chunks plus the mandatory context.

Readings where the page leaves a step open (each stated in the design notes):
- a segment is one shot: its video chunks, numbered in stream order;
- a query block is a query group: consecutive chunks whose queries share one
  anchor set (a shot in shot mode, a chunk in chunk mode, a run of frames with
  the same window in local mode); caption blocks are dense and not routed;
- both features are token means in fp64 - the block's queries, the segment's
  keys - and the score is their unscaled dot product (like the inner router);
- a block's candidate segments are the other segments, only the earlier ones
  when causal; its own segment is mandatory context and always kept;
- top-M by (score descending, segment ascending), all when fewer than M;
- the inner routing keeps its own rule (candidates, causal mask, top-k, ties to
  the lower chunk id), with candidates limited to chunks of kept segments.
"""
from __future__ import annotations

from typing import Dict, List

import numpy as np
import torch

ROLE_ANCHOR, ROLE_CAND = 1, 2
VIDEO = 1


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


def segments(lay) -> np.ndarray:
    """Segment (shot, numbered in stream order) of every chunk; -1 for captions."""
    seg = np.full(lay.C, -1, dtype=np.int64)
    cur, last = -1, None
    for c in range(lay.C):
        if lay.kind[c] != VIDEO:
            continue
        if lay.shot[c] != last:
            cur += 1
            last = lay.shot[c]
        seg[c] = cur
    return seg


def blocks(lay) -> List[List[int]]:
    """Query blocks: runs of consecutive chunks of one kind whose queries share
    one anchor set (the chunks with role ANCHOR)."""
    out: List[List[int]] = []
    for c in range(lay.C):
        anchors = tuple(np.nonzero(lay.role[c] == ROLE_ANCHOR)[0].tolist())
        if out:
            p = out[-1][-1]
            same_kind = lay.kind[p] == lay.kind[c]
            if same_kind and (lay.kind[c] != VIDEO or
                              tuple(np.nonzero(lay.role[p] == ROLE_ANCHOR)[0].tolist()) == anchors):
                out[-1].append(c)
                continue
        out.append([c])
    return out


def outer(wl, lay, Q: torch.Tensor, K: torch.Tensor, M: int) -> Dict[str, np.ndarray]:
    """Masks [B, H, G] (bit s = segment s kept), scores [B, H, G, S] (nan where
    not a candidate) and the blocks."""
    seg = segments(lay)
    S = int(seg.max()) + 1 if (seg >= 0).any() else 0
    blk = blocks(lay)
    G = len(blk)
    Qf, Kf = _f64(Q), _f64(K)
    masks = np.zeros((wl.B, wl.H, G), dtype=np.uint64)
    scores = np.full((wl.B, wl.H, G, S), np.nan)
    seg_tok = [np.concatenate([np.arange(lay.off[c], lay.off[c + 1]) for c in range(lay.C) if seg[c] == s])
               for s in range(S)]
    for b in range(wl.B):
        for h in range(wl.H):
            kfeat = [Kf[b, h, tok].mean(axis=0) for tok in seg_tok]
            for g, chunks in enumerate(blk):
                if lay.kind[chunks[0]] != VIDEO:
                    continue
                own = int(seg[chunks[0]])
                qtok = np.arange(lay.off[chunks[0]], lay.off[chunks[-1] + 1])
                qfeat = Qf[b, h, qtok].mean(axis=0)
                cands = [s for s in range(S) if s != own and (not wl.causal or s < own)]
                sc = {s: float(qfeat @ kfeat[s]) for s in cands}
                for s in cands:
                    scores[b, h, g, s] = sc[s]
                keep = sorted(cands, key=lambda s: (-sc[s], s))[:M]
                m = np.uint64(1) << np.uint64(own)
                for s in keep:
                    m |= np.uint64(1) << np.uint64(s)
                masks[b, h, g] = m
    return {"mask": masks, "scores": scores, "blocks": blk, "seg": seg}


def route_masked(wl, lay, Q: torch.Tensor, Kbar: np.ndarray, masks: np.ndarray, blk, seg, rows, k: int):
    """Inner routing of `rows` with candidates limited to kept segments.
    Returns sel [B, H, n, k] (-1 padded) and the sorted (score, chunk) lists
    [B][H][n] for near-tie checks."""
    block_of_chunk = np.zeros(lay.C, dtype=np.int64)
    for g, chunks in enumerate(blk):
        block_of_chunk[chunks] = g
    Qf = _f64(Q)
    sel = np.full((wl.B, wl.H, len(rows), k), -1, dtype=np.int32)
    lists = [[[None] * len(rows) for _ in range(wl.H)] for _ in range(wl.B)]
    for i, t in enumerate(rows):
        qc = int(lay.chunk_of_token[int(t)])
        if lay.kind[qc] != VIDEO:
            continue
        g = int(block_of_chunk[qc])
        base = np.nonzero(lay.role[qc] == ROLE_CAND)[0]
        for b in range(wl.B):
            for h in range(wl.H):
                m = int(masks[b, h, g])
                cands = [int(c) for c in base if (m >> int(seg[c])) & 1]
                sc = [(float(Qf[b, h, int(t)] @ Kbar[b, h, c]), c) for c in cands]
                sc.sort(key=lambda x: (-x[0], x[1]))
                lists[b][h][i] = sc
                for j, (_, c) in enumerate(sc[:k]):
                    sel[b, h, i, j] = c
    return sel, lists
