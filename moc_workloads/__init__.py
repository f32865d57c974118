"""Seeded synthetic workloads for the Mixture of Contexts (MoC) forward pass.

This module only *describes inputs*: the segment layout of a token stream
(caption segments and video frames / sub-frames, with their shot and frame
ids) and seeded random Q, K, V tensors. It holds none of the method's
arithmetic (no pooling, scoring, masking or attention), so that both the CUDA
path and the CPU oracle can consume the same bytes without sharing code.

The workloads mirror the scenes the pages measure on:

* "Mixture of Contexts for Long Video Generation | Summary" (§4): eight shots
  of 8 s at 480p / 12 fps, about 180k tokens; single-shot clips at 320x192
  with about 6.3k tokens (Appendix E).
* The MoC write-up on jxzklqfsx.com ("實驗"): LCT scenes of up to eight shots,
  about 22k tokens per shot.

There is no public dataset behind these kernels' measurement; the tensors are
N(0, 1) noise plus per-shot / per-frame mean offsets, so that mean-pooled keys
carry a routing signal the way real frame tokens do.

Recipes (every draw comes from a CPU ``torch.Generator``; the stream for
sample ``b``, head ``h`` is seeded with ``_slice_seed(seed, b, h)``):

* ``frame`` offsets (tiny, single): mu_f ~ N(0, 0.5^2 I) per (b, h, frame),
  added to every K row of the frame and to the Q rows of the frame picked by
  an independent Bernoulli(0.5) per token. Caption tokens get no offset.
* ``shot_frame`` offsets (eight, ragged, stress): mu_s ~ N(0, 0.5^2 I) per
  shot plus mu_sf ~ N(0, 0.25^2 I) per (shot, frame), both added to K and Q
  of every video token of that frame. Sub-chunks of one frame share its
  offset. Caption tokens get no offset.
* V is plain N(0, 1).
"""
from __future__ import annotations

import dataclasses
import random
from concurrent.futures import ThreadPoolExecutor
from typing import List, Optional, Sequence, Tuple

import torch

CAPTION = 0
VIDEO = 1


@dataclasses.dataclass(frozen=True)
class Segment:
    """One content-aligned segment of the flattened token stream.

    ``kind`` is CAPTION or VIDEO; ``shot`` is the shot the segment belongs to
    (for a caption: the shot it precedes, or -1 for a global caption);
    ``frame`` is the frame index within the shot (-1 for captions). A video
    frame may be cut into several segments (sub-chunks) that share ``frame``.
    """

    length: int
    kind: int
    shot: int
    frame: int


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    segments: Tuple[Segment, ...]
    anchor: str  # "shot" | "local" | "chunk"
    radius: int  # frame radius for anchor == "local"
    causal: bool
    k: int
    seed: int
    offsets: str  # "frame" | "shot_frame"

    @property
    def L(self) -> int:
        return sum(s.length for s in self.segments)

    @property
    def C(self) -> int:
        return len(self.segments)

    def seg_arrays(self):
        """Plain int lists (length, kind, shot, frame) in stream order."""
        return ([s.length for s in self.segments], [s.kind for s in self.segments],
                [s.shot for s in self.segments], [s.frame for s in self.segments])

    def with_k(self, k: int) -> "Workload":
        return dataclasses.replace(self, k=k)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _captions_then_shots(n_caps: int, cap_len: int, n_shots: int, frames: int,
                         frame_len: int) -> Tuple[Segment, ...]:
    segs: List[Segment] = [Segment(cap_len, CAPTION, s, -1) for s in range(n_caps)]
    for s in range(n_shots):
        for f in range(frames):
            segs.append(Segment(frame_len, VIDEO, s, f))
    return tuple(segs)


def tiny(k: int = 2) -> Workload:
    """64 caption tokens, then 2 shots x 4 frames x 256 tokens; B=1, H=2, d=64."""
    segs = [Segment(64, CAPTION, -1, -1)]
    for s in range(2):
        for f in range(4):
            segs.append(Segment(256, VIDEO, s, f))
    return Workload("tiny", 1, 2, 64, tuple(segs), "shot", 0, True, k, 101, "frame")


def single(k: int = 4) -> Workload:
    """Single-shot clip: 512 caption tokens + 21 frames x (30x52) tokens; H=12, d=128.

    The mandatory local anchor is the query's own frame +-1 (clipped)."""
    segs = [Segment(512, CAPTION, 0, -1)] + [Segment(30 * 52, VIDEO, 0, f) for f in range(21)]
    return Workload("single", 1, 12, 128, tuple(segs), "local", 1, True, k, 102, "frame")


def eight(k: int = 3) -> Workload:
    """Eight-shot scene: 8 x 64 caption tokens first, then 8 shots x 15 frames x
    (30x50) tokens = 180,512 tokens; H=24, d=128."""
    return Workload("eight", 1, 24, 128, _captions_then_shots(8, 64, 8, 15, 1500),
                    "shot", 0, True, k, 103, "shot_frame")


def stress(k: int = 8) -> Workload:
    """B=2, 16 x 64 caption tokens + 16 shots x 15 frames x 1500 tokens."""
    return Workload("stress", 2, 24, 128, _captions_then_shots(16, 64, 16, 15, 1500),
                    "shot", 0, True, k, 105, "shot_frame")


def ragged(k: int = 4, layout_seed: int = 1104, n_shots: int = 8, frame_len: int = 1500,
           H: int = 24, d: int = 128) -> Workload:
    """Ragged content-aligned chunks: shots of U{6..24} frames, each 1500-token
    frame cut at random into U{1..4} sub-chunks of at least 64 tokens, and a
    caption of U{32..128} tokens immediately before each shot."""
    rng = random.Random(layout_seed)
    segs: List[Segment] = []
    for s in range(n_shots):
        segs.append(Segment(rng.randint(32, 128), CAPTION, s, -1))
        for f in range(rng.randint(6, 24)):
            parts = rng.randint(1, 4)
            cuts = _random_cuts(rng, frame_len, parts, 64)
            for ln in cuts:
                segs.append(Segment(ln, VIDEO, s, f))
    return Workload("ragged", 1, H, d, tuple(segs), "shot", 0, True, k, 104, "shot_frame")


def _random_cuts(rng: random.Random, total: int, parts: int, min_len: int) -> List[int]:
    """Split ``total`` into ``parts`` positive lengths, each >= min_len."""
    spare = total - parts * min_len
    if parts == 1:
        return [total]
    pts = sorted(rng.randint(0, spare) for _ in range(parts - 1))
    bounds = [0] + pts + [spare]
    return [min_len + bounds[i + 1] - bounds[i] for i in range(parts)]


def custom(name: str, B: int, H: int, d: int, segments: Sequence[Segment], anchor: str = "shot",
           radius: int = 0, causal: bool = True, k: int = 2, seed: int = 7,
           offsets: str = "frame") -> Workload:
    return Workload(name, B, H, d, tuple(segments), anchor, radius, causal, k, seed, offsets)


CONFIGS = {"tiny": tiny, "single": single, "eight": eight, "ragged": ragged, "stress": stress}


def _slice_seed(seed: int, b: int, h: int) -> int:
    return (seed * 1_000_003 + b * 10_007 + h * 101 + 17) % (2 ** 62)


def _gen_slice(wl: Workload, b: int, h: int) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    g = torch.Generator().manual_seed(_slice_seed(wl.seed, b, h))
    L, d = wl.L, wl.d
    q = torch.randn(L, d, generator=g, dtype=torch.float32)
    k = torch.randn(L, d, generator=g, dtype=torch.float32)
    v = torch.randn(L, d, generator=g, dtype=torch.float32)
    # offsets, drawn in a fixed order after the noise
    shots = sorted({s.shot for s in wl.segments if s.kind == VIDEO})
    frames = sorted({(s.shot, s.frame) for s in wl.segments if s.kind == VIDEO})
    if wl.offsets == "frame":
        mu = {sf: 0.5 * torch.randn(d, generator=g) for sf in frames}
        pos = 0
        for s in wl.segments:
            if s.kind == VIDEO:
                m = mu[(s.shot, s.frame)]
                k[pos:pos + s.length] += m
                pick = torch.rand(s.length, generator=g) < 0.5
                q[pos:pos + s.length][pick] += m
            pos += s.length
    elif wl.offsets == "shot_frame":
        mu_s = {sh: 0.5 * torch.randn(d, generator=g) for sh in shots}
        mu_f = {sf: 0.25 * torch.randn(d, generator=g) for sf in frames}
        pos = 0
        for s in wl.segments:
            if s.kind == VIDEO:
                m = mu_s[s.shot] + mu_f[(s.shot, s.frame)]
                k[pos:pos + s.length] += m
                q[pos:pos + s.length] += m
            pos += s.length
    elif wl.offsets != "none":
        raise ValueError(f"unknown offset recipe {wl.offsets!r}")
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def make_qkv(wl: Workload, heads: Optional[Sequence[Tuple[int, int]]] = None, threads: int = 8):
    """Return bf16 CPU tensors Q, K, V of shape [B, H, L, d] (head-major).

    ``heads`` restricts generation to the listed (b, h) slices; the others stay
    zero. Each slice has its own generator, so a slice's bytes do not depend
    on which other slices are generated."""
    B, H, L, d = wl.B, wl.H, wl.L, wl.d
    Q = torch.zeros(B, H, L, d, dtype=torch.bfloat16)
    K = torch.zeros_like(Q)
    V = torch.zeros_like(Q)
    todo = list(heads) if heads is not None else [(b, h) for b in range(B) for h in range(H)]

    def one(bh):
        b, h = bh
        q, k, v = _gen_slice(wl, b, h)
        Q[b, h].copy_(q)
        K[b, h].copy_(k)
        V[b, h].copy_(v)

    if threads > 1 and len(todo) > 1:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(one, todo))
    else:
        for bh in todo:
            one(bh)
    return Q, K, V


def make_qkv_slices(wl: Workload, s0: int, s1: int, threads: int = 8):
    """Q, K, V of the flat (b, h) slices s0 .. s1-1 (slice i is b = i // H,
    h = i % H) as bf16 CPU tensors [1, s1 - s0, L, d]: the same bytes those
    slices have in ``make_qkv(wl)``, for a process that holds only a share of
    the heads."""
    n = s1 - s0
    Q = torch.zeros(1, n, wl.L, wl.d, dtype=torch.bfloat16)
    K = torch.zeros_like(Q)
    V = torch.zeros_like(Q)

    def one(i):
        q, k, v = _gen_slice(wl, i // wl.H, i % wl.H)
        Q[0, i - s0].copy_(q)
        K[0, i - s0].copy_(k)
        V[0, i - s0].copy_(v)

    if threads > 1 and n > 1:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(one, range(s0, s1)))
    else:
        for i in range(s0, s1):
            one(i)
    return Q, K, V


def bf16_bits(t: torch.Tensor) -> torch.Tensor:
    """View a bf16 tensor's storage as int16 (the raw bit patterns)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16)
