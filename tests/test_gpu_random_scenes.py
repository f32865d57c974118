"""GPU forward against the oracle on random small scenes: every row of every
head, for shots of sub-chunked frames with caption runs, every anchor mode,
window radius and causal flag (the layouts the layout-builder tests draw)."""
import numpy as np
import pytest
import torch

import moc_workloads as W

from test_gpu_parity import _check_full

pytestmark = pytest.mark.gpu


def _scene(i):
    rng = np.random.default_rng(5000 + i)
    segs = []
    for s in range(rng.integers(1, 6)):
        for _ in range(rng.integers(0, 3)):
            segs.append(W.Segment(int(rng.integers(1, 40)), W.CAPTION, s, -1))
        for f in range(rng.integers(1, 5)):
            for _ in range(rng.integers(1, 4)):
                segs.append(W.Segment(int(rng.integers(1, 200)), W.VIDEO, s, f))
    anchor = ["shot", "local", "chunk"][int(rng.integers(0, 3))]
    d = [64, 128][int(rng.integers(0, 2))]
    k = int(rng.integers(1, 5))
    return W.custom(f"rand{i}", 1, 2, d, segs, anchor, int(rng.integers(0, 3)), bool(rng.integers(0, 2)),
                    k, 900 + i, "shot_frame")


@pytest.mark.parametrize("i", range(12))
def test_random_scene_every_row(i):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    tot = _check_full(_scene(i))
    assert tot["max_abs"] <= 2e-2
