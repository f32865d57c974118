"""The allocation-free attention entry point (moc_attention_fwd_static).

It serves callers that cannot allocate device memory: its scratch is a static
64 MiB array inside the library instead of a caller workspace. Called twice in
a row through the C ABI, it must reproduce the workspace entry point
(moc_attention_fwd) within the parity tolerances of the other tests, and it
must reject a problem whose scratch does not fit. This file is collected last
so that a stop-at-first-failure run has already run every other test.
"""
import ctypes
import math

import pytest
import torch

import chunk_routed_sparse_b200 as moc
import moc_workloads as W
from parity import O_MAX_ABS, O_MEAN_ABS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _ragged_small():
    segs = [W.Segment(37, W.CAPTION, 0, -1)]
    for i, ln in enumerate([1, 64, 65, 127, 128, 129, 200, 3, 300, 17]):
        segs.append(W.Segment(ln, W.VIDEO, i // 4, i % 4))
    return W.custom("ragsmall", 2, 3, 128, segs, "shot", 0, True, 3, 31, "frame")


@pytest.mark.parametrize("wl", [W.tiny(), _ragged_small()], ids=["tiny_d64", "ragged_d128"])
def test_static_scratch_matches_workspace_entry_point(wl):
    B, H, L, d, k = wl.B, wl.H, wl.L, wl.d, wl.k
    Q, K, V = (t.cuda() for t in W.make_qkv(wl))
    lay = moc.Layout.from_workload(wl)
    kbar = moc.pool_keys(lay, K)
    sel = moc.route(lay, Q, kbar, k)
    O_ref, lse_ref = moc.attention_fwd(lay, Q, K, V, sel, k)
    torch.cuda.synchronize()
    lib = moc.lib()
    scale = 1.0 / math.sqrt(d)
    for _ in range(2):  # the scratch keeps the previous call's contents
        O = torch.full_like(Q, float("nan"))
        lse = torch.full((B, H, L), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.moc_attention_fwd_static(lay.handle, B, H, d, moc._ptr(Q), moc._ptr(K), moc._ptr(V),
                                          moc._ptr(sel), k, scale, moc._ptr(O), moc._ptr(lse),
                                          moc._stream())
        assert st == 0, moc.STATUS.get(st, st)
        torch.cuda.synchronize()
        diff = (O.double() - O_ref.double()).abs()
        assert diff.max().item() <= O_MAX_ABS and diff.mean().item() <= O_MEAN_ABS
        assert (lse - lse_ref).abs().max().item() <= 5e-3


def test_static_scratch_rejects_oversized_problem():
    wl = W.eight()
    lay = moc.Layout.from_workload(wl)
    assert lay.workspace_bytes(1, 24, 128, 3) > (64 << 20)
    lib = moc.lib()
    p = ctypes.c_void_p(256)  # never dereferenced: the size check fails first
    st = lib.moc_attention_fwd_static(lay.handle, 1, 24, 128, p, p, p, p, 3, 0.088, p, None,
                                      moc._stream())
    assert st == 3
