"""The allocation-free attention entry point (moc_attention_fwd_static).

It serves callers that cannot allocate device memory: its scratch is a static
64 MiB array inside the library instead of a caller workspace. Called twice in
a row through the C ABI, it must reproduce the workspace entry point
(moc_attention_fwd) bit for bit - both run the same deterministic kernels on
the same inputs, so any difference would be a scratch-layout fault - it must
report device-side errors through its own error-word call, and it must reject
a problem whose scratch does not fit. This file is collected last
so that a stop-at-first-failure run has already run every other test.
"""
import ctypes
import math

import pytest
import torch

import chunk_routed_sparse_b200 as moc
import moc_workloads as W

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
        assert torch.equal(O.view(torch.int16), O_ref.view(torch.int16))
        assert torch.equal(lse, lse_ref)
        assert lib.moc_check_device_error_static(None, moc._stream()) == 0


def test_static_scratch_rejects_oversized_problem():
    wl = W.eight()
    lay = moc.Layout.from_workload(wl)
    assert lay.workspace_bytes(1, 24, 128, 3) > (64 << 20)
    lib = moc.lib()
    p = ctypes.c_void_p(256)  # never dereferenced: the size check fails first
    st = lib.moc_attention_fwd_static(lay.handle, 1, 24, 128, p, p, p, p, 3, 0.088, p, None,
                                      moc._stream())
    assert st == 3


def test_static_scratch_reports_device_checks():
    """A selection entry that is not a chunk id is ignored by the query-list
    builder and recorded in the device error word; with the static scratch the
    word is read through moc_check_device_error_static (and cleared by it)."""
    wl = W.tiny()
    B, H, L, d, k = wl.B, wl.H, wl.L, wl.d, wl.k
    Q, K, V = (t.cuda() for t in W.make_qkv(wl))
    lay = moc.Layout.from_workload(wl)
    sel = moc.route(lay, Q, moc.pool_keys(lay, K), k)
    sel[0, 1, -5:, 0] = lay.C + 3
    O = torch.empty_like(Q)
    lib = moc.lib()
    st = lib.moc_attention_fwd_static(lay.handle, B, H, d, moc._ptr(Q), moc._ptr(K), moc._ptr(V),
                                      moc._ptr(sel), k, 1.0 / math.sqrt(d), moc._ptr(O), None,
                                      moc._stream())
    assert st == 0
    det = ctypes.c_int32(0)
    assert lib.moc_check_device_error_static(ctypes.byref(det), moc._stream()) == 7
    assert det.value == 3
    assert lib.moc_check_device_error_static(None, moc._stream()) == 0
