"""moc_forward_host (host buffers, chunks of heads pipelined over three
streams) against the device calls on whole tensors: every stage is
independent per (b, h), so the results must agree bit for bit whatever the
chunking; plus its argument checks."""
import ctypes

import pytest
import torch

import chunk_routed_sparse_b200 as moc
import moc_workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _device_reference(wl, Q, K, V):
    lay = moc.Layout.from_workload(wl)
    O, lse, sel, _ = moc.forward(lay, Q.cuda(), K.cuda(), V.cuda(), wl.k, causal=wl.causal)
    torch.cuda.synchronize()
    return lay, O.cpu(), lse.cpu(), sel.cpu()


SCENES = {
    "tiny": lambda: W.tiny(),
    "tiny_b2h3": lambda: W.tiny().replace(B=2, H=3),                # chunks cross the batch boundary
    "eight_h5": lambda: W.eight().replace(H=5),                     # full-length scene, 5 heads
}


@pytest.mark.parametrize("name,chunks", [("tiny", [0, 1, 2]), ("tiny_b2h3", [0, 1, 4, 6]),
                                         ("eight_h5", [0, 2, 5])])
def test_host_pipeline_matches_device_calls(name, chunks):
    wl = SCENES[name]()
    Q, K, V = W.make_qkv(wl)
    lay, O_ref, lse_ref, sel_ref = _device_reference(wl, Q, K, V)
    Qp, Kp, Vp = Q.pin_memory(), K.pin_memory(), V.pin_memory()
    for hc in chunks:
        O, lse, sel = moc.forward_host(lay, Qp, Kp, Vp, wl.k, causal=wl.causal, heads_per_chunk=hc,
                                       out=torch.empty_like(Q).pin_memory(), want_sel=True)
        assert torch.equal(O.view(torch.int16), O_ref.view(torch.int16)), hc
        assert torch.equal(lse, lse_ref), hc
        assert torch.equal(sel, sel_ref), hc


def test_host_pipeline_unpinned_and_k0():
    wl = W.tiny().with_k(0)
    Q, K, V = W.make_qkv(wl)
    lay, O_ref, lse_ref, _ = _device_reference(wl, Q, K, V)
    O, lse, sel = moc.forward_host(lay, Q, K, V, 0, causal=wl.causal, heads_per_chunk=1, want_sel=True)
    assert sel is None
    assert torch.equal(O.view(torch.int16), O_ref.view(torch.int16)) and torch.equal(lse, lse_ref)


def test_host_pipeline_argument_checks():
    wl = W.tiny()
    Q, K, V = W.make_qkv(wl)
    lay = moc.Layout.from_workload(wl)
    lib = moc.lib()
    n = moc.forward_host_device_bytes(lay, wl.B, wl.H, wl.d, wl.k, 1)
    dev = torch.empty(n, dtype=torch.uint8, device="cuda")
    O = torch.empty_like(Q)
    p = moc._ptr

    def call(dev_ptr, nbytes, scale=0.125, hc=1, q=Q):
        return lib.moc_forward_host(lay.handle, wl.B, wl.H, wl.d, wl.k, 1, scale, p(q), p(K), p(V), p(O),
                                    None, None, dev_ptr, nbytes, hc, moc._stream())

    assert call(p(dev), n - 256) == 3                                   # scratch too small
    assert call(ctypes.c_void_p(dev.data_ptr() + 16), n - 256) == 1     # scratch not 256-byte aligned
    assert call(p(dev), n, scale=0.0) == 1                              # scale must be > 0
    assert call(p(dev), n, q=None) == 1                                 # null input
    assert call(p(dev), n) == 0
    lay2, O_ref, _, _ = _device_reference(wl, Q, K, V)
    assert torch.equal(O.view(torch.int16), O_ref.view(torch.int16))
