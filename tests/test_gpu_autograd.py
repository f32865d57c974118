"""The differentiable wrapper (moc.moc_attention / moc.MoCAttention, a
torch.autograd.Function over the C ABI): PyTorch autograd through it gives exactly
the gradients of moc_attention_bwd on the forward pass's own O, lse and selection
(the same kernels on the same inputs, so bit for bit), and nothing else is
differentiated. The backward kernels themselves are checked against the oracle in
test_gpu_backward.py."""
import pytest
import torch

import chunk_routed_sparse_b200 as moc
import moc_workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _ragsmall():
    segs = [W.Segment(37, W.CAPTION, 0, -1)]
    for i, ln in enumerate([1, 64, 65, 127, 128, 129, 200, 3, 300, 17]):
        segs.append(W.Segment(ln, W.VIDEO, i // 4, i % 4))
    return W.custom("ragsmall", 2, 3, 128, segs, "shot", 0, True, 3, 31, "frame")


@pytest.mark.parametrize("which", ["tiny", "ragsmall"])
def test_autograd_equals_the_backward_call(which):
    wl = W.tiny() if which == "tiny" else _ragsmall()
    Q, K, V = (t.cuda() for t in W.make_qkv(wl))
    g = torch.Generator(device="cuda").manual_seed(3)
    G = torch.randn(Q.shape, device="cuda", generator=g).to(torch.bfloat16)
    lay = moc.Layout.from_workload(wl)
    Qr, Kr, Vr = (t.clone().requires_grad_(True) for t in (Q, K, V))
    O = moc.moc_attention(lay, Qr, Kr, Vr, wl.k, wl.causal)
    (O.float() * G.float()).sum().backward()
    torch.cuda.synchronize()
    O2, lse2, sel2, _ = moc.forward(lay, Q, K, V, wl.k, wl.causal)
    dQ, dK, dV = moc.attention_bwd(lay, Q, K, V, O2, lse2, G, sel2, wl.k)
    torch.cuda.synchronize()
    assert torch.equal(O.detach().view(torch.int16), O2.view(torch.int16))
    for got, want in ((Qr.grad, dQ), (Kr.grad, dK), (Vr.grad, dV)):
        assert got.dtype == torch.bfloat16 and got.shape == want.shape
        assert torch.equal(got.view(torch.int16), want.view(torch.int16))


def test_only_inputs_that_ask_for_it_get_gradients():
    wl = W.tiny()
    Q, K, V = (t.cuda() for t in W.make_qkv(wl))
    lay = moc.Layout.from_workload(wl)
    Vr = V.clone().requires_grad_(True)
    O = moc.moc_attention(lay, Q, K, Vr, wl.k)
    assert O.requires_grad
    O.float().sum().backward()
    assert Vr.grad is not None and torch.isfinite(Vr.grad.float()).all()
    # dV of sum(O) is sum over the queries attending each key of their weights: every
    # column of a key's gradient row is the same total weight, and the weights of
    # every query sum to one, so the grand total is (rows) x d
    tot = Vr.grad.float().sum().item()
    assert abs(tot - wl.B * wl.H * wl.L * wl.d) <= 2e-2 * wl.B * wl.H * wl.L * wl.d
