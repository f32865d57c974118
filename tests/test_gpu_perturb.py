"""moc_route_perturb (context drop-off / drop-in) against the oracle in
oracle/perturb.py, bit for bit, on selections routed by the oracle and random
words drawn by a seeded generator; and attention over a perturbed selection."""
import numpy as np
import pytest
import torch

import chunk_routed_sparse_b200 as moc
import moc_workloads as W
import oracle
from oracle import perturb as P
from parity import compare_attention, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _words(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(-(2 ** 31), 2 ** 31, shape, dtype=torch.int32, generator=g)


def _case(wl, rows, k, m_max, p_max, lam, seed, heads=None):
    """Oracle routing of `rows` (other rows -1), random words for every row; run
    the kernel on the whole tensor and the oracle on `rows`."""
    heads = heads or [(b, h) for b in range(wl.B) for h in range(wl.H)]
    Q, K, V = W.make_qkv(wl, heads=heads)
    orc = oracle.Layout(wl)
    kbar = oracle.pool(wl, K, orc)
    rt = oracle.route(wl, Q, kbar, rows=rows, k=k, lay=orc)
    sel = np.full((wl.B, wl.H, wl.L, k), -1, dtype=np.int32)
    sel[:, :, rows, :] = rt["sel"]
    rnd = _words((wl.B, wl.H, wl.L, 2 + k + m_max), seed)
    lay = moc.Layout.from_workload(wl)
    out = moc.route_perturb(lay, torch.from_numpy(sel).cuda() if k > 0 else None, rnd.cuda(), k, p_max, lam,
                            m_max, causal=wl.causal).cpu().numpy()
    ref = P.perturb(orc, rt["sel"], rnd[:, :, rows].numpy().view(np.uint32), k, p_max, lam, m_max, rows=rows)
    return out, ref, rt, (Q, K, V), orc, lay


def test_tiny_every_row_bitwise():
    wl = W.tiny()
    rows = np.arange(wl.L)
    out, ref, _, _, _, _ = _case(wl, rows, 2, 3, 0.7, 1.5, 1)
    assert np.array_equal(out, ref)


@pytest.mark.parametrize("causal,k,m_max,p_max,lam", [(True, 4, 2, 0.5, 0.8), (False, 8, 6, 1.0, 3.0),
                                                     (True, 0, 3, 0.3, 2.0)])
def test_ragged_sampled_rows_bitwise(causal, k, m_max, p_max, lam):
    wl = W.ragged().replace(causal=causal, H=3)
    rows = sample_rows(oracle.Layout(wl), 768, seed=7)
    out, ref, _, _, _, _ = _case(wl, rows, k, m_max, p_max, lam, 2)
    assert np.array_equal(out[:, :, rows], ref)


def test_eight_shot_sampled_rows_bitwise():
    wl = W.eight().replace(H=2)
    rows = sample_rows(oracle.Layout(wl), 1024, seed=9)
    out, ref, _, _, _, _ = _case(wl, rows, 3, 4, 0.6, 1.2, 3)
    assert np.array_equal(out[:, :, rows], ref)
    # rows the oracle did not route carry -1 selections: nothing to drop, only drop-ins
    assert (out >= -1).all()


def test_identity_when_rates_are_zero():
    wl = W.tiny()
    rows = np.arange(wl.L)
    out, ref, rt, _, _, _ = _case(wl, rows, 2, 3, 0.0, 0.0, 4)
    assert np.array_equal(out[..., :2], rt["sel"]) and (out[..., 2:] == -1).all()


def test_attention_over_a_perturbed_selection():
    """The attention calls take the perturbed selection with k + m_max slots."""
    wl = W.tiny()
    rows = np.arange(wl.L)
    k, m_max = 2, 3
    out, ref, _, (Q, K, V), orc, lay = _case(wl, rows, k, m_max, 0.7, 1.5, 5)
    O, lse = moc.attention_fwd(lay, Q.cuda(), K.cuda(), V.cuda(), torch.from_numpy(out).cuda(), k + m_max)
    torch.cuda.synchronize()
    O_o, lse_o, _ = oracle.attend(wl, Q, K, V, ref, rows=rows, lay=orc)
    compare_attention(O.cpu(), lse.cpu(), O_o, lse_o)


def test_argument_checks():
    wl = W.tiny()
    lay = moc.Layout.from_workload(wl)
    lib = moc.lib()
    sel = torch.full((1, 2, wl.L, 2), -1, dtype=torch.int32, device="cuda")
    rnd = torch.zeros(1, 2, wl.L, 2 + 2 + 3, dtype=torch.int32, device="cuda")
    out = torch.empty(1, 2, wl.L, 5, dtype=torch.int32, device="cuda")
    p = moc._ptr

    def call(k=2, p_max=0.5, lam=1.0, m_max=3):
        return lib.moc_route_perturb(lay.handle, 1, 2, k, 1, p(sel), p(rnd), p_max, lam, m_max, p(out),
                                     moc._stream())

    assert call() == 0
    assert call(p_max=1.5) == 1 and call(lam=-1.0) == 1 and call(lam=float("inf")) == 1
    assert call(m_max=30) == 1 and call(m_max=-1) == 1 and call(k=0, m_max=0) == 1
