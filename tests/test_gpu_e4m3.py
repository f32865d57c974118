"""The E4M3 attention variant (moc_quantize_e4m3, moc_attention_fwd_e4m3)
through the C ABI.

Quantisation: per (b, h) slice a power-of-two scale >= amax / 448 (and < twice
that), and E4M3 bytes equal to PyTorch's own round-to-nearest conversion of
X / scale (a library routine, independent of the kernel).

Attention: the oracle runs on the dequantised inputs X8 * scale, which are
exact bf16 values (the scales are powers of two), with the same selection, so
the only difference left is the kernel's own arithmetic: P written as E4M3 of
P * 2^6 before the P V product. For one row with weights w_u = p_u / l over
Omega (l >= 1: the element that set the running max has p = 1) the error is
  |O - O_ref| <= sum_u |p~_u - p_u| |v_u| / l
              <= 2^-4 * sum_u w_u |v_u|           (E4M3 rounding, normal range)
               + n * 2^-16 * max_u |v_u|          (subnormal or flushed P * 2^6)
plus the bf16 rounding of O (2^-8 |O|) and fp32 accumulation (1e-3 slack).
sum_u w_u |v_u| is the oracle's attention over |V|; n = |Omega|.
"""
import math

import numpy as np
import pytest
import torch

import chunk_routed_sparse_b200 as moc
import moc_workloads as W
import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _dequant(X8: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
    """bf16 values of E4M3 bytes times their slice's power-of-two scale (exact)."""
    f = X8.cpu().view(torch.float8_e4m3fn).float()
    return (f * scale.cpu()[:, :, None, None]).to(torch.bfloat16)


def _ragsmall(H=2):
    segs = [W.Segment(37, W.CAPTION, 0, -1)]
    for i, ln in enumerate([1, 64, 65, 127, 128, 129, 200, 3, 300, 17]):
        segs.append(W.Segment(ln, W.VIDEO, i // 4, i % 4))
        if i == 3:
            segs.append(W.Segment(5, W.CAPTION, 1, -1))
    return W.custom("ragsmall", 1, H, 128, segs, "shot", 0, True, 3, 31, "frame")


def test_quantisation_matches_torch_conversion():
    wl = _ragsmall(H=3)
    Q, _, _ = W.make_qkv(wl)
    Q = Q.clone()
    Q[0, 2] = 0  # an all-zero slice: scale 1, all bytes 0
    X8, scale = moc.quantize_e4m3(Q.cuda())
    torch.cuda.synchronize()
    sc = scale.cpu()
    for h in range(wl.H):
        amax = Q[0, h].float().abs().max().item()
        s = sc[0, h].item()
        assert math.log2(s) == int(math.log2(s))  # a power of two
        if amax == 0:
            assert s == 1.0
        else:
            assert amax / 448 <= s < 2 * amax / 448 or (s == 2 * amax / 448)
        want = (Q[0, h].float() / s).to(torch.float8_e4m3fn).view(torch.uint8)
        assert torch.equal(X8[0, h].cpu(), want), h


def _check(wl, rows=None, seed=0):
    Q, K, V = W.make_qkv(wl)
    orc = oracle.Layout(wl)
    sel = oracle.route(wl, Q, oracle.pool(wl, K, orc), lay=orc)["sel"]
    (Q8, qs), (K8, ks), (V8, vs) = (moc.quantize_e4m3(t.cuda()) for t in (Q, K, V))
    lay = moc.Layout.from_workload(wl)
    O, lse = moc.attention_fwd_e4m3(lay, Q8, K8, V8, qs, ks, vs, torch.from_numpy(sel).cuda(), wl.k)
    torch.cuda.synchronize()
    Qd, Kd, Vd = _dequant(Q8, qs), _dequant(K8, ks), _dequant(V8, vs)
    r = np.arange(wl.L) if rows is None else rows
    s_r = np.ascontiguousarray(sel[:, :, r])
    O_o, lse_o, nk = oracle.attend(wl, Qd, Kd, Vd, s_r, rows=r, lay=orc)
    A, _, _ = oracle.attend(wl, Qd, Kd, Vd.abs(), s_r, rows=r, lay=orc)
    vmax = Vd.float().abs().amax(dim=(2, 3)).numpy()[:, :, None, None]
    bound = 2.0 ** -4 * A + nk[..., None] * 2.0 ** -16 * vmax + 2.0 ** -8 * np.abs(O_o) + 1e-3
    og = O.cpu()[:, :, r].double().numpy()
    err = np.abs(og - O_o)
    assert np.all(err <= bound), f"worst excess {np.max(err - bound):.3e} at {np.unravel_index(np.argmax(err - bound), err.shape)}"
    assert np.abs(lse.cpu()[:, :, r].double().numpy() - lse_o).max() <= 5e-3
    return float(err.max()), float(err.mean())


def test_small_ragged_scene_every_row():
    mx, mean = _check(_ragsmall())
    assert mean <= 2e-3


def test_eight_shot_sampled_rows():
    wl = W.eight().replace(H=2)
    rng = np.random.default_rng(9)
    rows = np.unique(np.concatenate([[0, 511, 512, 513, 23011, 23012, wl.L - 1], rng.integers(0, wl.L, size=200)]))
    mx, mean = _check(wl, rows=rows)
    assert mean <= 2e-3
