"""Mixture of Contexts (MoC) sparse-attention forward pass on B200 (sm_100a).

Thin Python binding of the C ABI in ``include/moc.h`` (``libmoc.so``, built by
``chunk_routed_sparse_b200/build.py``). It only marshals arguments: PyTorch
provides device memory and the current CUDA stream, every step of the path
runs in the library's CUDA kernels, and there is no CPU fallback - if the
library is missing or a call fails, an exception is raised.

Pipeline (pages: "Mixture of Contexts for Long Video Generation | Summary"
§3.1-§3.3; the jxzklqfsx.com MoC write-up, "計算效率"):

    layout = Layout(seg_len, seg_kind, seg_shot, seg_frame, anchor="shot")
    kbar = pool_keys(layout, K)                  # (1) mean-pooled keys per chunk
    sel = route(layout, Q, kbar, k, causal=True) # (2) top-k chunks per query
    O, lse = attention_fwd(layout, Q, K, V, sel, k)  # (3) lists, (4) attend, (5) merge

Q, K, V are bf16 CUDA tensors [B, H, L, d] (head-major, contiguous), d in {64, 128}.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoc.so")

CAPTION, VIDEO = 0, 1
ANCHOR = {"shot": 0, "local": 1, "chunk": 2}
STATUS = {0: "ok", 1: "invalid argument", 2: "invalid layout description",
          3: "workspace too small", 4: "CUDA error", 5: "device-side wait timed out",
          6: "unsupported problem size", 7: "device-side consistency check failed"}


class MocError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)} (status {status})")
        self.status = status


class _Desc(ctypes.Structure):
    _fields_ = [("n_segments", ctypes.c_int32), ("seg_len", ctypes.c_void_p),
                ("seg_kind", ctypes.c_void_p), ("seg_shot", ctypes.c_void_p),
                ("seg_frame", ctypes.c_void_p), ("anchor_mode", ctypes.c_int32),
                ("local_radius", ctypes.c_int32)]


_lib = None

# name -> (restype, argtypes); every symbol include/moc.h declares
_I, _I64, _P, _F, _SZ = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "moc_status_string": (ctypes.c_char_p, [_I]),
    "moc_build_layout": (_I, [_P, _I, _P]),
    "moc_layout_destroy": (None, [_P]),
    "moc_layout_info": (_I, [_P, _P, _P, _P]),
    "moc_layout_table": (_I, [_P, _I, _P, _I64, _P]),
    "moc_pool_keys": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "moc_route": (_I, [_P, _I, _I, _I, _P, _P, _I, _I, _P, _P]),
    "moc_attention_workspace_bytes": (_SZ, [_P, _I, _I, _I, _I]),
    "moc_build_qlists": (_I, [_P, _I, _I, _I, _P, _P, _SZ, _P]),
    "moc_attend_partials": (_I, [_P, _I, _I, _I, _P, _P, _P, _I, _F, _P, _SZ, _P]),
    "moc_merge": (_I, [_P, _I, _I, _I, _I, _P, _P, _P, _P, _SZ, _P]),
    "moc_attend_merged": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _I, _F, _P, _P, _P, _SZ, _P]),
    "moc_quantize_e4m3": (_I, [_I, _I64, _I, _P, _P, _P, _P]),
    "moc_attend_partials_e4m3": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _I, _F, _P, _SZ, _P]),
    "moc_attention_fwd_e4m3": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _I, _F, _P, _P, _P, _SZ, _P]),
    "moc_attention_fwd": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _I, _F, _P, _P, _P, _SZ, _P]),
    "moc_attention_fwd_static": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _I, _F, _P, _P, _P]),
    "moc_attention_bwd_workspace_bytes": (_SZ, [_P, _I, _I, _I, _I]),
    "moc_attention_bwd": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _I, _F, _P, _P, _P, _P, _SZ,
                               _P]),
    "moc_check_device_error": (_I, [_P, _SZ, _P, _P]),
    "moc_check_device_error_static": (_I, [_P, _P]),
    "moc_layout_device_error": (_I, [_P, _P, _P]),
    "moc_selftest_bounded_wait": (_I, [_P, _P]),
    "moc_set_attend_schedule": (_I, [_I, _I]),
    "moc_set_attend_kernel": (_I, [_I]),
    "moc_forward_host": (_I, [_P, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P, _P, _P, _P, _SZ, _I, _P]),
    "moc_forward_host_device_bytes": (_SZ, [_P, _I, _I, _I, _I, _I]),
    "moc_route_perturb": (_I, [_P, _I, _I, _I, _I, _P, _P, _F, _F, _I, _P, _P]),
    "moc_outer_route": (_I, [_P, _I, _I, _I, _P, _P, _I, _I, _P, _P]),
    "moc_route_masked": (_I, [_P, _I, _I, _I, _P, _P, _I, _I, _P, _P, _P]),
}


def lib() -> ctypes.CDLL:
    """Load libmoc.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run chunk_routed_sparse_b200/build.py "
                              "(there is no fallback implementation)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != 0:
        raise MocError(status, where)


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _i32(xs: Sequence[int]):
    arr = (ctypes.c_int32 * len(xs))(*[int(x) for x in xs])
    return arr


class Layout:
    """A scene's chunk tables (moc_build_layout), on the current CUDA device
    by default, or host-only with ``device=-1`` (inspection only)."""

    def __init__(self, seg_len, seg_kind, seg_shot, seg_frame, anchor: str = "shot",
                 radius: int = 0, device: Optional[int] = None):
        n = len(seg_len)
        self._arrays = [_i32(seg_len), _i32(seg_kind), _i32(seg_shot), _i32(seg_frame)]
        desc = _Desc(n, *[ctypes.cast(a, ctypes.c_void_p) for a in self._arrays],
                     ANCHOR[anchor] if isinstance(anchor, str) else int(anchor), int(radius))
        if device is None:
            device = torch.cuda.current_device()
        self.device = device
        h = ctypes.c_void_p()
        _check(lib().moc_build_layout(ctypes.byref(desc), int(device), ctypes.byref(h)),
               "moc_build_layout")
        self._h = h
        L, C, S = ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
        _check(lib().moc_layout_info(h, ctypes.byref(L), ctypes.byref(C), ctypes.byref(S)),
               "moc_layout_info")
        self.L, self.C, self.n_shots = L.value, C.value, S.value

    @classmethod
    def from_workload(cls, wl, device: Optional[int] = None) -> "Layout":
        """From any object with seg_arrays(), ``anchor`` and ``radius``."""
        ln, kind, shot, frame = wl.seg_arrays()
        return cls(ln, kind, shot, frame, wl.anchor, wl.radius, device)

    @property
    def handle(self):
        return self._h

    def table(self, which: int):
        n = ctypes.c_int64()
        _check(lib().moc_layout_table(self._h, which, None, 0, ctypes.byref(n)), "moc_layout_table")
        buf = (ctypes.c_int32 * max(n.value, 1))()
        _check(lib().moc_layout_table(self._h, which, buf, n.value, ctypes.byref(n)),
               "moc_layout_table")
        return list(buf)[:n.value]

    def workspace_bytes(self, B: int, H: int, d: int, k: int) -> int:
        return int(lib().moc_attention_workspace_bytes(self._h, B, H, d, k))

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib().moc_layout_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _dims(Q: torch.Tensor) -> Tuple[int, int, int, int]:
    if Q.dim() != 4 or Q.dtype != torch.bfloat16 or not Q.is_cuda or not Q.is_contiguous():
        raise ValueError("expected a contiguous bf16 CUDA tensor [B, H, L, d]")
    return tuple(Q.shape)  # type: ignore


def pool_keys(layout: Layout, K: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    B, H, L, d = _dims(K)
    if out is None:
        out = torch.empty(B, H, layout.C, d, dtype=torch.float32, device=K.device)
    _check(lib().moc_pool_keys(layout.handle, B, H, d, _ptr(K), _ptr(out), _stream()),
           "moc_pool_keys")
    return out


def route(layout: Layout, Q: torch.Tensor, kbar: torch.Tensor, k: int, causal: bool = True,
          out: Optional[torch.Tensor] = None) -> torch.Tensor:
    B, H, L, d = _dims(Q)
    if out is None:
        out = torch.empty(B, H, L, k, dtype=torch.int32, device=Q.device)
    _check(lib().moc_route(layout.handle, B, H, d, _ptr(Q), _ptr(kbar), k, int(bool(causal)),
                           _ptr(out), _stream()), "moc_route")
    return out


def outer_route(layout: Layout, Qbar: torch.Tensor, Kbar: torch.Tensor, M: int, causal: bool = True,
                out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Outer-loop routing (moc_outer_route): Qbar = pool_keys(layout, Q), Kbar =
    pool_keys(layout, K), both fp32 [B, H, C, d]; returns int64 [B, H, G] masks
    (bit s = segment s allowed)."""
    B, H, C, d = Qbar.shape
    G = len(layout.table(1)) // 2
    if out is None:
        out = torch.empty(B, H, G, dtype=torch.int64, device=Qbar.device)
    _check(lib().moc_outer_route(layout.handle, B, H, d, _ptr(Qbar), _ptr(Kbar), M, 1 if causal else 0,
                                 _ptr(out), _stream()), "moc_outer_route")
    return out


def route_masked(layout: Layout, Q: torch.Tensor, kbar: torch.Tensor, k: int, seg_mask: torch.Tensor,
                 causal: bool = True, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    B, H, L, d = _dims(Q)
    if out is None:
        out = torch.empty(B, H, L, k, dtype=torch.int32, device=Q.device)
    _check(lib().moc_route_masked(layout.handle, B, H, d, _ptr(Q), _ptr(kbar), k, 1 if causal else 0,
                                  _ptr(seg_mask), _ptr(out), _stream()), "moc_route_masked")
    return out


def route_perturb(layout: Layout, sel: Optional[torch.Tensor], rnd: torch.Tensor, k: int, p_max: float,
                  lam: float, m_max: int, causal: bool = True, B: Optional[int] = None,
                  H: Optional[int] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Context drop-off / drop-in (moc_route_perturb): sel int32 [B, H, L, k] from
    route() (None when k == 0), rnd uint32-valued int32 [B, H, L, 2 + k + m_max]
    of random words; returns int32 [B, H, L, k + m_max]."""
    B = rnd.shape[0] if B is None else B
    H = rnd.shape[1] if H is None else H
    L = rnd.shape[2]
    if rnd.shape[3] != 2 + k + m_max or not rnd.is_cuda or rnd.dtype not in (torch.int32, torch.uint32):
        raise ValueError("rnd must be a CUDA int32/uint32 tensor [B, H, L, 2 + k + m_max]")
    if out is None:
        out = torch.empty(B, H, L, k + m_max, dtype=torch.int32, device=rnd.device)
    _check(lib().moc_route_perturb(layout.handle, B, H, k, 1 if causal else 0,
                                   _ptr(sel) if k > 0 else None, _ptr(rnd), float(p_max), float(lam),
                                   m_max, _ptr(out), _stream()), "moc_route_perturb")
    return out


def workspace(layout: Layout, B: int, H: int, d: int, k: int, device=None) -> torch.Tensor:
    n = layout.workspace_bytes(B, H, d, k)
    if n == 0:
        raise ValueError("invalid problem for the workspace size query")
    return torch.empty(n, dtype=torch.uint8, device=device or torch.cuda.current_device())


def build_qlists(layout, sel, B, H, k, ws):
    _check(lib().moc_build_qlists(layout.handle, B, H, k, _ptr(sel) if k > 0 else None, _ptr(ws),
                                  ws.numel(), _stream()), "moc_build_qlists")


def attend_partials(layout, Q, K, V, k, ws, scale=None):
    B, H, L, d = _dims(Q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    _check(lib().moc_attend_partials(layout.handle, B, H, d, _ptr(Q), _ptr(K), _ptr(V), k,
                                     float(scale), _ptr(ws), ws.numel(), _stream()),
           "moc_attend_partials")


def attend_merged(layout, Q, K, V, sel, k, ws, O, lse=None, scale=None):
    """(4) + (5) fused (moc_attend_merged); needs build_qlists first."""
    B, H, L, d = _dims(Q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    _check(lib().moc_attend_merged(layout.handle, B, H, d, _ptr(Q), _ptr(K), _ptr(V),
                                   _ptr(sel) if k > 0 else None, k, float(scale), _ptr(O), _ptr(lse),
                                   _ptr(ws), ws.numel(), _stream()), "moc_attend_merged")


def merge(layout, sel, k, ws, O, lse=None):
    B, H, L, d = _dims(O)
    _check(lib().moc_merge(layout.handle, B, H, d, k, _ptr(sel) if k > 0 else None, _ptr(O),
                           _ptr(lse), _ptr(ws), ws.numel(), _stream()), "moc_merge")


def attention_fwd(layout: Layout, Q, K, V, sel, k: int, scale: Optional[float] = None,
                  ws: Optional[torch.Tensor] = None, O: Optional[torch.Tensor] = None,
                  lse: Optional[torch.Tensor] = None, want_lse: bool = True):
    B, H, L, d = _dims(Q)
    for t in (K, V):
        if tuple(t.shape) != (B, H, L, d):
            raise ValueError("Q, K, V shapes differ")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if ws is None:
        ws = workspace(layout, B, H, d, k, Q.device)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty(B, H, L, dtype=torch.float32, device=Q.device)
    _check(lib().moc_attention_fwd(layout.handle, B, H, d, _ptr(Q), _ptr(K), _ptr(V),
                                   _ptr(sel) if k > 0 else None, k, float(scale), _ptr(O),
                                   _ptr(lse), _ptr(ws), ws.numel(), _stream()),
           "moc_attention_fwd")
    return O, lse


def attention_bwd(layout: Layout, Q, K, V, O, lse, dO, sel, k: int, scale: Optional[float] = None,
                  ws: Optional[torch.Tensor] = None, dQ: Optional[torch.Tensor] = None,
                  dK: Optional[torch.Tensor] = None, dV: Optional[torch.Tensor] = None):
    """Backward of attention_fwd (moc_attention_bwd): returns bf16 (dQ, dK, dV)
    for the upstream gradient dO, with the selection held constant."""
    B, H, L, d = _dims(Q)
    for t in (K, V, O, dO):
        if tuple(t.shape) != (B, H, L, d) or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("Q, K, V, O, dO must be contiguous bf16 [B, H, L, d] tensors")
    if tuple(lse.shape) != (B, H, L) or lse.dtype != torch.float32:
        raise ValueError("lse must be fp32 [B, H, L]")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if ws is None:
        n = int(lib().moc_attention_bwd_workspace_bytes(layout.handle, B, H, d, k))
        if n == 0:
            raise ValueError("invalid problem for the backward workspace size query")
        ws = torch.empty(n, dtype=torch.uint8, device=Q.device)
    dQ = torch.empty_like(Q) if dQ is None else dQ
    dK = torch.empty_like(Q) if dK is None else dK
    dV = torch.empty_like(Q) if dV is None else dV
    _check(lib().moc_attention_bwd(layout.handle, B, H, d, _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse),
                                   _ptr(dO), _ptr(sel) if k > 0 else None, k, float(scale), _ptr(dQ),
                                   _ptr(dK), _ptr(dV), _ptr(ws), ws.numel(), _stream()),
           "moc_attention_bwd")
    return dQ, dK, dV


def forward(layout: Layout, Q, K, V, k: int, causal: bool = True, scale=None, ws=None):
    """Pool -> route -> attention. Returns (O, lse, sel, kbar)."""
    kbar = pool_keys(layout, K)
    sel = route(layout, Q, kbar, k, causal) if k > 0 else \
        torch.empty(Q.shape[0], Q.shape[1], Q.shape[2], 0, dtype=torch.int32, device=Q.device)
    O, lse = attention_fwd(layout, Q, K, V, sel, k, scale=scale, ws=ws)
    return O, lse, sel, kbar


class MoCAttention(torch.autograd.Function):
    """The MoC attention as a torch.autograd.Function ("Mixture of Contexts for Long
    Video Generation | Summary", appendix on training: a custom autograd function
    carries the gradient of the attention over the selected keys and values).

    forward: pool -> route -> attention (moc_pool_keys, moc_route,
    moc_attention_fwd); backward: moc_attention_bwd for the upstream gradient of O.
    The top-k selection is discrete, so it is a constant of the backward pass: Q, K
    and V receive the gradient of the attention over each query's anchors and
    selected chunks, and nothing flows through the pooled keys or the scores. Every
    step runs in the library's kernels; this class only marshals arguments and
    keeps (Q, K, V, O, lse, sel) for the backward call.

    apply(layout, Q, K, V, k, causal=True, scale=None) -> O (bf16 [B, H, L, d])."""

    @staticmethod
    def forward(ctx, layout, Q, K, V, k, causal=True, scale=None):
        Q, K, V = Q.contiguous(), K.contiguous(), V.contiguous()
        O, lse, sel, _ = forward(layout, Q, K, V, k, causal, scale)
        ctx.layout, ctx.k, ctx.scale = layout, k, scale
        ctx.save_for_backward(Q, K, V, O, lse, sel)
        return O

    @staticmethod
    def backward(ctx, dO):
        Q, K, V, O, lse, sel = ctx.saved_tensors
        dQ, dK, dV = attention_bwd(ctx.layout, Q, K, V, O, lse, dO.contiguous().to(torch.bfloat16), sel,
                                   ctx.k, scale=ctx.scale)
        return None, dQ, dK, dV, None, None, None


def moc_attention(layout: Layout, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, k: int,
                  causal: bool = True, scale: Optional[float] = None) -> torch.Tensor:
    """Differentiable MoC attention (MoCAttention.apply): bf16 O with gradients for
    Q, K and V through the library's backward pass."""
    return MoCAttention.apply(layout, Q, K, V, k, causal, scale)


def quantize_e4m3(X: torch.Tensor):
    """Per-(b, h) power-of-two scale and E4M3 bytes of a bf16 [B, H, L, d] tensor
    (moc_quantize_e4m3). Returns (X8 uint8 [B, H, L, d], scale fp32 [B, H])."""
    B, H, L, d = _dims(X)
    X8 = torch.empty(B, H, L, d, dtype=torch.uint8, device=X.device)
    scale = torch.empty(B, H, dtype=torch.float32, device=X.device)
    _check(lib().moc_quantize_e4m3(B * H, L, d, _ptr(X), _ptr(X8), _ptr(scale), _stream()), "moc_quantize_e4m3")
    return X8, scale


def attention_fwd_e4m3(layout: Layout, Q8, K8, V8, q_scale, k_scale, v_scale, sel, k: int,
                       scale: Optional[float] = None, ws: Optional[torch.Tensor] = None,
                       O: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None):
    """The attention stage on E4M3 inputs (moc_attention_fwd_e4m3); bf16 O, fp32 lse."""
    B, H, L, d = Q8.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if ws is None:
        ws = workspace(layout, B, H, d, k, Q8.device)
    if O is None:
        O = torch.empty(B, H, L, d, dtype=torch.bfloat16, device=Q8.device)
    if lse is None:
        lse = torch.empty(B, H, L, dtype=torch.float32, device=Q8.device)
    _check(lib().moc_attention_fwd_e4m3(layout.handle, B, H, d, _ptr(Q8), _ptr(K8), _ptr(V8), _ptr(q_scale),
                                        _ptr(k_scale), _ptr(v_scale), _ptr(sel) if k > 0 else None, k,
                                        float(scale), _ptr(O), _ptr(lse), _ptr(ws), ws.numel(), _stream()),
           "moc_attention_fwd_e4m3")
    return O, lse


def forward_host_device_bytes(layout: Layout, B: int, H: int, d: int, k: int, heads_per_chunk: int = 0) -> int:
    return int(lib().moc_forward_host_device_bytes(layout.handle, B, H, d, k, heads_per_chunk))


def forward_host(layout: Layout, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, k: int,
                 causal: bool = True, scale=None, heads_per_chunk: int = 0,
                 dev: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                 want_lse: bool = True, want_sel: bool = False):
    """Whole forward pass on host tensors (moc_forward_host): Q, K, V are CPU bf16
    [B, H, L, d] (pinned for overlap); returns CPU (O, lse or None, sel or None)
    once complete. ``dev`` is the device scratch (allocated here if None)."""
    if Q.dim() != 4:
        raise ValueError("expected [B, H, L, d] tensors")
    B, H, L, d = tuple(Q.shape)
    for t in (Q, K, V):
        if t.device.type != "cpu" or not t.is_contiguous() or t.dtype != torch.bfloat16:
            raise ValueError("Q, K, V must be contiguous bf16 CPU tensors")
        if tuple(t.shape) != (B, H, L, d):
            raise ValueError("Q, K, V shapes differ")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if dev is None:
        n = forward_host_device_bytes(layout, B, H, d, k, heads_per_chunk)
        if n == 0:
            raise ValueError("invalid problem for moc_forward_host")
        dev = torch.empty(n, dtype=torch.uint8, device=torch.cuda.current_device())
    O = out if out is not None else torch.empty_like(Q)
    lse = torch.empty(B, H, L, dtype=torch.float32) if want_lse else None
    sel = torch.empty(B, H, L, k, dtype=torch.int32) if (want_sel and k > 0) else None
    _check(lib().moc_forward_host(layout.handle, B, H, d, k, 1 if causal else 0, float(scale),
                                  _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse), _ptr(sel),
                                  _ptr(dev), dev.numel(), heads_per_chunk, _stream()),
           "moc_forward_host")
    return O, lse, sel


def check_layout_error(layout: Layout) -> int:
    """Read and clear the layout's device error word (router); raises on error."""
    det = ctypes.c_int32()
    _check(lib().moc_layout_device_error(layout.handle, ctypes.byref(det), _stream()),
           "layout device error word")
    return det.value


def set_attend_kernel(variant: int = 0):
    """Kernel of the attention stage for the following calls
    (moc_set_attend_kernel): 0 default, 1 single CTA, 2 CTA pairs."""
    _check(lib().moc_set_attend_kernel(int(variant)), "moc_set_attend_kernel")


def set_attend_schedule(n_ctas: int = 0, reverse: bool = False):
    """Diagnostic: attention-kernel CTA count (0: one per SM) and item order for
    the following calls (moc_set_attend_schedule)."""
    _check(lib().moc_set_attend_schedule(int(n_ctas), 1 if reverse else 0), "moc_set_attend_schedule")


def check_device_error(ws: torch.Tensor) -> int:
    """Read and clear the workspace's device error word (synchronises); returns
    the detail code, raises MocError on a recorded device error."""
    det = ctypes.c_int32()
    st = lib().moc_check_device_error(_ptr(ws), ws.numel(), ctypes.byref(det), _stream())
    _check(st, "device error word")
    return det.value
