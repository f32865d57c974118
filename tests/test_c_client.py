"""The library used from plain C: ``include/moc.h`` compiles as strict C99, and
``tests/c/moc_client.c`` - a C program that links libmoc.so and the CUDA runtime
and calls the C ABI directly, with no Python in between - runs the forward pass
(pooling, routing, attention) whose outputs are then checked against the oracle
on every row."""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import chunk_routed_sparse_b200 as moc
import moc_workloads as W
import oracle
from conftest import ROOT
from parity import attend_reference, compare_attention, compare_routing

CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")
PKG = os.path.join(ROOT, "chunk_routed_sparse_b200")
ANCHOR = {"shot": 0, "local": 1, "chunk": 2}


def _need_toolchain():
    if shutil.which("gcc") is None:
        pytest.skip("gcc not found")
    if not os.path.exists(os.path.join(CUDA, "include", "cuda_runtime_api.h")):
        pytest.skip("CUDA headers not found")
    moc.lib()  # raises if libmoc.so is missing


def _build_client(tmp_path) -> str:
    _need_toolchain()
    exe = str(tmp_path / "moc_client")
    cmd = ["gcc", "-std=c11", "-O2", "-Wall", "-Wextra", "-pedantic", "-Werror",
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           os.path.join(ROOT, "tests", "c", "moc_client.c"), "-o", exe,
           "-L", PKG, "-lmoc", "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-lm",
           f"-Wl,-rpath,{PKG}", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    return exe


def test_header_compiles_as_strict_c99(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not found")
    src = tmp_path / "inc.c"
    src.write_text('#include "moc.h"\nint main(void) { return moc_status_string(MOC_OK) == 0; }\n')
    res = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-c",
                          "-I", os.path.join(ROOT, "include"), str(src), "-o", str(tmp_path / "inc.o")],
                         capture_output=True, text=True)
    assert res.returncode == 0, res.stderr


def test_c_client_host_only_calls(tmp_path):
    exe = _build_client(tmp_path)
    res = subprocess.run([exe, "--host-only"], capture_output=True, text=True, timeout=60)
    assert res.returncode == 0 and res.stdout.strip() == "ok", res.stderr


def _write_input(path, wl, Q, K, V):
    segs = wl.segments
    hdr = [0x4d6f4331, len(segs), ANCHOR[wl.anchor], wl.radius, wl.B, wl.H, wl.d, wl.k, int(wl.causal)]
    with open(path, "wb") as f:
        f.write(np.array(hdr, dtype="<i4").tobytes())
        for field in ("length", "kind", "shot", "frame"):
            f.write(np.array([getattr(s, field) for s in segs], dtype="<i4").tobytes())
        for t in (Q, K, V):
            f.write(t.contiguous().view(torch.int16).numpy().astype("<i2").tobytes())


@pytest.mark.gpu
@pytest.mark.parametrize("which", ["tiny", "ragged_d128"])
def test_c_client_forward_matches_oracle(tmp_path, which):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    if which == "tiny":
        wl = W.tiny()
    else:
        segs = [W.Segment(37, W.CAPTION, 0, -1)]
        for i, ln in enumerate([1, 64, 65, 127, 128, 129, 200, 3, 300, 17]):
            segs.append(W.Segment(ln, W.VIDEO, i // 4, i % 4))
        wl = W.custom("ragsmall", 2, 3, 128, segs, "shot", 0, True, 3, 31, "frame")
    exe = _build_client(tmp_path)
    Q, K, V = W.make_qkv(wl)
    _write_input(tmp_path / "in.bin", wl, Q, K, V)
    res = subprocess.run([exe, str(tmp_path / "in.bin"), str(tmp_path / "out.bin")],
                         capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr
    B, H, L, d, k = wl.B, wl.H, wl.L, wl.d, wl.k
    raw = (tmp_path / "out.bin").read_bytes()
    no, nl = B * H * L * d * 2, B * H * L * 4
    assert len(raw) == no + nl + B * H * L * k * 4
    O = torch.from_numpy(np.frombuffer(raw[:no], dtype="<i2").copy()).view(torch.bfloat16).view(B, H, L, d)
    lse = torch.from_numpy(np.frombuffer(raw[no:no + nl], dtype="<f4").copy()).view(B, H, L)
    sel = np.frombuffer(raw[no + nl:], dtype="<i4").reshape(B, H, L, k)
    orc = oracle.Layout(wl)
    w1 = wl.replace(B=1, H=1)
    for b in range(B):
        for h in range(H):
            q, kk, v = (t[b:b + 1, h:h + 1].contiguous() for t in (Q, K, V))
            kbar_o = oracle.pool(w1, kk, orc)
            rt = oracle.route(w1, q, kbar_o, lay=orc)
            r = rt["rows"]
            sel_g = np.ascontiguousarray(sel[b:b + 1, h:h + 1][:, :, r, :])
            rr = compare_routing(w1, q, kbar_o, sel_g, rt, orc)
            O_o, lse_o = attend_reference(w1, q, kk, v, rt["sel"], sel_g, r, orc, rr)
            compare_attention(O[b:b + 1, h:h + 1][:, :, r], lse[b:b + 1, h:h + 1][:, :, r], O_o, lse_o)
