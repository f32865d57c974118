"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): each rank
gets an independent scene, times are reduced with max over ranks, and the
reference arm prints one line from rank 0 while the other rank exits 0."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    import moc_workloads as W
    wl = bench.scene_for_rank(W.tiny(), rank)
    q, _, _ = W.make_qkv(wl)
    mx = bench.max_over_ranks([1.0 + rank, 10.0 - rank])
    out[rank] = (wl.seed, float(q.float().sum()), mx)
    dist.barrier()
    dist.destroy_process_group()


def test_ranks_get_independent_scenes_and_max_times():
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:  # no fork of this multi-threaded process
        out = m.dict()
        mp.start_processes(_worker, args=(2, port, out), nprocs=2, start_method="spawn")
        r0, r1 = out[0], out[1]
    assert r0[0] != r1[0] and r0[1] != r1[1]          # different scenes
    assert r0[2] == r1[2] == [2.0, 10.0]              # max over ranks, same on both


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "0", "--gpus", "2"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
