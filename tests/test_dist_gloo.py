"""Multi-rank host logic on CPU (gloo): in bench.py each replica rank gets an
independent scene, times are reduced with max over ranks, and the reference arm
prints one line from rank 0 while the other rank exits 0; the head split, the
all-gather of its shares and the sequence re-sharding of
chunk_routed_sparse_b200.sharding cover every slice and token exactly once."""
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


def test_head_split_covers_every_slice_once_and_balanced():
    from chunk_routed_sparse_b200 import sharding
    for B, H in [(1, 24), (2, 24), (1, 5), (3, 7)]:
        for world in (1, 2, 3, 4, 8):
            shares = [sharding.shard_slices(B, H, world, r) for r in range(world)]
            covered = [i for a, b in shares for i in range(a, b)]
            assert covered == list(range(B * H)), (B, H, world)
            sizes = [b - a for a, b in shares]
            assert max(sizes) - min(sizes) <= 1


def _gather_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import moc_workloads as W
    from chunk_routed_sparse_b200 import sharding
    wl = W.tiny().replace(B=2, H=3)            # 6 slices over `world` ranks
    s0, s1 = sharding.shard_slices(wl.B, wl.H, world, rank)
    q, _, _ = W.make_qkv_slices(wl, s0, s1)    # this rank's share of the scene's Q
    full = sharding.gather_slices(q.view(s1 - s0, wl.L, wl.d), wl.B * wl.H, world)
    out[rank] = full.view(torch.int16).numpy().tobytes()
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_head_split_shares_reassemble_the_whole_tensor(world):
    """Each rank generates only its slices; the all-gather of the shares must
    equal the whole tensor built by one process on the CPU."""
    import moc_workloads as W
    wl = W.tiny().replace(B=2, H=3)
    ref, _, _ = W.make_qkv(wl)
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_gather_worker, args=(world, port, out), nprocs=world, start_method="spawn")
        got = [out[r] for r in range(world)]
    want = ref.view(wl.B * wl.H, wl.L, wl.d).view(torch.int16).numpy().tobytes()
    assert all(g == want for g in got)


def _reshard_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import moc_workloads as W
    from chunk_routed_sparse_b200 import sharding
    wl = W.tiny().replace(B=2, H=3)
    q, _, _ = W.make_qkv(wl)
    full = q.view(wl.B * wl.H, wl.L, wl.d)
    t0, t1 = sharding.shard_slices(1, wl.L, world, rank)
    s0, s1 = sharding.shard_slices(wl.B, wl.H, world, rank)
    xs = full[:, t0:t1].contiguous()            # this rank's token share of every slice
    xh = sharding.seq_to_heads(xs, wl.B * wl.H, wl.L, world, rank)
    back = sharding.heads_to_seq(xh, wl.B * wl.H, wl.L, world, rank)
    lse = torch.arange(wl.B * wl.H * wl.L, dtype=torch.float32).view(wl.B * wl.H, wl.L)
    lh = sharding.seq_to_heads(lse[:, t0:t1].contiguous(), wl.B * wl.H, wl.L, world, rank)
    out[rank] = (torch.equal(xh.view(torch.int16), full[s0:s1].view(torch.int16)),
                 torch.equal(back.view(torch.int16), xs.view(torch.int16)),
                 torch.equal(lh, lse[s0:s1]), tuple(xh.shape))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 5])
def test_sequence_shards_reshard_to_the_head_split_and_back(world):
    """A caller holding sequence shards (contiguous token ranges of every slice,
    uneven at 5 ranks: 2,112 tokens, 6 slices) gets exactly the head split's
    slices over all tokens from seq_to_heads (one all-to-all), and heads_to_seq
    returns its own token share bit for bit; bf16 [.., L, d] and fp32 [.., L]
    tensors both."""
    from chunk_routed_sparse_b200 import sharding
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_reshard_worker, args=(world, port, out), nprocs=world, start_method="spawn")
        got = [out[r] for r in range(world)]
    for r, (heads_ok, back_ok, lse_ok, shape) in enumerate(got):
        s0, s1 = sharding.shard_slices(2, 3, world, r)
        assert heads_ok and back_ok and lse_ok, r
        assert shape == (s1 - s0, 2112, 64)
