"""Benchmark of the MoC sparse-attention forward pass (one JSON line on rank 0).

A step is one pass of the whole hot path over one scene: (1) pool keys,
(2) route, (3) build query lists, (4) attend, (5) merge - the stage calls
moc_attention_fwd makes. The variant with (5) fused into (4)
(moc_attend_merged) is timed once after the steps, beside it. Default workload:
the eight-shot 180,512-token scene (B=1, H=24, d=128, k=3). Inputs are larger
than L2 (3 x 1.1 GB), so no L2 flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--config eight|single|tiny|ragged|stress] [--k K]
                  [--shard heads|replicas] [--gather]

Under torchrun (N > 1) the ranks split one scene's B*H (b, h) slices into
contiguous shares (``--shard heads``, the default: strong scaling, the total
work is fixed) or each run an independent scene (``--shard replicas``: weak
scaling). Every stage is independent per slice, so neither has a collective on
the data path; ``--gather`` all-gathers the output shares afterwards, outside
the timed regions. Times are CUDA-event device times, max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moc_workloads as W  # noqa: E402
from chunk_routed_sparse_b200.sharding import (gather_slices, heads_to_seq, seq_to_heads,  # noqa: E402,F401
                                                shard_slices)

METRIC = "MoC fwd tokens/s and selected-pair TFLOP/s (% bf16 peak) at 180k tokens"
STAGES = ["pool", "route", "qlist", "attend", "merge"]
# kernel of the attention stage (moc_set_attend_kernel): the library's default, the
# single-CTA kernel, or the CTA-pair kernel (bf16, d = 128)
ATTEND_KERNELS = {"default": 0, "single": 1, "pair": 2}
LAUNCHES_PER_STEP = {"pool": 1, "route": 1, "qlist": 4, "attend": 1, "merge": 1}
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def workload(name: str, k, heads=None):
    wl = W.CONFIGS[name]()
    if heads is not None:  # fewer heads of the same scene (profiling captures)
        wl = wl.replace(H=heads)
    return wl.with_k(k) if k is not None else wl


def workload_string(wl, C: int) -> str:
    """The workload name both arms print in config.workload."""
    return (f"{wl.name}: B={wl.B} H={wl.H} L={wl.L} d={wl.d} k={wl.k} chunks={C} "
            f"anchor={wl.anchor} causal={wl.causal}")


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class ClockSampler:
    """nvidia-smi SM clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.skip = 0

    def start(self):
        """Start sampling every 100 ms and return once the first sample is in
        (nvidia-smi takes a while to start); mark() then sets where the counted
        samples begin."""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
            return
        t0 = time.time()
        while not self.lines and time.time() - t0 < 5.0 and self.proc.poll() is None:
            time.sleep(0.01)
        self.skip = len(self.lines)

    def mark(self):
        """Count only the samples taken from now on (the timed region)."""
        self.skip = len(self.lines)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = self.lines[self.skip:] or self.lines
        for ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


def kernel_traffic():
    """Per-launch DRAM bytes of the attend kernel from the committed ncu
    summary, if it was taken on the current kernel source (else None)."""
    src = os.path.join(ROOT, "chunk_routed_sparse_b200", "csrc", "k_attend_tc.cu")
    summ = os.path.join(ROOT, "profiles", "attend_traffic.txt")
    if not os.path.exists(summ):
        return None
    vals = {}
    with open(summ) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                a, b = line.split(":", 1)
                vals[a.strip()] = b.strip()
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if vals.get("source_sha256_16") != h or "dram_bytes_per_launch_full_scene" not in vals:
        return None
    return float(vals["dram_bytes_per_launch_full_scene"])


def selected_pairs(layout_tables, n_slices: int, wl, sel: torch.Tensor) -> int:
    """Kept (query, key) pairs of ``n_slices`` (b, h) slices: anchor pairs from
    the layout's group key counts plus the sizes of the selected chunks."""
    grp, ar, ar_off = layout_tables
    anchor = 0
    for g in range(len(grp) // 2):
        nq = grp[2 * g + 1] - grp[2 * g]
        keys = sum(ar[2 * x + 1] - ar[2 * x] for x in range(ar_off[g], ar_off[g + 1]))
        anchor += nq * keys
    anchor *= n_slices
    ln = torch.tensor([s.length for s in wl.segments], dtype=torch.int64, device=sel.device)
    routed = int(ln[sel[sel >= 0].long()].sum().item()) if sel.numel() else 0
    return anchor + routed


def scene_for_rank(wl, rank: int):
    """Weak scaling: every rank runs an independent scene of the same shape."""
    return wl.replace(seed=wl.seed + 1000 * rank)


def sum_over_ranks(values, device=None):
    """Element-wise sum of a list of floats over all ranks (identity at N=1)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return [float(v) for v in t.tolist()]


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity at N=1)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def run_ours(args):
    import chunk_routed_sparse_b200 as moc

    ws_, rank, local = dist_env()
    torch.cuda.set_device(local)
    if args.attend_kernel == "pair" and W.CONFIGS[args.config]().d != 128:
        raise SystemExit("--attend-kernel pair: the CTA-pair kernel is built for d = 128 only")
    moc.set_attend_kernel(ATTEND_KERNELS[args.attend_kernel])
    if ws_ > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    shard = args.shard if ws_ > 1 else "none"
    if shard == "heads":
        # one scene; this rank runs its share of the (b, h) slices (every stage is
        # independent per slice and the layout is shared, so a share runs as B=1,
        # H = its slice count)
        wl = workload(args.config, args.k, args.heads)
        s0, s1 = shard_slices(wl.B, wl.H, ws_, rank)
        Qh, Kh, Vh = W.make_qkv_slices(wl, s0, s1)
        B, H = 1, s1 - s0
    else:
        wl = scene_for_rank(workload(args.config, args.k, args.heads), rank)
        s0, s1 = 0, wl.B * wl.H
        Qh, Kh, Vh = W.make_qkv(wl)
        B, H = wl.B, wl.H
    L, d, k = wl.L, wl.d, wl.k
    Qh, Kh, Vh = Qh.pin_memory(), Kh.pin_memory(), Vh.pin_memory()
    dev = torch.device("cuda", local)
    Q, K, V = (t.to(dev, non_blocking=False) for t in (Qh, Kh, Vh))
    lay = moc.Layout.from_workload(wl, device=local)
    kbar = torch.empty(B, H, lay.C, d, dtype=torch.float32, device=dev)
    sel = torch.empty(B, H, L, k, dtype=torch.int32, device=dev)
    ws = moc.workspace(lay, B, H, d, k, dev)
    O = torch.empty_like(Q)
    lse = torch.empty(B, H, L, dtype=torch.float32, device=dev)
    scale = 1.0 / math.sqrt(d)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev: ev[0].record(stream)
        moc.pool_keys(lay, K, out=kbar)
        if ev: ev[1].record(stream)
        if k > 0:
            moc.route(lay, Q, kbar, k, wl.causal, out=sel)
        if ev: ev[2].record(stream)
        moc.build_qlists(lay, sel, B, H, k, ws)
        if ev: ev[3].record(stream)
        moc.attend_partials(lay, Q, K, V, k, ws, scale)
        if ev: ev[4].record(stream)
        moc.merge(lay, sel, k, ws, O, lse)
        if ev: ev[5].record(stream)

    # clocks are sampled from before the warm-up steps (the sampler takes a while to
    # start) and counted from the start of the timed region
    clocks = ClockSampler(local)
    clocks.start()
    for _ in range(args.warmup):
        step()
    moc.check_device_error(ws)
    torch.cuda.synchronize()
    pairs = selected_pairs((lay.table(1), lay.table(2), lay.table(3)), B * H, wl, sel)
    flops = 4.0 * d * pairs

    def barrier():
        if ws_ > 1:
            torch.distributed.barrier()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(STAGES) + 1)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    clocks.mark()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    stage_ms = {s: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs)
                for j, s in enumerate(STAGES)}
    moc.check_device_error(ws)
    fused = fused_timing(moc, lay, Q, K, V, sel, k, ws, scale, stream, B, H, L)

    # end to end through the C ABI's host-buffer call (moc_forward_host): pinned host
    # Q, K, V in, host O back; inside, chunks of heads are uploaded, computed and
    # downloaded on three streams so that the copies overlap the kernels
    Oh = torch.empty_like(Qh).pin_memory()
    devbuf = torch.empty(moc.forward_host_device_bytes(lay, B, H, d, k), dtype=torch.uint8, device=dev)
    moc.forward_host(lay, Qh, Kh, Vh, k, causal=wl.causal, scale=scale, dev=devbuf, out=Oh,
                     want_lse=False)  # untimed first call
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = args.steps
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e2e_steps):
        moc.forward_host(lay, Qh, Kh, Vh, k, causal=wl.causal, scale=scale, dev=devbuf, out=Oh,
                         want_lse=False)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    del devbuf

    gather = None
    if shard == "heads" and args.gather:
        # the whole O on every rank, outside the timed regions (NCCL all-gather of
        # the slice shares, which sit in rank order in the [B*H, L, d] layout)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        O_all = gather_slices(O.view(H, L, d), wl.B * wl.H, ws_)
        g1.record(stream)
        torch.cuda.synchronize()
        gather = {"ms": g0.elapsed_time(g1), "bytes_per_rank_in": O.numel() * 2,
                  "shape": list(O_all.shape)}
        del O_all

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dev)
    job_pairs = int(sum_over_ranks([float(pairs)], dev)[0])

    ms_per_step = total_ms / args.steps
    tokens = B * L
    # whole-job tokens per step: the head shares of one scene add up to that scene;
    # replicas each run a scene of their own
    job_tokens = wl.B * L if shard == "heads" else ws_ * tokens
    peaks, peak_src = load_peaks()
    att_s = stage_ms["attend"] / 1e3
    achieved_tf = flops / att_s / 1e12
    peak_tf = float(peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"]))
    traffic = kernel_traffic()
    # dense pairs of everything the job computed (the whole scene for a head split)
    dense_pairs = (wl.B * wl.H if shard == "heads" else ws_ * B * H) * L * L
    parallelism = {"none": "single GPU",
                   "heads": f"head split x{ws_}: slices [{s0}, {s1}) of {wl.B * wl.H} on rank {rank}; "
                            "no collective on the data path",
                   "replicas": f"replicas x{ws_} (independent scenes, no collective)"}[shard]
    line = {
        "metric": METRIC,
        "value": job_tokens / (ms_per_step / 1e3),
        "unit": "tokens/s",
        "n_gpus": ws_,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        # the series the same command forms over N: --shard heads splits one scene
        # (total work fixed, also at N = 1), --shard replicas adds a scene per rank
        "scaling": "strong" if args.shard == "heads" else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) + per-shot/per-frame mean offsets; no dataset)",
        "config": {"workload": workload_string(wl, lay.C),
                   "tokens_per_step_per_gpu": tokens if shard != "heads" else wl.B * L * H / (wl.B * wl.H),
                   "l2": "inputs larger than L2 (3 x %.2f GB), no flush" % (Q.numel() * 2 / 1e9),
                   "parallelism": parallelism,
                   "attend_kernel": args.attend_kernel},
        "selected_pair_tflops_attend": achieved_tf,
        "selected_pair_tflops_step": 4.0 * d * job_pairs / (ms_per_step / 1e3) / 1e12,
        "pct_bf16_peak_attend": 100.0 * achieved_tf / peak_tf,
        "stage_ms": stage_ms,
        "pruned_fraction": 1.0 - job_pairs / dense_pairs,
        "kept_pairs": job_pairs,
        "roofline": {"bound": "tensor", "kernel": "attend (4)", "achieved": achieved_tf,
                     "peak": peak_tf, "unit": "TFLOP/s", "frac": achieved_tf / peak_tf,
                     "peak_kind": f"bf16_tflops_sustained ({peak_src})",
                     "frac_of_burst": achieved_tf / float(peaks.get("bf16_tflops", 1590.0)),
                     "traffic": traffic},
        "hbm_kernels": hbm_fracs(stage_ms, B, H, L, lay.C, d, k, peaks, routed_rows(lay, wl),
                                 int((sel >= 0).sum().item()) if k > 0 else 0),
        "fused_attend_merge": fused,
        "clocks": clk,
        "e2e": {"value": job_tokens / (e2e_ms / 1e3), "unit": "tokens/s",
                "ms_per_step": e2e_ms,
                "path": "moc_forward_host: host buffers, 12 chunks of heads, copies overlapped",
                "h2d_bytes_per_step": 3 * Q.numel() * 2, "d2h_bytes_per_step": O.numel() * 2},
        "gpu_launches": args.steps * sum(LAUNCHES_PER_STEP.values()),
        "gpu_launches_breakdown": {"per_step": LAUNCHES_PER_STEP,
                                   "note": "kernels of this library in the device-timed steps"},
    }
    if gather is not None:
        line["gather"] = gather
    if not args.no_backward:
        line["backward"] = backward_timing(moc, lay, Q, K, V, O, lse, sel, k, pairs, d, stream, peak_tf)
    if d == 128 and not args.no_e4m3:
        line["e4m3_variant"] = e4m3_timing(moc, lay, Q, K, V, O, sel, k, ws, scale, stream, pairs, peak_tf)
    if ws_ == 1 and not args.no_dense_compare:
        line["dense_compare"] = dense_compare(moc, wl, Q, K, V, O, lse, stream, pairs,
                                              stage_ms, ms_per_step, peak_tf)
    if rank == 0 and ws_ == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, Qh, Kh, Vh, budget_s=args.cpu_budget)
        line["routing_check"] = routing_check(wl, Qh, Kh, sel.cpu().numpy())
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws_ > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def flop_matched_blocks(L: int, pairs_per_head: float):
    """Equal video blocks of s tokens (n of them, plus one block of the r left over)
    whose block-diagonal dense attention keeps as many (query, key) pairs per head as
    the MoC scene: n s^2 + r^2 closest to pairs_per_head, with n s + r = L."""
    s0 = max(1, int(pairs_per_head // L))
    best = None
    for s_ in range(max(1, s0 - 4000), min(L, s0 + 4000) + 1):
        n, r = divmod(L, s_)
        err = abs(n * s_ * s_ + r * r - pairs_per_head)
        if best is None or err < best[0]:
            best = (err, s_, n, r)
    return best[1], best[2], best[3]


def dense_compare(moc, wl, Q, K, V, O, lse, stream, moc_pairs, stage_ms, moc_step_ms, peak_tf):
    """The same attention kernel on two anchor-only layouts of the scene's length
    (k = 0, so no routing and one partial per row):
      dense - one caption segment and one shot holding every frame, so every
              query attends every key (L^2 pairs per head);
      flop_matched - equal video blocks (``flop_matched_blocks``), block-diagonal
              dense attention with the MoC scene's kept-pair count per head (within
              0.1 %), which separates the pruning gain from the cost of routing,
              query lists, gathered tiles and the merge.
    Pool -> attention (query lists, attend, merge) is timed with CUDA events over
    3 runs after 2 warm-up runs, on the resident Q, K, V."""
    import moc_workloads as Wm
    B, L, d, H = wl.B, wl.L, wl.d, wl.H
    n_cap = sum(sg.length for sg in wl.segments if sg.kind == Wm.CAPTION)
    n_fr, rest = divmod(L - n_cap, 1500)
    blk, n_blk, r_blk = flop_matched_blocks(L, moc_pairs / (B * H))
    scenes = {
        "dense": [Wm.Segment(n_cap, Wm.CAPTION, -1, -1)]
                 + [Wm.Segment(1500 + (rest if f == n_fr - 1 else 0), Wm.VIDEO, 0, f) for f in range(n_fr)],
        "flop_matched": [Wm.Segment(blk, Wm.VIDEO, s_, 0) for s_ in range(n_blk)]
                        + ([Wm.Segment(r_blk, Wm.VIDEO, n_blk, 0)] if r_blk else []),
    }
    out = {}
    for name, segs in scenes.items():
        assert sum(sg.length for sg in segs) == L
        w2 = Wm.custom(name, B, H, d, segs, anchor="shot", causal=True, k=0)
        lay = moc.Layout.from_workload(w2, device=Q.device.index)
        ws = moc.workspace(lay, B, H, d, 0, Q.device)
        kbar = torch.empty(B, H, lay.C, d, dtype=torch.float32, device=Q.device)
        # dense: every query sees every key; block-diagonal: every query its own block
        pairs = B * H * L * L if name == "dense" else B * H * sum(sg.length ** 2 for sg in segs)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        att, tot = [], []
        for it in range(5):
            ev[0].record(stream)
            moc.pool_keys(lay, K, out=kbar)
            ev[1].record(stream)
            moc.attention_fwd(lay, Q, K, V, None, 0, ws=ws, O=O, lse=lse)
            ev[2].record(stream)
            torch.cuda.synchronize()
            if it >= 2:
                tot.append(ev[0].elapsed_time(ev[2]))
                att.append(ev[1].elapsed_time(ev[2]))
        moc.check_device_error(ws)
        a, t = statistics.mean(att), statistics.mean(tot)
        out[name] = {"pairs": pairs, "attention_ms": a, "step_ms": t,
                     "tflops": 4.0 * d * pairs / (a / 1e3) / 1e12,
                     "frac_sustained": 4.0 * d * pairs / (a / 1e3) / 1e12 / peak_tf}
        del ws
    moc_attention_ms = stage_ms["qlist"] + stage_ms["attend"] + stage_ms["merge"]
    out["flop_matched"]["blocks"] = {"tokens": blk, "count": n_blk, "rest": r_blk}
    out["moc_pairs"] = moc_pairs
    out["moc_step_speedup_vs_dense"] = out["dense"]["step_ms"] / moc_step_ms
    out["moc_attention_vs_flop_matched"] = moc_attention_ms / out["flop_matched"]["attention_ms"]
    return out


def fused_timing(moc, lay, Q, K, V, sel, k, ws, scale, stream, B, H, L, reps=3):
    """(4) with the merge (5) fused into its anchor items' epilogue
    (moc_attend_merged) after the timed steps, on the same query lists; mean of
    ``reps`` after one untimed run, against the step's (4) + (5)."""
    O2 = torch.empty_like(Q)
    lse2 = torch.empty(B, H, L, dtype=torch.float32, device=Q.device)
    ts = []
    moc.build_qlists(lay, sel, B, H, k, ws)
    for it in range(1 + reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        moc.attend_merged(lay, Q, K, V, sel, k, ws, O2, lse2, scale)
        e1.record(stream)
        torch.cuda.synchronize()
        if it >= 1:
            ts.append(e0.elapsed_time(e1))
    moc.check_device_error(ws)
    del O2, lse2
    return {"attend_merged_ms": statistics.mean(ts)}


def e4m3_timing(moc, lay, Q, K, V, O_ref, sel, k, ws, scale, stream, pairs, peak_tf, reps=3):
    """The E4M3 variant of the attention stage on the step's inputs and
    selection: per-slice quantisation of Q, K, V (moc_quantize_e4m3), then
    query lists, the E4M3 attention and the merge (moc_attention_fwd_e4m3);
    CUDA events, mean of ``reps`` after one untimed run. Its output is compared
    with the bf16 path's O of the same step (the effect of E4M3 inputs)."""
    B, H, L, d = Q.shape
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record(stream)
    (Q8, qs), (K8, ks), (V8, vs) = (moc.quantize_e4m3(t) for t in (Q, K, V))
    ev[1].record(stream)
    torch.cuda.synchronize()
    quant_ms = ev[0].elapsed_time(ev[1])
    O8 = torch.empty_like(Q)
    lse8 = torch.empty(B, H, L, dtype=torch.float32, device=Q.device)
    att, tot = [], []
    for it in range(1 + reps):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        e[0].record(stream)
        moc.build_qlists(lay, sel, B, H, k, ws)
        e[1].record(stream)
        moc.lib().moc_attend_partials_e4m3(lay.handle, B, H, d, moc._ptr(Q8), moc._ptr(K8), moc._ptr(V8),
                                           moc._ptr(qs), moc._ptr(ks), moc._ptr(vs), k, float(scale),
                                           moc._ptr(ws), ws.numel(), moc._stream())
        e[2].record(stream)
        moc.merge(lay, sel, k, ws, O8, lse8)
        e[3].record(stream)
        torch.cuda.synchronize()
        if it >= 1:
            att.append(e[1].elapsed_time(e[2]))
            tot.append(e[0].elapsed_time(e[3]))
    moc.check_device_error(ws)
    diff = (O8.float() - O_ref.float()).abs()
    a_ms = statistics.mean(att)
    tf = 4.0 * d * pairs / (a_ms / 1e3) / 1e12
    # the E4M3 MMAs' peak: the measured sustained bf16 peak times the nominal fp8 / bf16
    # dense ratio (4.5 / 2.25 PFLOP/s)
    fp8_peak = 2.0 * peak_tf
    out = {"quantize_ms": quant_ms, "attend_ms": a_ms, "attention_stage_ms": statistics.mean(tot),
           "tflops_selected_pairs": tf,
           "roofline": {"bound": "tensor", "achieved": tf, "peak": fp8_peak, "unit": "TFLOP/s",
                        "frac": tf / fp8_peak,
                        "peak_kind": "e4m3: measured sustained bf16 peak x 2 (nominal fp8/bf16 ratio)"},
           "o_vs_bf16_path": {"max_abs": diff.max().item(), "mean_abs": diff.mean().item()}}
    del Q8, K8, V8, O8, lse8
    return out


def backward_timing(moc, lay, Q, K, V, O, lse, sel, k, pairs, d, stream, peak_tf, reps=5):
    """The backward pass (moc_attention_bwd: query lists, D = dO . o, the dQ
    kernel, the dQ reduce, the dK / dV kernel) for a seeded upstream gradient,
    over the forward pass's selection and outputs; CUDA events around each
    call after 2 untimed calls, mean of ``reps``. Selected-pair FLOPs follow the
    usual 2.5x-forward count (10 d per kept pair: S, dP, dV, dK, dQ); the
    kernels execute 14 d (S and dP are formed once per side)."""
    B, H, L, _ = Q.shape
    g = torch.Generator(device=Q.device).manual_seed(99)
    dO = torch.randn(Q.shape, device=Q.device, generator=g).to(torch.bfloat16)
    n = int(moc.lib().moc_attention_bwd_workspace_bytes(lay.handle, B, H, d, k))
    ws = torch.empty(n, dtype=torch.uint8, device=Q.device)
    dQ, dK, dV = torch.empty_like(Q), torch.empty_like(Q), torch.empty_like(Q)
    ts = []
    for it in range(2 + reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        moc.attention_bwd(lay, Q, K, V, O, lse, dO, sel, k, ws=ws, dQ=dQ, dK=dK, dV=dV)
        e1.record(stream)
        torch.cuda.synchronize()
        if it >= 2:
            ts.append(e0.elapsed_time(e1))
    moc.check_device_error(ws)
    ms = statistics.mean(ts)
    del ws, dO, dQ, dK, dV
    t10 = 10.0 * d * pairs / (ms / 1e3) / 1e12
    t14 = 14.0 * d * pairs / (ms / 1e3) / 1e12
    return {"ms": ms, "tflops_selected_pairs_10d": t10, "tflops_executed_14d": t14,
            "frac_sustained_10d": t10 / peak_tf, "frac_sustained_executed_14d": t14 / peak_tf,
            "launches": 4 + 4, "workspace_bytes": n}


def routed_rows(lay, wl) -> int:
    """Query rows (one head) that have at least one routing candidate."""
    grp = lay.table(1)
    cand_off = lay.table(5)
    ncausal = lay.table(6)
    rows = 0
    for g in range(len(grp) // 2):
        n = ncausal[g] if wl.causal else cand_off[g + 1] - cand_off[g]
        if n > 0:
            rows += grp[2 * g + 1] - grp[2 * g]
    return rows


def hbm_fracs(stage_ms, B, H, L, C, d, k, peaks, n_routed_rows, n_valid_sel):
    """Achieved GB/s of the HBM-bound kernels on their algorithmic bytes:
    pool reads K and writes Kbar; route reads the Q rows that have candidates
    and writes sel; merge reads sel, the anchor partial of every row and one
    partial per valid selection (fp32 row + lse), and writes bf16 O + lse."""
    hbm = float(peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"]))
    BH = B * H
    alg = {
        "pool": BH * L * 2 * d + BH * C * d * 4,
        "route": BH * n_routed_rows * 2 * d + BH * L * 4 * k,
        "merge": BH * L * (4 * k + 4 * d + 4 + 2 * d + 4) + n_valid_sel * (4 * d + 4),
    }
    out = {}
    for s, b in alg.items():
        gbs = b / (stage_ms[s] / 1e3) / 1e9
        out[s] = {"bytes": b, "GB/s": gbs, "frac_measured_hbm": gbs / hbm, "frac_8TBs": gbs / 8000.0}
    return out


def cpu_baseline(wl, Qh, Kh, Vh, budget_s: float = 20.0, rows_per_round: int = 64, seed: int = 0):
    """The oracle as it stands, on this host's cores, on a bounded sample: one
    head's pooling plus routing and attention of uniformly drawn query rows
    until ~budget_s of work; scaled to tokens/s of the whole problem."""
    import oracle

    w1 = wl.replace(B=1, H=1)
    q, kk, v = (t[0:1, 0:1].contiguous() for t in (Qh, Kh, Vh))
    lay = oracle.Layout(w1)
    t0 = time.perf_counter()
    kbar = oracle.pool(w1, kk, lay)
    t_pool = time.perf_counter() - t0
    rng = np.random.default_rng(seed)
    n, t_rows = 0, 0.0
    while t_rows < budget_s:
        rows = np.sort(rng.integers(0, lay.L, size=rows_per_round))
        t1 = time.perf_counter()
        rt = oracle.route(w1, q, kbar, rows=rows, lay=lay)
        oracle.attend(w1, q, kk, v, rt["sel"], rows=rows, lay=lay)
        t_rows += time.perf_counter() - t1
        n += len(rows)
    per_head = t_pool + t_rows * lay.L / n
    value = wl.B * wl.L / (per_head * wl.B * wl.H)
    return {"value": value, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": f"head (0,0): pool all {lay.C} chunks ({t_pool:.2f} s) + route/attend "
                      f"{n} uniform query rows ({t_rows:.1f} s); extrapolated to {wl.B}x{wl.H} "
                      f"heads x {lay.L} rows"}


def routing_check(wl, Qh, Kh, sel_gpu, max_heads: int = 24):
    """Routing of the timed run against the oracle (part of the oracle leg):
    every row of up to ``max_heads`` heads, each classified as exact, or as a
    near-tie swap the contract admits (the oracle's near-tie rule; every pick a
    routing candidate of the query, same count, scores in order up to near
    ties), or as inadmissible. Near-tie rows are those whose adjacent sorted
    candidate scores (the k-th and (k+1)-th, or two selected ones) are within
    the tie tolerance, whether or not the GPU's order differs there."""
    import oracle

    t0 = time.perf_counter()
    heads = [(b, h) for b in range(wl.B) for h in range(wl.H)]
    if len(heads) > max_heads:
        step = len(heads) / max_heads
        heads = [heads[int(i * step)] for i in range(max_heads)]
    w1 = wl.replace(B=1, H=1)
    lay = oracle.Layout(w1)
    tot = {"exact": 0, "mismatch": 0, "near_tie_rows": 0, "inadmissible": 0}
    first_bad = None
    for b, h in heads:
        q, kk = (t[b:b + 1, h:h + 1].contiguous() for t in (Qh, Kh))
        kbar = oracle.pool(w1, kk, lay)
        rt = oracle.route(w1, q, kbar, lay=lay)
        res = oracle.check_selection(w1, q, kbar, np.ascontiguousarray(sel_gpu[b:b + 1, h:h + 1]), rt, lay)
        for key in ("exact", "mismatch", "near_tie_rows"):
            tot[key] += res[key]
        tot["inadmissible"] += len(res["bad"])
        if res["bad"] and first_bad is None:
            first_bad = dict(res["bad"][0], b=b, h=h)
    out = {"heads_checked": len(heads), "rows_checked": len(heads) * wl.L, **tot,
           "rule": "near tie: adjacent sorted candidate scores within 1e-4 relative (or 1e-5 of "
                   "sum |q_e Kbar_e|)", "seconds": round(time.perf_counter() - t0, 2)}
    if first_bad is not None:
        out["first_inadmissible"] = first_bad
    return out


def run_reference(args):
    """Reference arm: the CPU oracle, timed on this host's cores (rank 0 only).
    Each step is a bounded sample of the same workload: routing and attention
    of ``rows_per_step`` uniformly drawn query rows of head (0, 0), after the
    head's pooling (done once, before the timed steps). ``value`` is the
    sample's own throughput in whole-problem tokens (a token is one query row
    of every head: rows / (B*H) tokens per step), so value * ms_per_step / 1e3
    is the tokens one step processes; the time the oracle would need for the
    whole scene is reported beside it."""
    ws_, rank, _ = dist_env()
    if rank != 0:
        return
    wl = workload(args.config, args.k, args.heads)
    Qh, Kh, Vh = W.make_qkv(wl, heads=[(0, 0)])
    import oracle
    w1 = wl.replace(B=1, H=1)
    q, kk, v = (t[0:1, 0:1].contiguous() for t in (Qh, Kh, Vh))
    lay = oracle.Layout(w1)
    rng = np.random.default_rng(1)
    rows_per_step = 48
    t0 = time.perf_counter()
    kbar = oracle.pool(w1, kk, lay)
    t_pool = time.perf_counter() - t0
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        rows = np.sort(rng.integers(0, lay.L, size=rows_per_step))
        rt = oracle.route(w1, q, kbar, rows=rows, lay=lay)
        oracle.attend(w1, q, kk, v, rt["sel"], rows=rows, lay=lay)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    step_s = sum(times) / len(times)
    tokens_per_step = rows_per_step / (wl.B * wl.H)
    value = tokens_per_step / step_s
    scene_s = (t_pool + step_s * lay.L / rows_per_step) * wl.B * wl.H
    sample = (f"per step {rows_per_step} uniform query rows of head (0,0) (route + attend) = "
              f"{tokens_per_step:.3f} tokens of the {wl.B}x{wl.H}-head problem; head pooling once "
              f"before timing ({t_pool:.3f} s)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": ws_, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "strong" if args.shard == "heads" else "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_string(wl, lay.C),
                       "tokens_per_step": tokens_per_step},
            "extrapolated_ms_per_scene": scene_s * 1e3,
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="eight", choices=sorted(W.CONFIGS))
    ap.add_argument("--k", type=int, default=None)
    ap.add_argument("--heads", type=int, default=None,
                    help="run the scene with this many heads instead (small profiling captures)")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-e4m3", action="store_true",
                    help="skip the timing of the E4M3 variant of the attention stage")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the timing of the backward pass (moc_attention_bwd) after the forward steps")
    ap.add_argument("--shard", default="heads", choices=["heads", "replicas"],
                    help="N > 1: split one scene's (b, h) slices over the ranks (strong scaling), "
                         "or run an independent scene per rank (weak scaling)")
    ap.add_argument("--gather", action="store_true",
                    help="with --shard heads: all-gather the output slices after the timed steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--attend-kernel", default="default", choices=sorted(ATTEND_KERNELS),
                    help="kernel of the attention stage (the CTA-pair kernel is a measured alternative)")
    ap.add_argument("--no-dense-compare", action="store_true",
                    help="skip the dense and FLOP-matched block-diagonal runs of the attention kernel")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be at least 3 (timing rule: three untimed steps before the timed ones)")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
