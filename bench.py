#!/usr/bin/env python
"""Benchmark: tile-sparse attention forward (FG-Attn style) on B200.

One step = the whole hot path over one attention call of the workload:
mask compaction (packed tile bitmask -> kept key lists) followed by the
tile-sparse attention forward.  Default workload: the Wan-480p-like layer
(B1 H40 L32760 d128, M64 N16, window + temporal stripe + random tiles at 70%
score sparsity).  Metric: effective TFLOP/s counted on unskipped work
(4 d FLOP per kept score) and ms per attention call.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

N > 1 runs under torch.distributed (one process per GPU); every rank owns its
own 40 heads (weak scaling, no collective on the data path); timing is the max
over ranks.  `--impl reference` times the plain CPU oracle on the host cores
on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "effective TFLOP/s (unskipped) & ms per attention call; % of B200 BF16 TC peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_setup(n):
    if n <= 1 or "RANK" not in os.environ:
        return 0, 1, None
    import datetime
    import torch.distributed as dist
    rank = int(os.environ["RANK"])
    world = int(os.environ["WORLD_SIZE"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    backend = "nccl" if torch.cuda.is_available() else "gloo"
    if backend == "nccl":
        torch.cuda.set_device(local)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, dist


def head_shard(H: int, rank: int) -> range:
    """Weak scaling: rank r owns heads [r*H, (r+1)*H) of an (N*H)-head job."""
    return range(rank * H, (rank + 1) * H)


def reduce_max(x: float, dist) -> float:
    """Max of a per-rank scalar (device time of the slowest rank)."""
    if dist is None:
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, flops_per_rank: float, max_ms_per_step: float) -> float:
    """Whole-job effective TFLOP/s: every rank does the same work (weak scaling),
    timed by the slowest rank."""
    return world * flops_per_rank / (max_ms_per_step * 1e-3) / 1e12


def barrier(dist):
    if dist is not None:
        dist.barrier()


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.file = None

    def __enter__(self):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.dev)], stdout=self.file,
                                         stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.file.flush()

    def summary(self):
        self.file.seek(0)
        rows = [r.strip().split(", ") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        rows = [r for r in rows if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        load = sorted(sm)[len(sm) // 4:] if sm else []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


# ---------------------------------------------------------------------------
# traffic figure from the committed ncu summary (valid only for the same kernel source)
# ---------------------------------------------------------------------------
def ncu_traffic(workload, src_hash: str, prefix: str = "fgattn_fwd"):
    if workload is None:
        return None, None
    path = os.path.join(ROOT, "profiles", f"{prefix}_{workload}.json")
    if not os.path.exists(path):
        return None, None
    with open(path) as f:
        prof = json.load(f)
    if prof.get("src_hash") != src_hash:
        return None, prof
    return prof.get("dram_bytes_per_launch"), prof


# ---------------------------------------------------------------------------
# oracle (CPU baseline) on a bounded sample
# ---------------------------------------------------------------------------
class OracleSampler:
    """The plain CPU oracle on seeded query blocks of the workload's first heads."""

    def __init__(self, w: W.Workload, seed: int, nheads: int = 2):
        import oracle as O
        self.w = w
        self.orc = O.get()
        heads = range(min(w.H, nheads))
        self.H = len(heads)
        self.q, self.k, self.v = W.make_qkv(w, seed, heads=heads)
        self.mask = W.make_mask(w, seed, heads=heads)
        _, cnt = self.orc.compact(self.mask, w.B, self.H, w.L, w.M, w.N)  # kept keys per block (FLOP count)
        self.kept_cnt = cnt.reshape(-1)
        self.rows = np.minimum(w.M, w.L - np.arange(w.QB) * w.M)
        self.cores = os.cpu_count() or 1
        self.order = np.random.default_rng(seed + 99).permutation(w.B * self.H * w.QB)
        self.next = 0

    def run(self, min_s: float, max_s: float):
        """Run block batches until min_s of wall time has passed; returns (flops, seconds, blocks)."""
        w = self.w
        flops, nblocks = 0.0, 0
        t0 = time.perf_counter()
        batch = max(self.cores, 8)
        while True:
            if self.next >= self.order.size:
                self.next = 0
            blocks = self.order[self.next:self.next + batch]
            self.next += len(blocks)
            self.orc.attention(self.q, self.k, self.v, self.mask, w.M, w.N, w.scale, blocks=blocks,
                               nthreads=self.cores)
            for blk in blocks:
                flops += 4.0 * w.d * self.rows[int(blk) % w.QB] * float(self.kept_cnt[int(blk)])
            nblocks += len(blocks)
            el = time.perf_counter() - t0
            if el >= min_s or el >= max_s:
                break
        return flops, time.perf_counter() - t0, nblocks


def run_reference(args, w):
    # Under torchrun only rank 0 times the oracle; the other ranks exit without work.
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    samp = OracleSampler(w, args.seed)
    per = max(1.0, 90.0 / max(1, args.steps + args.warmup))  # whole run stays within a few minutes
    flops_total, secs, blocks_total = 0.0, 0.0, 0
    for i in range(args.warmup + args.steps):
        fl, sec, nb = samp.run(min_s=per, max_s=2 * per)
        if i >= args.warmup:
            flops_total += fl
            secs += sec
            blocks_total += nb
    value = flops_total / secs / 1e12
    # one step = one whole attention call; the oracle's time for it is extrapolated
    # from the sample's throughput and the kept work of the sampled heads
    sample_heads_flops = 4.0 * w.d * float((samp.kept_cnt.reshape(-1, w.QB) * samp.rows[None, :]).sum())
    call_flops = sample_heads_flops * w.B * w.H / (w.B * samp.H)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * call_flops / (value * 1e12),
        "ms_per_step_kind": "extrapolated from the sample throughput to one whole attention call",
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": cfg_dict(w, args, False),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": samp.cores, "kind": "oracle",
                         "sample": f"{blocks_total} seeded query blocks of heads 0-1 over {args.steps} steps"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


L2_BYTES = 126 * 1024 * 1024
FLUSH_BYTES = 256 * 1024 * 1024


def cfg_dict(w, args, flush):
    l2 = ("L2 flushed before every step (256 MB write, outside the kernel events)" if flush
          else "inputs larger than L2 (no flush needed)")
    return {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "grid": list(w.grid), "d": w.d, "M": w.M, "N": w.N,
            "sparsity_target": w.sparsity, "mask": w.mask, "qkv": w.qkv, "seed": args.seed,
            "l2": l2, "parallelism": f"heads x{args.gpus} (weak)",
            "path": "dense (no kept lists)" if getattr(args, "dense", False) else
            "tile-sparse, fused (the forward reads the mask; no kept lists)" if getattr(args, "fused", False) else
            "tile-sparse (compaction + forward)",
            "layout": "[B][L][H][d]" if getattr(args, "layout", "bhld") == "blhd" else "[B][H][L][d]"}


def profile_key(w, args):
    """Name of the committed ncu summary for this exact workload (None when overridden)."""
    if args.N is not None or args.sparsity is not None or args.heads is not None or args.dense or \
            args.layout != "bhld" or args.fused:
        return None
    return w.name


# ---------------------------------------------------------------------------
# backward mode: gradients of one attention call over the forward's kept lists
# ---------------------------------------------------------------------------
BWD_METRIC = "effective TFLOP/s of the backward (unskipped; 10 d FLOP per kept score) & ms per call"


def run_backward(args, w, F):
    """One step = fgattn_backward on resident q, k, v, out, dO, lse and kept lists
    (the delta pass, zeroing dk/dv and the gradient kernel).  The forward and the
    compaction that produce its inputs run once, before timing."""
    rank, world, dist = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    heads = head_shard(w.H, rank)
    B, H, L, d, M, N = w.B, w.H, w.L, w.d, w.M, w.N
    QB = w.QB
    q_h, k_h, v_h = W.make_qkv(w, args.seed, heads=heads)
    g_h = W.random_grad(B, H, L, d, seed=args.seed + 17)
    mask_h = W.make_mask(w, args.seed, heads=heads)
    q, k, v, g = (t.to(dev) for t in (q_h, k_h, v_h, g_h))
    mask = torch.from_numpy(mask_h.view(np.int32)).to(dev)
    cap = F.kept_capacity(L)
    kept_idx = torch.empty((B, H, QB, cap), dtype=torch.int32, device=dev)
    kept_cnt = torch.empty((B, H, QB), dtype=torch.int32, device=dev)
    F.compact_mask(mask, B, H, L, M, N, kept_idx=kept_idx, kept_cnt=kept_cnt, cap=cap)
    out, lse = F.forward(q, k, v, kept_idx, kept_cnt, M, N, w.scale)
    dq, dk, dv = (torch.empty((B, H, L, d), dtype=torch.float32, device=dev) for _ in range(3))
    delta = torch.empty((B, H, L), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        F.backward(q, k, v, out, g, lse, kept_idx, kept_cnt, M, N, w.scale, dq=dq, dk=dk, dv=dv, delta=delta)

    step()
    assert F.device_error() == 0, "device error on the first step"
    rows = torch.clamp(L - torch.arange(QB, device=dev) * M, max=M).to(torch.float64)
    kept_scores = float((kept_cnt.to(torch.float64) * rows).sum().item())
    flops_per_step = 10.0 * d * kept_scores
    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v, out, g, kept_idx))
    flush = in_bytes < 2 * L2_BYTES
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if flush else None
    for _ in range(args.warmup):
        if flush:
            flush_buf.zero_()
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    barrier(dist)
    torch.cuda.synchronize()
    with sampler:
        t_start.record(stream)
        for i in range(args.steps):
            if flush:
                flush_buf.zero_()
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier(dist)
    bwd_ms = reduce_max(statistics.mean(a.elapsed_time(b) for a, b in ev), dist)
    total_ms = reduce_max(t_start.elapsed_time(t_end), dist)
    clocks = sampler.summary()
    assert F.device_error() == 0, "device error in the timed region"
    ms_per_step = bwd_ms if flush else total_ms / args.steps
    value = job_throughput(world, flops_per_step, ms_per_step)

    # ---- end to end: pinned host inputs -> compaction + backward -> gradients on the host
    pins = [t.pin_memory() for t in (q_h, k_h, v_h, g_h)]
    out_p, lse_p = out.cpu().pin_memory(), lse.cpu().pin_memory()
    mask_p = torch.from_numpy(mask_h.view(np.int32)).pin_memory()
    grads_h = [torch.empty((B, H, L, d), dtype=torch.float32).pin_memory() for _ in range(3)]
    out_d, lse_d = torch.empty_like(out), torch.empty_like(lse)
    h2d = sum(t.numel() * t.element_size() for t in pins + [out_p, lse_p, mask_p])
    d2h = sum(t.numel() * t.element_size() for t in grads_h)

    def e2e_step():
        for dst, src in zip((q, k, v, g, out_d, lse_d, mask), pins + [out_p, lse_p, mask_p]):
            dst.copy_(src, non_blocking=True)
        F.compact_mask(mask, B, H, L, M, N, kept_idx=kept_idx, kept_cnt=kept_cnt, cap=cap)
        F.backward(q, k, v, out_d, g, lse_d, kept_idx, kept_cnt, M, N, w.scale, dq=dq, dk=dk, dv=dv, delta=delta)
        for dst, src in zip(grads_h, (dq, dk, dv)):
            dst.copy_(src, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier(dist)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1), dist) / args.e2e_steps
    assert F.device_error() == 0, "device error in the end-to-end steps"

    peaks, peak_kind = load_peaks()
    achieved = flops_per_step / (bwd_ms * 1e-3) / 1e12
    from fine_grained_sparse_fgattn_b200 import _build
    traffic, _ = ncu_traffic(profile_key(w, args), _build.kernel_hash("bwd"), "fgattn_bwd")
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "traffic": traffic,
                "peak_kind": f"{peak_kind} bf16 burst", "kernel": f"fgattn_bwd_kernel<{d},{M}>",
                "frac_of_sustained": achieved / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]),
                "flops_per_launch": flops_per_step,
                "timed": "delta pass + dk/dv zeroing + gradient kernel (one fgattn_backward call)"}
    if rank == 0:
        cfg = cfg_dict(w, args, flush)
        cfg["path"] = "tile-sparse backward (fgattn_backward over the forward's kept lists)"
        line = {
            "metric": BWD_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
            "backward_ms": bwd_ms, "achieved_sparsity": 1.0 - kept_scores / (B * H * float(L) * L),
            "roofline": roofline, "cpu_baseline": None,
            "e2e": {"value": job_throughput(world, flops_per_step, e2e_ms), "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "mode": "copy in, compaction + backward, copy dq/dk/dv out (serial)"},
            "gpu_launches": 2 * args.steps, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="wan480p")
    ap.add_argument("--N", type=int, default=None, help="override the tile width N")
    ap.add_argument("--sparsity", type=float, default=None)
    ap.add_argument("--heads", type=int, default=None, help="override H (smaller cases for profiling)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--heads-per-group", type=int, default=2,
                    help="head-group size of the pipelined host-to-host call used for the e2e figure")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layout", default="bhld", choices=["bhld", "blhd"],
                    help="memory layout of q, k, v, out: [B][H][L][d] (contiguous entry point) or "
                         "[B][L][H][d] (strided entry point)")
    ap.add_argument("--dense", action="store_true",
                    help="dense run of the same kernel (no kept lists: every key of every block)")
    ap.add_argument("--fused", action="store_true",
                    help="one kernel per step: the forward reads the mask in place of kept lists "
                         "(fgattn_masked_forward; compaction fused into the forward)")
    ap.add_argument("--backward", action="store_true",
                    help="time the gradients (fgattn_backward) of the workload's attention call instead")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = W.get(args.workload)
    if args.N is not None:
        w = w.with_(N=args.N)
    if args.sparsity is not None:
        w = w.with_(sparsity=args.sparsity)
    if args.heads is not None:
        w = w.with_(H=args.heads)
    if args.impl == "reference":
        return run_reference(args, w)

    import fine_grained_sparse_fgattn_b200 as F  # fails loudly without the CUDA library

    if args.backward:
        return run_backward(args, w, F)
    rank, world, dist = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    heads = head_shard(w.H, rank)
    B, H, L, d, M, N = w.B, w.H, w.L, w.d, w.M, w.N
    QB = w.QB

    # ---- inputs: seeded on the host, then resident in HBM before timing
    q_h, k_h, v_h = W.make_qkv(w, args.seed, heads=heads)
    if args.layout == "blhd":  # [B][L][H][d] storage, used through [B][H][L][d] views
        q_h, k_h, v_h = (t.transpose(1, 2).contiguous().transpose(1, 2) for t in (q_h, k_h, v_h))
    mask_h = W.make_mask(w, args.seed, heads=heads)
    q, k, v = (t.transpose(1, 2).to(dev).transpose(1, 2) if args.layout == "blhd" else t.to(dev)
               for t in (q_h, k_h, v_h))
    mask = torch.from_numpy(mask_h.view(np.int32)).to(dev)
    cap = F.kept_capacity(L)
    kept_idx = torch.empty((B, H, QB, cap), dtype=torch.int32, device=dev)
    kept_cnt = torch.empty((B, H, QB), dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, H, L), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def compact():
        if not args.dense and not args.fused:
            F.compact_mask(mask, B, H, L, M, N, kept_idx=kept_idx, kept_cnt=kept_cnt, cap=cap)

    def forward():
        if args.dense:
            F.forward(q, k, v, None, None, M, N, w.scale, out=out, lse=lse)
        elif args.fused:
            F.masked_forward(q, k, v, mask, M, N, w.scale, out=out, lse=lse)
        else:
            F.forward(q, k, v, kept_idx, kept_cnt, M, N, w.scale, out=out, lse=lse)

    def step():
        compact()
        forward()

    if args.fused:  # the kept-key counts for the FLOP figure, once, outside any timing
        F.compact_mask(mask, B, H, L, M, N, kept_idx=kept_idx, kept_cnt=kept_cnt, cap=cap)
    step()
    assert F.device_error() == 0, "device error on the first step"
    if args.dense:
        kept_cnt.fill_(L)
    rows = torch.clamp(L - torch.arange(QB, device=dev) * M, max=M).to(torch.float64)
    kept_scores = float((kept_cnt.to(torch.float64) * rows).sum().item())
    flops_per_step = 4.0 * d * kept_scores
    sparsity = 1.0 - kept_scores / (B * H * float(L) * L)

    # Inputs (and the kept lists) smaller than twice the L2 would stay cached between
    # steps: flush L2 before every step instead, outside the per-kernel events.
    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v, mask, kept_idx))
    flush = in_bytes < 2 * L2_BYTES
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if flush else None

    for _ in range(args.warmup):
        if flush:
            flush_buf.zero_()
        step()
    torch.cuda.synchronize()

    # ---- device-timed region: K steps, events per kernel on the launching stream
    ev_c = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    ev_f = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    barrier(dist)
    torch.cuda.synchronize()
    with sampler:
        t_start.record(stream)
        for i in range(args.steps):
            if flush:
                flush_buf.zero_()
            ev_c[i][0].record(stream)
            compact()
            ev_c[i][1].record(stream)
            ev_f[i][0].record(stream)
            forward()
            ev_f[i][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier(dist)
    total_ms = reduce_max(t_start.elapsed_time(t_end), dist)
    fwd_ms = statistics.mean(a.elapsed_time(b) for a, b in ev_f)
    cmp_ms = statistics.mean(a.elapsed_time(b) for a, b in ev_c)
    fwd_ms = reduce_max(fwd_ms, dist)
    cmp_ms = reduce_max(cmp_ms, dist)
    clocks = sampler.summary()
    assert F.device_error() == 0, "device error in the timed region"
    # with a flush between steps the step time is the two kernels' event time
    ms_per_step = (reduce_max(fwd_ms + cmp_ms, dist) if flush else total_ms / args.steps)
    value = job_throughput(world, flops_per_step, ms_per_step)

    # ---- end to end through the public API: pinned host inputs -> device -> host results
    if args.layout == "blhd":
        qp, kp, vp = (t.transpose(1, 2).pin_memory().transpose(1, 2) for t in (q_h, k_h, v_h))
    else:
        qp, kp, vp = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
    mp = torch.from_numpy(mask_h.view(np.int32)).pin_memory()
    out_h = torch.empty_like(out, device="cpu").pin_memory() if args.layout == "bhld" else \
        torch.empty((B, L, H, d), dtype=out.dtype).pin_memory().transpose(1, 2)
    lse_h = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (qp, kp, vp, mp))
    d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * lse_h.element_size()

    # Contiguous tile-sparse runs go through the host-to-host entry point, which overlaps
    # the copies of one head group with the kernels of another; dense and strided runs
    # copy in, run and copy out one after the other.
    pipelined = args.layout == "bhld" and not args.dense and not args.fused
    buffers = {"q": q, "k": k, "v": v, "mask": mask, "kept_idx": kept_idx, "kept_cnt": kept_cnt, "out": out,
               "lse": lse}

    def e2e_step():
        if pipelined:
            F.attention_from_host(qp, kp, vp, mp, M, N, w.scale, buffers=buffers, out=out_h, lse=lse_h,
                                  heads_per_group=args.heads_per_group)
            return
        q.copy_(qp, non_blocking=True)
        k.copy_(kp, non_blocking=True)
        v.copy_(vp, non_blocking=True)
        mask.copy_(mp, non_blocking=True)
        step()
        out_h.copy_(out, non_blocking=True)
        lse_h.copy_(lse, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier(dist)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1), dist) / args.e2e_steps
    e2e_value = job_throughput(world, flops_per_step, e2e_ms)

    # ---- roofline for the dominant kernel (the forward): tensor-bound on kept FLOPs
    peaks, peak_kind = load_peaks()
    achieved = flops_per_step / (fwd_ms * 1e-3) / 1e12
    from fine_grained_sparse_fgattn_b200 import _build
    # 128-row query blocks (M = 128 lists, dense runs) run the query-major kernel
    qm = args.dense or M == 128
    gather = not args.dense and min(N, L) % 16 != 0
    strided = args.layout != "bhld"
    tf = lambda x: str(bool(x)).lower()
    if qm:
        kname = f"fgattn_fwd_qm_kernel<{d},{tf(gather)},{tf(strided)},{tf(args.fused)}>"
        traffic, _ = ncu_traffic(profile_key(w, args), _build.kernel_hash("fwd_qm"), "fgattn_fwd_qm")
    else:
        kname = f"fgattn_fwd_kernel<{d},{M},{tf(gather)},{tf(strided)},{tf(args.fused)}>"
        traffic, _ = ncu_traffic(profile_key(w, args), _build.kernel_hash("fwd"))
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "traffic": traffic,
                "peak_kind": f"{peak_kind} bf16 burst",
                "kernel": kname,
                "frac_of_sustained": achieved / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]),
                "flops_per_launch": flops_per_step}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        samp = OracleSampler(w, args.seed)
        fl, sec, nb = samp.run(min_s=12.0, max_s=30.0)
        cpu = {"value": fl / sec / 1e12, "unit": "TFLOP/s", "cores": samp.cores, "kind": "oracle",
               "sample": f"{nb} seeded query blocks of heads 0-1 ({sec:.1f} s wall)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg_dict(w, args, flush),
            "forward_ms": fwd_ms, "compact_ms": cmp_ms, "achieved_sparsity": sparsity,
            "pct_of_bf16_peak": 100.0 * value / peaks["bf16_tflops"],
            "roofline": roofline, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "mode": (f"fgattn_attention_from_host: copies overlapped with the kernels, "
                             f"{args.heads_per_group} heads per group") if pipelined
                    else "copy in, run, copy out (serial)"},
            "gpu_launches": (1 if args.dense or args.fused else 2) * args.steps, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
