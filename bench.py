#!/usr/bin/env python3
"""Benchmark of Re-ttention's reshaped block-sparse attention hot path on B200.

One step = one pass of the whole hot path over one calibration cycle of the
workload: build the CSR block index of the static mask, one calibration
(full-attention) step on X_0, then the workload's sparse steps on the drifted
inputs X_1..X_n with step distance k = 1..n.  Inputs (all steps' Q/K/V) are
resident in HBM when the timed region starts; each step's inputs (2.1 GB per
attention call for the default long-video workload, 205 MB for CogVideoX)
exceed the 126 MB L2, so no explicit flush is done.

Default workload: the long-video sweep at 3.1 % density (B=1, H=24, L=115200,
d=128, 28 of 900 key blocks kept per query block = 96.9 % sparsity), the
largest configuration; the other workloads run with --workload.

Metric: executed-block TFLOP/s (4 * block^2 * d * kept blocks * B * H per
attention call, true d; calibration executes every block).  The line also
carries per-kernel latency/TFLOP/s, the roofline object of the dominant
kernel, the CPU oracle baseline, the end-to-end number through the public API
with host buffers, one denoising-schedule cycle (call by call and as a captured
CUDA graph, with each step's error against full attention), the token
reordering (the permutation's bandwidth and the mask's locality on raster vs
Hilbert-ordered tokens), and the SM clocks seen during the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
Multi-GPU (weak scaling, independent replicas, no data-path collective):
    python -m torch.distributed.run --nproc-per-node N bench.py --gpus N ...
"""

from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import re
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_attention_diffusion_rt_b200 import inputs  # noqa: E402

METRIC = "sparse-step attention latency & TFLOP/s (executed blocks), % bf16 peak, 1 B200"
DEFAULT_WORKLOAD = "longvideo-3.1"
KERNEL_SOURCES = ("attn_kernel.cuh", "ptx.cuh", "softmax.cuh", "sparse_kernel.cuh", "pp_sparse.cuh",
                  "pp_calibrate.cuh", "cal_kernel.cuh", "attn_launch.h")


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_source_hash():
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "sparse_attention_diffusion_rt_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_tag: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (its 'source_hash' line matches), else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}_{workload}.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m_hash = re.search(r"source_hash:\s*([0-9a-f]+)", txt)
    m_bytes = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    if not m_hash or not m_bytes or m_hash.group(1) != kernel_source_hash():
        return None
    return float(m_bytes.group(1))


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of every rank's x (one all-reduce; every rank must call it)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, flops_per_rank_step: float, ms_per_step: float) -> float:
    """Whole-job throughput of weak-scaled replicas: every rank does the same
    work per step, and a step lasts as long as the slowest rank's."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


class ClockSampler:
    """nvidia-smi SM clock / throttle-reason sampling during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def executed_flops(w: inputs.Workload, nnz_per_head: int) -> float:
    return 4.0 * w.block * w.block * w.d * nnz_per_head * w.B * w.H


# ---------------------------------------------------------------------------
# the step
# ---------------------------------------------------------------------------

class Step:
    """One calibration cycle through the C ABI, with per-kernel CUDA events."""

    def __init__(self, w, mask_dev, qkv_steps, rt):
        self.w, self.mask, self.qkv, self.rt = w, mask_dev, qkv_steps, rt
        q = qkv_steps[0][0]
        like_q = lambda: torch.empty_strided(q.shape, q.stride(), dtype=q.dtype, device=q.device)
        self.o = [like_q() for _ in qkv_steps]          # same strides as the inputs (head-shard views too)
        self.rho = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=q.device)
        self.r = like_q()
        n = len(qkv_steps)
        self.ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        self.times = {"calibrate": [], "sparse": []}
        self.launches = 0

    def run(self, record=False, before=None, after=None):
        """before(s) / after(s), when given, run on the host right before the
        call of sub-step s is enqueued and right after (stream waits and
        event records of a pipelined caller)."""
        rt, w = self.rt, self.w
        idx = rt.rt_build_block_index(self.mask)
        self.launches += 3
        for s in range(len(self.qkv)):
            q, k, v = self.qkv[s]
            if before is not None:
                before(s)
            if record:
                self.ev[s][0].record()
            if s == 0:
                rt.rt_calibrate(q, k, v, idx, block=w.block, o=self.o[0], rho=self.rho, r=self.r)
            else:
                rt.rt_sparse_step(q, k, v, idx, self.rho, self.r, block=w.block, lam=w.lam, step_distance=s,
                                  o=self.o[s])
            if record:
                self.ev[s][1].record()
            if after is not None:
                after(s)
            self.launches += 1
        self.idx = idx

    def collect(self):
        self.times["calibrate"].append(self.ev[0][0].elapsed_time(self.ev[0][1]))
        for s in range(1, len(self.qkv)):
            self.times["sparse"].append(self.ev[s][0].elapsed_time(self.ev[s][1]))


def cpu_oracle_sample(w, qkv_steps_cpu, mask, budget_s=15.0):
    """Time the oracle (as it stands) on a bounded sample of the workload:
    query blocks of head (0, 0), sparse step first, then calibration rows, until
    ~budget_s of CPU time.  Returns (executed-block TFLOP/s, description, cores)."""
    from oracle import reference as ref
    q0, k0, v0 = (x[0, 0].double().numpy() for x in qkv_steps_cpu[0])
    q1, k1, v1 = (x[0, 0].double().numpy() for x in qkv_steps_cpu[min(1, len(qkv_steps_cpu) - 1)])
    L, blk = w.L, w.block
    nqb = w.nqb
    bm = mask[0]
    flops, n_sp, n_cal = 0.0, 0, 0
    t0 = time.perf_counter()
    order = np.random.default_rng(0).permutation(nqb)
    for qb in order:
        rows = np.arange(qb * blk, min(L, (qb + 1) * blk))
        O, RHO, R = ref.calibrate_rows_ref(q0, k0, v0, bm, blk, rows)
        flops += 4.0 * blk * blk * w.d * w.nkb
        n_cal += 1
        ref.sparse_step_rows_ref(q1, k1, v1, bm, blk, rows, RHO, R, w.lam, 1)
        flops += 4.0 * blk * blk * w.d * int(bm[qb].sum())
        n_sp += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    desc = (f"head (0,0) of {w.name}: {n_cal} query blocks calibrated + sparse-stepped "
            f"({n_cal}/{w.B * w.H * nqb} of the cycle's calibration units) in {dt:.1f} s; "
            f"executed-block FLOPs of the sample / CPU time")
    return flops / dt / 1e12, desc, cores


def mask_locality(w, mask, perm=None):
    """How local a static block mask is on the latent grid: the fraction of
    each visual token's 26 grid neighbours that lie in the key blocks kept for
    its query block (neighbour recall), and the mean bounding-box volume, in
    grid cells, of the visual tokens of a block."""
    coords = inputs.token_coords(w, perm)
    F, Y, X = w.grid
    raster = np.arange(w.L) if perm is None else np.asarray(perm, dtype=np.int64)
    pos = np.empty(w.L, dtype=np.int64)
    pos[raster] = np.arange(w.L)                      # raster index -> position
    vis = np.nonzero(~np.isnan(coords[:, 0]))[0]
    c = coords[vis].astype(np.int64)
    m = mask[0].astype(bool)
    hit = total = 0
    for df in (-1, 0, 1):
        for dy in (-1, 0, 1):
            for dx in (-1, 0, 1):
                if df == dy == dx == 0:
                    continue
                nb = c + np.array([df, dy, dx])
                ok = ((nb >= 0) & (nb < np.array([F, Y, X]))).all(axis=1)
                j = pos[w.n_text + (nb[ok, 0] * Y + nb[ok, 1]) * X + nb[ok, 2]]
                hit += int(m[vis[ok] // w.block, j // w.block].sum())
                total += int(ok.sum())
    blk = vis // w.block
    vols = []
    for b in np.unique(blk):
        cb = c[blk == b]
        vols.append(float(np.prod(cb.max(axis=0) - cb.min(axis=0) + 1)))
    return hit / max(total, 1), float(np.mean(vols))


def measure_token_order(w, rt, reps=5):
    """The reordering row: the Hilbert token order, the device permutation's
    bandwidth on one [B, H, L, d] tensor (read + write), and the mask's
    locality on raster vs reordered tokens at the same kept blocks per row."""
    if w.grid is None:
        return None
    perm_h = rt.rt_hilbert_token_order(w.n_text, *w.grid)
    perm = perm_h.cuda()
    x = inputs.initial_qkv(w, device="cuda")[0]
    y = torch.empty_like(x)
    for _ in range(2):
        rt.rt_permute_tokens(x, perm, dst=y)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        rt.rt_permute_tokens(x, perm, dst=y)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    nbytes = 2 * x.numel() * x.element_size()
    ok = bool(torch.equal(y, x[:, :, perm.long()]))
    st = rt.rt_check_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the permutation: {rt.rt_status_string(st)}")
    gbs = nbytes / (ms * 1e-3) / 1e9
    peaks = load_peaks()
    rec_r, vol_r = mask_locality(w, inputs.block_mask(w))
    rec_h, vol_h = mask_locality(w, inputs.block_mask(w, perm_h.numpy()), perm_h.numpy())
    return {"order": "text first, then the grid along its Hilbert curve",
            "permute_ms": ms, "permute_bytes": nbytes, "permute_gbs": gbs,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"]},
            "permute_matches_torch_indexing": ok, "kept_blocks_per_row": w.kept,
            "neighbour_recall": {"raster": rec_r, "hilbert": rec_h},
            "block_bbox_cells": {"raster": vol_r, "hilbert": vol_h}}


def measure_schedule(w, mask, rt, period=5, reps=3):
    """One calibration cycle of the denoising-schedule driver on drifting inputs:
    the cycle run call by call and as one captured CUDA graph (device time per
    cycle), and each step's relative L2 error against full attention on that
    step's inputs, for Re-ttention, the no-rho ablation and DiTFastAttn."""
    dev = mask.device
    steps = inputs.qkv_steps(w, period, device=dev)
    idx = rt.rt_build_block_index(mask)
    q0 = steps[0][0]
    rho = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=dev)
    r = torch.empty_like(q0)
    outs = [torch.empty_like(q0) for _ in range(period)]
    s = torch.cuda.Stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def eager(epilogue=rt.RT_EPI_RESHAPED, residual=rt.RT_RES_MASKED):
        for t, (q, k, v) in enumerate(steps):
            rt.rt_schedule_step(q, k, v, idx, t, block=w.block, period=period, lam=w.lam, o=outs[t], rho=rho,
                                r=r, epilogue=epilogue, residual=residual, stream=s)

    with torch.cuda.stream(s):
        eager()
        s.synchronize()
        e0, e1 = ev(), ev()
        e0.record(s)
        for _ in range(reps):
            eager()
        e1.record(s)
        s.synchronize()
        eager_ms = e0.elapsed_time(e1) / reps
    graph = rt.CycleGraph(steps, idx, block=w.block, outs=outs, rho=rho, r=r, lam=w.lam, stream=s)
    try:
        graph.launch(stream=s)
        s.synchronize()
        e0, e1 = ev(), ev()
        e0.record(s)
        for _ in range(reps):
            graph.launch(stream=s)
        e1.record(s)
        s.synchronize()
        graph_ms = e0.elapsed_time(e1) / reps
    finally:
        graph.close()
    # full attention of every step (the calibration kernel's O), then each method's outputs
    full = []
    for q, k, v in steps:
        o_full, _, _ = rt.rt_calibrate(q, k, v, idx, block=w.block)
        full.append(o_full.float())
    errs = {}
    for name, epi, res in (("rettention", rt.RT_EPI_RESHAPED, rt.RT_RES_MASKED),
                           ("no_rho", rt.RT_EPI_NO_RHO, rt.RT_RES_MASKED),
                           ("ditfastattn", rt.RT_EPI_NO_RHO, rt.RT_RES_SUBTRACTIVE)):
        with torch.cuda.stream(s):
            eager(epi, res)
        s.synchronize()
        errs[name] = [float(torch.linalg.vector_norm(o.float() - f) / torch.linalg.vector_norm(f))
                      for o, f in zip(outs, full)]
    st = rt.rt_check_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the schedule run: {rt.rt_status_string(st)}")
    return {"period": period, "cycle": f"1 calibration + {period - 1} sparse steps (k = 1..{period - 1})",
            "cycle_ms_call_by_call": eager_ms, "cycle_ms_graph": graph_ms, "launches_per_cycle_graph": 1,
            "rel_l2_err_vs_full_per_step": errs,
            "inputs": "synthetic, each step adds 0.05*N(0,1) to Q/K/V (errors are of the synthetic drift)"}


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------

def run_reference(args, rank, world):
    """The oracle timed on the host cores (rank 0 only)."""
    if rank != 0:
        return
    w = inputs.WORKLOADS[args.workload]
    # the timed sample covers head (0, 0) only: draw a one-head problem of the same shape
    steps = inputs.qkv_steps(dataclasses.replace(w, B=1, H=1), 2, device="cpu")
    mask = inputs.block_mask(w)
    budget = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    vals = []
    for i in range(args.warmup + args.steps):
        v, desc, cores = cpu_oracle_sample(w, steps, mask, budget_s=budget)
        if i >= args.warmup:
            vals.append(v)
    value = float(np.median(vals))
    nnz = int(mask.sum())
    step_flops = executed_flops(w, w.nqb * w.nkb) + w.n_sparse_steps * executed_flops(w, nnz)
    ms_step = step_flops / (value * 1e12) * 1e3        # the whole step at the sample's rate (extrapolated)
    desc += f"; ms_per_step extrapolated from the sample's rate to the whole step ({step_flops / 1e12:.1f} TFLOP)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "d": w.d, "block": w.block,
                   "kept_blocks_per_row": w.kept, "sparse_steps": w.n_sparse_steps},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    from sparse_attention_diffusion_rt_b200 import rt
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    rt.load_library()
    w = inputs.WORKLOADS[args.workload]
    if args.heads:
        w = dataclasses.replace(w, H=args.heads, name=f"{w.name}-h{args.heads}")
    peaks = load_peaks()
    n_steps = 1 + w.n_sparse_steps
    qkv = inputs.qkv_steps(w, n_steps, device=dev)
    w_job = w
    sharded = args.shard == "heads" and world > 1
    if sharded:
        # one problem split by heads: this rank's heads as strided views, no collective
        from sparse_attention_diffusion_rt_b200 import shard
        h0, h1 = shard.head_range(w.H, world, rank)
        qkv = [tuple(shard.shard_heads(x, h0, h1) for x in s) for s in qkv]
        w = dataclasses.replace(w, H=h1 - h0)
    mask_np = inputs.block_mask(w)
    mask = torch.from_numpy(mask_np).to(dev)
    nnz = int(mask_np.sum())
    cal_flops = executed_flops(w, w.nqb * w.nkb)
    sp_flops = executed_flops(w, nnz)
    step_flops = cal_flops + w.n_sparse_steps * sp_flops
    # whole-job work per step: N replicas, or the one problem the shards split
    job_step_flops = (executed_flops(w_job, w.nqb * w.nkb) + w.n_sparse_steps * executed_flops(w_job, nnz)
                      if sharded else world * step_flops)
    step = Step(w, mask, qkv, rt)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    st = rt.rt_check_device_error()
    if st != 0:
        raise RuntimeError(f"device error during warm-up: {rt.rt_status_string(st)}")

    # ---- device-timed region: all K steps, events on the launching stream
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    step.launches = 0
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    start.record()
    for _ in range(args.steps):
        step.run()
    end.record()
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    total_ms = start.elapsed_time(end)
    launches = step.launches
    st = rt.rt_check_device_error()
    if st != 0:
        raise RuntimeError(f"device error in timed region: {rt.rt_status_string(st)}")
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / args.steps
    value = job_tflops(1, job_step_flops, ms_per_step)

    # ---- per-kernel timing: separate pass, each kernel bracketed by events
    step.times = {"calibrate": [], "sparse": []}
    for _ in range(max(3, min(args.steps, 10))):
        step.run(record=True)
        torch.cuda.synchronize()
        step.collect()
    cal_ms = float(np.median(step.times["calibrate"]))
    sp_ms = float(np.median(step.times["sparse"]))
    cal_tf = cal_flops / (cal_ms * 1e-3) / 1e12
    sp_tf = sp_flops / (sp_ms * 1e-3) / 1e12
    share_cal = cal_ms / (cal_ms + w.n_sparse_steps * sp_ms)
    dominant = ("calibrate", cal_ms, cal_flops, cal_tf) if share_cal >= 0.5 else ("sparse_step", sp_ms, sp_flops, sp_tf)
    # The denominator matches the power regime the kernels ran in: the measured
    # cuBLAS rate held back to back under the power cap when the cap limited the
    # clocks during the timed region, else the burst rate.
    capped = "sw_power_cap" in (clocks.get("reasons") or [])
    peak = peaks["bf16_tflops_sustained"] if capped else peaks["bf16_tflops"]
    peak_source = peaks["source"] + (" (sustained: sw_power_cap active in the timed region)" if capped
                                     else " (burst)")

    def roof(tag, ms, fl, tf):
        return {"kernel": tag, "bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s",
                "frac": tf / peak, "frac_of_burst": tf / peaks["bf16_tflops"],
                "frac_of_sustained": tf / peaks["bf16_tflops_sustained"],
                "peak_source": peak_source, "algorithmic_flops_per_launch": fl,
                "launch_ms": ms, "traffic": profiled_traffic(tag, w.name)}

    # ---- end to end through the public API from pinned host buffers
    e2e = None
    if not args.no_e2e:
        # Every step copies its inputs from pinned host memory and reads every
        # output back.  Like a caller that pipelines steps, it does so on two
        # copy streams (one per direction) with two device buffer sets, so that
        # step n's copies overlap the kernels of steps n-1 and n+1.
        host_in = [tuple(x.cpu().pin_memory() for x in s) for s in qkv]
        host_out = [torch.empty_like(o, device="cpu").pin_memory() for o in step.o]
        h2d = sum(x.numel() * x.element_size() for s in host_in for x in s)
        d2h = sum(o.numel() * o.element_size() for o in host_out)
        sets = [Step(w, mask, [tuple(torch.empty_like(x) for x in s) for s in qkv], rt) for _ in range(2)]
        cs = torch.cuda.current_stream()
        hs, ds = torch.cuda.Stream(), torch.cuda.Stream()
        nsub = len(qkv)
        ev = lambda: torch.cuda.Event()
        in_ready = [[ev() for _ in range(nsub)] for _ in range(2)]
        out_ready = [[ev() for _ in range(nsub)] for _ in range(2)]
        in_free = [[ev() for _ in range(nsub)] for _ in range(2)]
        out_free = [[ev() for _ in range(nsub)] for _ in range(2)]
        used = [False, False]
        n_e2e = max(2, min(args.steps, 5))

        def e2e_once(n):
            b = n & 1
            st_b = sets[b]
            with torch.cuda.stream(hs):
                for sidx in range(nsub):
                    if used[b]:
                        hs.wait_event(in_free[b][sidx])      # step n-2 is done reading these inputs
                    for xh, xd in zip(host_in[sidx], st_b.qkv[sidx]):
                        xd.copy_(xh, non_blocking=True)
                    in_ready[b][sidx].record(hs)

            def before(sidx):
                cs.wait_event(in_ready[b][sidx])
                if used[b]:
                    cs.wait_event(out_free[b][sidx])          # step n-2's output has been read back

            def after(sidx):
                in_free[b][sidx].record(cs)
                out_ready[b][sidx].record(cs)
                with torch.cuda.stream(ds):
                    ds.wait_event(out_ready[b][sidx])
                    host_out[sidx].copy_(st_b.o[sidx], non_blocking=True)
                    out_free[b][sidx].record(ds)
            st_b.run(before=before, after=after)
            used[b] = True

        def drain():
            cs.wait_stream(hs)
            cs.wait_stream(ds)
        e2e_once(0)
        e2e_once(1)
        drain()
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        hs.wait_event(e0)
        ds.wait_event(e0)
        for n in range(n_e2e):
            e2e_once(n)
        drain()
        e1.record()
        torch.cuda.synchronize()
        barrier()
        e_ms = e0.elapsed_time(e1) / n_e2e
        e_ms = max_over_ranks(e_ms, world, dev)
        # the outputs read back equal the device-resident path's on the same inputs
        match = all(torch.equal(ho, o.cpu()) for ho, o in zip(host_out, step.o))
        e2e = {"value": job_tflops(1, job_step_flops, e_ms), "unit": "TFLOP/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "copies": "H2D and D2H on their own streams, 2 device buffer sets, overlapping the kernels",
               "outputs_match_device_path": bool(match)}
        del host_in, host_out, sets

    # context only: torch's fused SDPA (the pages' speed reference) on the calibration inputs
    sdpa = None
    try:
        q0, k0, v0 = qkv[0]
        for _ in range(2):
            torch.nn.functional.scaled_dot_product_attention(q0, k0, v0)
        torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        for _ in range(3):
            torch.nn.functional.scaled_dot_product_attention(q0, k0, v0)
        s1.record()
        torch.cuda.synchronize()
        sdpa_ms = s0.elapsed_time(s1) / 3
        sdpa_flops = 4.0 * w.L * w.L * w.d * w.B * w.H
        sdpa = {"what": "torch.nn.functional.scaled_dot_product_attention full attention, same Q/K/V (context only)",
                "ms": sdpa_ms, "tflops_true_L": sdpa_flops / (sdpa_ms * 1e-3) / 1e12}
    except Exception as exc:  # noqa: BLE001
        sdpa = {"error": str(exc)[:200]}

    schedule = None
    if not args.no_schedule and not sharded:
        try:
            schedule = measure_schedule(w, mask, rt)
        except torch.cuda.OutOfMemoryError as exc:
            schedule = {"error": str(exc)[:200]}

    token_order = None
    if not args.no_schedule and not sharded:
        token_order = measure_token_order(w, rt)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        steps_cpu = [tuple(x[:, :1].cpu() for x in qkv[0]), tuple(x[:, :1].cpu() for x in qkv[1])]
        v, desc, cores = cpu_oracle_sample(w, steps_cpu, mask_np, budget_s=args.cpu_budget)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "strong" if sharded else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w_job.name, "B": w_job.B, "H": w_job.H, "L": w.L, "d": w.d, "block": w.block,
                       "kept_blocks_per_row": w.kept, "sparsity": 1 - nnz / (w.nqb * w.nkb),
                       "sparse_steps": w.n_sparse_steps, "lambda": w.lam,
                       "l2": "inputs larger than L2 (no flush)",
                       "parallelism": f"heads x{world} (one problem)" if sharded else f"replicas x{world}"},
            "step": "block index + 1 calibration + %d sparse steps" % w.n_sparse_steps,
            "sparse_step": {"latency_us": sp_ms * 1e3, "tflops": sp_tf, "frac_of_peak": sp_tf / peak,
                            "executed_gflop": sp_flops / 1e9},
            "calibrate": {"latency_us": cal_ms * 1e3, "tflops": cal_tf, "frac_of_peak": cal_tf / peak,
                          "executed_gflop": cal_flops / 1e9},
            "roofline": roof(*dominant),
            "roofline_sparse_step": roof("sparse_step", sp_ms, sp_flops, sp_tf),
            "cpu_baseline": cpu,
            "context_torch_sdpa": sdpa,
            "schedule": schedule,
            "token_order": token_order,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-schedule", action="store_true",
                    help="skip the denoising-schedule and token-order measurements")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="N > 1: independent replicas (weak scaling, default) or one problem split by heads")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the workload's head count (a smaller case for profiling)")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
