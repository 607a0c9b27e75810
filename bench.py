#!/usr/bin/env python3
"""Benchmark of Re-ttention's reshaped block-sparse attention hot path on B200.

Headline (the metric): the reshaped sparse step, rt_sparse_step, on the
workload's drifted inputs at step distance k = 1, reading the cached rho and R
of a calibration made during warm-up.  The timed region is K sparse steps
back to back, bracketed by a barrier and a device synchronisation, timed with
CUDA events on the launching stream (max over ranks).  `value` is the
executed-block TFLOP/s of the whole job (4 * block^2 * d * kept blocks * B * H
per call, true d) and `ms_per_step` the sparse step's latency.  Each call
reads more than the 126 MB L2 for the default workload (2.8 GB); smaller
workloads rotate over enough input sets to exceed it.

Default workload: the long-video sweep at 3.1 % density (B=1, H=24, L=115200,
d=128, 28 of 900 key blocks kept per query block = 96.9 % sparsity), the
largest configuration that fits one GPU.

The same JSON line also carries:
  cycle        the whole hot path of one calibration cycle (CSR block index,
               calibration, the workload's sparse steps), device-timed, with
               per-kernel events; `roofline_calibrate` is the calibration's
  per_config   every configuration (tiny, PixArt-, Hunyuan-, CogVideoX-like and
               the long-video sweep at 25 / 12.5 / 6.25 / 3.1 %): calibration
               and sparse-step latency, executed-block TFLOP/s and fractions of
               the measured bf16 peaks, the sparse step's HBM rate on its
               compulsory bytes, and the cost of the residual/rho epilogue
  e2e          the sparse step through the C ABI with host buffers (H2D of its
               Q/K/V and D2H of its output inside the timed region); e2e_cycle
               the same for a whole cycle
  cpu_baseline the float64 CPU oracle's sparse step on a bounded sample
  schedule, token_order, context_torch_sdpa, clocks (NVML samples taken during
               the timed region), gpu_launches

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
PER_CONFIG = ("tiny", "pixart", "hunyuan", "cogvideox", "longvideo-25", "longvideo-12.5", "longvideo-6.25",
              "longvideo-3.1")
KERNEL_SOURCES = ("attn_kernel.cuh", "ptx.cuh", "softmax.cuh", "sparse_kernel.cuh", "pp_sparse.cuh",
                  "pp_calibrate.cuh", "cal_kernel.cuh", "attn_launch.h")
L2_BYTES = 126 * 1024 * 1024


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
    """DRAM bytes per launch of one kernel on one workload, from the ncu
    capture recorded in profiles/traffic.json, if that capture was taken on
    the current kernel source (its source_hash matches), else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        table = json.load(f)
    rec = table.get(kernel_tag, {}).get(workload)
    if not rec or rec.get("source_hash") != kernel_source_hash():
        return None
    return float(rec["dram_bytes_per_launch"])


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


def executed_flops(w: inputs.Workload, nnz_per_head: int) -> float:
    """QK^T and PV of every executed (query block, key block) pair, true d."""
    return 4.0 * w.block * w.block * w.d * nnz_per_head * w.B * w.H


def compulsory_bytes(w: inputs.Workload, r_bytes: int = 2):
    """Bytes a sparse step must move at least: Q, K, V, R in and O out
    ([B, H, L, d] each; R in r_bytes per element), rho in (fp32 [B, H, L]).
    Returns (total, R + rho part)."""
    elems = w.B * w.H * w.L * w.d
    r_rho = elems * r_bytes + w.B * w.H * w.L * 4
    return 4 * elems * 2 + r_rho, r_rho


def frac_block(tflops, peaks, peak):
    return {"tflops": tflops, "frac_of_burst": tflops / peaks["bf16_tflops"],
            "frac_of_sustained": tflops / peaks["bf16_tflops_sustained"], "frac_of_peak": tflops / peak}


# SM clock and clock-event reasons, read through NVML during a timed region.
_REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}


class ClockSampler:
    """Samples the SM clock, power and clock-event reasons of this process's
    GPU every few milliseconds while running (NVML; nvidia-smi as fallback)."""

    def __init__(self, device_index: int, period_s: float = 0.004):
        self.dev, self.period = device_index, period_s
        self.samples = []
        self._stop = threading.Event()
        self._thread = None
        self._smi = None

    def _handle(self, nv):
        try:
            uuid = torch.cuda.get_device_properties(self.dev).uuid
            return nv.nvmlDeviceGetHandleByUUID(("GPU-" + str(uuid)).encode())
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.dev)

    def start(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            reasons_fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            self.sm_max = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))

            def loop():
                while not self._stop.is_set():
                    try:
                        self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                             int(reasons_fn(h)), nv.nvmlDeviceGetPowerUsage(h) / 1000.0))
                    except Exception:
                        pass
                    self._stop.wait(self.period)
            self._thread = threading.Thread(target=loop, daemon=True)
            self._thread.start()
        except Exception:
            self._start_smi()

    def _start_smi(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self._smi = subprocess.Popen(["nvidia-smi", f"--id={self.dev}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

            def read():
                for line in self._smi.stdout:
                    p = [x.strip() for x in line.split(",")]
                    try:
                        bits = sum(_REASON_BITS[n] for n, v in zip(names, p[3:7]) if v.lower() == "active")
                        self.sm_max = float(p[1])
                        self.samples.append((float(p[0]), bits, float(p[2])))
                    except (ValueError, IndexError):
                        continue
            self._thread = threading.Thread(target=read, daemon=True)
            self._thread.start()
        except Exception:
            self._smi = None

    def stop(self):
        self._stop.set()
        if self._smi is not None:
            time.sleep(0.15)
            self._smi.terminate()
        if self._thread is not None:
            self._thread.join(timeout=2)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock samples"], "samples": 0}
        sm = [s[0] for s in self.samples]
        bits = 0
        for s in self.samples:
            bits |= s[1]
        reasons = sorted(n for n, b in _REASON_BITS.items() if bits & b)
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": getattr(self, "sm_max", None),
                "sm_mhz_min": float(min(sm)), "reasons": reasons, "samples": len(sm),
                "power_w_max": float(max(s[2] for s in self.samples)),
                "source": "nvml" if self._smi is None else "nvidia-smi"}


def peak_for(clocks, peaks):
    """bf16 peak that matches the power regime a region ran in: the measured
    cuBLAS rate held back to back under the power cap when the cap limited the
    clocks, else the burst rate."""
    capped = "sw_power_cap" in (clocks.get("reasons") or [])
    if capped:
        return peaks["bf16_tflops_sustained"], peaks["source"] + " (sustained: sw_power_cap active in the region)"
    return peaks["bf16_tflops"], peaks["source"] + " (burst)"


class L2Flush:
    """Writes a buffer twice the size of L2 so that the next kernel starts cold."""

    def __init__(self, device):
        self.buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)

    def __call__(self):
        self.buf.fill_(1.0)


def time_each(fn, reps, warm=1, flush=None):
    """Median device time (ms) of fn() over reps calls, each bracketed by its
    own CUDA events on the current stream, with an optional L2 flush before
    each (outside the events)."""
    for _ in range(warm):
        fn()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for e0, e1 in ev:
        if flush is not None:
            flush()
        e0.record()
        fn()
        e1.record()
    torch.cuda.synchronize()
    return float(np.median([e0.elapsed_time(e1) for e0, e1 in ev]))


def sets_for_l2(bytes_per_call: int) -> int:
    """Input sets to rotate over so that back-to-back calls never find their
    operands in L2."""
    return max(1, -(-2 * L2_BYTES // max(1, bytes_per_call)))


def cpu_oracle_sparse(w, mask, budget_s=15.0, n_blocks=8, steps_cpu=None):
    """The oracle's sparse step, as it stands, on a bounded sample of the
    workload: query blocks of head (0, 0).  Their cached rho and R come from
    the oracle's calibration rows (not timed).  Returns a callable that times
    sparse_step_rows_ref over the sampled query blocks for about budget_s and
    gives (executed-block TFLOP/s, description, cores)."""
    from oracle import reference as ref
    if steps_cpu is None:
        steps_cpu = inputs.qkv_steps(dataclasses.replace(w, B=1, H=1), 2, device="cpu")
    q0, k0, v0 = (x[0, 0].double().numpy() for x in steps_cpu[0])
    q1, k1, v1 = (x[0, 0].double().numpy() for x in steps_cpu[1])
    bm = mask[0]
    order = np.random.default_rng(0).permutation(w.nqb)[:n_blocks]
    cached = []
    for qb in order:
        rows = np.arange(qb * w.block, min(w.L, (qb + 1) * w.block))
        _, rho, r = ref.calibrate_rows_ref(q0, k0, v0, bm, w.block, rows)
        cached.append((qb, rows, rho, r))

    def run(budget=budget_s):
        flops, n = 0.0, 0
        t0 = time.perf_counter()
        while True:
            qb, rows, rho, r = cached[n % len(cached)]
            ref.sparse_step_rows_ref(q1, k1, v1, bm, w.block, rows, rho, r, w.lam, 1)
            flops += 4.0 * w.block * w.block * w.d * int(bm[qb].sum())
            n += 1
            if time.perf_counter() - t0 > budget:
                break
        dt = time.perf_counter() - t0
        cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
        desc = (f"head (0,0) of {w.name}: {n} query-block sparse steps over {len(cached)} sampled query blocks "
                f"(of {w.B * w.H * w.nqb} per call) in {dt:.1f} s; executed-block FLOPs of the sample / CPU time")
        return flops / dt / 1e12, desc, cores
    return run


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
# per-configuration measurements
# ---------------------------------------------------------------------------

def measure_config(name, rt, peaks, flush, cache):
    """Device-timed calibration and sparse step of one configuration (each
    call bracketed by its own events, L2 flushed before each), with the
    sparse step's HBM rate on its compulsory bytes and the cost of the
    residual read (the same step with the RT_EPI_NO_R epilogue)."""
    w = inputs.WORKLOADS[name]
    key = (w.B, w.H, w.L, w.d, w.seed)
    if cache.get("key") != key:
        cache.clear()
        torch.cuda.empty_cache()
        cache["key"] = key
        cache["qkv"] = inputs.qkv_steps(w, 2, device="cuda")
    (q0, k0, v0), (q1, k1, v1) = cache["qkv"]
    mask_np = inputs.block_mask(w)
    nnz = int(mask_np.sum())
    idx = rt.rt_build_block_index(torch.from_numpy(mask_np).cuda())
    o0, o1, r = torch.empty_like(q0), torch.empty_like(q0), torch.empty_like(q0)
    rho = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=q0.device)

    def reps_for(ms):
        return int(max(3, min(20, 400.0 / max(ms, 1e-3))))

    cal = lambda: rt.rt_calibrate(q0, k0, v0, idx, block=w.block, o=o0, rho=rho, r=r)
    first = time_each(cal, 1, warm=1, flush=flush)
    cal_ms = time_each(cal, reps_for(first), warm=0, flush=flush)
    sp = lambda: rt.rt_sparse_step(q1, k1, v1, idx, rho, r, block=w.block, lam=w.lam, step_distance=1, o=o1)
    first = time_each(sp, 1, warm=2, flush=flush)
    sp_ms = time_each(sp, reps_for(first), warm=0, flush=flush)
    no_r = lambda: rt.rt_sparse_step(q1, k1, v1, idx, rho, None, block=w.block, lam=w.lam, step_distance=1, o=o1,
                                     epilogue=rt.RT_EPI_NO_R)
    no_r_ms = time_each(no_r, reps_for(first), warm=1, flush=flush)
    st = rt.rt_check_device_error()
    if st != 0:
        raise RuntimeError(f"device error in {name}: {rt.rt_status_string(st)}")
    cal_flops = executed_flops(w, w.nqb * w.nkb)
    sp_flops = executed_flops(w, nnz)
    cal_tf = cal_flops / (cal_ms * 1e-3) / 1e12
    sp_tf = sp_flops / (sp_ms * 1e-3) / 1e12
    comp, r_rho = compulsory_bytes(w)
    gbs = comp / (sp_ms * 1e-3) / 1e9
    # min(tensor peak, arithmetic intensity x HBM): the sparse step's own roofline
    ceiling_tf = min(peaks["bf16_tflops"], sp_flops / comp * peaks["hbm_gbs"] / 1e3)
    inc_ms = sp_ms - no_r_ms
    return {
        "B": w.B, "H": w.H, "L": w.L, "d": w.d, "block": w.block, "kept_blocks_per_row": w.kept,
        "sparsity": 1 - nnz / (w.nqb * w.nkb), "sparse_steps_per_cycle": w.n_sparse_steps,
        "calibrate": {"us": cal_ms * 1e3, "executed_gflop": cal_flops / 1e9,
                      **frac_block(cal_tf, peaks, peaks["bf16_tflops"])},
        "sparse_step": {"us": sp_ms * 1e3, "executed_gflop": sp_flops / 1e9,
                        **frac_block(sp_tf, peaks, peaks["bf16_tflops"]),
                        "compulsory_mb": comp / 1e6, "hbm_gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"],
                        "roofline_tflops": ceiling_tf, "roofline_bound": "tensor" if ceiling_tf >= peaks[
                            "bf16_tflops"] else "hbm",
                        "frac_of_roofline": sp_tf / ceiling_tf},
        "residual_and_rho": {"bytes": r_rho, "share_of_compulsory": r_rho / comp,
                             "sparse_step_without_r_us": no_r_ms * 1e3, "incremental_us": inc_ms * 1e3,
                             "incremental_gbs": (r_rho / (inc_ms * 1e-3) / 1e9) if inc_ms > 0 else None},
        "cycle_us": (cal_ms + w.n_sparse_steps * sp_ms) * 1e3,
        "cycle": f"1 calibration + {w.n_sparse_steps} sparse steps (sum of the medians)",
    }


def measure_per_config(rt, peaks, names=PER_CONFIG):
    flush = L2Flush("cuda")
    cache = {}
    out = {}
    for name in names:
        try:
            out[name] = measure_config(name, rt, peaks, flush, cache)
        except torch.cuda.OutOfMemoryError as exc:
            out[name] = {"error": str(exc)[:200]}
    cache.clear()
    del flush
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------
# the cycle (block index + calibration + sparse steps)
# ---------------------------------------------------------------------------

class Cycle:
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


def pipelined_e2e(n_steps, host_in, dev_sets, host_out, dev_out, launch, world, dev, barrier):
    """End-to-end time per step through the public API: every step copies its
    inputs from pinned host memory (host_in[i]: list of tensors) into one of
    two device buffer sets, runs launch(set, i) on the current stream and reads
    its outputs back (dev_out(set) -> host_out).  Copies run on their own
    streams, one per direction, so that a step's copies overlap the kernels of
    its neighbours (as a caller that pipelines steps would).  Returns ms per
    step (max over ranks)."""
    cs = torch.cuda.current_stream()
    hs, ds = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_ready, in_free = [ev(), ev()], [ev(), ev()]
    out_ready, out_free = [ev(), ev()], [ev(), ev()]
    used = [False, False]

    def once(n):
        b = n & 1
        with torch.cuda.stream(hs):
            if used[b]:
                hs.wait_event(in_free[b])
            for xh, xd in zip(host_in[n % len(host_in)], dev_sets[b]):
                xd.copy_(xh, non_blocking=True)
            in_ready[b].record(hs)
        cs.wait_event(in_ready[b])
        if used[b]:
            cs.wait_event(out_free[b])
        launch(b, n)
        in_free[b].record(cs)
        out_ready[b].record(cs)
        with torch.cuda.stream(ds):
            ds.wait_event(out_ready[b])
            for xh, xd in zip(host_out, dev_out(b)):
                xh.copy_(xd, non_blocking=True)
            out_free[b].record(ds)
        used[b] = True

    def drain():
        cs.wait_stream(hs)
        cs.wait_stream(ds)
    once(0)
    once(1)
    drain()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    hs.wait_event(e0)
    ds.wait_event(e0)
    for n in range(n_steps):
        once(n)
    drain()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    return max_over_ranks(e0.elapsed_time(e1) / n_steps, world, dev)


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------

def run_reference(args, rank, world):
    """The oracle's sparse step timed on the host cores (rank 0 only)."""
    if rank != 0:
        return
    w = inputs.WORKLOADS[args.workload]
    mask = inputs.block_mask(w)
    budget = max(1.0, 45.0 / max(1, args.steps + args.warmup))
    run = cpu_oracle_sparse(w, mask, n_blocks=4)
    vals = []
    for i in range(args.warmup + args.steps):
        v, desc, cores = run(budget)
        if i >= args.warmup:
            vals.append(v)
    value = float(np.median(vals))
    sp_flops = executed_flops(w, int(mask.sum()))
    ms_step = sp_flops / (value * 1e12) * 1e3          # the whole sparse step at the sample's rate (extrapolated)
    desc += f"; ms_per_step extrapolated from the sample's rate to the whole sparse step ({sp_flops / 1e12:.2f} TFLOP)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "d": w.d, "block": w.block,
                   "kept_blocks_per_row": w.kept, "sparsity": 1 - int(mask.sum()) / (w.nqb * w.nkb),
                   "lambda": w.lam, "step_distance": 1},
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
    w_job = w
    sharded = args.shard == "heads" and world > 1
    heads = None
    if sharded:
        # one problem split by heads: this rank draws and runs only its own heads, no collective
        from sparse_attention_diffusion_rt_b200 import shard
        heads = shard.head_range(w.H, world, rank)
        w = dataclasses.replace(w, H=heads[1] - heads[0])
    n_steps = 1 + w.n_sparse_steps
    qkv = inputs.qkv_steps(w_job, n_steps, device=dev, heads=heads)
    mask_np = inputs.block_mask(w)
    mask = torch.from_numpy(mask_np).to(dev)
    nnz = int(mask_np.sum())
    cal_flops = executed_flops(w, w.nqb * w.nkb)
    sp_flops = executed_flops(w, nnz)
    # whole-job work of one sparse step: N replicas, or the one problem the shards split
    job_sp_flops = executed_flops(w_job, nnz) if sharded else world * sp_flops

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    # ---- warm-up: the calibration that fills the cache, then W sparse steps
    idx = rt.rt_build_block_index(mask)
    q0, k0, v0 = qkv[0]
    q1, k1, v1 = qkv[1]
    like = lambda t: torch.empty_strided(t.shape, t.stride(), dtype=t.dtype, device=t.device)
    rho = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=dev)
    r, o0 = like(q0), like(q0)
    rt.rt_calibrate(q0, k0, v0, idx, block=w.block, o=o0, rho=rho, r=r)
    per_call = sum(x.numel() * x.element_size() for x in (q1, k1, v1, r, rho, o0))
    n_sets = sets_for_l2(per_call)
    sets = [(q1, k1, v1, rho, r, like(q0))]
    for _ in range(n_sets - 1):
        sets.append(tuple(x.clone() for x in (q1, k1, v1, rho, r)) + (like(q0),))

    def sparse(i):
        q, k, v, rh, rr, o = sets[i % n_sets]
        rt.rt_sparse_step(q, k, v, idx, rh, rr, block=w.block, lam=w.lam, step_distance=1, o=o)

    for i in range(args.warmup):
        sparse(i)
    torch.cuda.synchronize()
    st = rt.rt_check_device_error()
    if st != 0:
        raise RuntimeError(f"device error during warm-up: {rt.rt_status_string(st)}")

    # ---- device-timed region: K sparse steps back to back
    sampler = ClockSampler(local_rank)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    start.record()
    for i in range(args.steps):
        sparse(i)
    end.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier()
    launches = args.steps                      # one kernel launch per sparse step
    st = rt.rt_check_device_error()
    if st != 0:
        raise RuntimeError(f"device error in timed region: {rt.rt_status_string(st)}")
    sp_ms = max_over_ranks(start.elapsed_time(end) / args.steps, world, dev)
    value = job_tflops(1, job_sp_flops, sp_ms)
    sp_tf_rank = sp_flops / (sp_ms * 1e-3) / 1e12
    peak, peak_source = peak_for(clocks, peaks)
    comp, r_rho = compulsory_bytes(w, r.element_size())
    hbm_gbs = comp / (sp_ms * 1e-3) / 1e9
    roofline = {"kernel": "sparse_step", "bound": "tensor", "achieved": sp_tf_rank, "peak": peak,
                "unit": "TFLOP/s", "frac": sp_tf_rank / peak, "frac_of_burst": sp_tf_rank / peaks["bf16_tflops"],
                "frac_of_sustained": sp_tf_rank / peaks["bf16_tflops_sustained"], "peak_source": peak_source,
                "algorithmic_flops_per_launch": sp_flops, "launch_ms": sp_ms,
                "traffic": profiled_traffic("sparse_step", w.name), "compulsory_bytes": comp,
                "hbm_gbs_on_compulsory_bytes": hbm_gbs, "hbm_frac": hbm_gbs / peaks["hbm_gbs"]}
    sparse_obj = {"latency_us": sp_ms * 1e3, "executed_gflop": sp_flops / 1e9,
                  **frac_block(sp_tf_rank, peaks, peak),
                  "residual_and_rho_bytes": r_rho, "residual_and_rho_share": r_rho / comp,
                  "input_sets_rotated": n_sets}
    del sets
    torch.cuda.empty_cache()

    # ---- the whole cycle: block index + calibration + sparse steps, per-kernel events
    cyc = Cycle(w, mask, qkv, rt)
    cyc.run()
    torch.cuda.synchronize()
    n_cyc = max(3, min(args.steps, 5))
    csampler = ClockSampler(local_rank)
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    csampler.start()
    c0.record()
    for _ in range(n_cyc):
        cyc.run(record=True)
        # the event pairs are reused each cycle: read them before the next one records
        torch.cuda.synchronize()
        cyc.collect()
    c1.record()
    torch.cuda.synchronize()
    cclocks = csampler.stop()
    barrier()
    st = rt.rt_check_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the cycle: {rt.rt_status_string(st)}")
    cyc_ms = max_over_ranks(c0.elapsed_time(c1) / n_cyc, world, dev)
    cal_ms = max_over_ranks(float(np.median(cyc.times["calibrate"])), world, dev)
    csp_ms = max_over_ranks(float(np.median(cyc.times["sparse"])), world, dev)
    cal_tf = cal_flops / (cal_ms * 1e-3) / 1e12
    cpeak, cpeak_source = peak_for(cclocks, peaks)
    cyc_flops = cal_flops + w.n_sparse_steps * sp_flops
    cyc_job_flops = (executed_flops(w_job, w.nqb * w.nkb) + w.n_sparse_steps * executed_flops(w_job, nnz)
                     if sharded else world * cyc_flops)
    cycle = {"what": f"CSR block index + 1 calibration + {w.n_sparse_steps} sparse steps (k = 1..{w.n_sparse_steps})",
             "cycles": n_cyc, "ms": cyc_ms, "tflops": job_tflops(1, cyc_job_flops, cyc_ms),
             "calibrate_ms": cal_ms, "sparse_step_ms_in_cycle": csp_ms,
             "calibrate_share": cal_ms / (cal_ms + w.n_sparse_steps * csp_ms), "clocks": cclocks,
             "launches_per_cycle": 3 + n_steps}
    calibrate_obj = {"latency_us": cal_ms * 1e3, "executed_gflop": cal_flops / 1e9,
                     **frac_block(cal_tf, peaks, cpeak)}
    roofline_cal = {"kernel": "calibrate", "bound": "tensor", "achieved": cal_tf, "peak": cpeak, "unit": "TFLOP/s",
                    "frac": cal_tf / cpeak, "frac_of_burst": cal_tf / peaks["bf16_tflops"],
                    "frac_of_sustained": cal_tf / peaks["bf16_tflops_sustained"], "peak_source": cpeak_source,
                    "algorithmic_flops_per_launch": cal_flops, "launch_ms": cal_ms,
                    "traffic": profiled_traffic("calibrate", w.name)}

    # ---- end to end through the public API from pinned host buffers
    e2e = e2e_cycle = None
    if not args.no_e2e:
        # the sparse step: its Q, K, V come from the host and its output goes back;
        # rho and R stay resident, where the calibration that made them left them
        host_in = [[x.cpu().pin_memory() for x in (q1, k1, v1)]]
        dsets = [[like(x) for x in (q1, k1, v1)] for _ in range(2)]
        douts = [like(q1) for _ in range(2)]
        host_o = [torch.empty_like(q1, device="cpu").pin_memory()]

        def launch_sp(b, n):
            q, k, v = dsets[b]
            rt.rt_sparse_step(q, k, v, idx, rho, r, block=w.block, lam=w.lam, step_distance=1, o=douts[b])
        e_ms = pipelined_e2e(max(3, min(args.steps, 10)), host_in, dsets, host_o, lambda b: [douts[b]], launch_sp,
                             world, dev, barrier)
        ref_o = like(q1)
        rt.rt_sparse_step(q1, k1, v1, idx, rho, r, block=w.block, lam=w.lam, step_distance=1, o=ref_o)
        torch.cuda.synchronize()
        match = bool(torch.equal(host_o[0], ref_o.cpu()))
        h2d = sum(x.numel() * x.element_size() for x in host_in[0])
        e2e = {"value": job_tflops(1, job_sp_flops, e_ms), "unit": "TFLOP/s", "ms_per_step": e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": host_o[0].numel() * host_o[0].element_size(),
               "what": "rt_sparse_step with its Q/K/V copied in from pinned host memory and its output read back; "
                       "rho and R resident on the device (the calibration's cache)",
               "copies": "H2D and D2H on their own streams, 2 device buffer sets, overlapping the kernels",
               "outputs_match_device_path": match}
        del host_in, dsets, douts, host_o, ref_o

        # the whole cycle: every step's inputs in, every output out
        host_cyc = [[x.cpu().pin_memory() for s in qkv for x in s]]
        csets = [Cycle(w, mask, [tuple(like(x) for x in s) for s in qkv], rt) for _ in range(2)]
        dflat = [[x for s in c.qkv for x in s] for c in csets]
        host_co = [torch.empty_like(o, device="cpu").pin_memory() for o in cyc.o]
        e_ms_c = pipelined_e2e(max(2, min(args.steps, 4)), host_cyc, dflat, host_co, lambda b: csets[b].o,
                               lambda b, n: csets[b].run(), world, dev, barrier)
        match_c = all(torch.equal(ho, o.cpu()) for ho, o in zip(host_co, cyc.o))
        e2e_cycle = {"value": job_tflops(1, cyc_job_flops, e_ms_c), "unit": "TFLOP/s (calibration + sparse steps)",
                     "ms_per_cycle": e_ms_c,
                     "h2d_bytes_per_cycle": sum(x.numel() * x.element_size() for x in host_cyc[0]),
                     "d2h_bytes_per_cycle": sum(o.numel() * o.element_size() for o in host_co),
                     "outputs_match_device_path": bool(match_c)}
        del host_cyc, csets, dflat, host_co
        torch.cuda.empty_cache()

    # context only: torch's fused SDPA (the pages' speed reference) on the calibration inputs
    sdpa = None
    try:
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

    del cyc
    torch.cuda.empty_cache()
    schedule = token_order = None
    if not args.no_schedule and not sharded:
        try:
            schedule = measure_schedule(w, mask, rt)
        except torch.cuda.OutOfMemoryError as exc:
            schedule = {"error": str(exc)[:200]}
        token_order = measure_token_order(w, rt)

    per_config = None
    if world == 1 and not args.no_per_config:
        del qkv, q0, k0, v0, q1, k1, v1, r, o0, rho
        torch.cuda.empty_cache()
        per_config = measure_per_config(rt, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc, cores = cpu_oracle_sparse(w, mask_np, n_blocks=8)(args.cpu_budget)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": sp_ms, "higher_is_better": True,
            "scaling": "strong" if sharded else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w_job.name, "B": w_job.B, "H": w_job.H, "L": w.L, "d": w.d, "block": w.block,
                       "kept_blocks_per_row": w.kept, "sparsity": 1 - nnz / (w.nqb * w.nkb),
                       "lambda": w.lam, "step_distance": 1,
                       "timed": "K sparse steps back to back (rt_sparse_step at k = 1 on the drifted inputs, "
                                "reading the cached rho/R of a calibration made during warm-up)",
                       "l2": ("inputs larger than L2 (no flush)" if n_sets == 1 else
                              f"{n_sets} input sets rotated so that each call's operands are not in L2"),
                       "parallelism": f"heads x{world} (one problem)" if sharded else f"replicas x{world}"},
            "sparse_step": sparse_obj,
            "roofline": roofline,
            "calibrate": calibrate_obj,
            "roofline_calibrate": roofline_cal,
            "cycle": cycle,
            "per_config": per_config,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "e2e_cycle": e2e_cycle,
            "context_torch_sdpa": sdpa,
            "schedule": schedule,
            "token_order": token_order,
            "gpu_launches": launches,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-schedule", action="store_true",
                    help="skip the denoising-schedule and token-order measurements")
    ap.add_argument("--no-per-config", action="store_true", help="skip the per-configuration block")
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
