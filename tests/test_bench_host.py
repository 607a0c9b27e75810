"""Host-side pieces of bench.py that need no GPU: the executed-block FLOP count,
the lookup of DRAM traffic in the committed ncu summaries (taken only when the
summary was made on the current kernel source), and the mask-locality figures
of the token-reordering row, checked against a brute-force count."""
import numpy as np

import bench
from oracle.reference import hilbert_order_ref
from sparse_attention_diffusion_rt_b200 import inputs


def test_executed_flops_counts_qk_and_pv_of_every_executed_block():
    w = inputs.Workload("t", 2, 3, 512, 72, 128, kept=2, n_sparse_steps=1, seed=0)
    nnz = 7
    # QK^T and PV: 2 * 128 * 128 * d multiply-adds each, per executed block, per (b, h)
    assert bench.executed_flops(w, nnz) == 2 * (2 * 128 * 128 * 72) * nnz * 2 * 3


def test_profiled_traffic_only_for_the_current_source(tmp_path, monkeypatch):
    import json
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"calibrate": {"w": {"source_hash": "0123abcd", "dram_bytes_per_launch": 123456789}}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0123abcd")
    assert bench.profiled_traffic("calibrate", "w") == 123456789.0
    assert bench.profiled_traffic("sparse_step", "w") is None          # no capture of that kernel
    assert bench.profiled_traffic("calibrate", "other") is None        # nor of that workload
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "ffff0000")
    assert bench.profiled_traffic("calibrate", "w") is None            # kernel changed since


def test_committed_traffic_records_are_well_formed():
    import json
    import os
    path = os.path.join(bench.ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return
    table = json.load(open(path))
    for kernel, per_w in table.items():
        assert kernel in ("calibrate", "sparse_step")
        for wname, rec in per_w.items():
            assert wname in inputs.WORKLOADS or wname.rsplit("-h", 1)[0] in inputs.WORKLOADS
            assert len(rec["source_hash"]) == 16 and rec["dram_bytes_per_launch"] > 0
            assert "command" in rec


def test_compulsory_bytes_and_l2_rotation():
    w = inputs.WORKLOADS["pixart"]
    elems = 2 * 16 * 4096 * 72
    total, r_rho = bench.compulsory_bytes(w)
    assert r_rho == elems * 2 + 2 * 16 * 4096 * 4                      # R bf16 + rho fp32
    assert total == 4 * elems * 2 + r_rho                              # Q, K, V in, O out, plus R and rho
    assert bench.compulsory_bytes(w, 4)[1] == elems * 4 + 2 * 16 * 4096 * 4
    # rotated sets always exceed L2 twice over; a call larger than that needs one set
    for per_call in (1, 10 ** 6, 90 * 10 ** 6, 3 * 10 ** 9):
        n = bench.sets_for_l2(per_call)
        assert n * per_call >= 2 * bench.L2_BYTES and (n == 1 or (n - 1) * per_call < 2 * bench.L2_BYTES)


def test_peak_follows_the_power_regime():
    peaks = {"bf16_tflops": 1646.8, "bf16_tflops_sustained": 1398.0, "hbm_gbs": 6551.0, "source": "measured"}
    assert bench.peak_for({"reasons": ["sw_power_cap"]}, peaks)[0] == 1398.0
    assert bench.peak_for({"reasons": []}, peaks)[0] == 1646.8
    assert bench.peak_for({"reasons": ["hw_slowdown"]}, peaks)[0] == 1646.8


def test_kernel_source_hash_covers_every_kernel_file():
    import os
    csrc = os.path.join(bench.ROOT, "sparse_attention_diffusion_rt_b200", "csrc")
    kernel_files = {f for f in os.listdir(csrc) if f.endswith(".cuh")}
    assert kernel_files <= set(bench.KERNEL_SOURCES)
    h = bench.kernel_source_hash()
    assert len(h) == 16 and int(h, 16) >= 0


def _brute_recall(w, mask, perm):
    """Fraction of (visual token, grid neighbour) pairs whose key block is kept
    for the token's query block: plain loops over the tokens."""
    F, Y, X = w.grid
    pos_of = {}
    for i, r in enumerate(perm):
        pos_of[int(r)] = i
    hit = total = 0
    for i, r in enumerate(perm):
        r = int(r)
        if r < w.n_text:
            continue
        g = r - w.n_text
        f, y, x = g // (Y * X), (g // X) % Y, g % X
        for df in (-1, 0, 1):
            for dy in (-1, 0, 1):
                for dx in (-1, 0, 1):
                    if df == dy == dx == 0:
                        continue
                    ff, yy, xx = f + df, y + dy, x + dx
                    if not (0 <= ff < F and 0 <= yy < Y and 0 <= xx < X):
                        continue
                    j = pos_of[w.n_text + (ff * Y + yy) * X + xx]
                    total += 1
                    hit += int(mask[0, i // w.block, j // w.block])
    return hit / total


def test_mask_locality_against_brute_force_and_hilbert_bricks():
    w = inputs.Workload("g", 1, 1, 64, 64, 16, kept=1, n_sparse_steps=1, seed=0,
                        grid=(1, 8, 8), diagonal=True)
    own = inputs.block_mask(w)                       # each query block keeps only itself
    dense = np.ones_like(own)
    raster = np.arange(w.L)
    hil = hilbert_order_ref(0, 1, 8, 8)
    for perm in (raster, hil):
        r, vol = bench.mask_locality(w, own, None if perm is raster else perm)
        assert abs(r - _brute_recall(w, own, perm)) < 1e-12
        assert vol == 16.0                           # a 2 x 8 strip or a 4 x 4 brick
        assert bench.mask_locality(w, dense, None if perm is raster else perm)[0] == 1.0
    # a 4 x 4 brick keeps more of each token's neighbours than a 2 x 8 strip
    assert bench.mask_locality(w, own, hil)[0] > bench.mask_locality(w, own, None)[0]
