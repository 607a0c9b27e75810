"""GPU parity: the C-ABI kernels against the float64 CPU oracle, element by
element, on identical seeded bf16 inputs.

Sizes the oracle finishes in seconds are checked in full (several tiles and a
ragged tail); the full-size CogVideoX-like and long-video workloads, launched
exactly as bench.py launches them, are checked on sampled rows.
"""

import math

import numpy as np
import pytest
import torch

from helpers import check_out, check_rho, f64
from oracle import reference as ref
from sparse_attention_diffusion_rt_b200 import inputs
from sparse_attention_diffusion_rt_b200 import rt

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _index(mask_np):
    return rt.rt_build_block_index(torch.from_numpy(np.ascontiguousarray(mask_np)).to(DEV))


def _ok():
    st = rt.rt_check_device_error()
    assert st == rt.RT_OK, rt.rt_status_string(st)


def _stats_inputs(shape, seed, r_dtype=torch.bfloat16):
    """Synthetic cached statistics for isolated sparse-step parity (not from the CUDA path)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    B, H, L, d = shape
    rho = torch.rand((B, H, L), generator=g, dtype=torch.float32)
    r = (0.1 * torch.randn(shape, generator=g, dtype=torch.float32)).to(r_dtype)
    return rho.to(DEV), r.to(DEV)


# ---------------------------------------------------------------------------
# block index
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", list(inputs.WORKLOADS))
def test_block_index_workload_masks_bit_exact(name):
    mask = inputs.block_mask(inputs.WORKLOADS[name])
    idx = _index(mask)
    rp, ci = ref.build_block_index_ref(mask)
    assert idx.nnz == len(ci)
    np.testing.assert_array_equal(idx.row_ptr.cpu().numpy(), rp)
    np.testing.assert_array_equal(idx.col_idx.cpu().numpy(), ci)


@pytest.mark.parametrize("Hm,nqb,nkb,dens,seed", [(1, 1, 1, 1.0, 0), (3, 17, 33, 0.2, 1), (2, 50, 70, 0.0, 2),
                                                   (4, 300, 300, 0.05, 3), (1, 1100, 1000, 0.5, 4),
                                                   (2, 7, 1, 0.5, 5)])
def test_block_index_random_bit_exact(Hm, nqb, nkb, dens, seed):
    mask = inputs.random_block_mask(Hm, nqb, nkb, dens, seed)
    idx = _index(mask)
    rp, ci = ref.build_block_index_ref(mask)
    np.testing.assert_array_equal(idx.row_ptr.cpu().numpy(), rp)
    np.testing.assert_array_equal(idx.col_idx.cpu().numpy(), ci)


def test_block_index_capacity_error():
    mask = torch.ones((1, 4, 4), dtype=torch.uint8, device=DEV)
    row_ptr = torch.empty(5, dtype=torch.int32, device=DEV)
    col = torch.full((10,), -7, dtype=torch.int32, device=DEV)
    lib = rt.load_library()
    import ctypes
    nnz = ctypes.c_int64(0)
    st = lib.rt_build_block_index(mask.data_ptr(), 1, 4, 4, row_ptr.data_ptr(), col.data_ptr(), 10,
                                  ctypes.byref(nnz), rt._stream_ptr(None))
    assert st == rt.RT_ERR_CAPACITY and nnz.value == 16
    assert row_ptr.cpu().tolist() == [0, 4, 8, 12, 16]
    assert col.cpu().tolist() == [0, 1, 2, 3] * 2 + [0, 1]      # only positions that fit


# ---------------------------------------------------------------------------
# small problems, full tensors
# ---------------------------------------------------------------------------

def _run_cycle_full(q, k, v, q2, k2, v2, mask, block, lam=0.04, kdist=1, ramp=rt.RT_RAMP_MUL_LINEAR,
                    r_dtype=torch.bfloat16, scale=0.0, Hm_mask=None, rel=0.0):
    idx = _index(mask)
    o, rho, r = rt.rt_calibrate(q, k, v, idx, block=block, r_dtype=r_dtype, softmax_scale=scale)
    o2 = rt.rt_sparse_step(q2, k2, v2, idx, rho, r, block=block, lam=lam, step_distance=kdist, ramp=ramp,
                           softmax_scale=scale)
    torch.cuda.synchronize()
    _ok()
    sc = scale if scale else None
    O, RHO, R = ref.calibrate_ref(f64(q), f64(k), f64(v), mask, block, scale=sc)
    check_out(f64(o), O, "calibrate O", rel=rel)
    check_out(f64(r), R, "calibrate R", rel=rel)
    check_rho(f64(rho), RHO)
    O2 = ref.sparse_step_ref(f64(q2), f64(k2), f64(v2), mask, block, RHO, R, lam, kdist, ramp, scale=sc)
    check_out(f64(o2), O2, "sparse O (end to end)", rel=rel)
    # isolated sparse step on synthetic statistics
    rho_s, r_s = _stats_inputs(tuple(q.shape), 99, r_dtype)
    o3 = rt.rt_sparse_step(q2, k2, v2, idx, rho_s, r_s, block=block, lam=lam, step_distance=kdist, ramp=ramp,
                           softmax_scale=scale)
    torch.cuda.synchronize()
    _ok()
    O3 = ref.sparse_step_ref(f64(q2), f64(k2), f64(v2), mask, block, f64(rho_s), f64(r_s), lam, kdist, ramp,
                             scale=sc)
    check_out(f64(o3), O3, "sparse O (isolated)", rel=rel)


@pytest.mark.parametrize("name", ["tiny", "pixart", "hunyuan"])
def test_workload_cycle_full(name):
    w = inputs.WORKLOADS[name]
    steps = inputs.qkv_steps(w, 2, device=DEV)
    mask = inputs.block_mask(w)
    _run_cycle_full(*steps[0], *steps[1], mask, w.block, lam=w.lam, kdist=1)


@pytest.mark.parametrize("d", [16, 32, 48, 64, 72, 88, 96, 104, 120, 128])
def test_head_dims_ragged_tail(d):
    B, H, L, blk = 1, 2, 300, 128              # 3 query blocks, tail of 44
    q, k, v = inputs.random_qkv(B, H, L, d, seed=d, device=DEV)
    q2, k2, v2 = inputs.random_qkv(B, H, L, d, seed=1000 + d, device=DEV)
    mask = inputs.random_block_mask(1, 3, 3, 0.5, seed=d, ensure_nonempty=True)
    _run_cycle_full(q, k, v, q2, k2, v2, mask, blk)


@pytest.mark.parametrize("ramp", [rt.RT_RAMP_MUL_LINEAR, rt.RT_RAMP_ADD_LINEAR, rt.RT_RAMP_GEOMETRIC])
def test_ramp_modes_and_fp32_residual(ramp):
    B, H, L, d, blk = 2, 3, 520, 64, 128
    q, k, v = inputs.random_qkv(B, H, L, d, seed=5, device=DEV)
    q2, k2, v2 = inputs.random_qkv(B, H, L, d, seed=6, device=DEV)
    mask = inputs.random_block_mask(H, 5, 5, 0.4, seed=7)           # per-head masks, some empty rows
    _run_cycle_full(q, k, v, q2, k2, v2, mask, blk, lam=0.04, kdist=3, ramp=ramp, r_dtype=torch.float32)


@pytest.mark.parametrize("d", [72, 88, 128])
def test_fp32_residual_padded_dims(d):
    B, H, L, blk = 1, 2, 400, 128
    q, k, v = inputs.random_qkv(B, H, L, d, seed=11, device=DEV)
    q2, k2, v2 = inputs.random_qkv(B, H, L, d, seed=12, device=DEV)
    mask = inputs.random_block_mask(1, 4, 4, 0.5, seed=13, ensure_nonempty=True)
    _run_cycle_full(q, k, v, q2, k2, v2, mask, blk, r_dtype=torch.float32)


def test_block64_and_scale_override():
    B, H, L, d, blk = 1, 2, 200, 64, 64        # 4 query blocks of 64, tail of 8
    q, k, v = inputs.random_qkv(B, H, L, d, seed=21, device=DEV)
    q2, k2, v2 = inputs.random_qkv(B, H, L, d, seed=22, device=DEV)
    mask = inputs.random_block_mask(1, 4, 4, 0.5, seed=23)
    _run_cycle_full(q, k, v, q2, k2, v2, mask, blk, scale=0.1)


def _climbing_qkv(B, H, L, d, blk, step_log2, seed):
    """Q along one unit direction u per head, K = c_j u + N(0, 1) noise with c_j
    growing by step_log2 (in log2 units of the logits) per key block j, V ~ N(0, 1):
    the row max rises block after block, so the online softmax must rescale
    whenever a block raises it by more than 2^8."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    u = torch.randn((B, H, 1, d), generator=g, dtype=torch.float64)
    u = u / u.norm(dim=-1, keepdim=True)
    q = math.sqrt(d) * u + 0.3 * torch.randn((B, H, L, d), generator=g, dtype=torch.float64)
    c = (step_log2 * math.log(2.0)) * (torch.arange(L, dtype=torch.float64) // blk)
    k = c.view(1, 1, L, 1) * u + torch.randn((B, H, L, d), generator=g, dtype=torch.float64)
    v = torch.randn((B, H, L, d), generator=g, dtype=torch.float64)
    drift = [0.05 * torch.randn((B, H, L, d), generator=g, dtype=torch.float64) for _ in range(3)]
    bf = lambda t: t.to(torch.bfloat16).to(DEV)
    return (bf(q), bf(k), bf(v)), (bf(q + drift[0]), bf(k + drift[1]), bf(v + drift[2]))


@pytest.mark.parametrize("d", [64, 88, 128])
@pytest.mark.parametrize("case", ["climbing_keys", "large_scale"])
def test_lazy_rescale_paths(d, case):
    """Blocks that raise the running row max by more than 2^8 take the rescale
    path of every kernel: in the calibration also at the switch from masked to
    kept blocks (row 0 keeps only the highest block, visited after all the
    masked ones), and with every row shape (one kept block, the first block
    only, a mixed row, a dense row, an empty row)."""
    B, H, L, blk = 1, 2, 600, 128               # 5 blocks, tail of 88
    mask = np.array([[[0, 0, 0, 0, 1],
                      [1, 0, 0, 0, 0],
                      [0, 0, 1, 0, 1],
                      [1, 1, 1, 1, 1],
                      [0, 0, 0, 0, 0]]], dtype=np.uint8)
    if case == "climbing_keys":
        (q, k, v), (q2, k2, v2) = _climbing_qkv(B, H, L, d, blk, step_log2=6.0, seed=d)
        _run_cycle_full(q, k, v, q2, k2, v2, mask, blk)
    else:
        # Logits of standard deviation sqrt(d): block maxima differ by far more
        # than 2^8, and the softmax is close to one-hot, so O copies single V
        # entries, some beyond 4 in magnitude, where half a bf16 ulp of the
        # output alone is 2^-6 > 1e-2.  The bounds add 2^-8 |O| (element-wise)
        # and 2^-8 mean |O| (mean): the bf16 rounding of O and of the
        # probabilities P, 2^-9 each.
        q, k, v = inputs.random_qkv(B, H, L, d, seed=40 + d, device=DEV)
        q2, k2, v2 = inputs.random_qkv(B, H, L, d, seed=50 + d, device=DEV)
        _run_cycle_full(q, k, v, q2, k2, v2, mask, blk, scale=1.0, rel=2.0 ** -8)


def test_dense_and_empty_masks():
    B, H, L, d, blk = 1, 2, 384, 64, 128
    q, k, v = inputs.random_qkv(B, H, L, d, seed=31, device=DEV)
    dense = np.ones((1, 3, 3), dtype=np.uint8)
    idx = _index(dense)
    o, rho, r = rt.rt_calibrate(q, k, v, idx, block=blk)
    torch.cuda.synchronize()
    _ok()
    assert torch.all(rho == 1.0)
    assert torch.all(r == 0)
    o_full = ref.full_attention_ref(f64(q), f64(k), f64(v))
    check_out(f64(o), o_full, "dense calibrate O")
    empty = np.zeros((1, 3, 3), dtype=np.uint8)
    idx0 = _index(empty)
    assert idx0.nnz == 0
    o, rho, r = rt.rt_calibrate(q, k, v, idx0, block=blk)
    torch.cuda.synchronize()
    _ok()
    assert torch.all(rho == 0.0)
    check_out(f64(r), o_full, "empty-mask R is the full output")
    rho_s, r_s = _stats_inputs((B, H, L, d), 5)
    o2 = rt.rt_sparse_step(q, k, v, idx0, rho_s, r_s, block=blk)
    torch.cuda.synchronize()
    _ok()
    assert torch.equal(o2, r_s)                # empty kept set: O' = R exactly


@pytest.mark.parametrize("d", [72, 88, 128])
@pytest.mark.parametrize("r_dtype", [torch.bfloat16, torch.float32])
def test_dense_empty_and_mixed_rows_padded_dims(d, r_dtype):
    """The d > 64 calibration keeps one accumulator and orders masked blocks
    before kept ones: a row with no masked block, a row with no kept block and
    rows with both take different paths through it."""
    B, H, L, blk = 1, 2, 4 * 128 - 30, 128               # 4 query blocks, ragged tail
    q, k, v = inputs.random_qkv(B, H, L, d, seed=60 + d, device=DEV)
    q2, k2, v2 = inputs.random_qkv(B, H, L, d, seed=160 + d, device=DEV)
    mixed = np.array([[[1, 1, 1, 1],                      # dense row: no masked block
                       [0, 0, 0, 0],                      # empty row: no kept block
                       [0, 1, 0, 1],                      # kept blocks include the tail block
                       [1, 0, 1, 0]]], dtype=np.uint8)    # the tail block is masked
    _run_cycle_full(q, k, v, q2, k2, v2, mixed, blk, r_dtype=r_dtype)
    o_full = ref.full_attention_ref(f64(q), f64(k), f64(v))
    for mask, rho_want in ((np.ones((1, 4, 4), np.uint8), 1.0), (np.zeros((1, 4, 4), np.uint8), 0.0)):
        o, rho, r = rt.rt_calibrate(q, k, v, _index(mask), block=blk, r_dtype=r_dtype)
        torch.cuda.synchronize()
        _ok()
        assert torch.all(rho == rho_want)
        check_out(f64(o), o_full, "calibrate O")
        if rho_want == 1.0:
            assert torch.all(r == 0)
        else:
            check_out(f64(r), o_full, "all-masked R is the full output")


@pytest.mark.parametrize("vscale", [1e-3, 300.0])
def test_residual_copy_row_scale_extremes(vscale):
    """At d = 128 with a bf16 residual the masked-block accumulator is kept as
    f16 with a power-of-two row scale; very small and very large V exercise
    that scale.  Errors are compared in units of the V scale."""
    B, H, L, d, blk = 1, 2, 3 * 128, 128, 128
    q, k, v = inputs.random_qkv(B, H, L, d, seed=71, device=DEV)
    v = (v.float() * vscale).to(torch.bfloat16)
    mask = np.array([[[1, 0, 0], [0, 1, 0], [1, 0, 1]]], dtype=np.uint8)
    o, rho, r = rt.rt_calibrate(q, k, v, _index(mask), block=blk)
    torch.cuda.synchronize()
    _ok()
    O, RHO, R = ref.calibrate_ref(f64(q), f64(k), f64(v), mask, blk)
    check_out(f64(o) / vscale, O / vscale, "calibrate O / vscale")
    check_out(f64(r) / vscale, R / vscale, "calibrate R / vscale")
    check_rho(f64(rho), RHO)


@pytest.mark.parametrize("d,blk,r_dtype", [(64, 128, torch.bfloat16), (88, 128, torch.bfloat16),
                                           (128, 128, torch.bfloat16), (128, 128, torch.float32),
                                           (64, 64, torch.float32)])
def test_epilogue_variants_and_subtractive_residual(d, blk, r_dtype):
    """The ablation epilogues (no rho, no R) and DiTFastAttn's subtractive
    residual with its reconstruction, on every kernel family (d = 64 ping-pong,
    d > 64 persistent, 64-token blocks)."""
    B, H, L = 1, 2, 3 * blk + 17
    q, k, v = inputs.random_qkv(B, H, L, d, seed=80 + d + blk, device=DEV)
    q2, k2, v2 = inputs.random_qkv(B, H, L, d, seed=180 + d + blk, device=DEV)
    nb = -(-L // blk)
    mask = inputs.random_block_mask(1, nb, nb, 0.4, seed=81)
    mask[0, 1, :] = 0                                   # one query block with no kept key block
    idx = _index(mask)
    lam, kd = 0.04, 2
    # Re-ttention's residual, then the two ablations of the sparse step
    o, rho, r = rt.rt_calibrate(q, k, v, idx, block=blk, r_dtype=r_dtype)
    o_norho = rt.rt_sparse_step(q2, k2, v2, idx, None, r, block=blk, lam=lam, step_distance=kd,
                                epilogue=rt.RT_EPI_NO_RHO)
    o_nor = rt.rt_sparse_step(q2, k2, v2, idx, rho, None, block=blk, lam=lam, step_distance=kd,
                              epilogue=rt.RT_EPI_NO_R)
    # DiTFastAttn: subtractive residual at calibration, attn + R_sub later
    o_s, rho_s, r_sub = rt.rt_calibrate(q, k, v, idx, block=blk, r_dtype=r_dtype,
                                        residual=rt.RT_RES_SUBTRACTIVE)
    o_dfa = rt.rt_sparse_step(q2, k2, v2, idx, None, r_sub, block=blk, lam=lam, step_distance=kd,
                              epilogue=rt.RT_EPI_NO_RHO)
    torch.cuda.synchronize()
    _ok()
    O, RHO, R = ref.calibrate_ref(f64(q), f64(k), f64(v), mask, blk)
    check_out(f64(o_s), O, "calibrate O (subtractive residual)")
    check_rho(f64(rho_s), RHO)
    R_SUB = ref.ditfastattn_residual_ref(f64(q), f64(k), f64(v), mask, blk)
    check_out(f64(r_sub), R_SUB, "subtractive residual O - O_sparse")
    args = (f64(q2), f64(k2), f64(v2), mask, blk)
    check_out(f64(o_norho), ref.sparse_step_epilogue_ref(*args, None, f64(r), lam, kd, ref.EPI_NO_RHO),
              "sparse O, no rho")
    check_out(f64(o_nor), ref.sparse_step_epilogue_ref(*args, f64(rho), None, lam, kd, ref.EPI_NO_R),
              "sparse O, no R")
    check_out(f64(o_dfa), ref.sparse_step_epilogue_ref(*args, None, R_SUB, lam, kd, ref.EPI_NO_RHO),
              "DiTFastAttn reconstruction")


def _drifting_steps(B, H, L, d, n, seed):
    x = inputs.random_qkv(B, H, L, d, seed=seed, device=DEV)
    steps = [x]
    g = torch.Generator(device=DEV).manual_seed(seed + 1)
    for _ in range(n - 1):
        x = tuple((t.float() + 0.05 * torch.randn(t.shape, generator=g, device=DEV)).to(torch.bfloat16)
                  for t in x)
        steps.append(x)
    return steps


@pytest.mark.parametrize("d,epilogue,residual", [(64, rt.RT_EPI_RESHAPED, rt.RT_RES_MASKED),
                                                 (128, rt.RT_EPI_RESHAPED, rt.RT_RES_MASKED),
                                                 (88, rt.RT_EPI_NO_RHO, rt.RT_RES_SUBTRACTIVE)])
def test_schedule_steps_match_oracle_schedule(d, epilogue, residual):
    """Seven denoising steps with a calibration every three, on inputs that
    drift from step to step: Re-ttention's schedule and DiTFastAttn's."""
    B, H, L, blk, period, lam = 1, 2, 3 * 128 - 40, 128, 3, 0.04
    steps = _drifting_steps(B, H, L, d, 7, seed=90 + d)
    mask = inputs.random_block_mask(1, 3, 3, 0.5, seed=91, ensure_nonempty=True)
    idx = _index(mask)
    rho = torch.empty((B, H, L), dtype=torch.float32, device=DEV)
    r = torch.empty_like(steps[0][0])
    outs = []
    for t, (q, k, v) in enumerate(steps):
        outs.append(rt.rt_schedule_step(q, k, v, idx, t, block=blk, period=period, lam=lam, o=torch.empty_like(q),
                                        rho=rho, r=r, epilogue=epilogue, residual=residual))
    torch.cuda.synchronize()
    _ok()
    want = ref.schedule_ref([tuple(f64(x) for x in s) for s in steps], mask, blk, period, lam,
                            epilogue=epilogue, residual=residual)
    for t, (o, w) in enumerate(zip(outs, want)):
        check_out(f64(o), w, f"schedule step {t}")


def test_cycle_graph_replays_the_eager_cycle_bit_exactly():
    """A captured calibration cycle launched twice gives exactly the outputs of
    the same steps run one call at a time (one launch per cycle instead of
    `period`)."""
    B, H, L, d, blk, period = 1, 2, 4 * 128, 128, 128, 4
    steps = _drifting_steps(B, H, L, d, period, seed=95)
    mask = inputs.random_block_mask(1, 4, 4, 0.4, seed=96, ensure_nonempty=True)
    idx = _index(mask)
    rho = torch.empty((B, H, L), dtype=torch.float32, device=DEV)
    r = torch.empty_like(steps[0][0])
    eager = [rt.rt_schedule_step(q, k, v, idx, t, block=blk, period=period, o=torch.empty_like(q), rho=rho, r=r)
             for t, (q, k, v) in enumerate(steps)]
    torch.cuda.synchronize()
    _ok()
    eager = [o.clone() for o in eager]
    outs = [torch.zeros_like(steps[0][0]) for _ in range(period)]
    rho_g, r_g = torch.empty_like(rho), torch.empty_like(r)
    s = torch.cuda.Stream()
    graph = rt.CycleGraph(steps, idx, block=blk, outs=outs, rho=rho_g, r=r_g, stream=s)
    try:
        torch.cuda.synchronize()
        assert all(torch.count_nonzero(o) == 0 for o in outs)      # capturing launched nothing
        for _ in range(2):
            graph.launch(stream=s)
            s.synchronize()
            _ok()
            for o, e in zip(outs, eager):
                assert torch.equal(o, e)
            assert torch.equal(rho_g, rho) and torch.equal(r_g, r)
            for o in outs:
                o.zero_()
            torch.cuda.synchronize()                              # zeroed before the next replay writes
    finally:
        graph.close()


def test_invariant_same_inputs_lambda0_gives_full_attention():
    w = inputs.WORKLOADS["pixart"]
    q, k, v = inputs.initial_qkv(w, device=DEV)
    idx = _index(inputs.block_mask(w))
    o, rho, r = rt.rt_calibrate(q, k, v, idx, block=w.block, r_dtype=torch.float32)
    o2 = rt.rt_sparse_step(q, k, v, idx, rho, r, block=w.block, lam=0.0, step_distance=1)
    torch.cuda.synchronize()
    _ok()
    full = torch.nn.functional.scaled_dot_product_attention(q.float(), k.float(), v.float())
    check_out(f64(o2), f64(full), "sparse(lambda=0) vs full attention")
    check_out(f64(o), f64(full), "calibrate O vs full attention")


def test_strided_layout_bsHd():
    """[B, L, H, d] storage viewed as [B, H, L, d] (non-contiguous strides)."""
    B, H, L, d, blk = 2, 4, 256, 64, 128
    g = torch.Generator(device=DEV).manual_seed(41)
    base = [torch.randn((B, L, H, d), generator=g, device=DEV).to(torch.bfloat16) for _ in range(6)]
    q, k, v, q2, k2, v2 = (t.permute(0, 2, 1, 3) for t in base)
    mask = inputs.random_block_mask(1, 2, 2, 0.5, seed=42, ensure_nonempty=True)
    idx = _index(mask)
    o = torch.empty_like(base[0]).permute(0, 2, 1, 3)
    r = torch.empty_like(base[0]).permute(0, 2, 1, 3)
    o, rho, r = rt.rt_calibrate(q, k, v, idx, block=blk, o=o, r=r)
    o2 = torch.empty_like(base[0]).permute(0, 2, 1, 3)
    o2 = rt.rt_sparse_step(q2, k2, v2, idx, rho, r, block=blk, o=o2)
    torch.cuda.synchronize()
    _ok()
    O, RHO, R = ref.calibrate_ref(f64(q), f64(k), f64(v), mask, blk)
    check_out(f64(o), O, "strided O")
    check_out(f64(r), R, "strided R")
    check_rho(f64(rho), RHO)
    O2 = ref.sparse_step_ref(f64(q2), f64(k2), f64(v2), mask, blk, RHO, R, 0.04, 1)
    check_out(f64(o2), O2, "strided sparse O")


# ---------------------------------------------------------------------------
# full-size workloads, sampled rows (launched as bench.py launches them)
# ---------------------------------------------------------------------------

def _sample_rows(L, block, rng, n_mid=6):
    nqb = -(-L // block)
    blocks = sorted(set([0, 1, nqb - 1] + list(rng.integers(0, nqb, n_mid))))
    rows = []
    for qb in blocks:
        lo, hi = qb * block, min(L, (qb + 1) * block)
        rows += [lo, hi - 1, int(rng.integers(lo, hi))]
    return np.array(sorted(set(rows)))


@pytest.mark.parametrize("name", ["pixart", "hunyuan"])
def test_workload_schedule_full_tensors(name):
    """The configuration's own cycle, 1 calibration + 4 sparse steps at
    k = 1..4 on inputs that drift from step to step, through the schedule
    driver, against the oracle's schedule on every element."""
    w = inputs.WORKLOADS[name]
    period = 1 + w.n_sparse_steps
    steps = inputs.qkv_steps(w, period, device=DEV)
    mask = inputs.block_mask(w)
    idx = _index(mask)
    rho = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=DEV)
    r = torch.empty_like(steps[0][0])
    outs = [rt.rt_schedule_step(q, k, v, idx, t, block=w.block, period=period, lam=w.lam, o=torch.empty_like(q),
                                rho=rho, r=r) for t, (q, k, v) in enumerate(steps)]
    torch.cuda.synchronize()
    _ok()
    want = ref.schedule_ref([tuple(f64(x) for x in s) for s in steps], mask, w.block, period, w.lam)
    for t, (o, wt) in enumerate(zip(outs, want)):
        check_out(f64(o), wt, f"{name} schedule step {t} (k = {t})")


def test_cogvideox_cycle_sampled_rows_k1_and_k9():
    """CogVideoX-like cycle, 1 calibration + 9 sparse steps through the
    schedule driver at full size; sampled rows of the calibration and of the
    sparse steps at k = 1 and k = 9 against the oracle."""
    w = inputs.WORKLOADS["cogvideox"]
    period = 1 + w.n_sparse_steps
    steps = inputs.qkv_steps(w, period, device=DEV)
    mask = inputs.block_mask(w)
    idx = _index(mask)
    rho = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=DEV)
    r = torch.empty_like(steps[0][0])
    outs = [rt.rt_schedule_step(q, k, v, idx, t, block=w.block, period=period, lam=w.lam, o=torch.empty_like(q),
                                rho=rho, r=r) for t, (q, k, v) in enumerate(steps)]
    torch.cuda.synchronize()
    _ok()
    rng = np.random.default_rng(33)
    for b, h in [(0, 0), (0, w.H - 1), (0, int(rng.integers(w.H)))]:
        rows = _sample_rows(w.L, w.block, rng)
        O, RHO, R = ref.calibrate_rows_ref(*(f64(x[b, h]) for x in steps[0]), mask[0], w.block, rows)
        check_out(f64(outs[0][b, h, rows]), O, f"cogvideox calibrate O (h{h})")
        check_out(f64(r[b, h, rows]), R, f"cogvideox calibrate R (h{h})")
        check_rho(f64(rho[b, h, rows]), RHO, f"cogvideox rho (h{h})")
        for t in (1, w.n_sparse_steps):
            O2 = ref.sparse_step_rows_ref(*(f64(x[b, h]) for x in steps[t]), mask[0], w.block, rows, RHO, R,
                                          w.lam, t)
            check_out(f64(outs[t][b, h, rows]), O2, f"cogvideox sparse O at k = {t} (h{h})")
    del steps, outs
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["cogvideox", "longvideo-3.1", "longvideo-6.25", "longvideo-12.5", "longvideo-25"])
def test_full_size_sampled_rows(name):
    w = inputs.WORKLOADS[name]
    steps = inputs.qkv_steps(w, 2, device=DEV)
    mask = inputs.block_mask(w)
    idx = _index(mask)
    (q, k, v), (q2, k2, v2) = steps
    o, rho, r = rt.rt_calibrate(q, k, v, idx, block=w.block)
    o2 = rt.rt_sparse_step(q2, k2, v2, idx, rho, r, block=w.block, lam=w.lam, step_distance=1)
    torch.cuda.synchronize()
    _ok()
    rng = np.random.default_rng(w.seed)
    heads = [(0, 0), (w.B - 1, w.H - 1), (0, int(rng.integers(w.H)))]
    for b, h in heads:
        rows = _sample_rows(w.L, w.block, rng)
        qf, kf, vf = f64(q[b, h]), f64(k[b, h]), f64(v[b, h])
        O, RHO, R = ref.calibrate_rows_ref(qf, kf, vf, mask[0], w.block, rows)
        check_out(f64(o[b, h, rows]), O, f"{name} calibrate O (b{b} h{h})")
        check_out(f64(r[b, h, rows]), R, f"{name} calibrate R (b{b} h{h})")
        check_rho(f64(rho[b, h, rows]), RHO, f"{name} rho")
        O2 = ref.sparse_step_rows_ref(f64(q2[b, h]), f64(k2[b, h]), f64(v2[b, h]), mask[0], w.block, rows,
                                      RHO, R, w.lam, 1)
        check_out(f64(o2[b, h, rows]), O2, f"{name} sparse O (b{b} h{h})")
    # properties that hold at any size
    assert torch.all(torch.isfinite(o.float())) and torch.all(torch.isfinite(o2.float()))
    assert torch.all((rho >= 0) & (rho <= 1.0 + 1e-6))
    del steps, q, k, v, q2, k2, v2, o, o2, r, rho
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# device-side error paths (never fault: bad index is detected and recorded)
# ---------------------------------------------------------------------------

def _bad_index_run(row_ptr, col_idx, nqb):
    B, H, L, d, blk = 1, 2, nqb * 128, 64, 128
    q, k, v = inputs.random_qkv(B, H, L, d, seed=3, device=DEV)
    idx = rt.make_block_index(torch.tensor(row_ptr, dtype=torch.int32, device=DEV),
                              torch.tensor(col_idx, dtype=torch.int32, device=DEV), 1, nqb, nqb)
    rt.rt_calibrate(q, k, v, idx, block=blk)
    return rt.rt_check_device_error()


def test_bad_col_idx_out_of_range_recorded():
    assert _bad_index_run([0, 1, 2], [0, 5], 2) == rt.RT_ERR_BAD_INDEX
    assert rt.rt_check_device_error() == rt.RT_OK            # cleared


def test_bad_col_idx_not_ascending_recorded():
    assert _bad_index_run([0, 2, 3], [1, 0, 1], 2) == rt.RT_ERR_BAD_INDEX


def test_bad_row_ptr_recorded():
    assert _bad_index_run([0, 3, 2], [0, 1], 2) == rt.RT_ERR_BAD_INDEX


def test_sparse_step_bad_row_recorded_good_rows_correct():
    """One corrupt CSR row among good ones: the persistent sparse kernel records
    RT_ERR_BAD_INDEX, skips that tile and still computes every other tile."""
    B, H, L, d, blk = 1, 2, 512, 64, 128
    q, k, v = inputs.random_qkv(B, H, L, d, seed=51, device=DEV)
    mask = np.array([[[1, 0, 0, 0], [1, 1, 0, 0], [0, 1, 1, 0], [0, 0, 1, 1]]], dtype=np.uint8)
    rp, ci = ref.build_block_index_ref(mask)
    ci_bad = ci.copy()
    ci_bad[rp[2]] = 9                                         # row 2 points past nkb
    idx = rt.make_block_index(torch.from_numpy(rp).to(DEV), torch.from_numpy(ci_bad).to(DEV), 1, 4, 4)
    rho_s, r_s = _stats_inputs((B, H, L, d), 52)
    o = torch.zeros_like(q)
    rt.rt_sparse_step(q, k, v, idx, rho_s, r_s, block=blk, lam=0.04, step_distance=2, o=o)
    assert rt.rt_check_device_error() == rt.RT_ERR_BAD_INDEX
    want = ref.sparse_step_ref(f64(q), f64(k), f64(v), mask, blk, f64(rho_s), f64(r_s), 0.04, 2)
    got = f64(o)
    good = np.r_[0:256, 384:512]
    check_out(got[:, :, good], want[:, :, good], "good rows")
    assert np.all(got[:, :, 256:384] == 0)                   # the bad tile wrote nothing


def test_good_index_after_errors_still_correct():
    test_workload_cycle_full("tiny")


def test_bounded_wait_reports_timeout():
    rt.rt_debug_wait_timeout(2_000_000)                     # 2 ms on a barrier nobody completes
    assert rt.rt_check_device_error() == rt.RT_ERR_TIMEOUT
    assert rt.rt_check_device_error() == rt.RT_OK


def test_host_validation_rejects_before_launch():
    q, k, v = inputs.random_qkv(1, 1, 128, 64, seed=0, device=DEV)
    idx = _index(np.ones((1, 1, 1), dtype=np.uint8))
    with pytest.raises(rt.RtError) as e:
        rt.rt_calibrate(q, k, v, idx, block=32)
    assert e.value.status == rt.RT_ERR_UNSUPPORTED
    q20, k20, v20 = inputs.random_qkv(1, 1, 128, 20, seed=0, device=DEV)
    with pytest.raises(rt.RtError) as e:
        rt.rt_calibrate(q20, k20, v20, idx, block=128)
    assert e.value.status == rt.RT_ERR_UNSUPPORTED
    bad_idx = rt.BlockIndex(idx.row_ptr, idx.col_idx, 1, 2, 2, idx.nnz)      # nqb inconsistent with L
    with pytest.raises(rt.RtError) as e:
        rt.rt_calibrate(q, k, v, bad_idx, block=128)
    assert e.value.status == rt.RT_ERR_INVALID_ARGUMENT
    _ok()


# ---------------------------------------------------------------------------
# token reordering
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("B,H,L,d,strided", [(1, 2, 300, 72, False), (2, 3, 1000, 128, False), (2, 4, 256, 64, True)])
def test_permute_tokens_bit_exact(B, H, L, d, strided):
    g = torch.Generator(device=DEV).manual_seed(L + d)
    if strided:                                      # [B, L, H, d] storage viewed as [B, H, L, d]
        x = torch.randn((B, L, H, d), generator=g, device=DEV).to(torch.bfloat16).transpose(1, 2)
    else:
        x = torch.randn((B, H, L, d), generator=g, device=DEV).to(torch.bfloat16)
    perm = torch.randperm(L, generator=g, device=DEV).to(torch.int32)
    y = rt.rt_permute_tokens(x, perm)
    z = rt.rt_permute_tokens(y, perm, inverse=True)
    torch.cuda.synchronize()
    _ok()
    assert torch.equal(y, x[:, :, perm.long()])
    assert torch.equal(z, x)


def test_permute_tokens_bad_entry_recorded():
    L = 200
    x = torch.randn((1, 2, L, 64), device=DEV).to(torch.bfloat16)
    perm = torch.arange(L, device=DEV, dtype=torch.int32)
    perm[7] = L                                      # out of range: recorded, row skipped
    y = torch.zeros_like(x)
    rt.rt_permute_tokens(x, perm, dst=y)
    assert rt.rt_check_device_error() == rt.RT_ERR_BAD_INDEX
    keep = torch.ones(L, dtype=torch.bool, device=DEV)
    keep[7] = False
    assert torch.equal(y[:, :, keep], x[:, :, keep])
    assert torch.count_nonzero(y[:, :, 7]) == 0


def test_reordered_tokens_calibrate_and_sparse_step():
    """Hilbert-ordered tokens with the block mask built on them: the GPU cycle
    matches the oracle on the reordered problem, and with a dense mask the
    reordered full attention scattered back equals raster full attention."""
    w = inputs.Workload("grid", 1, 2, 4 * 8 * 16 + 64, 64, 128, kept=2, n_sparse_steps=1, seed=7,
                        n_text=64, grid=(4, 8, 16))
    perm_h = rt.rt_hilbert_token_order(w.n_text, *w.grid)
    perm = perm_h.to(DEV)
    (q, k, v), (q2, k2, v2) = inputs.qkv_steps(w, 2, device=DEV)
    qp, kp, vp, q2p, k2p, v2p = (rt.rt_permute_tokens(t, perm) for t in (q, k, v, q2, k2, v2))
    mask = inputs.block_mask(w, perm_h.numpy())
    _run_cycle_full(qp, kp, vp, q2p, k2p, v2p, mask, w.block)
    dense = np.ones((1, w.nqb, w.nkb), dtype=np.uint8)
    o_p, _, _ = rt.rt_calibrate(qp, kp, vp, _index(dense), block=w.block)
    o_back = rt.rt_permute_tokens(o_p, perm, inverse=True)
    torch.cuda.synchronize()
    _ok()
    check_out(f64(o_back), ref.full_attention_ref(f64(q), f64(k), f64(v)), "reordered full attention, back")


# ---------------------------------------------------------------------------
# head sharding
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("per_head_mask,d", [(False, 128), (True, 64), (True, 88)])
def test_head_shards_reproduce_the_whole_problem(per_head_mask, d):
    """Each rank of a head-sharded run calls the library on strided views of
    its heads (and the slice of a per-head mask); the pieces equal the
    unsharded outputs exactly, since heads are independent."""
    from sparse_attention_diffusion_rt_b200 import shard
    B, H, L, blk, world = 2, 5, 3 * 128 - 20, 128, 2
    q, k, v = inputs.random_qkv(B, H, L, d, seed=120 + d, device=DEV)
    q2, k2, v2 = inputs.random_qkv(B, H, L, d, seed=121 + d, device=DEV)
    mask = inputs.random_block_mask(H if per_head_mask else 1, 3, 3, 0.5, seed=122, ensure_nonempty=True)
    idx = _index(mask)
    o, rho, r = rt.rt_calibrate(q, k, v, idx, block=blk)
    o2 = rt.rt_sparse_step(q2, k2, v2, idx, rho, r, block=blk, step_distance=2)
    for rank in range(world):
        h0, h1 = shard.head_range(H, world, rank)
        sl = lambda t: shard.shard_heads(t, h0, h1)
        idx_s = _index(shard.shard_mask(mask, h0, h1))
        o_s, rho_s, r_s = rt.rt_calibrate(sl(q), sl(k), sl(v), idx_s, block=blk)
        o2_s = rt.rt_sparse_step(sl(q2), sl(k2), sl(v2), idx_s, rho_s, r_s, block=blk, step_distance=2)
        torch.cuda.synchronize()
        _ok()
        assert torch.equal(o_s, sl(o)) and torch.equal(rho_s, sl(rho)) and torch.equal(r_s, sl(r))
        assert torch.equal(o2_s, sl(o2))
        # and each shard against the oracle on its own heads
        mask_s = shard.shard_mask(mask, h0, h1)
        O, RHO, R = ref.calibrate_ref(f64(sl(q)), f64(sl(k)), f64(sl(v)), mask_s, blk)
        check_out(f64(o_s), O, f"shard {rank} calibrate O")
        check_out(f64(r_s), R, f"shard {rank} calibrate R")
        check_rho(f64(rho_s), RHO, f"shard {rank} rho")
        O2 = ref.sparse_step_ref(f64(sl(q2)), f64(sl(k2)), f64(sl(v2)), mask_s, blk, RHO, R, 0.04, 2)
        check_out(f64(o2_s), O2, f"shard {rank} sparse O")
