"""Pins for the CPU oracle (no GPU).

Each test checks the oracle against something other than itself: values the
Re-ttention pages print (the worked 4-key example), a library routine (torch's
float64 softmax / scaled_dot_product_attention), a closed form (uniform logits,
dense mask), or an independent plain-C brute force on tiny inputs.  The last
tests plant mistakes in the oracle and check that the pins catch them.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from oracle import reference as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _worked_example():
    with open(os.path.join(GOLDEN, "worked_example_4key.json")) as f:
        return json.load(f)


def _example_inputs(p_row, d=4):
    """q = ln(p), K = sqrt(d) I, V = I: with c = 1/sqrt(d) the logits are ln(p)
    and every output row is the attention-probability row itself."""
    L = len(p_row)
    q = np.tile(np.log(np.asarray(p_row, dtype=np.float64)), (L, 1))[None, None]
    k = (math.sqrt(d) * np.eye(L))[None, None]
    v = np.eye(L)[None, None]
    return q, k, v


def _window_mask(keys, L=4):
    m = np.zeros((1, L, L), dtype=np.uint8)
    m[0, :, keys] = 1
    return m


# ---------------------------------------------------------------------------
# the pages' worked example
# ---------------------------------------------------------------------------

def test_worked_example_rettention():
    g = _worked_example()
    mask = _window_mask(g["window_keys"])
    q_t, k, v = _example_inputs(g["step_t"]["full"])
    o, rho, r = ref.calibrate_ref(q_t, k, v, mask, block=1)
    np.testing.assert_allclose(o[0, 0, 0], g["step_t"]["full"], atol=1e-14)
    np.testing.assert_allclose(r[0, 0, 0], g["step_t"]["rettention_residual"], atol=1e-14)
    np.testing.assert_allclose(rho[0, 0, 0], 0.8, atol=1e-14)
    # reshaped sparse row at step t (residual left out)
    zero = np.zeros_like(r)
    resh_t = ref.sparse_step_ref(q_t, k, v, mask, 1, rho, zero, 0.0, 0)
    np.testing.assert_allclose(resh_t[0, 0, 0], g["step_t"]["rettention_reshaped_sparse"], atol=1e-14)

    q_t1, _, _ = _example_inputs(g["step_t_plus_1"]["full"])
    ones = np.ones_like(rho)
    sparse_t1 = ref.sparse_step_ref(q_t1, k, v, mask, 1, ones, zero, 0.0, 0)
    np.testing.assert_allclose(sparse_t1[0, 0, 0], g["step_t_plus_1"]["sparse"], atol=1e-14)
    resh_t1 = ref.sparse_step_ref(q_t1, k, v, mask, 1, rho, zero, 0.0, 0)
    np.testing.assert_allclose(resh_t1[0, 0, 0], g["step_t_plus_1"]["rettention_reshaped_sparse"], atol=1e-14)
    rec = ref.sparse_step_ref(q_t1, k, v, mask, 1, rho, r, 0.0, 0)
    np.testing.assert_allclose(rec[0, 0, 0], g["step_t_plus_1"]["rettention_reconstruction"], atol=1e-14)
    np.testing.assert_allclose(rec[0, 0, 0], g["step_t_plus_1"]["full"], atol=1e-14)


def test_worked_example_ditfastattn_contrast():
    g = _worked_example()
    mask = _window_mask(g["window_keys"])
    q_t, k, v = _example_inputs(g["step_t"]["full"])
    ones = np.ones((1, 1, 4))
    zero = np.zeros((1, 1, 4, 4))
    sp_t = ref.sparse_step_ref(q_t, k, v, mask, 1, ones, zero, 0.0, 0)
    np.testing.assert_allclose(sp_t[0, 0, 0], g["step_t"]["ditfastattn_sparse"], atol=1e-14)
    r_sub = ref.ditfastattn_residual_ref(q_t, k, v, mask, 1)
    np.testing.assert_allclose(r_sub[0, 0, 0], g["step_t"]["ditfastattn_residual"], atol=1e-14)
    q_t1, _, _ = _example_inputs(g["step_t_plus_1"]["full"])
    rec = ref.sparse_step_ref(q_t1, k, v, mask, 1, ones, r_sub, 0.0, 0)
    np.testing.assert_allclose(rec[0, 0, 0], g["step_t_plus_1"]["ditfastattn_reconstruction"], atol=1e-14)


def test_worked_example_epilogue_variants():
    """The named epilogues reproduce the worked example's rows: without R the
    reshaped sparse row, without rho and with DiTFastAttn's R_sub its
    reconstruction, and the full Re-ttention epilogue the full row."""
    g = _worked_example()
    mask = _window_mask(g["window_keys"])
    q_t, k, v = _example_inputs(g["step_t"]["full"])
    _, rho, r = ref.calibrate_ref(q_t, k, v, mask, 1)
    r_sub = ref.ditfastattn_residual_ref(q_t, k, v, mask, 1)
    q_t1, _, _ = _example_inputs(g["step_t_plus_1"]["full"])
    no_r = ref.sparse_step_epilogue_ref(q_t1, k, v, mask, 1, rho, None, 0.0, 0, ref.EPI_NO_R)
    np.testing.assert_allclose(no_r[0, 0, 0], g["step_t_plus_1"]["rettention_reshaped_sparse"], atol=1e-14)
    no_rho = ref.sparse_step_epilogue_ref(q_t1, k, v, mask, 1, None, r_sub, 0.0, 0, ref.EPI_NO_RHO)
    np.testing.assert_allclose(no_rho[0, 0, 0], g["step_t_plus_1"]["ditfastattn_reconstruction"], atol=1e-14)
    full = ref.sparse_step_epilogue_ref(q_t1, k, v, mask, 1, rho, r, 0.0, 0, ref.EPI_RESHAPED)
    np.testing.assert_allclose(full[0, 0, 0], g["step_t_plus_1"]["full"], atol=1e-14)
    with pytest.raises(ValueError):
        ref.sparse_step_epilogue_ref(q_t1, k, v, mask, 1, rho, r, 0.0, 0, 7)


def test_worked_example_as_a_schedule():
    """The worked example is a two-step schedule: a calibration at t, then the
    step t+1 from the cached statistics.  Re-ttention reconstructs the full row
    exactly; DiTFastAttn's residual caching gives its printed row."""
    g = _worked_example()
    mask = _window_mask(g["window_keys"])
    q_t, k, v = _example_inputs(g["step_t"]["full"])
    q_t1, _, _ = _example_inputs(g["step_t_plus_1"]["full"])
    steps = [(q_t, k, v), (q_t1, k, v)]
    outs = ref.schedule_ref(steps, mask, 1, 2, 0.0)
    np.testing.assert_allclose(outs[0][0, 0, 0], g["step_t"]["full"], atol=1e-14)
    np.testing.assert_allclose(outs[1][0, 0, 0], g["step_t_plus_1"]["rettention_reconstruction"], atol=1e-14)
    dfa = ref.schedule_ref(steps, mask, 1, 2, 0.0, epilogue=ref.EPI_NO_RHO, residual=ref.RES_SUBTRACTIVE)
    np.testing.assert_allclose(dfa[1][0, 0, 0], g["step_t_plus_1"]["ditfastattn_reconstruction"], atol=1e-14)


def test_schedule_period_one_is_full_attention_and_static_inputs_stay_exact():
    q, k, v = (_rand((1, 2, 96, 8), s) for s in (1, 2, 3))
    q2 = q + 0.1 * _rand(q.shape, 4)
    mask = np.array([[[1, 0, 0], [0, 1, 1], [1, 0, 1]]], dtype=np.uint8)
    full = [ref.full_attention_ref(*x) for x in ((q, k, v), (q2, k, v))]
    outs = ref.schedule_ref([(q, k, v), (q2, k, v)], mask, 32, 1, 0.04)       # every step calibrates
    for o, f in zip(outs, full):
        np.testing.assert_allclose(o, f, atol=1e-12)
    # unchanged inputs and no ramp: every sparse step reproduces full attention
    outs = ref.schedule_ref([(q, k, v)] * 4, mask, 32, 4, 0.0)
    for o in outs:
        np.testing.assert_allclose(o, full[0], atol=1e-12)
    # with a ramp the sparse steps move away from it, more with the step distance
    outs = ref.schedule_ref([(q, k, v)] * 4, mask, 32, 4, 0.04)
    errs = [np.abs(o - full[0]).max() for o in outs]
    assert errs[0] < 1e-12 and 0 < errs[1] < errs[2] < errs[3]


# ---------------------------------------------------------------------------
# library routines and closed forms
# ---------------------------------------------------------------------------

def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(q, k, v, scale=None):
    t = [torch.from_numpy(x) for x in (q, k, v)]
    return torch.nn.functional.scaled_dot_product_attention(*t, scale=scale).numpy()


@pytest.mark.parametrize("L,d", [(70, 24), (128, 64), (33, 72)])
def test_full_attention_matches_torch_sdpa(L, d):
    q, k, v = (_rand((1, 2, L, d), s) for s in (1, 2, 3))
    np.testing.assert_allclose(ref.full_attention_ref(q, k, v), _sdpa(q, k, v), atol=1e-12)


def test_rho_and_residual_match_library_softmax():
    """rho_i = sum of the full softmax over the window; R_i = (full softmax
    outside the window) . V -- computed here with torch's float64 softmax."""
    B, H, L, d, blk = 1, 2, 50, 16, 8
    q, k, v = (_rand((B, H, L, d), s) for s in (4, 5, 6))
    mask = ref_mask = np.random.default_rng(7).random((1, 7, 7)) < 0.4
    o, rho, r = ref.calibrate_ref(q, k, v, mask.astype(np.uint8), blk)
    p = torch.softmax(torch.from_numpy(q) @ torch.from_numpy(k).transpose(-1, -2) / math.sqrt(d), dim=-1)
    keep = torch.from_numpy(ref.token_keep_mask(ref_mask[0], blk, L))
    rho_lib = (p * keep).sum(-1).numpy()
    r_lib = ((p * ~keep) @ torch.from_numpy(v)).numpy()
    np.testing.assert_allclose(rho, rho_lib, atol=1e-13)
    np.testing.assert_allclose(r, r_lib, atol=1e-13)
    np.testing.assert_allclose(o, _sdpa(q, k, v), atol=1e-12)


def test_invariant_same_inputs_no_ramp_is_full_attention():
    """O' = rho * sparse softmax . V + R equals full attention when the inputs
    have not changed and no ramp is applied."""
    B, H, L, d, blk = 2, 3, 61, 8, 16
    q, k, v = (_rand((B, H, L, d), s) for s in (8, 9, 10))
    mask = (np.random.default_rng(11).random((H, 4, 4)) < 0.5).astype(np.uint8)
    o, rho, r = ref.calibrate_ref(q, k, v, mask, blk)
    full = _sdpa(q, k, v)
    for mode in (ref.RAMP_MUL_LINEAR, ref.RAMP_ADD_LINEAR, ref.RAMP_GEOMETRIC):
        np.testing.assert_allclose(ref.sparse_step_ref(q, k, v, mask, blk, rho, r, 0.0, 3, mode), full, atol=1e-12)
        np.testing.assert_allclose(ref.sparse_step_ref(q, k, v, mask, blk, rho, r, 0.04, 0, mode), full, atol=1e-12)


def test_dense_mask_rho_one_residual_zero():
    B, H, L, d, blk = 1, 2, 40, 8, 16
    q, k, v = (_rand((B, H, L, d), s) for s in (12, 13, 14))
    mask = np.ones((1, 3, 3), dtype=np.uint8)
    o, rho, r = ref.calibrate_ref(q, k, v, mask, blk)
    assert np.all(rho == 1.0)
    assert np.all(r == 0.0)
    np.testing.assert_allclose(ref.sparse_step_ref(q, k, v, mask, blk, rho, r, 0.04, 2), _sdpa(q, k, v), atol=1e-12)


def test_uniform_logits_closed_form():
    """q = 0: every logit is 0, so rho_i = |M(i)| / L and R_i = sum_{j not in M(i)} v_j / L."""
    B, H, L, d, blk = 1, 1, 45, 8, 8
    q = np.zeros((B, H, L, d))
    k, v = _rand((B, H, L, d), 15), _rand((B, H, L, d), 16)
    mask = (np.random.default_rng(17).random((1, 6, 6)) < 0.5).astype(np.uint8)
    o, rho, r = ref.calibrate_ref(q, k, v, mask, blk)
    keep = ref.token_keep_mask(mask[0], blk, L)
    np.testing.assert_allclose(rho[0, 0], keep.sum(1) / L, atol=1e-15)
    np.testing.assert_allclose(r[0, 0], (~keep).astype(float) @ v[0, 0] / L, atol=1e-14)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(v[0, 0].mean(0), (L, d)), atol=1e-14)


def test_empty_row_returns_residual():
    B, H, L, d, blk = 1, 1, 32, 8, 8
    q, k, v = (_rand((B, H, L, d), s) for s in (18, 19, 20))
    mask = np.ones((1, 4, 4), dtype=np.uint8)
    mask[0, 2] = 0
    rho = np.random.default_rng(21).random((B, H, L))
    r = _rand((B, H, L, d), 22)
    out = ref.sparse_step_ref(q, k, v, mask, blk, rho, r, 0.04, 1)
    np.testing.assert_array_equal(out[0, 0, 16:24], r[0, 0, 16:24])


def test_ramp_modes():
    rho = np.array([0.0, 0.2, 0.5, 0.9, 1.0])
    for mode in (ref.RAMP_MUL_LINEAR, ref.RAMP_ADD_LINEAR, ref.RAMP_GEOMETRIC):
        np.testing.assert_array_equal(ref.ramp_ref(rho, 0.0, 4, mode), rho)
        np.testing.assert_array_equal(ref.ramp_ref(rho, 0.04, 0, mode), rho)
        prev = rho
        for k in range(1, 12):
            cur = ref.ramp_ref(rho, 0.04, k, mode)
            assert np.all(cur >= prev) and np.all(cur <= 1.0)
            prev = cur
    np.testing.assert_allclose(ref.ramp_ref(0.5, 0.04, 2, ref.RAMP_MUL_LINEAR), 0.54, rtol=1e-15)
    np.testing.assert_allclose(ref.ramp_ref(0.5, 0.04, 2, ref.RAMP_ADD_LINEAR), 0.58, rtol=1e-15)
    np.testing.assert_allclose(ref.ramp_ref(0.5, 0.04, 2, ref.RAMP_GEOMETRIC), 0.5 * 1.04 ** 2, rtol=1e-15)
    assert ref.ramp_ref(0.99, 0.5, 5, ref.RAMP_MUL_LINEAR) == 1.0


# ---------------------------------------------------------------------------
# independent brute force (plain C, token-level mask)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("L,d,blk,dens,seed", [(48, 16, 8, 0.4, 0), (45, 12, 8, 0.5, 1),
                                                (64, 8, 16, 0.3, 2), (17, 8, 4, 0.6, 3)])
def test_calibrate_and_sparse_match_brute_force(L, d, blk, dens, seed):
    H = 2
    q, k, v = (_rand((1, H, L, d), 100 * seed + s) for s in range(3))
    q2, k2, v2 = (x + 0.05 * _rand(x.shape, 100 * seed + 10 + i) for i, x in enumerate((q, k, v)))
    nb = -(-L // blk)
    mask = (np.random.default_rng(seed).random((H, nb, nb)) < dens).astype(np.uint8)
    mask[1, 0] = 0                        # one empty row
    scale = 0.3 if seed == 3 else None
    o, rho, r = ref.calibrate_ref(q, k, v, mask, blk, scale=scale)
    out = ref.sparse_step_ref(q2, k2, v2, mask, blk, rho, r, 0.04, 2, ref.RAMP_MUL_LINEAR, scale=scale)
    c = scale if scale else 1.0 / math.sqrt(d)
    for h in range(H):
        keep = ref.token_keep_mask(mask[h], blk, L)
        bo, brho, br = brute.calibrate(q[0, h], k[0, h], v[0, h], keep, c)
        np.testing.assert_allclose(o[0, h], bo, atol=1e-12)
        np.testing.assert_allclose(rho[0, h], brho, atol=1e-13)
        np.testing.assert_allclose(r[0, h], br, atol=1e-12)
        rho_hat = ref.ramp_ref(brho, 0.04, 2)
        bout = brute.sparse_step(q2[0, h], k2[0, h], v2[0, h], keep, c, rho_hat, br)
        np.testing.assert_allclose(out[0, h], bout, atol=1e-12)


def test_row_sampled_variants_match_full():
    B, H, L, d, blk = 1, 2, 100, 16, 16
    q, k, v = (_rand((B, H, L, d), s) for s in (30, 31, 32))
    mask = (np.random.default_rng(33).random((1, 7, 7)) < 0.4).astype(np.uint8)
    o, rho, r = ref.calibrate_ref(q, k, v, mask, blk)
    out = ref.sparse_step_ref(q, k, v, mask, blk, rho, r, 0.04, 3)
    rows = np.array([0, 5, 17, 63, 99])
    so, srho, sr = ref.calibrate_rows_ref(q[0, 1], k[0, 1], v[0, 1], mask[0], blk, rows)
    np.testing.assert_allclose(so, o[0, 1, rows], atol=1e-14)
    np.testing.assert_allclose(srho, rho[0, 1, rows], atol=1e-15)
    np.testing.assert_allclose(sr, r[0, 1, rows], atol=1e-14)
    sout = ref.sparse_step_rows_ref(q[0, 1], k[0, 1], v[0, 1], mask[0], blk, rows, rho[0, 1, rows],
                                    r[0, 1, rows], 0.04, 3)
    np.testing.assert_allclose(sout, out[0, 1, rows], atol=1e-14)


# ---------------------------------------------------------------------------
# CSR block index
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("Hm,nqb,nkb,dens,seed", [(1, 4, 4, 0.25, 0), (3, 17, 33, 0.2, 1),
                                                   (1, 139, 139, 0.03, 2), (2, 5, 7, 0.0, 3),
                                                   (2, 6, 5, 1.0, 4)])
def test_block_index_matches_loops(Hm, nqb, nkb, dens, seed):
    mask = (np.random.default_rng(seed).random((Hm, nqb, nkb)) < dens).astype(np.uint8)
    row_ptr, col_idx = ref.build_block_index_ref(mask)
    exp_ptr, exp_col = [0], []
    for h in range(Hm):
        for qb in range(nqb):
            for kb in range(nkb):
                if mask[h, qb, kb]:
                    exp_col.append(kb)
            exp_ptr.append(len(exp_col))
    assert row_ptr.dtype == np.int32 and col_idx.dtype == np.int32
    np.testing.assert_array_equal(row_ptr, exp_ptr)
    np.testing.assert_array_equal(col_idx, np.asarray(exp_col, dtype=np.int32))


# ---------------------------------------------------------------------------
# planted mistakes: each must be caught by one of the pins above
# ---------------------------------------------------------------------------

def _mutant_residual_over_kept(q_rows, k, v, keep, c):
    s = c * (q_rows @ k.T)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    e_in = np.where(keep, e, 0.0)
    z = e.sum(axis=1)
    return (e @ v) / z[:, None], e_in.sum(1) / z, (e_in @ v) / z[:, None]   # wrong set for R


def _mutant_wrong_sign(q_rows, k, v, keep, c):
    s = c * (q_rows @ k.T)
    e = np.exp(s.max(axis=1, keepdims=True) - s)                              # sign flipped
    e_in = np.where(keep, e, 0.0)
    z = e.sum(axis=1)
    return (e @ v) / z[:, None], e_in.sum(1) / z, ((e - e_in) @ v) / z[:, None]


def _mutant_no_max_over_all_keys(q_rows, k, v, keep, c):
    s = c * (q_rows @ k.T)
    e = np.exp(s - np.where(keep, s, -np.inf).max(axis=1, keepdims=True, initial=-np.inf))
    e_in = np.where(keep, e, 0.0)
    z = e_in.sum(axis=1)                                                       # dropped masked term
    return (e @ v) / z[:, None], e_in.sum(1) / z, ((e - e_in) @ v) / z[:, None]


@pytest.mark.parametrize("mutant", [_mutant_residual_over_kept, _mutant_wrong_sign,
                                    _mutant_no_max_over_all_keys])
def test_pins_catch_planted_mistakes(monkeypatch, mutant):
    monkeypatch.setattr(ref, "_calibrate_rows", mutant)
    caught = 0
    for pin in (test_worked_example_rettention, test_rho_and_residual_match_library_softmax,
                lambda: test_calibrate_and_sparse_match_brute_force(48, 16, 8, 0.4, 0)):
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1


def test_oracle_exports():
    for name in ("full_attention_ref", "calibrate_ref", "sparse_step_ref", "ramp_ref",
                 "build_block_index_ref", "ditfastattn_residual_ref"):
        assert callable(getattr(oracle, name))


# ---------------------------------------------------------------------------
# token reordering (Hilbert order of the latent grid)
# ---------------------------------------------------------------------------

def _grid_points(perm, n_text, F, Y, X):
    r = np.asarray(perm[n_text:]) - n_text
    return np.stack([r // (Y * X), (r // X) % Y, r % X], axis=1)


@pytest.mark.parametrize("shape", [(1, 2, 2), (1, 4, 4), (1, 8, 8), (1, 16, 16), (2, 2, 2), (4, 4, 4), (8, 8, 8)])
def test_hilbert_order_is_a_unit_step_curve_on_full_cubes(shape):
    """On a full 2^b cube the order is a Hamiltonian path of unit steps that
    starts at the origin: the defining property of a Hilbert curve."""
    perm = ref.hilbert_order_ref(0, *shape)
    assert sorted(perm.tolist()) == list(range(int(np.prod(shape))))
    pts = _grid_points(perm, 0, *shape)
    assert (pts[0] == 0).all()
    steps = np.abs(np.diff(pts, axis=0)).sum(axis=1)
    assert (steps == 1).all()


@pytest.mark.parametrize("shape,sub", [((8, 8, 8), 4), ((1, 16, 16), 4), ((16, 16, 16), 8)])
def test_hilbert_order_visits_aligned_subcubes_contiguously(shape, sub):
    """Consecutive runs of sub^n points are aligned sub-cubes: a block of the
    reordered tokens is a compact brick, which is what the reordering is for."""
    perm = ref.hilbert_order_ref(0, *shape)
    pts = _grid_points(perm, 0, *shape)
    n = sum(1 for e in shape if e > 1)
    run = sub ** n
    for s0 in range(0, len(pts), run):
        chunk = pts[s0:s0 + run]
        ext = chunk.max(axis=0) - chunk.min(axis=0) + 1
        assert all(e == (sub if full > 1 else 1) for e, full in zip(ext, shape))
        assert (chunk.min(axis=0) % sub == 0).all()


def test_hilbert_order_keeps_text_first_and_restricts_the_cube():
    perm = ref.hilbert_order_ref(5, 3, 6, 5)
    assert perm[:5].tolist() == list(range(5))
    assert sorted(perm.tolist()) == list(range(5 + 90))
    # the order of a grid is the enclosing cube's order with the outside points dropped
    cube = ref.hilbert_order_ref(0, 8, 8, 8)
    cube_pts = _grid_points(cube, 0, 8, 8, 8)
    inside = cube_pts[(cube_pts[:, 0] < 3) & (cube_pts[:, 1] < 6) & (cube_pts[:, 2] < 5)]
    np.testing.assert_array_equal(_grid_points(perm, 5, 3, 6, 5), inside)


def test_permute_tokens_ref_gathers_and_scatters():
    x = np.arange(2 * 3 * 5 * 2).reshape(2, 3, 5, 2).astype(np.float64)
    perm = np.array([3, 0, 4, 1, 2])
    y = ref.permute_tokens_ref(x, perm)
    for i in range(5):
        np.testing.assert_array_equal(y[:, :, i], x[:, :, perm[i]])
    np.testing.assert_array_equal(ref.permute_tokens_ref(y, perm, inverse=True), x)
