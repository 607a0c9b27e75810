"""CPU checks of the C-ABI library (no GPU, no compute calls): it loads, it
exports every entry point include/rt.h declares, the ctypes structures match
the C layout, and host-side validation rejects bad arguments before any CUDA
call is made."""

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from sparse_attention_diffusion_rt_b200 import build as rtbuild
from sparse_attention_diffusion_rt_b200 import rt

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rt.h")


@pytest.fixture(scope="module")
def lib():
    rtbuild.build()
    return rt.load_library()


def _declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"RT_API\s+[\w\s\*]+?\b(rt_\w+)\s*\(", txt)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("rt_build_block_index", "rt_calibrate", "rt_sparse_step", "rt_check_device_error",
              "rt_status_string"):
        assert n in names
    assert sorted(rt.EXPORTED) == names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", rt.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s(\w+)$", out, re.M))
    for n in _declared():
        assert n in exported, n
        assert hasattr(lib, n)
    assert {s for s in exported if s.startswith("rt_")} == set(_declared())


def test_status_strings_and_arch(lib):
    assert rt.rt_status_string(0) == "RT_OK"
    assert rt.rt_status_string(6) == "RT_ERR_BAD_INDEX"
    assert rt.rt_status_string(99) == "RT_ERR_UNKNOWN"
    assert rt.rt_build_arch() == 1000


def test_struct_layout_matches_c(tmp_path):
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "rt.h"\n'
        "int main(void){printf(\"%zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\\n\", sizeof(rt_attn_desc),"
        " offsetof(rt_attn_desc, stride_b), offsetof(rt_attn_desc, softmax_scale), offsetof(rt_attn_desc, r_dtype),"
        " sizeof(rt_block_index), offsetof(rt_block_index, nnz), offsetof(rt_block_index, col_idx),"
        " sizeof(rt_schedule), offsetof(rt_schedule, lambda), offsetof(rt_schedule, epilogue),"
        " offsetof(rt_schedule, residual));return 0;}\n")
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)])
    got = list(map(int, subprocess.check_output([str(exe)]).split()))
    want = [ctypes.sizeof(rt.RtAttnDesc), rt.RtAttnDesc.stride_b.offset, rt.RtAttnDesc.softmax_scale.offset,
            rt.RtAttnDesc.r_dtype.offset, ctypes.sizeof(rt.RtBlockIndex), rt.RtBlockIndex.nnz.offset,
            rt.RtBlockIndex.col_idx.offset, ctypes.sizeof(rt.RtSchedule), rt.RtSchedule.lambda_.offset,
            rt.RtSchedule.epilogue.offset, rt.RtSchedule.residual.offset]
    assert got == want


def test_host_validation_without_gpu(lib):
    """Argument errors are returned before any CUDA call (safe without a device)."""
    vp = ctypes.c_void_p
    assert lib.rt_calibrate(None, vp(16), vp(16), vp(16), None, vp(16), vp(16), vp(16), None) == rt.RT_ERR_INVALID_ARGUMENT
    desc = rt.RtAttnDesc(1, 1, 128, 64, 128, 8192, 8192, 64, 0.0, 0)
    idx = rt.RtBlockIndex(1, 1, 1, 1, 4096, 4096)
    # q, k, v, idx, o, rho, r at disjoint (never dereferenced) addresses
    args = (vp(1 << 20), vp(2 << 20), vp(3 << 20), ctypes.byref(idx), vp(4 << 20), vp(5 << 20), vp(6 << 20), None)
    bad = rt.RtAttnDesc(1, 1, 128, 20, 128, 8192, 8192, 64, 0.0, 0)          # d % 8 != 0
    assert lib.rt_calibrate(ctypes.byref(bad), *args) == rt.RT_ERR_UNSUPPORTED
    bad = rt.RtAttnDesc(1, 1, 128, 64, 32, 8192, 8192, 64, 0.0, 0)           # block 32
    assert lib.rt_calibrate(ctypes.byref(bad), *args) == rt.RT_ERR_UNSUPPORTED
    bad = rt.RtAttnDesc(1, 1, 128, 64, 128, 8192, 8192, 64, -1.0, 0)         # negative scale
    assert lib.rt_calibrate(ctypes.byref(bad), *args) == rt.RT_ERR_INVALID_ARGUMENT
    mis = (vp(4096 + 8),) + args[1:]                                          # misaligned q
    assert lib.rt_calibrate(ctypes.byref(desc), *mis) == rt.RT_ERR_INVALID_ARGUMENT
    idx2 = rt.RtBlockIndex(1, 2, 2, 1, 4096, 4096)                           # nqb != ceil(L/block)
    assert lib.rt_calibrate(ctypes.byref(desc), vp(4096), vp(4096), vp(4096), ctypes.byref(idx2), vp(4096),
                            vp(4096), vp(4096), None) == rt.RT_ERR_INVALID_ARGUMENT
    assert lib.rt_sparse_step(ctypes.byref(desc), *args[:4], vp(4096), vp(4096), ctypes.c_float(0.04), 1, 7,
                              vp(4096), None) == rt.RT_ERR_INVALID_ARGUMENT     # unknown ramp
    assert lib.rt_sparse_step(ctypes.byref(desc), *args[:4], vp(4096), vp(4096), ctypes.c_float(0.04), -1, 0,
                              vp(4096), None) == rt.RT_ERR_INVALID_ARGUMENT     # negative step distance
    # extended entry points: the residual kind and the epilogue are checked, and
    # rho / r may be NULL only for the epilogue that does not read them
    c_lam = ctypes.c_float(0.04)
    assert lib.rt_calibrate_ex(ctypes.byref(desc), *args[:7], 5, None) == rt.RT_ERR_INVALID_ARGUMENT
    sp = (ctypes.byref(desc), *args[:4])
    assert lib.rt_sparse_step_ex(*sp, vp(4096), vp(4096), c_lam, 1, 0, 9, vp(4096), None) == \
        rt.RT_ERR_INVALID_ARGUMENT                                           # unknown epilogue
    for epi in (rt.RT_EPI_RESHAPED, rt.RT_EPI_NO_R):                         # these read rho
        assert lib.rt_sparse_step_ex(*sp, None, vp(4096), c_lam, 1, 0, epi, vp(4096), None) == \
            rt.RT_ERR_INVALID_ARGUMENT
    for epi in (rt.RT_EPI_RESHAPED, rt.RT_EPI_NO_RHO):                       # these read r
        assert lib.rt_sparse_step_ex(*sp, vp(4096), None, c_lam, 1, 0, epi, vp(4096), None) == \
            rt.RT_ERR_INVALID_ARGUMENT
    bad = rt.RtAttnDesc(1, 1, 128, 20, 128, 8192, 8192, 64, 0.0, 0)
    assert lib.rt_sparse_step_ex(ctypes.byref(bad), *args[:4], None, vp(4096), c_lam, 1, 0, rt.RT_EPI_NO_RHO,
                                 vp(4096), None) == rt.RT_ERR_UNSUPPORTED   # NULL rho accepted, shape checked
    # schedule driver: the schedule and t are checked before any CUDA call
    sched = rt.RtSchedule(5, 0.04, 0, 0, 0)
    cal_args = (vp(4096), vp(4096), vp(4096), ctypes.byref(idx), vp(4096), vp(4096), vp(4096), None)
    assert lib.rt_schedule_step(ctypes.byref(desc), None, 0, *cal_args) == rt.RT_ERR_INVALID_ARGUMENT
    assert lib.rt_schedule_step(ctypes.byref(desc), ctypes.byref(sched), -1, *cal_args) == rt.RT_ERR_INVALID_ARGUMENT
    zero = rt.RtSchedule(0, 0.04, 0, 0, 0)
    assert lib.rt_schedule_step(ctypes.byref(desc), ctypes.byref(zero), 3, *cal_args) == rt.RT_ERR_INVALID_ARGUMENT
    bad = rt.RtAttnDesc(1, 1, 128, 20, 128, 8192, 8192, 64, 0.0, 0)
    assert lib.rt_schedule_step(ctypes.byref(bad), ctypes.byref(sched), 0, *cal_args) == rt.RT_ERR_UNSUPPORTED
    assert lib.rt_schedule_step(ctypes.byref(bad), ctypes.byref(sched), 2, *cal_args) == rt.RT_ERR_UNSUPPORTED
    h = ctypes.c_void_p(1)
    assert lib.rt_schedule_capture(ctypes.byref(desc), ctypes.byref(sched), None, None, None, ctypes.byref(idx),
                                   None, vp(4096), vp(4096), None, ctypes.byref(h)) == rt.RT_ERR_INVALID_ARGUMENT
    assert h.value is None                                                   # the handle is cleared on error
    assert lib.rt_cycle_graph_launch(None, None) == rt.RT_ERR_INVALID_ARGUMENT
    assert lib.rt_cycle_graph_destroy(None) == rt.RT_OK
    nnz = ctypes.c_int64(0)
    assert lib.rt_build_block_index(None, 1, 1, 1, vp(16), vp(16), 1, ctypes.byref(nnz), None) == \
        rt.RT_ERR_INVALID_ARGUMENT
    assert lib.rt_build_block_index(vp(16), 1, 0, 1, vp(16), vp(16), 1, ctypes.byref(nnz), None) == \
        rt.RT_ERR_INVALID_ARGUMENT


def test_host_validation_rejects_aliasing_layouts_and_overlaps(lib):
    """Layouts whose (b, h, l) rows share elements, and outputs that overlap an
    input or another output, are refused before any CUDA call."""
    vp = ctypes.c_void_p
    idx = rt.RtBlockIndex(1, 1, 1, 1, 4096, 4096)
    q, k, v, o, rho, r = (vp(i << 20) for i in range(1, 7))
    # two heads on the same rows (stride_h < L * stride_l, and not a [B, L, H, d] interleave)
    alias = rt.RtAttnDesc(1, 2, 128, 64, 128, 16384, 64, 64, 0.0, 0)
    assert lib.rt_calibrate(ctypes.byref(alias), q, k, v, ctypes.byref(idx), o, rho, r, None) == \
        rt.RT_ERR_INVALID_ARGUMENT
    alias_b = rt.RtAttnDesc(2, 2, 128, 64, 128, 8192, 8192, 64, 0.0, 0)     # batches alias the heads
    assert lib.rt_calibrate(ctypes.byref(alias_b), q, k, v, ctypes.byref(idx), o, rho, r, None) == \
        rt.RT_ERR_INVALID_ARGUMENT
    assert lib.rt_permute_tokens(ctypes.byref(alias), q, k, vp(64), 0, None) == rt.RT_ERR_INVALID_ARGUMENT
    desc = rt.RtAttnDesc(1, 1, 128, 64, 128, 8192, 8192, 64, 0.0, 0)       # 16 KiB per tensor
    near = lambda p, off: vp(p.value + off)
    bad_calls = [
        (near(q, 4096), rho, r),        # o overlaps q
        (o, rho, near(k, 1024)),        # r overlaps k (the calibration writes r)
        (o, near(v, 16), r),            # rho overlaps v
        (o, rho, near(o, 8192)),        # r overlaps o
        (o, near(r, 64), r),            # rho overlaps r
    ]
    for oo, rr, res in bad_calls:
        assert lib.rt_calibrate(ctypes.byref(desc), q, k, v, ctypes.byref(idx), oo, rr, res, None) == \
            rt.RT_ERR_INVALID_ARGUMENT
    lam = ctypes.c_float(0.04)
    assert lib.rt_sparse_step(ctypes.byref(desc), q, k, v, ctypes.byref(idx), rho, near(o, 32), lam, 1, 0, o,
                              None) == rt.RT_ERR_INVALID_ARGUMENT                 # o overlaps r
    span = 16384
    assert lib.rt_permute_tokens(ctypes.byref(desc), q, near(q, span - 16), vp(64), 0, None) == \
        rt.RT_ERR_INVALID_ARGUMENT                                            # dst overlaps src
    # a [B, L, H, d] interleave has disjoint rows: accepted by validation (the
    # call then needs a device, so without one it fails later, not as invalid)
    blhd = rt.RtAttnDesc(1, 2, 128, 64, 128, 16384, 64, 128, 0.0, 0)
    assert lib.rt_calibrate(ctypes.byref(blhd), q, k, v, ctypes.byref(idx), o, rho, r, None) != \
        rt.RT_ERR_INVALID_ARGUMENT


def test_binding_checks_dtypes_and_layouts_before_launch(lib):
    """Every entry point of the binding refuses a wrong dtype or layout of
    rho, r or o with ValueError before anything is launched (these checks do
    not need a device)."""
    import torch
    q = torch.zeros(1, 2, 256, 64, dtype=torch.bfloat16)
    good_rho = torch.zeros(1, 2, 256, dtype=torch.float32)
    good_r = torch.zeros_like(q)
    bad = {
        "bf16 rho": dict(rho=good_rho.to(torch.bfloat16), r=good_r),
        "non-contiguous rho": dict(rho=torch.zeros(1, 2, 512, dtype=torch.float32)[:, :, ::2], r=good_r),
        "short rho": dict(rho=torch.zeros(1, 2, 255, dtype=torch.float32), r=good_r),
        "fp16 r": dict(rho=good_rho, r=good_r.to(torch.float16)),
        "r in another layout": dict(rho=good_rho, r=good_r.transpose(1, 2).contiguous().transpose(1, 2)),
    }
    idx = rt.BlockIndex(torch.zeros(3, dtype=torch.int32), torch.zeros(0, dtype=torch.int32), 1, 2, 2, 0)
    for what, kw in bad.items():
        with pytest.raises(ValueError):
            rt.rt_schedule_step(q, q, q, idx, 0, block=128, period=5, o=torch.empty_like(q), **kw)
        with pytest.raises(ValueError):
            rt.rt_schedule_step(q, q, q, idx, 2, block=128, period=5, o=torch.empty_like(q), **kw)
        with pytest.raises(ValueError):
            rt.rt_sparse_step(q, q, q, idx, kw["rho"], kw["r"], block=128)
        with pytest.raises(ValueError):
            rt.CycleGraph([(q, q, q)] * 2, idx, block=128, outs=[torch.empty_like(q)] * 2, stream=None, **kw)
        with pytest.raises(ValueError):
            rt.rt_calibrate(q, q, q, idx, block=128, rho=kw["rho"], r=kw["r"], r_dtype=kw["r"].dtype)
    with pytest.raises(ValueError):
        rt.rt_schedule_step(q, q, q, idx, 0, block=128, period=5, o=q.float(), rho=good_rho, r=good_r)
    with pytest.raises(ValueError):
        rt.rt_calibrate(q.float(), q, q, idx, block=128)


def test_binding_refuses_without_cuda(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("CUDA present")
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(RuntimeError):
        rt.rt_calibrate(q, q, q, None, block=128)


@pytest.mark.parametrize("n_text,F,Y,X", [(0, 13, 30, 45), (226, 13, 30, 45), (0, 32, 45, 80), (256, 1, 64, 64),
                                          (0, 1, 64, 64), (3, 5, 1, 7), (0, 1, 1, 1)])
def test_hilbert_token_order_matches_oracle(lib, n_text, F, Y, X):
    """The library's (host, C++) token order equals the oracle's on the
    workload grids, bit for bit."""
    from oracle import reference as ref
    got = rt.rt_hilbert_token_order(n_text, F, Y, X).numpy()
    np.testing.assert_array_equal(got, ref.hilbert_order_ref(n_text, F, Y, X))


def test_token_order_validation_without_gpu(lib):
    vp = ctypes.c_void_p
    buf = (ctypes.c_int32 * 8)()
    assert lib.rt_hilbert_token_order(0, 0, 2, 2, buf) == rt.RT_ERR_INVALID_ARGUMENT
    assert lib.rt_hilbert_token_order(-1, 1, 2, 2, buf) == rt.RT_ERR_INVALID_ARGUMENT
    assert lib.rt_hilbert_token_order(0, 1, 2, 2, None) == rt.RT_ERR_INVALID_ARGUMENT
    desc = rt.RtAttnDesc(1, 1, 128, 64, 128, 8192, 8192, 64, 0.0, 0)
    assert lib.rt_permute_tokens(ctypes.byref(desc), vp(4096), vp(8192), None, 0, None) == rt.RT_ERR_INVALID_ARGUMENT
    assert lib.rt_permute_tokens(ctypes.byref(desc), vp(4096), vp(8192), vp(4096), 2, None) == \
        rt.RT_ERR_INVALID_ARGUMENT                                            # inverse must be 0 or 1
    assert lib.rt_permute_tokens(ctypes.byref(desc), vp(4096), vp(4096), vp(64), 0, None) == \
        rt.RT_ERR_INVALID_ARGUMENT                                            # in place
    assert lib.rt_permute_tokens(ctypes.byref(desc), vp(4096 + 8), vp(8192), vp(64), 0, None) == \
        rt.RT_ERR_INVALID_ARGUMENT                                            # misaligned
    bad = rt.RtAttnDesc(1, 1, 128, 20, 128, 8192, 8192, 64, 0.0, 0)
    assert lib.rt_permute_tokens(ctypes.byref(bad), vp(4096), vp(8192), vp(64), 0, None) == \
        rt.RT_ERR_INVALID_ARGUMENT                                            # d % 8 != 0
