"""ctypes binding of the C ABI in ``include/rt.h`` (``librt_b200.so``).

Argument marshalling only: the functions here carry the C entry points'
names, check that tensors are CUDA tensors of the right dtype and layout,
allocate outputs with torch when the caller gives none, and pass raw device
pointers and the current CUDA stream.  Every step of the computation runs in
the library's kernels.  There is no CPU fallback: without the built library
or a CUDA device these functions raise.
"""

from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librt_b200.so")

RT_OK = 0
RT_ERR_INVALID_ARGUMENT = 1
RT_ERR_UNSUPPORTED = 2
RT_ERR_CAPACITY = 3
RT_ERR_CUDA = 4
RT_ERR_TIMEOUT = 5
RT_ERR_BAD_INDEX = 6

RT_RAMP_MUL_LINEAR = 0
RT_RAMP_ADD_LINEAR = 1
RT_RAMP_GEOMETRIC = 2

RT_BF16 = 0
RT_F32 = 1

RT_RES_MASKED = 0          # Re-ttention's residual (masked tokens' part of O)
RT_RES_SUBTRACTIVE = 1     # DiTFastAttn's residual O - O_sparse

RT_EPI_RESHAPED = 0        # O' = ramp(rho) * attn + R
RT_EPI_NO_RHO = 1          # O' = attn + R
RT_EPI_NO_R = 2            # O' = ramp(rho) * attn

EXPORTED = (
    "rt_build_block_index", "rt_calibrate", "rt_sparse_step", "rt_calibrate_ex", "rt_sparse_step_ex",
    "rt_check_device_error", "rt_status_string", "rt_last_cuda_error", "rt_set_wait_limit_ns",
    "rt_debug_wait_timeout", "rt_build_arch", "rt_schedule_step", "rt_schedule_capture",
    "rt_cycle_graph_launch", "rt_cycle_graph_destroy", "rt_hilbert_token_order", "rt_permute_tokens",
)


class RtAttnDesc(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("L", ctypes.c_int32), ("d", ctypes.c_int32),
        ("block", ctypes.c_int32),
        ("stride_b", ctypes.c_int64), ("stride_h", ctypes.c_int64), ("stride_l", ctypes.c_int64),
        ("softmax_scale", ctypes.c_float), ("r_dtype", ctypes.c_int),
    ]


class RtBlockIndex(ctypes.Structure):
    _fields_ = [
        ("Hm", ctypes.c_int32), ("nqb", ctypes.c_int32), ("nkb", ctypes.c_int32),
        ("nnz", ctypes.c_int64),
        ("row_ptr", ctypes.c_void_p), ("col_idx", ctypes.c_void_p),
    ]


class RtSchedule(ctypes.Structure):
    _fields_ = [("period", ctypes.c_int32), ("lambda_", ctypes.c_float), ("ramp", ctypes.c_int),
                ("epilogue", ctypes.c_int), ("residual", ctypes.c_int)]


class RtError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        lib = _lib
        name = lib.rt_status_string(status).decode() if lib else str(status)
        extra = lib.rt_last_cuda_error().decode() if (lib and status == RT_ERR_CUDA) else ""
        super().__init__(f"{where}: {name}" + (f" ({extra})" if extra else ""))


_lib = None


def load_library() -> ctypes.CDLL:
    """Load librt_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m sparse_attention_diffusion_rt_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    lib.rt_build_block_index.argtypes = [vp, i32, i32, i32, vp, vp, i64, ctypes.POINTER(i64), vp]
    lib.rt_calibrate.argtypes = [ctypes.POINTER(RtAttnDesc), vp, vp, vp, ctypes.POINTER(RtBlockIndex),
                                 vp, vp, vp, vp]
    lib.rt_sparse_step.argtypes = [ctypes.POINTER(RtAttnDesc), vp, vp, vp, ctypes.POINTER(RtBlockIndex),
                                   vp, vp, ctypes.c_float, i32, ctypes.c_int, vp, vp]
    lib.rt_calibrate_ex.argtypes = [ctypes.POINTER(RtAttnDesc), vp, vp, vp, ctypes.POINTER(RtBlockIndex),
                                    vp, vp, vp, ctypes.c_int, vp]
    lib.rt_sparse_step_ex.argtypes = [ctypes.POINTER(RtAttnDesc), vp, vp, vp, ctypes.POINTER(RtBlockIndex),
                                      vp, vp, ctypes.c_float, i32, ctypes.c_int, ctypes.c_int, vp, vp]
    lib.rt_schedule_step.argtypes = [ctypes.POINTER(RtAttnDesc), ctypes.POINTER(RtSchedule), i32, vp, vp, vp,
                                     ctypes.POINTER(RtBlockIndex), vp, vp, vp, vp]
    vpp = ctypes.POINTER(vp)
    lib.rt_schedule_capture.argtypes = [ctypes.POINTER(RtAttnDesc), ctypes.POINTER(RtSchedule), vpp, vpp, vpp,
                                        ctypes.POINTER(RtBlockIndex), vpp, vp, vp, vp, ctypes.POINTER(vp)]
    lib.rt_cycle_graph_launch.argtypes = [vp, vp]
    lib.rt_hilbert_token_order.argtypes = [i32, i32, i32, i32, vp]
    lib.rt_permute_tokens.argtypes = [ctypes.POINTER(RtAttnDesc), vp, vp, vp, i32, vp]
    lib.rt_cycle_graph_destroy.argtypes = [vp]
    lib.rt_check_device_error.argtypes = [vp]
    lib.rt_status_string.argtypes = [ctypes.c_int]
    lib.rt_status_string.restype = ctypes.c_char_p
    lib.rt_last_cuda_error.argtypes = []
    lib.rt_last_cuda_error.restype = ctypes.c_char_p
    lib.rt_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.rt_debug_wait_timeout.argtypes = [ctypes.c_uint64, vp]
    lib.rt_build_arch.argtypes = []
    for name in ("rt_build_block_index", "rt_calibrate", "rt_sparse_step", "rt_calibrate_ex", "rt_sparse_step_ex",
                 "rt_schedule_step", "rt_schedule_capture", "rt_cycle_graph_launch", "rt_cycle_graph_destroy",
                 "rt_hilbert_token_order", "rt_permute_tokens",
                 "rt_check_device_error",
                 "rt_set_wait_limit_ns", "rt_debug_wait_timeout", "rt_build_arch"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _require_cuda(*tensors):
    if not torch.cuda.is_available():
        raise RuntimeError("librt_b200 needs a CUDA device; there is no CPU fallback")
    for t in tensors:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")


def _stream_ptr(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, where: str):
    if status != RT_OK:
        raise RtError(status, where)


@dataclasses.dataclass
class BlockIndex:
    """CSR block index on the device (see rt_block_index in include/rt.h)."""
    row_ptr: torch.Tensor      # int32 [Hm*nqb + 1]
    col_idx: torch.Tensor      # int32 [nnz]
    Hm: int
    nqb: int
    nkb: int
    nnz: int

    def as_c(self) -> RtBlockIndex:
        return RtBlockIndex(self.Hm, self.nqb, self.nkb, self.nnz, self.row_ptr.data_ptr(),
                            self.col_idx.data_ptr() if self.nnz > 0 else None)


def rt_build_block_index(mask: torch.Tensor, stream=None) -> BlockIndex:
    """Dense uint8 block mask [Hm, nqb, nkb] (CUDA) -> CSR BlockIndex."""
    lib = load_library()
    _require_cuda(mask)
    if mask.dtype != torch.uint8 or mask.dim() != 3 or not mask.is_contiguous():
        raise ValueError("mask must be a contiguous uint8 [Hm, nqb, nkb] tensor")
    Hm, nqb, nkb = mask.shape
    row_ptr = torch.empty(Hm * nqb + 1, dtype=torch.int32, device=mask.device)
    cap = Hm * nqb * nkb
    col = torch.empty(max(cap, 1), dtype=torch.int32, device=mask.device)
    nnz = ctypes.c_int64(0)
    _check(lib.rt_build_block_index(mask.data_ptr(), Hm, nqb, nkb, row_ptr.data_ptr(), col.data_ptr(),
                                    cap, ctypes.byref(nnz), _stream_ptr(stream)),
           "rt_build_block_index")
    return BlockIndex(row_ptr, col[: nnz.value], Hm, nqb, nkb, nnz.value)


def make_block_index(row_ptr: torch.Tensor, col_idx: torch.Tensor, Hm: int, nqb: int, nkb: int) -> BlockIndex:
    """Wrap caller-made CSR arrays (CUDA int32) without validating them here;
    the kernels validate every row they use and record RT_ERR_BAD_INDEX."""
    return BlockIndex(row_ptr, col_idx, Hm, nqb, nkb, int(col_idx.numel()))


def _desc(q: torch.Tensor, block: int, softmax_scale: float, r_dtype: torch.dtype) -> RtAttnDesc:
    if q.dim() != 4 or q.stride(3) != 1:
        raise ValueError("q/k/v/o/r must be [B, H, L, d] with d contiguous")
    if r_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("r must be bf16 or fp32")
    B, H, L, d = q.shape
    sb, sh, sl, _ = q.stride()
    rd = RT_F32 if r_dtype == torch.float32 else RT_BF16
    return RtAttnDesc(B, H, L, d, block, sb, sh, sl, float(softmax_scale), rd)


def _same_layout(ref: torch.Tensor, *ts):
    for t in ts:
        if t.shape != ref.shape or t.stride() != ref.stride():
            raise ValueError("q, k, v, o and r must share shape and strides")


def _check_attn_tensors(q, k, v, o=None, rho=None, r=None, *, need_rho=True, need_r=True):
    """The checks every attention entry point makes before anything launches:
    q, k, v (and o) bf16 [B, H, L, d] with d contiguous and one shared layout,
    r bf16 or fp32 in that layout, rho a contiguous fp32 [B, H, L] tensor.
    The C side cannot see dtypes or allocation sizes (it writes B*H*L floats
    of rho), so these are refused here with ValueError."""
    for t in (q, k, v):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16:
            raise ValueError("q, k, v must be bfloat16 tensors")
    if q.dim() != 4 or q.stride(3) != 1:
        raise ValueError("q/k/v/o/r must be [B, H, L, d] with d contiguous")
    if o is not None and o.dtype != torch.bfloat16:
        raise ValueError("o must be bfloat16")
    if need_rho and rho is None:
        raise ValueError("rho is required")
    if need_r and r is None:
        raise ValueError("r is required")
    if r is not None and r.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("r must be bf16 or fp32")
    if rho is not None:
        B, H, L, _ = q.shape
        if rho.dtype != torch.float32 or tuple(rho.shape) != (B, H, L) or not rho.is_contiguous():
            raise ValueError("rho must be a contiguous fp32 [B, H, L] tensor")
    _same_layout(q, k, v, *(t for t in (o, r) if t is not None))


def rt_calibrate(q, k, v, index: BlockIndex, *, block: int, o=None, rho=None, r=None,
                 r_dtype=torch.bfloat16, softmax_scale: float = 0.0, residual: int = RT_RES_MASKED,
                 stream=None):
    """Calibration step: returns (O bf16, rho fp32 [B,H,L], R r_dtype).
    residual selects Re-ttention's R (default) or DiTFastAttn's O - O_sparse."""
    lib = load_library()
    _check_attn_tensors(q, k, v, o, rho, r, need_rho=False, need_r=False)
    if r is not None and r.dtype != r_dtype:
        raise ValueError("r must have dtype r_dtype")
    _require_cuda(q, k, v, o, rho, r)
    B, H, L, d = q.shape
    o = torch.empty_strided(q.shape, q.stride(), dtype=q.dtype, device=q.device) if o is None else o
    r = torch.empty_strided(q.shape, q.stride(), dtype=r_dtype, device=q.device) if r is None else r
    rho = torch.empty((B, H, L), dtype=torch.float32, device=q.device) if rho is None else rho
    desc = _desc(q, block, softmax_scale, r_dtype)
    idx = index.as_c()
    _check(lib.rt_calibrate_ex(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(idx),
                               o.data_ptr(), rho.data_ptr(), r.data_ptr(), int(residual), _stream_ptr(stream)),
           "rt_calibrate")
    return o, rho, r


def rt_sparse_step(q, k, v, index: BlockIndex, rho, r, *, block: int, lam: float = 0.04,
                   step_distance: int = 1, ramp: int = RT_RAMP_MUL_LINEAR, o=None,
                   softmax_scale: float = 0.0, epilogue: int = RT_EPI_RESHAPED, stream=None):
    """Reshaped sparse step: returns O' (bf16).  epilogue selects the
    Re-ttention epilogue (default) or an ablation; rho may be None with
    RT_EPI_NO_RHO and r may be None with RT_EPI_NO_R."""
    lib = load_library()
    _check_attn_tensors(q, k, v, o, rho, r, need_rho=epilogue != RT_EPI_NO_RHO, need_r=epilogue != RT_EPI_NO_R)
    _require_cuda(q, k, v, rho, r, o)
    o = torch.empty_strided(q.shape, q.stride(), dtype=q.dtype, device=q.device) if o is None else o
    desc = _desc(q, block, softmax_scale, torch.bfloat16 if r is None else r.dtype)
    idx = index.as_c()
    _check(lib.rt_sparse_step_ex(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(idx),
                                 None if rho is None else rho.data_ptr(), None if r is None else r.data_ptr(),
                                 float(lam), int(step_distance), int(ramp), int(epilogue),
                                 o.data_ptr(), _stream_ptr(stream)),
           "rt_sparse_step")
    return o


def rt_check_device_error(stream=None) -> int:
    """Synchronise, return and clear the first device-side status (0 = none)."""
    lib = load_library()
    _require_cuda()
    return lib.rt_check_device_error(_stream_ptr(stream))


def rt_set_wait_limit_ns(limit_ns: int) -> None:
    _check(load_library().rt_set_wait_limit_ns(int(limit_ns)), "rt_set_wait_limit_ns")


def rt_debug_wait_timeout(limit_ns: int, stream=None) -> None:
    lib = load_library()
    _require_cuda()
    _check(lib.rt_debug_wait_timeout(int(limit_ns), _stream_ptr(stream)), "rt_debug_wait_timeout")


def rt_status_string(status: int) -> str:
    return load_library().rt_status_string(int(status)).decode()


def rt_build_arch() -> int:
    return load_library().rt_build_arch()


def _schedule(period, lam, ramp, epilogue, residual) -> RtSchedule:
    return RtSchedule(int(period), float(lam), int(ramp), int(epilogue), int(residual))


def rt_schedule_step(q, k, v, index: BlockIndex, t: int, *, block: int, period: int, o, rho, r,
                     lam: float = 0.04, ramp: int = RT_RAMP_MUL_LINEAR, epilogue: int = RT_EPI_RESHAPED,
                     residual: int = RT_RES_MASKED, softmax_scale: float = 0.0, stream=None):
    """Step t of a denoising schedule: a calibration into (o, rho, r) when
    t % period == 0, else a sparse step reading (rho, r) into o."""
    lib = load_library()
    _check_attn_tensors(q, k, v, o, rho, r)
    _require_cuda(q, k, v, o, rho, r)
    desc = _desc(q, block, softmax_scale, r.dtype)
    sched = _schedule(period, lam, ramp, epilogue, residual)
    idx = index.as_c()
    _check(lib.rt_schedule_step(ctypes.byref(desc), ctypes.byref(sched), int(t), q.data_ptr(), k.data_ptr(),
                                v.data_ptr(), ctypes.byref(idx), o.data_ptr(), rho.data_ptr(), r.data_ptr(),
                                _stream_ptr(stream)),
           "rt_schedule_step")
    return o


class CycleGraph:
    """One calibration cycle (steps 0 .. period-1) captured as a CUDA graph.
    steps[t] = (q, k, v) and outs[t] = o of step t; rho and r are the cache.
    The buffers must stay alive (and at the same addresses) while the graph
    is used.  Capture needs a created stream (not the default stream)."""

    def __init__(self, steps, index: BlockIndex, *, block: int, outs, rho, r, lam: float = 0.04,
                 ramp: int = RT_RAMP_MUL_LINEAR, epilogue: int = RT_EPI_RESHAPED, residual: int = RT_RES_MASKED,
                 softmax_scale: float = 0.0, stream: torch.cuda.Stream):
        lib = load_library()
        period = len(steps)
        if period < 1 or len(outs) != period:
            raise ValueError("one (q, k, v) and one output per step of the cycle")
        for (q, k, v), o in zip(steps, outs):
            _check_attn_tensors(q, k, v, o, rho, r)
            _same_layout(steps[0][0], q)
        for (q, k, v), o in zip(steps, outs):
            _require_cuda(q, k, v, o)
        _require_cuda(rho, r)
        if stream is None or stream.cuda_stream == 0:
            raise ValueError("capture needs a created stream")
        desc = _desc(steps[0][0], block, softmax_scale, r.dtype)
        sched = _schedule(period, lam, ramp, epilogue, residual)
        arr = lambda xs: (ctypes.c_void_p * period)(*[x.data_ptr() for x in xs])
        self._keep = (steps, outs, rho, r, index)       # keep the captured buffers alive
        idx = index.as_c()
        h = ctypes.c_void_p()
        _check(lib.rt_schedule_capture(ctypes.byref(desc), ctypes.byref(sched), arr([s[0] for s in steps]),
                                       arr([s[1] for s in steps]), arr([s[2] for s in steps]), ctypes.byref(idx),
                                       arr(outs), rho.data_ptr(), r.data_ptr(), ctypes.c_void_p(stream.cuda_stream),
                                       ctypes.byref(h)),
               "rt_schedule_capture")
        self._h = h
        self.period = period

    def launch(self, stream=None):
        _check(load_library().rt_cycle_graph_launch(self._h, _stream_ptr(stream)), "rt_cycle_graph_launch")

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            _check(load_library().rt_cycle_graph_destroy(self._h), "rt_cycle_graph_destroy")
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def rt_hilbert_token_order(n_text: int, F: int, Y: int, X: int) -> torch.Tensor:
    """Host int32 [n_text + F*Y*X]: perm[i] = raster index of the token at
    position i of the Hilbert order (text tokens first)."""
    lib = load_library()
    perm = torch.empty(n_text + F * Y * X, dtype=torch.int32)
    _check(lib.rt_hilbert_token_order(int(n_text), int(F), int(Y), int(X), perm.data_ptr()),
           "rt_hilbert_token_order")
    return perm


def rt_permute_tokens(src, perm, *, inverse: bool = False, dst=None, stream=None):
    """dst[:, :, i] = src[:, :, perm[i]] (inverse=False) or
    dst[:, :, perm[i]] = src[:, :, i] (inverse=True); src bf16 [B, H, L, d]."""
    lib = load_library()
    _require_cuda(src, perm, dst)
    if src.dtype != torch.bfloat16 or src.dim() != 4:
        raise ValueError("src must be a bf16 [B, H, L, d] tensor")
    if perm.dtype != torch.int32 or perm.dim() != 1 or perm.numel() != src.shape[2] or not perm.is_contiguous():
        raise ValueError("perm must be a contiguous int32 [L] tensor")
    dst = torch.empty_like(src) if dst is None else dst
    _same_layout(src, dst)
    desc = _desc(src, 128, 0.0, torch.bfloat16)
    _check(lib.rt_permute_tokens(ctypes.byref(desc), src.data_ptr(), dst.data_ptr(), perm.data_ptr(),
                                 1 if inverse else 0, _stream_ptr(stream)),
           "rt_permute_tokens")
    return dst
