// C ABI of the library (declared in include/rt.h): argument validation, TMA
// descriptor encoding, kernel dispatch and the device status word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "attn_launch.h"
#include "layout.h"
#include "nvtx_range.h"
#include "rt.h"

namespace rtb {
cudaError_t launch_block_index(const uint8_t* mask, int rows, int nkb, int32_t* row_ptr,
                               int32_t* col_idx, long long capacity, cudaStream_t s);
}

using namespace rtb;

namespace rtb {
rt_status api_cuda_fail(cudaError_t e, const char* where);
rt_status api_status_word(unsigned int** out);
}

namespace {

// One status word per device (first device-side error since the last check).
__device__ unsigned int g_rt_status;

thread_local char g_last_cuda_error[256] = "";
std::atomic<unsigned long long> g_wait_limit_ns{4000000000ull};
constexpr unsigned long long kDefaultWaitLimitNs = 4000000000ull;

rt_status cuda_fail(cudaError_t e, const char* where) {
  std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s (%d)", where,
                cudaGetErrorString(e), static_cast<int>(e));
  return RT_ERR_CUDA;
}

rt_status status_word(unsigned int** out) {
  static std::mutex mu;
  static unsigned int* cache[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return RT_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_rt_status);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status)");
    cache[dev] = static_cast<unsigned int*>(p);
  }
  *out = cache[dev];
  return RT_OK;
}

}  // namespace

// Records a CUDA error for rt_last_cuda_error (used by the other translation units).
rt_status rtb::api_cuda_fail(cudaError_t e, const char* where) { return cuda_fail(e, where); }
// The device status word of the current device (for the other translation units).
rt_status rtb::api_status_word(unsigned int** out) { return status_word(out); }

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int dpad_of(int d) { return d <= 64 ? 64 : d <= 80 ? 80 : d <= 96 ? 96 : 128; }

// 4-D map over [B, H, L, d] (innermost first) with a box of (box_inner, box_rows, 1, 1).
rt_status make_map(CUtensorMap* m, const void* ptr, const rt_attn_desc& d, bool f32,
                   uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cuTensorMapEncodeTiled unavailable");
    return RT_ERR_CUDA;
  }
  const uint64_t es = f32 ? 4 : 2;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d.d), static_cast<cuuint64_t>(d.L),
                        static_cast<cuuint64_t>(d.H), static_cast<cuuint64_t>(d.B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d.stride_l) * es, static_cast<cuuint64_t>(d.stride_h) * es,
                           static_cast<cuuint64_t>(d.stride_b) * es};
  cuuint32_t box[4] = {box_inner, box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                  const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cuTensorMapEncodeTiled failed (%d)",
                  static_cast<int>(r));
    return RT_ERR_CUDA;
  }
  return RT_OK;
}

CUtensorMapSwizzle c1_swizzle(int c1) {
  return c1 == 16 ? CU_TENSOR_MAP_SWIZZLE_32B : c1 == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
}

// bf16 tile maps: chunk 0 = 64 columns (128B swizzle), chunk 1 = dpad-64 columns.
rt_status make_chunk_maps(CUtensorMap (&m)[2], const void* ptr, const rt_attn_desc& d, int dpad,
                          uint32_t rows) {
  rt_status s = make_map(&m[0], ptr, d, false, 64, rows, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != RT_OK || dpad == 64) return s;
  return make_map(&m[1], ptr, d, false, static_cast<uint32_t>(dpad - 64), rows, c1_swizzle(dpad - 64));
}

rt_status make_residual_maps(CUtensorMap (&m)[4], const void* ptr, const rt_attn_desc& d, int dpad) {
  const uint32_t rows = static_cast<uint32_t>(d.block);
  if (d.r_dtype == RT_F32) {
    for (int c = 0; c < (dpad + 31) / 32; ++c) {
      rt_status s = make_map(&m[c], ptr, d, true, 32, rows, CU_TENSOR_MAP_SWIZZLE_128B);
      if (s != RT_OK) return s;
    }
    return RT_OK;
  }
  CUtensorMap two[2];
  rt_status s = make_chunk_maps(two, ptr, d, dpad, rows);
  m[0] = two[0];
  m[1] = two[1];
  return s;
}

// need_rho / need_r: whether the call reads (or writes) rho and R.
// stats_out: the call writes rho and R (calibration) rather than reading them.
rt_status validate(const rt_attn_desc* desc, const void* q, const void* k, const void* v,
                   const rt_block_index* idx, const void* o, const void* rho, const void* r,
                   bool stats_out, bool need_rho = true, bool need_r = true) {
  if (!desc || !idx || !q || !k || !v || !o) return RT_ERR_INVALID_ARGUMENT;
  if ((need_rho && !rho) || (need_r && !r)) return RT_ERR_INVALID_ARGUMENT;
  const rt_attn_desc& d = *desc;
  if (d.B < 1 || d.H < 1 || d.L < 1 || d.d < 1) return RT_ERR_INVALID_ARGUMENT;
  if (d.stride_b < 1 || d.stride_h < 1 || d.stride_l < 1) return RT_ERR_INVALID_ARGUMENT;
  if (!(d.softmax_scale >= 0.f) || !std::isfinite(d.softmax_scale)) return RT_ERR_INVALID_ARGUMENT;
  if (d.r_dtype != RT_BF16 && d.r_dtype != RT_F32) return RT_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (need_r && !aligned16(r)) ||
      (need_rho && !aligned16(rho)))
    return RT_ERR_INVALID_ARGUMENT;
  if (d.d < 16 || d.d > 128 || d.d % 8 != 0) return RT_ERR_UNSUPPORTED;
  if (d.block != 64 && d.block != 128) return RT_ERR_UNSUPPORTED;
  if (d.block == 64 && d.d > 64) return RT_ERR_UNSUPPORTED;
  if (d.stride_l % 8 || d.stride_h % 8 || d.stride_b % 8) return RT_ERR_UNSUPPORTED;
  if (d.stride_l < d.d) return RT_ERR_INVALID_ARGUMENT;
  if (d.B > 65535 || d.H > 65535) return RT_ERR_UNSUPPORTED;
  const long long nb = (static_cast<long long>(d.L) + d.block - 1) / d.block;
  if (nb > kMaxKeyBlocks) return RT_ERR_UNSUPPORTED;
  if (idx->nqb != nb || idx->nkb != nb) return RT_ERR_INVALID_ARGUMENT;
  if (idx->Hm != 1 && idx->Hm != d.H) return RT_ERR_INVALID_ARGUMENT;
  if (idx->nnz < 0 || !idx->row_ptr || (idx->nnz > 0 && !idx->col_idx)) return RT_ERR_INVALID_ARGUMENT;
  if (idx->nnz > static_cast<long long>(idx->Hm) * nb * nb) return RT_ERR_INVALID_ARGUMENT;
  // strides below 2^40 bytes (tensor-map limit)
  const long long lim = 1ll << 38;
  if (d.stride_b >= lim || d.stride_h >= lim || d.stride_l >= lim) return RT_ERR_UNSUPPORTED;
  // distinct (b, h, l) rows must not share elements: different CTAs store them
  if (!layout_rows_disjoint(d)) return RT_ERR_INVALID_ARGUMENT;
  // what the call writes overlaps nothing else it reads or writes
  const long long span2 = layout_span_bytes(d, 2);
  const long long span_r = layout_span_bytes(d, d.r_dtype == RT_F32 ? 4 : 2);
  const long long span_rho = static_cast<long long>(d.B) * d.H * d.L * 4;
  const void* ins[3] = {q, k, v};
  for (const void* in : ins) {
    if (ranges_overlap(o, span2, in, span2)) return RT_ERR_INVALID_ARGUMENT;
    if (stats_out && (ranges_overlap(r, span_r, in, span2) || ranges_overlap(rho, span_rho, in, span2)))
      return RT_ERR_INVALID_ARGUMENT;
  }
  if (ranges_overlap(o, span2, need_r ? r : nullptr, span_r) ||
      ranges_overlap(o, span2, need_rho ? rho : nullptr, span_rho) ||
      (need_r && need_rho && ranges_overlap(r, span_r, rho, span_rho)))
    return RT_ERR_INVALID_ARGUMENT;
  return RT_OK;
}

rt_status fill_common(const rt_attn_desc& d, const rt_block_index& idx, AttnParams& p) {
  std::memset(&p, 0, sizeof(p));
  p.B = d.B; p.H = d.H; p.L = d.L; p.d = d.d; p.block = d.block;
  p.nqb = idx.nqb; p.nkb = idx.nkb; p.Hm = idx.Hm; p.nnz = idx.nnz;
  p.row_ptr = idx.row_ptr; p.col_idx = idx.col_idx;
  const double c = d.softmax_scale > 0.f ? static_cast<double>(d.softmax_scale) : 1.0 / std::sqrt(static_cast<double>(d.d));
  p.scale_log2 = static_cast<float>(c * 1.4426950408889634);   // c * log2(e)
  p.r_f32 = d.r_dtype == RT_F32;
  p.use_rho = 1;
  p.use_r = 1;
  p.r_sub = 0;
  p.wait_limit_ns = g_wait_limit_ns.load();
  return status_word(&p.status);
}

cudaError_t dispatch(int dpad, bool cal, const rt_attn_desc& d, const TmaSet& tm, const AttnParams& p,
                     cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>(p.nqb), static_cast<unsigned>(d.H), static_cast<unsigned>(d.B));
  switch (dpad) {
    case 64: return launch_attn_d64(cal, d.block, tm, p, grid, s);
    case 80: return launch_attn_d80(cal, d.block, tm, p, grid, s);
    case 96: return launch_attn_d96(cal, d.block, tm, p, grid, s);
    default: return launch_attn_d128(cal, d.block, tm, p, grid, s);
  }
}

__global__ void debug_wait_kernel(unsigned long long limit_ns, unsigned int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = globaltimer_ns();
    bool done = false;
    while (!(done = mbar_try_wait(&bar, 0))) {
      if (globaltimer_ns() - t0 > limit_ns) break;
    }
    if (!done) atomicCAS(status, 0u, static_cast<unsigned int>(RT_ERR_TIMEOUT));
    mbar_arrive(&bar);      // complete the phase so nothing is left pending
  }
}

}  // namespace

extern "C" {

const char* rt_status_string(rt_status s) {
  switch (s) {
    case RT_OK: return "RT_OK";
    case RT_ERR_INVALID_ARGUMENT: return "RT_ERR_INVALID_ARGUMENT";
    case RT_ERR_UNSUPPORTED: return "RT_ERR_UNSUPPORTED";
    case RT_ERR_CAPACITY: return "RT_ERR_CAPACITY";
    case RT_ERR_CUDA: return "RT_ERR_CUDA";
    case RT_ERR_TIMEOUT: return "RT_ERR_TIMEOUT";
    case RT_ERR_BAD_INDEX: return "RT_ERR_BAD_INDEX";
  }
  return "RT_ERR_UNKNOWN";
}

const char* rt_last_cuda_error(void) { return g_last_cuda_error; }

int32_t rt_build_arch(void) { return 1000; }

rt_status rt_set_wait_limit_ns(uint64_t limit_ns) {
  g_wait_limit_ns.store(limit_ns ? limit_ns : kDefaultWaitLimitNs);
  return RT_OK;
}

rt_status rt_build_block_index(const uint8_t* d_mask, int32_t Hm, int32_t nqb, int32_t nkb,
                               int32_t* d_row_ptr, int32_t* d_col_idx, int64_t col_capacity,
                               int64_t* h_nnz, void* stream) {
  RT_RANGE("rt_build_block_index");
  if (!d_mask || !d_row_ptr || !h_nnz || Hm < 1 || nqb < 1 || nkb < 1 || col_capacity < 0)
    return RT_ERR_INVALID_ARGUMENT;
  if (col_capacity > 0 && !d_col_idx) return RT_ERR_INVALID_ARGUMENT;
  const long long total = static_cast<long long>(Hm) * nqb * nkb;
  if (total >= (1ll << 31)) return RT_ERR_UNSUPPORTED;
  const int rows = Hm * nqb;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_block_index(d_mask, rows, nkb, d_row_ptr, d_col_idx, col_capacity, s);
  if (e != cudaSuccess) return cuda_fail(e, "block index launch");
  int32_t nnz = 0;
  e = cudaMemcpyAsync(&nnz, d_row_ptr + rows, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "nnz readback");
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "nnz sync");
  *h_nnz = nnz;
  return nnz > col_capacity ? RT_ERR_CAPACITY : RT_OK;
}

rt_status rt_calibrate(const rt_attn_desc* desc, const void* q, const void* k, const void* v,
                       const rt_block_index* idx, void* o, float* rho, void* r, void* stream) {
  return rt_calibrate_ex(desc, q, k, v, idx, o, rho, r, RT_RES_MASKED, stream);
}

rt_status rt_calibrate_ex(const rt_attn_desc* desc, const void* q, const void* k, const void* v,
                          const rt_block_index* idx, void* o, float* rho, void* r, rt_residual kind,
                          void* stream) {
  RT_RANGE("rt_calibrate_ex");
  if (kind != RT_RES_MASKED && kind != RT_RES_SUBTRACTIVE) return RT_ERR_INVALID_ARGUMENT;
  rt_status st = validate(desc, q, k, v, idx, o, rho, r, true);
  if (st != RT_OK) return st;
  const rt_attn_desc& d = *desc;
  const int dpad = dpad_of(d.d);
  AttnParams p;
  if ((st = fill_common(d, *idx, p)) != RT_OK) return st;
  p.rho_out = rho;
  p.r_sub = kind == RT_RES_SUBTRACTIVE;
  TmaSet tm;
  std::memset(&tm, 0, sizeof(tm));
  if ((st = make_chunk_maps(tm.q, q, d, dpad, 128)) != RT_OK) return st;
  if ((st = make_chunk_maps(tm.k, k, d, dpad, static_cast<uint32_t>(d.block))) != RT_OK) return st;
  if ((st = make_chunk_maps(tm.v, v, d, dpad, static_cast<uint32_t>(d.block))) != RT_OK) return st;
  if ((st = make_chunk_maps(tm.o, o, d, dpad, static_cast<uint32_t>(d.block))) != RT_OK) return st;
  if ((st = make_residual_maps(tm.r, r, d, dpad)) != RT_OK) return st;
  cudaError_t e = dispatch(dpad, true, d, tm, p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RT_OK : cuda_fail(e, "rt_calibrate launch");
}

rt_status rt_sparse_step(const rt_attn_desc* desc, const void* q, const void* k, const void* v,
                         const rt_block_index* idx, const float* rho, const void* r, float lambda,
                         int32_t step_distance, rt_ramp ramp, void* o, void* stream) {
  return rt_sparse_step_ex(desc, q, k, v, idx, rho, r, lambda, step_distance, ramp, RT_EPI_RESHAPED, o, stream);
}

rt_status rt_sparse_step_ex(const rt_attn_desc* desc, const void* q, const void* k, const void* v,
                            const rt_block_index* idx, const float* rho, const void* r, float lambda,
                            int32_t step_distance, rt_ramp ramp, rt_epilogue epi, void* o, void* stream) {
  RT_RANGE("rt_sparse_step_ex");
  if (epi != RT_EPI_RESHAPED && epi != RT_EPI_NO_RHO && epi != RT_EPI_NO_R) return RT_ERR_INVALID_ARGUMENT;
  const bool use_rho = epi != RT_EPI_NO_RHO, use_r = epi != RT_EPI_NO_R;
  rt_status st = validate(desc, q, k, v, idx, o, rho, r, false, use_rho, use_r);
  if (st != RT_OK) return st;
  if (!std::isfinite(lambda) || step_distance < 0) return RT_ERR_INVALID_ARGUMENT;
  double mul = 1.0, add = 0.0;
  const double lam = lambda, kd = step_distance;
  switch (ramp) {
    case RT_RAMP_MUL_LINEAR: mul = 1.0 + lam * kd; break;
    case RT_RAMP_ADD_LINEAR: add = lam * kd; break;
    case RT_RAMP_GEOMETRIC: mul = std::pow(1.0 + lam, kd); break;
    default: return RT_ERR_INVALID_ARGUMENT;
  }
  const rt_attn_desc& d = *desc;
  const int dpad = dpad_of(d.d);
  AttnParams p;
  if ((st = fill_common(d, *idx, p)) != RT_OK) return st;
  p.rho_in = use_rho ? rho : nullptr;
  p.r_in = use_r ? r : nullptr;
  p.use_rho = use_rho;
  p.use_r = use_r;
  p.stride_b = d.stride_b;
  p.stride_h = d.stride_h;
  p.stride_l = d.stride_l;
  p.ramp_mul = static_cast<float>(mul);
  p.ramp_add = static_cast<float>(add);
  TmaSet tm;
  std::memset(&tm, 0, sizeof(tm));
  if ((st = make_chunk_maps(tm.q, q, d, dpad, 128)) != RT_OK) return st;
  if ((st = make_chunk_maps(tm.k, k, d, dpad, static_cast<uint32_t>(d.block))) != RT_OK) return st;
  if ((st = make_chunk_maps(tm.v, v, d, dpad, static_cast<uint32_t>(d.block))) != RT_OK) return st;
  if ((st = make_chunk_maps(tm.o, o, d, dpad, static_cast<uint32_t>(d.block))) != RT_OK) return st;
  if (use_r && (st = make_residual_maps(tm.r, r, d, dpad)) != RT_OK) return st;
  cudaError_t e = dispatch(dpad, false, d, tm, p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RT_OK : cuda_fail(e, "rt_sparse_step launch");
}

rt_status rt_check_device_error(void* stream) {
  unsigned int* w = nullptr;
  rt_status st = status_word(&w);
  if (st != RT_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int val = 0;
  cudaError_t e = cudaMemcpyAsync(&val, w, sizeof(val), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "status readback");
  if (val != 0) {
    e = cudaMemsetAsync(w, 0, sizeof(unsigned int), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "status clear");
  }
  return static_cast<rt_status>(val);
}

rt_status rt_debug_wait_timeout(uint64_t limit_ns, void* stream) {
  unsigned int* w = nullptr;
  rt_status st = status_word(&w);
  if (st != RT_OK) return st;
  if (limit_ns > 10000000000ull) return RT_ERR_INVALID_ARGUMENT;   // at most 10 s
  debug_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, w);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? RT_OK : cuda_fail(e, "rt_debug_wait_timeout launch");
}

}  // extern "C"
