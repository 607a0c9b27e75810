// Token reordering for the static block mask.  The pages lay the video tokens
// of a 3-D latent grid out in a space-filling (Hilbert) order so that every
// 128-token block is a compact brick of the grid and a local window of key
// blocks covers a compact neighbourhood (DFSAttn and the 3-D sparse-attention
// pages reorder tokens this way).  Attention, and every per-token operation of
// the model, commute with a fixed permutation of the tokens, so the order is
// applied once where the tokens are formed and undone where they are
// unpatchified; the attention kernels then run unchanged on reordered tokens.
//
//   rt_hilbert_token_order  host: the permutation (text tokens first, then the
//                           grid in Hilbert order, restricted to the grid)
//   rt_permute_tokens       device: gather rows by the permutation, or scatter
//                           them back (HBM-bound copy, 16-byte accesses)
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <numeric>
#include <vector>

#include "attn_kernel.cuh"
#include "layout.h"
#include "nvtx_range.h"
#include "rt.h"

namespace rtb {
rt_status api_cuda_fail(cudaError_t e, const char* where);
rt_status api_status_word(unsigned int** out);
}

namespace {

// Index of point a[0..n) (n = 1..3 axes) along the n-dimensional Hilbert
// curve of the cube of side 2^bits.  Skilling's transpose method
// ("Programming the Hilbert curve", AIP Conf. Proc. 707, 2004): undo the
// per-level reflections and exchanges from the coarsest level down, Gray-code
// the result, then read the transposed bits out most significant level first,
// axis 0 first.
uint64_t hilbert_index(uint32_t* a, int n, int bits) {
  for (uint32_t q = bits > 0 ? 1u << (bits - 1) : 0u; q > 1; q >>= 1) {
    const uint32_t low = q - 1;
    for (int i = 0; i < n; ++i) {
      if (a[i] & q) {
        a[0] ^= low;                                    // reflect the lower levels of axis 0
      } else {
        const uint32_t t = (a[0] ^ a[i]) & low;         // exchange the lower levels of axes 0 and i
        a[0] ^= t;
        a[i] ^= t;
      }
    }
  }
  for (int i = 1; i < n; ++i) a[i] ^= a[i - 1];
  uint32_t t = 0;
  for (uint32_t q = bits > 0 ? 1u << (bits - 1) : 0u; q > 1; q >>= 1)
    if (a[n - 1] & q) t ^= q - 1;
  for (int i = 0; i < n; ++i) a[i] ^= t;
  uint64_t h = 0;
  for (int j = bits - 1; j >= 0; --j)
    for (int i = 0; i < n; ++i) h = (h << 1) | ((a[i] >> j) & 1u);
  return h;
}

// dst row i <- src row perm[i] (inverse = 0) or dst row perm[i] <- src row i
// (inverse = 1), for every (b, h); one thread per 16-byte chunk of a row (a
// four-deep unrolled variant measured slower on the long-video tensor).
// A perm entry outside [0, L) records RT_ERR_BAD_INDEX and its row is skipped.
__global__ void permute_rows_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst,
                                    const int32_t* __restrict__ perm, int B, int H, int L, int chunks,
                                    long long sb, long long sh, long long sl, int inverse, unsigned int* status) {
  const long long total = static_cast<long long>(B) * H * L * chunks;
  for (long long u = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(u % chunks);
    const long long row = u / chunks;
    const int i = static_cast<int>(row % L);
    const long long bh = row / L;
    const int j = __ldg(perm + i);
    if (j < 0 || j >= L) {
      if (c == 0) atomicCAS(status, 0u, static_cast<unsigned int>(RT_ERR_BAD_INDEX));
      continue;
    }
    const int si = inverse ? i : j, di = inverse ? j : i;
    const long long base = (bh / H) * sb + (bh % H) * sh;       // bytes
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + base + si * sl) + c);
    reinterpret_cast<uint4*>(dst + base + di * sl)[c] = v;
  }
}

}  // namespace

extern "C" {

rt_status rt_hilbert_token_order(int32_t n_text, int32_t F, int32_t Y, int32_t X, int32_t* h_perm) {
  if (!h_perm || n_text < 0 || F < 1 || Y < 1 || X < 1) return RT_ERR_INVALID_ARGUMENT;
  const long long n = static_cast<long long>(F) * Y * X;
  if (n + n_text > (1ll << 31) - 1) return RT_ERR_UNSUPPORTED;
  int bits = 0;
  while ((1ll << bits) < std::max({F, Y, X})) ++bits;
  // the curve runs over the axes longer than 1 (a single frame is a 2-D grid)
  const int32_t ext[3] = {F, Y, X};
  std::vector<uint64_t> key(static_cast<size_t>(n));
  for (int32_t f = 0; f < F; ++f)
    for (int32_t y = 0; y < Y; ++y)
      for (int32_t x = 0; x < X; ++x) {
        const uint32_t c[3] = {static_cast<uint32_t>(f), static_cast<uint32_t>(y), static_cast<uint32_t>(x)};
        uint32_t a[3];
        int na = 0;
        for (int k = 0; k < 3; ++k)
          if (ext[k] > 1) a[na++] = c[k];
        key[(static_cast<size_t>(f) * Y + y) * X + x] = na > 0 ? hilbert_index(a, na, bits) : 0;
      }
  std::vector<int32_t> order(static_cast<size_t>(n));
  std::iota(order.begin(), order.end(), 0);
  std::sort(order.begin(), order.end(), [&](int32_t a, int32_t b) { return key[a] < key[b]; });
  for (int32_t i = 0; i < n_text; ++i) h_perm[i] = i;
  for (long long i = 0; i < n; ++i) h_perm[n_text + i] = n_text + order[static_cast<size_t>(i)];
  return RT_OK;
}

rt_status rt_permute_tokens(const rt_attn_desc* desc, const void* src, void* dst, const int32_t* d_perm,
                            int32_t inverse, void* stream) {
  RT_RANGE("rt_permute_tokens");
  if (!desc || !src || !dst || !d_perm || (inverse != 0 && inverse != 1) || src == dst)
    return RT_ERR_INVALID_ARGUMENT;
  const rt_attn_desc& d = *desc;
  if (d.B < 1 || d.H < 1 || d.L < 1 || d.d < 8 || d.d % 8 != 0) return RT_ERR_INVALID_ARGUMENT;
  if (d.stride_b < 1 || d.stride_h < 1 || d.stride_l < d.d) return RT_ERR_INVALID_ARGUMENT;
  if (d.stride_b % 8 || d.stride_h % 8 || d.stride_l % 8) return RT_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15u) return RT_ERR_INVALID_ARGUMENT;
  // every destination row is written by one thread group: rows must be disjoint,
  // and the source must not be overwritten while it is read
  if (!rtb::layout_rows_disjoint(d)) return RT_ERR_INVALID_ARGUMENT;
  const long long span = rtb::layout_span_bytes(d, 2);
  if (rtb::ranges_overlap(src, span, dst, span)) return RT_ERR_INVALID_ARGUMENT;
  unsigned int* status = nullptr;
  rt_status st = rtb::api_status_word(&status);
  if (st != RT_OK) return st;
  const int chunks = d.d / 8;                       // 16-byte chunks of a bf16 row
  const long long total = static_cast<long long>(d.B) * d.H * d.L * chunks;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (total + 255) / 256;
  const int grid = static_cast<int>(std::min<long long>(want, static_cast<long long>(sms) * 16));
  permute_rows_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(src), static_cast<uint8_t*>(dst), d_perm, d.B, d.H, d.L, chunks,
      d.stride_b * 2, d.stride_h * 2, d.stride_l * 2, inverse, status);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? RT_OK : rtb::api_cuda_fail(e, "rt_permute_tokens launch");
}

}  // extern "C"
