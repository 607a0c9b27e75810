// CSR block index of a dense static block mask.
//
// Re-ttention uses one static mask of spatially/temporally local windows for
// all denoising steps (OpenReview reply to W2: a static mask adds no overhead
// at inference), so this runs once per mask, off the per-step path.  The
// result is bit-exact: row_ptr is the exclusive prefix sum of the per-row
// counts, col_idx lists each row's kept key blocks in ascending order.
//
// Three launches, no scratch memory:
//   count  one warp per row writes its popcount into row_ptr[row + 1];
//   scan   one CTA turns row_ptr[1..rows] into inclusive sums in place, row_ptr[0] = 0;
//   fill   one warp per row compacts its kept block ids with ballots, writing
//          only positions below the caller's capacity.
#include <cstdint>

#include <cuda_runtime.h>

namespace rtb {

namespace {

__global__ void bi_count_kernel(const uint8_t* __restrict__ mask, int rows, int nkb,
                                int32_t* __restrict__ row_ptr) {
  const int warps_per_cta = blockDim.x >> 5;
  const int row = blockIdx.x * warps_per_cta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint8_t* m = mask + static_cast<size_t>(row) * nkb;
  int cnt = 0;
  for (int kb = lane; kb < nkb; kb += 32) cnt += m[kb] != 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) row_ptr[row + 1] = cnt;
}

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) bi_scan_kernel(int32_t* __restrict__ row_ptr, int rows) {
  __shared__ int32_t warp_sums[kScanThreads / 32];
  const int t = threadIdx.x;
  const int per = (rows + kScanThreads - 1) / kScanThreads;
  const int r0 = t * per;
  const int r1 = min(rows, r0 + per);
  int local = 0;
  for (int r = r0; r < r1; ++r) local += row_ptr[r + 1];
  // inclusive scan of the per-thread sums across the CTA
  const int lane = t & 31, warp = t >> 5;
  int x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  int run = x - local + (warp > 0 ? warp_sums[warp - 1] : 0);   // exclusive prefix of this thread
  for (int r = r0; r < r1; ++r) {
    run += row_ptr[r + 1];
    row_ptr[r + 1] = run;
  }
  if (t == 0) row_ptr[0] = 0;
}

__global__ void bi_fill_kernel(const uint8_t* __restrict__ mask, int rows, int nkb,
                               const int32_t* __restrict__ row_ptr, int32_t* __restrict__ col_idx,
                               long long capacity) {
  const int warps_per_cta = blockDim.x >> 5;
  const int row = blockIdx.x * warps_per_cta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint8_t* m = mask + static_cast<size_t>(row) * nkb;
  long long pos = row_ptr[row];
  for (int kb0 = 0; kb0 < nkb; kb0 += 32) {
    const int kb = kb0 + lane;
    const bool kept = kb < nkb && m[kb] != 0;
    const unsigned bal = __ballot_sync(0xffffffffu, kept);
    const long long my = pos + __popc(bal & ((1u << lane) - 1u));
    if (kept && my < capacity) col_idx[my] = kb;
    pos += __popc(bal);
  }
}

}  // namespace

cudaError_t launch_block_index(const uint8_t* mask, int rows, int nkb, int32_t* row_ptr,
                               int32_t* col_idx, long long capacity, cudaStream_t s) {
  constexpr int kWarps = 8;
  const int grid = (rows + kWarps - 1) / kWarps;
  bi_count_kernel<<<grid, kWarps * 32, 0, s>>>(mask, rows, nkb, row_ptr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bi_scan_kernel<<<1, kScanThreads, 0, s>>>(row_ptr, rows);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (capacity > 0 && col_idx != nullptr) {
    bi_fill_kernel<<<grid, kWarps * 32, 0, s>>>(mask, rows, nkb, row_ptr, col_idx, capacity);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace rtb
