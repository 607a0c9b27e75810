// Host-side launch interface shared by the C-ABI layer and the per-head-dim
// kernel instantiation units.
#pragma once
#include <cuda_runtime.h>

#include <atomic>

#include "attn_kernel.cuh"

namespace rtb {

// Every launch asks for at least this much shared memory so that no two CTAs
// share an SM (each allocates all 512 TMEM columns).
constexpr int kMinSmem = 120 * 1024;

// Dynamic shared memory the launch needs (bytes).
int attn_smem_bytes(int dpad, bool cal, bool r_f32);

// Launch the attention kernel instantiated for (dpad, block, cal).
// Returns cudaErrorInvalidValue for an instantiation that does not exist.
cudaError_t launch_attn_d64(bool cal, int block, const TmaSet& tm, const AttnParams& p, dim3 grid,
                            int smem, cudaStream_t s);
cudaError_t launch_attn_d80(bool cal, int block, const TmaSet& tm, const AttnParams& p, dim3 grid,
                            int smem, cudaStream_t s);
cudaError_t launch_attn_d96(bool cal, int block, const TmaSet& tm, const AttnParams& p, dim3 grid,
                            int smem, cudaStream_t s);
cudaError_t launch_attn_d128(bool cal, int block, const TmaSet& tm, const AttnParams& p, dim3 grid,
                             int smem, cudaStream_t s);

template <int DPAD, int BN, bool CAL>
cudaError_t launch_attn_impl(const TmaSet& tm, const AttnParams& p, dim3 grid, int smem,
                             cudaStream_t s) {
  auto kern = attn_kernel<DPAD, BN, CAL>;
  // the shared-memory opt-in is a per-device function attribute: set it once per device
  static std::atomic<unsigned long long> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg<DPAD, BN>::SMEM_SPARSE > kMinSmem ? Cfg<DPAD, BN>::SMEM_SPARSE : kMinSmem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  kern<<<grid, kThreads, smem, s>>>(tm, p);
  return cudaGetLastError();
}

}  // namespace rtb
