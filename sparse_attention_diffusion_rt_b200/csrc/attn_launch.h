// Host-side launch interface shared by the C-ABI layer and the per-head-dim
// kernel instantiation units.
#pragma once
#include <cuda_runtime.h>

#include <atomic>

#include "attn_kernel.cuh"
#include "sparse_kernel.cuh"
#include "pp_sparse.cuh"
#include "pp_calibrate.cuh"
#include "cal_kernel.cuh"

namespace rtb {

// Every launch asks for at least this much shared memory so that no two CTAs
// share an SM (each allocates all 512 TMEM columns).
constexpr int kMinSmem = 120 * 1024;

// Dynamic shared memory one launch of attn_kernel<DPAD, BN, CAL> needs (bytes),
// never below kMinSmem.
template <int DPAD, int BN>
constexpr int attn_smem_bytes(bool cal, bool r_f32) {
  using C = Cfg<DPAD, BN>;
  const int need = cal ? C::SMEM_CAL : C::OFF_R + (r_f32 ? C::R_MAX_BYTES : C::Q_BYTES) + 1024;
  return need > kMinSmem ? need : kMinSmem;
}

// Launch the attention kernel instantiated for (dpad, block, cal).
// Returns cudaErrorInvalidValue for an instantiation that does not exist.
cudaError_t launch_attn_d64(bool cal, int block, const TmaSet& tm, const AttnParams& p, dim3 grid,
                            cudaStream_t s);
cudaError_t launch_attn_d80(bool cal, int block, const TmaSet& tm, const AttnParams& p, dim3 grid,
                            cudaStream_t s);
cudaError_t launch_attn_d96(bool cal, int block, const TmaSet& tm, const AttnParams& p, dim3 grid,
                            cudaStream_t s);
cudaError_t launch_attn_d128(bool cal, int block, const TmaSet& tm, const AttnParams& p, dim3 grid,
                             cudaStream_t s);

template <int DPAD, int BN, bool CAL>
cudaError_t launch_attn_impl(const TmaSet& tm, const AttnParams& p, dim3 grid, cudaStream_t s) {
  constexpr int kMaxSmem = attn_smem_bytes<DPAD, BN>(CAL, true) > attn_smem_bytes<DPAD, BN>(CAL, false)
                               ? attn_smem_bytes<DPAD, BN>(CAL, true) : attn_smem_bytes<DPAD, BN>(CAL, false);
  const int smem = attn_smem_bytes<DPAD, BN>(CAL, p.r_f32 != 0);
  auto kern = attn_kernel<DPAD, BN, CAL>;
  // the shared-memory opt-in is a per-device function attribute: set it once per device
  static std::atomic<unsigned long long> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  kern<<<grid, kThreads, smem, s>>>(tm, p);
  return cudaGetLastError();
}

// Calibration kernel with one TMEM accumulator (d > 64, 128-token blocks):
// one CTA per (query block, head, batch); QT = Q in TMEM.
template <int DPAD, bool QT>
cudaError_t launch_cal_impl(const TmaSet& tm, const AttnParams& p, dim3 grid, cudaStream_t s) {
  auto kern = cal_kernel<DPAD, QT>;
  constexpr int smem = CalCfg<DPAD, QT>::SMEM > kMinSmem ? CalCfg<DPAD, QT>::SMEM : kMinSmem;
  static std::atomic<unsigned long long> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  kern<<<grid, kThreads, smem, s>>>(tm, p);
  return cudaGetLastError();
}

// Persistent sparse-step kernel (128-token blocks): one CTA per SM.
template <int DPAD>
cudaError_t launch_sparse_impl(const TmaSet& tm, const AttnParams& p, cudaStream_t s) {
  auto kern = sparse_kernel<DPAD>;
  constexpr int smem = SpCfg<DPAD>::SMEM > kMinSmem ? SpCfg<DPAD>::SMEM : kMinSmem;
  static std::atomic<unsigned long long> configured{0};
  static int sm_count[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sm_count[dev & 63], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  const long long ntiles = static_cast<long long>(p.B) * p.H * p.nqb;
  const int grid = static_cast<int>(ntiles < sm_count[dev & 63] ? ntiles : sm_count[dev & 63]);
  kern<<<grid, kSpThreads, smem, s>>>(tm, p, static_cast<int>(ntiles));
  return cudaGetLastError();
}

// Ping-pong persistent sparse-step kernel (d <= 64, 128-token blocks).
template <int DPAD>
cudaError_t launch_pp_sparse(const TmaSet& tm, const AttnParams& p, cudaStream_t s) {
  static std::atomic<unsigned long long> configured{0};
  static int sm_count[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(pp_sparse_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, PpCfg::SMEM);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sm_count[dev & 63], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  const long long ntiles = static_cast<long long>(p.B) * p.H * p.nqb;
  const long long half = (ntiles + 1) / 2;
  const int grid = static_cast<int>(half < sm_count[dev & 63] ? half : sm_count[dev & 63]);
  pp_sparse_kernel<64><<<grid, kPpThreads, PpCfg::SMEM, s>>>(tm, p, static_cast<int>(ntiles));
  return cudaGetLastError();
}

// Ping-pong calibration kernel (d <= 64, 128-token blocks): two query tiles per CTA.
template <int DPAD>
cudaError_t launch_pp_calibrate(const TmaSet& tm, const AttnParams& p, cudaStream_t s) {
  static std::atomic<unsigned long long> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(pp_calibrate_kernel<DPAD>, cudaFuncAttributeMaxDynamicSharedMemorySize, PcCfg::SMEM);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  const dim3 grid(static_cast<unsigned>((p.nqb + 1) / 2), static_cast<unsigned>(p.H), static_cast<unsigned>(p.B));
  pp_calibrate_kernel<DPAD><<<grid, 352, PcCfg::SMEM, s>>>(tm, p);
  return cudaGetLastError();
}

}  // namespace rtb
