// Instantiation of the attention kernel for head dimensions padded to 128.
#include "attn_launch.h"

namespace rtb {

cudaError_t launch_attn_d128(bool cal, int block, const TmaSet& tm, const AttnParams& p, dim3 grid,
                           cudaStream_t s) {
  if (block != 128) return cudaErrorInvalidValue;
  return cal ? (p.r_f32 ? launch_cal_impl<128, false>(tm, p, grid, s) : launch_cal_impl<128, true>(tm, p, grid, s)) : launch_sparse_impl<128>(tm, p, s);
}

}  // namespace rtb
