// Instantiation of the attention kernel for head dimensions padded to 96.
#include "attn_launch.h"

namespace rtb {

cudaError_t launch_attn_d96(bool cal, int block, const TmaSet& tm, const AttnParams& p, dim3 grid,
                           cudaStream_t s) {
  if (block != 128) return cudaErrorInvalidValue;
  return cal ? launch_cal_impl<96, true>(tm, p, grid, s) : launch_sparse_impl<96>(tm, p, s);
}

}  // namespace rtb
