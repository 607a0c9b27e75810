// Instantiation of the attention kernel for head dimensions padded to 80.
#include "attn_launch.h"

namespace rtb {

cudaError_t launch_attn_d80(bool cal, int block, const TmaSet& tm, const AttnParams& p, dim3 grid,
                           cudaStream_t s) {
  if (block != 128) return cudaErrorInvalidValue;
  return cal ? launch_cal_impl<80, true>(tm, p, grid, s) : launch_sparse_impl<80>(tm, p, s);
}

}  // namespace rtb
