// Instantiation of the attention kernel for head dimensions padded to 64.
#include "attn_launch.h"

namespace rtb {

cudaError_t launch_attn_d64(bool cal, int block, const TmaSet& tm, const AttnParams& p, dim3 grid,
                           cudaStream_t s) {
  if (block == 64) return cal ? launch_attn_impl<64, 64, true>(tm, p, grid, s)
                            : launch_attn_impl<64, 64, false>(tm, p, grid, s);
  if (block != 128) return cudaErrorInvalidValue;
  return cal ? launch_pp_calibrate<64>(tm, p, s) : launch_pp_sparse<64>(tm, p, s);
}

}  // namespace rtb
