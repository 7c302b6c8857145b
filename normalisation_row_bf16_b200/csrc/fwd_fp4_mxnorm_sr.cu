// MXNorm forward kernels with E2M1 (MXFP4) codes, stochastic rounding; see row_fwd.cuh.
#include "fwd_dispatch.h"
#include "row_fwd.cuh"

namespace mxn {
const void* fwd_kernel_mxnorm_fp4_sr(int bpt, int tpr, bool has_gamma) {
  return has_gamma ? pick_fwd_shape<kModeMXNorm, true, true, kElemE2M1>(bpt, tpr)
                   : pick_fwd_shape<kModeMXNorm, true, false, kElemE2M1>(bpt, tpr);
}
}  // namespace mxn
