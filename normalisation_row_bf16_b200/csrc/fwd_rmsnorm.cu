// RMSNorm kernels of the two-pass comparator (see row_fwd.cuh).
#include "fwd_dispatch.h"
#include "row_fwd.cuh"

namespace mxn {
const void* fwd_kernel_rmsnorm(int bpt, int tpr, bool has_gamma) {
  return has_gamma ? pick_fwd_shape<kModeRMSNorm, false, true>(bpt, tpr)
                   : pick_fwd_shape<kModeRMSNorm, false, false>(bpt, tpr);
}
}  // namespace mxn
