// MXCast kernels, nearest-even and stochastic (see row_fwd.cuh).
#include "fwd_dispatch.h"
#include "row_fwd.cuh"

namespace mxn {
const void* fwd_kernel_cast(int bpt, int tpr, bool sr) {
  return sr ? pick_fwd_shape<kModeCast, true, false>(bpt, tpr)
            : pick_fwd_shape<kModeCast, false, false>(bpt, tpr);
}
}  // namespace mxn
