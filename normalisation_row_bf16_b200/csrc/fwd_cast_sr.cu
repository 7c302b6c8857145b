// MXCast kernels, stochastic rounding, with and without a gain along the row;
// see row_fwd.cuh.
#include "fwd_dispatch.h"
#include "row_fwd.cuh"

namespace mxn {
const void* fwd_kernel_cast_sr(int bpt, int tpr, bool has_gamma) {
  return has_gamma ? pick_fwd_shape<kModeCast, true, true>(bpt, tpr)
                   : pick_fwd_shape<kModeCast, true, false>(bpt, tpr);
}
}  // namespace mxn
