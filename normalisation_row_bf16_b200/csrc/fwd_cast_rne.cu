// MXCast kernels, nearest-even, with and without a gain along the row (the
// folded MXNormLinear weight); see row_fwd.cuh.
#include "fwd_dispatch.h"
#include "row_fwd.cuh"

namespace mxn {
const void* fwd_kernel_cast_rne(int bpt, int tpr, bool has_gamma) {
  return has_gamma ? pick_fwd_shape<kModeCast, false, true>(bpt, tpr)
                   : pick_fwd_shape<kModeCast, false, false>(bpt, tpr);
}
}  // namespace mxn
