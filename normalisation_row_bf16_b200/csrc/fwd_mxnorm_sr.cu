// MXNorm forward kernels, stochastic-rounding cast (see row_fwd.cuh).
#include "fwd_dispatch.h"
#include "row_fwd.cuh"

namespace mxn {
const void* fwd_kernel_mxnorm_sr(int bpt, int tpr, bool has_gamma) {
  return has_gamma ? pick_fwd_shape<kModeMXNorm, true, true>(bpt, tpr)
                   : pick_fwd_shape<kModeMXNorm, true, false>(bpt, tpr);
}
}  // namespace mxn
