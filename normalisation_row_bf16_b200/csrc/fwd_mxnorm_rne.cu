// MXNorm forward kernels, nearest-even cast (see row_fwd.cuh).
#include "fwd_dispatch.h"
#include "row_fwd.cuh"

namespace mxn {
const void* fwd_kernel_mxnorm_rne(int bpt, int tpr, bool has_gamma) {
  return has_gamma ? pick_fwd_shape<kModeMXNorm, false, true>(bpt, tpr)
                   : pick_fwd_shape<kModeMXNorm, false, false>(bpt, tpr);
}
}  // namespace mxn
