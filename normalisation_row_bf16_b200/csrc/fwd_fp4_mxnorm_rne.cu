// MXNorm forward kernels with E2M1 (MXFP4) codes, nearest-even; see row_fwd.cuh.
#include "fwd_dispatch.h"
#include "row_fwd.cuh"

namespace mxn {
const void* fwd_kernel_mxnorm_fp4_rne(int bpt, int tpr, bool has_gamma) {
  return has_gamma ? pick_fwd_shape<kModeMXNorm, false, true, kElemE2M1>(bpt, tpr)
                   : pick_fwd_shape<kModeMXNorm, false, false, kElemE2M1>(bpt, tpr);
}
}  // namespace mxn
