// MXCast kernels with E2M1 (MXFP4) codes, both roundings, with and without a
// gain along the row; see row_fwd.cuh.
#include "fwd_dispatch.h"
#include "row_fwd.cuh"

namespace mxn {
const void* fwd_kernel_cast_fp4(int bpt, int tpr, bool sr, bool has_gamma) {
  if (sr)
    return has_gamma ? pick_fwd_shape<kModeCast, true, true, kElemE2M1>(bpt, tpr)
                     : pick_fwd_shape<kModeCast, true, false, kElemE2M1>(bpt, tpr);
  return has_gamma ? pick_fwd_shape<kModeCast, false, true, kElemE2M1>(bpt, tpr)
                   : pick_fwd_shape<kModeCast, false, false, kElemE2M1>(bpt, tpr);
}
}  // namespace mxn
