// MXNorm forward and MXCast kernels with NVFP4 codes (E2M1, one E4M3 scale
// per 16 elements), both roundings, with and without gamma; see row_fwd.cuh.
#include "fwd_dispatch.h"
#include "row_fwd.cuh"

namespace mxn {
const void* fwd_kernel_nvfp4(int mode, int bpt, int tpr, bool sr, bool has_gamma) {
  if (mode == kModeMXNorm) {
    if (sr)
      return has_gamma ? pick_fwd_shape<kModeMXNorm, true, true, kElemNVFP4>(bpt, tpr)
                       : pick_fwd_shape<kModeMXNorm, true, false, kElemNVFP4>(bpt, tpr);
    return has_gamma ? pick_fwd_shape<kModeMXNorm, false, true, kElemNVFP4>(bpt, tpr)
                     : pick_fwd_shape<kModeMXNorm, false, false, kElemNVFP4>(bpt, tpr);
  }
  if (mode == kModeCast) {
    if (sr)
      return has_gamma ? pick_fwd_shape<kModeCast, true, true, kElemNVFP4>(bpt, tpr)
                       : pick_fwd_shape<kModeCast, true, false, kElemNVFP4>(bpt, tpr);
    return has_gamma ? pick_fwd_shape<kModeCast, false, true, kElemNVFP4>(bpt, tpr)
                     : pick_fwd_shape<kModeCast, false, false, kElemNVFP4>(bpt, tpr);
  }
  return nullptr;
}
}  // namespace mxn
