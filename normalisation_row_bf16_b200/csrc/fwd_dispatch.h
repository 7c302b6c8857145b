// fwd_dispatch.h -- the forward kernel instantiations, one translation unit
// per (mode, rounding) so that they compile in parallel.
#pragma once

namespace mxn {

const void* fwd_kernel_mxnorm_rne(int bpt, int tpr, bool has_gamma);
const void* fwd_kernel_mxnorm_sr(int bpt, int tpr, bool has_gamma);
const void* fwd_kernel_cast(int bpt, int tpr, bool sr);
const void* fwd_kernel_rmsnorm(int bpt, int tpr, bool has_gamma);

}  // namespace mxn
