// fwd_dispatch.h -- the forward kernel instantiations, one translation unit
// per (mode, rounding, element format) so that they compile in parallel.
#pragma once

namespace mxn {

const void* fwd_kernel_mxnorm_rne(int bpt, int tpr, bool has_gamma);
const void* fwd_kernel_mxnorm_sr(int bpt, int tpr, bool has_gamma);
const void* fwd_kernel_cast_rne(int bpt, int tpr, bool has_gamma);
const void* fwd_kernel_cast_sr(int bpt, int tpr, bool has_gamma);
const void* fwd_kernel_rmsnorm(int bpt, int tpr, bool has_gamma);
// E2M1 (MXFP4) codes: MXNorm and MXCast.
const void* fwd_kernel_mxnorm_fp4_rne(int bpt, int tpr, bool has_gamma);
const void* fwd_kernel_mxnorm_fp4_sr(int bpt, int tpr, bool has_gamma);
const void* fwd_kernel_cast_fp4(int bpt, int tpr, bool sr, bool has_gamma);
// NVFP4 codes (E2M1, E4M3 scale per 16): MXNorm and MXCast.
const void* fwd_kernel_nvfp4(int mode, int bpt, int tpr, bool sr, bool has_gamma);

}  // namespace mxn
