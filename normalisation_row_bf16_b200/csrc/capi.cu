// capi.cu -- the C ABI declared in include/mxnorm.h: argument checks, launch
// planning and error reporting around the row kernels.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <map>
#include <mutex>
#include <string>
#include <tuple>

#include "fwd_dispatch.h"
#include "gemm_mxfp8.h"
#include "mxnorm.h"
#include "row_bwd.cuh"
#include "row_fwd.cuh"

// Device status word: kernels record a bounded wait that gave up here.
__device__ unsigned g_mxn_status;

namespace {

using namespace mxn;

constexpr int kMaxDevices = 64;
constexpr int kMaxBwdD = 16384;

thread_local std::string t_err;
thread_local int t_fail_next = 0;

struct Tuning {
  int consumer_threads = 0, stages = 0, ctas_per_sm = 0;
} g_tuning;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_err = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(MXN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DeviceInfo {
  int sms = 0;
  unsigned* status = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// SM count and the status word's device address for the current device,
// looked up once per device.
int device_info(DeviceInfo* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MXN_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.sms == 0) {
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_mxn_status);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status)");
    d.status = static_cast<unsigned*>(p);
    d.sms = sms;
  }
  *out = d;
  return MXN_OK;
}

int injected() {
  if (t_fail_next > 0) {
    --t_fail_next;
    return fail(MXN_ERR_CUDA, "injected failure (mxnorm_debug_fail_next)");
  }
  return MXN_OK;
}

int next_pow2(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

int ilog2(int v) {
  int l = 0;
  while ((1 << l) < v) ++l;
  return l;
}

// Resident CTAs per SM of (kernel, threads, dynamic shared memory) on the
// current device.  The first use of a combination sets the kernel's dynamic
// shared-memory limit and queries the occupancy; later launches reuse both,
// so a launch costs one map lookup on the host.
std::map<std::tuple<int, const void*, int, size_t>, int> g_occ;
std::mutex g_occ_mu;

int occupancy(const void* kernel, int threads, size_t smem, int* occ) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  const auto key = std::make_tuple(dev, kernel, threads, smem);
  {
    std::lock_guard<std::mutex> lk(g_occ_mu);
    auto it = g_occ.find(key);
    if (it != g_occ.end()) {
      *occ = it->second;
      return MXN_OK;
    }
  }
  // Raise the kernel's dynamic shared-memory limit to the device maximum, so
  // that no plan can shrink it below what another cached plan launches with.
  int optin = 0;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(smem optin)");
  if (smem > (size_t)optin) return fail(MXN_ERR_UNSUPPORTED, "%zu bytes of shared memory > %d", smem, optin);
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  int n = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
  std::lock_guard<std::mutex> lk(g_occ_mu);
  g_occ[key] = n;
  *occ = n;
  return MXN_OK;
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel in the stream drains; every row kernel waits
// (griddepcontrol.wait) before it reads or writes a tensor.
int launch_pdl(const void* kernel, int grid, int threads, size_t smem, void** argv, cudaStream_t stream,
               const char* what) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelExC(&cfg, kernel, argv);
  if (e != cudaSuccess) return cuda_fail(e, what);
  return MXN_OK;
}

// Pointer checks are skipped for T = 0 (an empty tensor may have no storage);
// shape checks always run.
thread_local bool t_empty = false;

int check_common(const void* x, int64_t T, int64_t D, int64_t ld_x) {
  t_empty = (T == 0);
  if (!x && !t_empty) return fail(MXN_ERR_ARG, "x is NULL");
  if (T < 0) return fail(MXN_ERR_ARG, "T = %lld < 0", (long long)T);
  if (D <= 0 || D % kBlock != 0) return fail(MXN_ERR_ARG, "D = %lld is not a positive multiple of 32", (long long)D);
  if (D > MXN_MAX_D) return fail(MXN_ERR_UNSUPPORTED, "D = %lld > %d", (long long)D, MXN_MAX_D);
  if (ld_x < D || ld_x % 8 != 0)
    return fail(MXN_ERR_ARG, "ld_x = %lld must be >= D and a multiple of 8", (long long)ld_x);
  if (!aligned16(x)) return fail(MXN_ERR_ARG, "x is not 16-byte aligned");
  return MXN_OK;
}

int check_out(const void* p, const char* name) {
  if (!p && t_empty) return MXN_OK;
  if (!p) return fail(MXN_ERR_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(MXN_ERR_ARG, "%s is not 16-byte aligned", name);
  return MXN_OK;
}

int check_opt(const void* p, const char* name) {
  if (p && !aligned16(p)) return fail(MXN_ERR_ARG, "%s is not 16-byte aligned", name);
  return MXN_OK;
}

const void* fwd_kernel(int mode, bool sr, bool has_gamma, int elem, int bpt, int tpr) {
  if (elem == kElemNVFP4) return fwd_kernel_nvfp4(mode, bpt, tpr, sr, has_gamma);
  if (elem == kElemE2M1) {
    switch (mode) {
      case kModeMXNorm:
        return sr ? fwd_kernel_mxnorm_fp4_sr(bpt, tpr, has_gamma) : fwd_kernel_mxnorm_fp4_rne(bpt, tpr, has_gamma);
      case kModeCast: return fwd_kernel_cast_fp4(bpt, tpr, sr, has_gamma);
      default: return nullptr;
    }
  }
  switch (mode) {
    case kModeMXNorm:
      return sr ? fwd_kernel_mxnorm_sr(bpt, tpr, has_gamma) : fwd_kernel_mxnorm_rne(bpt, tpr, has_gamma);
    case kModeCast:
      return sr ? fwd_kernel_cast_sr(bpt, tpr, has_gamma) : fwd_kernel_cast_rne(bpt, tpr, has_gamma);
    case kModeRMSNorm: return fwd_kernel_rmsnorm(bpt, tpr, has_gamma);
    default: return nullptr;
  }
}

// Launch plan for the forward row kernels (row_fwd.cuh).
struct FwdPlan {
  FwdCfg C;
  const void* kernel = nullptr;
  int threads = 0;
  size_t smem = 0;
  int grid = 0;
};

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

int plan_fwd(int mode, bool sr, bool gamma_smem, int elem, int64_t T, int D, int64_t ld_x, int sms,
             FwdPlan* P) {
  FwdCfg& C = P->C;
  C = FwdCfg{};
  C.T = T;
  C.ld_x = ld_x;
  C.D = D;
  C.K = D / kBlock;
  // Blocks per thread and threads per row: rows of up to 128 blocks take one
  // warp (1, 2 or 4 blocks per thread), longer rows 4 blocks per thread over
  // 64..256 threads, rows under 32 blocks a power-of-two segment of a warp.
  // Stochastic rounding spreads rows wider: one block per thread up to 64
  // blocks, two up to 512 (over 64..256 threads; measured 8% faster than one
  // block per thread at 128 blocks), then 4 over 256 threads.
  int bpt;
  if (C.K <= 32) { bpt = 1; C.tpr = next_pow2(C.K); }
  else if (sr && C.K <= 64) { bpt = 1; C.tpr = next_pow2(C.K); }
  else if (sr && C.K <= 512) { bpt = 2; C.tpr = next_pow2((C.K + 1) / 2); }
  else if (C.K <= 64) { bpt = 2; C.tpr = 32; }
  else if (C.K <= 128) { bpt = 4; C.tpr = 32; }
  else { bpt = 4; C.tpr = next_pow2((C.K + 3) / 4); }
  C.log2_tpr = ilog2(C.tpr);
  C.gthreads = C.tpr < 32 ? 32 : C.tpr;
  C.rps = C.gthreads / C.tpr;
  C.row_bytes = 2u * (uint32_t)D;
  C.stage_bytes = (uint32_t)C.rps * C.row_bytes;
  // Defaults measured on B200 with whole input and output sets rotating
  // through HBM (T = 8192 and 16384): one stage per group, and 512 threads
  // per CTA for rows of 33..64 blocks and of more than 256, 384 for 65..256
  // blocks of E4M3 codes (12 one-warp rows or 6 two-warp rows in flight per
  // SM).  The FP4 formats do more arithmetic per byte and want the warps:
  // 512 threads there too (MXFP4 / NVFP4 at 16384 x 8192: 65.5 -> 57.8 and
  // 100.1 -> 85.6 us; at 8192 x 4096: 17.8 -> 17.4 and 27.2 -> 26.0 us).
  // Rows under 33 blocks, and stochastic rounding (bound by the Philox
  // arithmetic), keep the largest CTA the kernel is compiled for
  // (fwd_launch_threads) with extra stages while 176 KB covers them.
  const bool widest = bpt == 1 || sr;
  const bool fp4 = elem != kElemE4M3;
  const int def_threads = widest ? fwd_max_threads(bpt) : (bpt == 2 || C.tpr > 64 || fp4 ? 512 : 384);
  if (g_tuning.stages) {
    C.stages = g_tuning.stages;
  } else if (widest) {
    const int gmax = fwd_max_threads(bpt) / (C.tpr < 32 ? 32 : C.tpr);
    int st = (int)((176u * 1024u) / ((size_t)gmax * C.rps * 2u * (uint32_t)D));
    C.stages = st < 1 ? 1 : (st > 3 ? 3 : st);
  } else {
    C.stages = 1;
  }
  // gamma in shared memory: fp32 for up to 64 threads per row (D <= 8192), else bf16
  C.gamma_bytes = gamma_smem ? (uint32_t)align_up((gamma_fp32(C.tpr) ? 4u : 2u) * (uint32_t)D, 128) : 0u;
  size_t per_group = (size_t)C.stages * C.stage_bytes;
  // MXNorm and MXCast rows of several warps stage each row's codes in shared
  // memory and write them with one bulk copy (D bytes of E4M3, half that of
  // E2M1); see kFwdBulkStores.
  C.code_row_bytes = elem == kElemE4M3 ? (uint32_t)D : (uint32_t)D / 2u;
  C.ostage_bytes = (mode == kModeRMSNorm || C.tpr <= 32 || sr) ? 0u : (uint32_t)align_up((size_t)C.rps * C.code_row_bytes, 128);
  // Shared memory per group: its ring, its code staging buffer, its 2 * stages
  // barriers and its two reduction slot arrays; plus gamma and 16 bytes of
  // alignment once.
  size_t per_group_base = per_group + (size_t)2 * C.stages * sizeof(uint64_t) +
                          (size_t)2 * kRedSlots * sizeof(float2);
  int ng;
  if (g_tuning.consumer_threads) {
    ng = g_tuning.consumer_threads / C.gthreads;
  } else {
    ng = def_threads / C.gthreads;
  }
  int ng_max = fwd_launch_threads(bpt, C.tpr, sr, elem) / C.gthreads;
  const size_t fixed = C.gamma_bytes + 16 + (elem == kElemNVFP4 ? 128u * sizeof(float) : 0u);
  const size_t smem_cap = 227u * 1024u;
  if (fixed + per_group_base > smem_cap)
    return fail(MXN_ERR_UNSUPPORTED, "row of %d elements does not fit in shared memory", D);
  int ng_fit = (int)((smem_cap - fixed) / per_group_base);
  if (ng_fit < ng_max) ng_max = ng_fit;
  ng = ng < 1 ? 1 : (ng > ng_max ? ng_max : ng);
  // Few rows for the device (full CTAs would not reach every SM): fewer row
  // groups per CTA, at least 4, so that the rows spread over (nearly) every SM,
  // and one stage, since each group then gets about one row.  Measured on
  // B200: 256 x 1024 4.06 -> 2.52 us, 1024 x 1024 4.30 -> 2.91, 256 x 4096
  // 5.87 -> 4.28, 1024 x 4096 6.44 -> 5.07; shapes that fill every SM as
  // planned are unchanged.
  const int64_t n_rb = (T + C.rps - 1) / C.rps;
  if (!g_tuning.consumer_threads && !g_tuning.stages && (n_rb + ng - 1) / ng < sms) {
    int64_t ng_small = (n_rb + sms - 1) / sms;
    if (ng_small < 4) ng_small = 4;
    if (ng_small < ng) {
      ng = (int)ng_small;
      C.stages = 1;
      per_group = C.stage_bytes;
      per_group_base = per_group + 2 * sizeof(uint64_t) + (size_t)2 * kRedSlots * sizeof(float2);
    }
  }
  // The staging buffers must not cost row groups: where they would, codes are
  // stored directly.
  if (C.ostage_bytes && fixed + (size_t)ng * (per_group_base + C.ostage_bytes) > smem_cap) C.ostage_bytes = 0;
  if (C.tpr > 32 && ng > 15) ng = 15;  // named barriers 1..15
  C.ng = ng;
  C.n_row_blocks = n_rb;
  C.ring_off = C.gamma_bytes;
  C.out_off = (uint32_t)align_up(C.ring_off + (size_t)ng * per_group, 128);
  C.bar_off = (uint32_t)align_up(C.out_off + (size_t)ng * C.ostage_bytes, 16);
  C.red_off = C.bar_off + (uint32_t)(ng * 2 * C.stages * sizeof(uint64_t));
  C.rcp_off = (uint32_t)(C.red_off + (size_t)ng * 2 * kRedSlots * sizeof(float2));
  P->smem = C.rcp_off + (elem == kElemNVFP4 ? 128u * sizeof(float) : 0u);
  P->threads = ng * C.gthreads;
  P->kernel = fwd_kernel(mode, sr, gamma_smem, elem, bpt, C.tpr);
  if (!P->kernel) return fail(MXN_ERR_UNSUPPORTED, "no kernel for D = %d", D);
  int occ = 0;
  int rc = occupancy(P->kernel, P->threads, P->smem, &occ);
  if (rc) return rc;
  if (occ < 1) return fail(MXN_ERR_UNSUPPORTED, "row kernel does not fit on an SM (D = %d)", D);
  if (g_tuning.ctas_per_sm && g_tuning.ctas_per_sm < occ) occ = g_tuning.ctas_per_sm;
  // One CTA per resident slot (fewer when there are fewer row blocks than groups).
  const int64_t max_ctas = (int64_t)sms * occ;
  const int64_t need_ctas = (C.n_row_blocks + ng - 1) / ng;
  const int64_t ctas = need_ctas < max_ctas ? need_ctas : max_ctas;
  // Nearest-even E4M3 codes (memory-bound): every active group gets R or R - 1
  // row blocks with R = ceil(blocks / groups), only as many groups as R rounds
  // need take rows, so no round runs on a fraction of the groups while the
  // rest idle.  Stochastic rounding and the FP4 formats (bound by their
  // arithmetic): row blocks dealt round-robin over every group, which spreads
  // them evenly over the SMs (within one block per SM) -- measured on B200 at
  // 8192 x 4096: SR 55.4 -> 53.1, MXFP4 18.3 -> 17.6, NVFP4 24.8 -> 23.9 us,
  // while the E4M3 forward ran 18.8 -> 19.5 us that way.
  if (sr || elem != kElemE4M3) {
    C.ngt = ctas * ng;
  } else {
    const int64_t R = (C.n_row_blocks + ctas * ng - 1) / (ctas * ng);
    C.ngt = R > 0 ? (C.n_row_blocks + R - 1) / R : 0;
  }
  P->grid = (int)ctas;
  return MXN_OK;
}

int launch_fwd(int mode, bool sr, const FwdArgs& A, int64_t T, int D, int64_t ld_x,
               cudaStream_t stream) {
  DeviceInfo dev;
  int rc = device_info(&dev);
  if (rc) return rc;
  FwdPlan P;
  rc = plan_fwd(mode, sr, A.gamma != nullptr, A.elem, T, D, ld_x, dev.sms, &P);
  if (rc) return rc;
  FwdArgs a = A;
  a.status = dev.status;
  a.n_stat = A.elem == kElemNVFP4 ? D / 16 : D / kBlock;   // statistic blocks per row
  a.inv_n_stat = 1.0 / (double)a.n_stat;
  a.inv_k_pow2 = (a.n_stat & (a.n_stat - 1)) == 0 ? (float)a.inv_n_stat : 0.0f;
  void* argv[] = {&a, &P.C};
  return launch_pdl(P.kernel, P.grid, P.threads, P.smem, argv, stream, "row_fwd_kernel launch");
}

int pmode_of(float p) {
  if (std::isinf(p)) return kPInf;
  if (p == 1.0f) return kP1;
  if (p == 2.0f) return kP2;
  if (p == 4.0f) return kP4;
  return kPGeneral;
}

// Launch plan of the backward row kernel (row_bwd.cuh).
struct BwdPlan {
  BwdCfg C;
  const void* kernel = nullptr;
  int threads = 0;
  size_t smem = 0;
  int grid = 0;
  size_t partial_rows() const { return (size_t)grid; }   // one per CTA
};

// Rows of up to 256 blocks: one block per thread (tpr = K, several rows per
// warp below 32 blocks); 257..512 blocks: 256 threads with two blocks each.
// Row groups per CTA fill the register budget (512 threads, or 256 with two
// blocks), one stage each by default; one CTA per SM.
// max_partial_rows > 0 caps the groups that get rows (the allocation-free
// entry point's scratch).
int plan_bwd(int64_t T, int D, int sms, BwdPlan* P, int64_t max_partial_rows = 0) {
  BwdCfg& C = P->C;
  C = BwdCfg{};
  C.T = T;
  C.D = D;
  C.K = D / kBlock;
  int bpt;
  if (C.K <= 256) { bpt = 1; C.tpr = next_pow2(C.K); }
  else if (C.K <= 512) { bpt = 2; C.tpr = 256; }
  else return fail(MXN_ERR_UNSUPPORTED, "mxnorm_bwd: D = %d > %d", D, kMaxBwdD);
  C.log2_tpr = ilog2(C.tpr);
  C.gthreads = C.tpr < 32 ? 32 : C.tpr;
  C.rps = C.gthreads / C.tpr;
  C.row_bytes = 2u * (uint32_t)D;
  C.stage_bytes = 2u * (uint32_t)C.rps * C.row_bytes;
  const int max_threads = bwd_max_threads(bpt);
  int threads = g_tuning.consumer_threads ? g_tuning.consumer_threads : max_threads;
  if (threads > max_threads) threads = max_threads;
  int ng = threads / C.gthreads;
  if (ng < 1) ng = 1;
  if (C.tpr > 32 && ng > 15) ng = 15;  // named barriers 1..15
  const size_t smem_cap = 227u * 1024u;
  const size_t per_group_fixed = (size_t)2 * kRedSlots * sizeof(float2) + 16;
  // One stage per group measured best on B200 (8192 x 4096: 47.4 us against
  // 49.1 with two stages and 51.6 with three groups of two stages).
  const int stages = g_tuning.stages ? g_tuning.stages : 1;
  C.gamma_bytes = (uint32_t)align_up(4u * (uint32_t)D, 128);   // fp32
  // dx staged per group and written with one bulk copy per row block, while
  // the buffers fit beside the rings of the planned groups.
  C.ostage_bytes = (uint32_t)align_up((size_t)C.rps * C.row_bytes, 128);
  auto smem_of = [&](int n) {
    return (size_t)C.gamma_bytes + (size_t)n * stages * (C.stage_bytes + 2 * sizeof(uint64_t) + sizeof(uint32_t)) +
           (size_t)n * (per_group_fixed + C.ostage_bytes) + 128 + 16;
  };
  {
    const uint32_t keep = C.ostage_bytes;
    C.ostage_bytes = 0;
    while (ng > 1 && smem_of(ng) > smem_cap) --ng;
    C.ostage_bytes = keep;
    if (smem_of(ng) > smem_cap) C.ostage_bytes = 0;
  }
  if (smem_of(ng) > smem_cap)
    return fail(MXN_ERR_UNSUPPORTED, "mxnorm_bwd: a row of %d elements does not fit in shared memory", D);
  C.ng = ng;
  C.stages = stages;
  C.n_row_blocks = (T + C.rps - 1) / C.rps;
  C.ring_off = C.gamma_bytes;
  C.out_off = (uint32_t)align_up(C.ring_off + (size_t)ng * stages * C.stage_bytes, 128);
  C.bar_off = (uint32_t)align_up(C.out_off + (size_t)ng * C.ostage_bytes, 16);
  C.red_off = C.bar_off + (uint32_t)(ng * 2 * stages * sizeof(uint64_t));
  C.cnt_off = C.red_off + (uint32_t)(ng * 2 * kRedSlots * sizeof(float2));
  P->smem = C.cnt_off + (size_t)ng * stages * sizeof(uint32_t);
  P->threads = ng * C.gthreads;
  P->kernel = pick_bwd_shape(bpt, C.tpr);
  if (!P->kernel) return fail(MXN_ERR_UNSUPPORTED, "mxnorm_bwd: no kernel for D = %d", D);
  int occ = 0;
  int rc = occupancy(P->kernel, P->threads, P->smem, &occ);
  if (rc) return rc;
  if (occ < 1) return fail(MXN_ERR_UNSUPPORTED, "mxnorm_bwd: row kernel does not fit on an SM (D = %d)", D);
  if (g_tuning.ctas_per_sm && g_tuning.ctas_per_sm < occ) occ = g_tuning.ctas_per_sm;
  int64_t ctas = (C.n_row_blocks + ng - 1) / ng;
  if (ctas > (int64_t)sms * occ) ctas = (int64_t)sms * occ;
  if (max_partial_rows > 0 && ctas > max_partial_rows) ctas = max_partial_rows;   // one partial row per CTA
  const int64_t R = (C.n_row_blocks + ctas * ng - 1) / (ctas * ng);
  C.ngt = R > 0 ? (C.n_row_blocks + R - 1) / R : 0;
  P->grid = (int)ctas;
  return MXN_OK;
}

// Backward row kernel, then (when partial is set) the fixed-order dgamma sum.
int launch_bwd(const BwdPlan& P, const BwdArgs& A, uint16_t* dgamma, cudaStream_t s) {
  void* argv[] = {const_cast<BwdArgs*>(&A), const_cast<BwdCfg*>(&P.C)};
  int rc = launch_pdl(P.kernel, P.grid, P.threads, P.smem, argv, s, "row_bwd_kernel launch");
  if (rc) return rc;
  if (A.partial) {
    const float* part = A.partial;
    int64_t n_part = (int64_t)P.partial_rows();
    int D = P.C.D;
    void* rargv[] = {&part, &n_part, &D, &dgamma};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((D + 31) / 32));
    cfg.blockDim = dim3(32, 32);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelExC(&cfg, (const void*)dgamma_reduce_kernel, rargv);
    if (e != cudaSuccess) return cuda_fail(e, "dgamma_reduce_kernel launch");
  }
  return MXN_OK;
}

// ----------------------------------------------- allocation-free backward
//
// Scratch for mxnorm_bwd_noalloc: the per-CTA dgamma partial sums, 2^21 fp32
// (8 MiB).  The runtime reserves it on a device when the library's kernels are
// first used there (whether or not mxnorm_bwd_noalloc is called) and holds it
// until the process exits.  In host code the name is only a host-side stand-in; its device
// address comes from cudaGetSymbolAddress, looked up once per device with
// that device current.
constexpr size_t kNoAllocScratchFloats = size_t(1) << 21;
static __device__ __align__(256) float g_bwd_noalloc_scratch[kNoAllocScratchFloats];

float* g_noalloc_scratch_ptr[kMaxDevices];
std::mutex g_noalloc_mu;

int noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MXN_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_bwd_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(noalloc scratch)");
    g_noalloc_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_scratch_ptr[dev];
  return MXN_OK;
}

// Test kernel for the bounded-wait mechanism: one thread initialises an
// mbarrier that expects one arrival, never arrives, and waits on it for at most
// limit_ns; the wait gives up, records itself in the status word and returns.
__global__ void wait_timeout_probe_kernel(uint64_t limit_ns, unsigned* status, int* gave_up) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    *gave_up = mbar_wait_limit(&bar, 0, limit_ns, status) ? 0 : 1;
  }
}

}  // namespace

extern "C" {

size_t mxnorm_scales_bytes(int64_t T, int64_t D, int layout) {
  if (T < 0 || D <= 0 || D % kBlock != 0) return 0;
  const int64_t K = D / kBlock;
  if (layout == MXN_SCALES_ROWMAJOR) return (size_t)(T * K);
  if (layout == MXN_SCALES_MMA) return (size_t)(((T + 127) / 128) * 128 * ((K + 3) / 4) * 4);
  return 0;
}

static int fwd_like(int mode, const void* x, const void* gamma, void* q, void* scales, float* G_out,
                    int64_t T, int64_t D, int64_t ld_x, float p, int rounding, uint64_t seed,
                    int scale_layout, int elem, int stat, void* stream) {
  t_err.clear();
  int rc = check_common(x, T, D, ld_x);
  if (!rc) rc = check_out(q, "q");
  if (!rc) rc = check_out(scales, "scales");
  if (!rc) rc = check_opt(gamma, "gamma");
  if (!rc) rc = check_opt(G_out, "G_out");
  if (rc) return rc;
  if (mode == kModeMXNorm && !(p > 0.0f)) return fail(MXN_ERR_ARG, "p = %g must be > 0", (double)p);
  if (rounding != MXN_ROUND_RNE && rounding != MXN_ROUND_SR)
    return fail(MXN_ERR_ARG, "rounding = %d", rounding);
  if (scale_layout != MXN_SCALES_ROWMAJOR && scale_layout != MXN_SCALES_MMA)
    return fail(MXN_ERR_ARG, "scale_layout = %d", scale_layout);
  if (elem != MXN_ELEM_E4M3 && elem != MXN_ELEM_E2M1 && elem != MXN_ELEM_NVFP4)
    return fail(MXN_ERR_ARG, "elem_format = %d", elem);
  if (elem == MXN_ELEM_NVFP4 && scale_layout != MXN_SCALES_ROWMAJOR)
    return fail(MXN_ERR_UNSUPPORTED, "NVFP4 scales are row-major only");
  if (stat != MXN_STAT_ABSMAX && stat != MXN_STAT_SCALE_EXP) return fail(MXN_ERR_ARG, "statistic = %d", stat);
  if ((rc = injected())) return rc;
  if (T == 0) return MXN_OK;
  FwdArgs A{};
  A.elem = elem == MXN_ELEM_NVFP4 ? kElemNVFP4 : (elem == MXN_ELEM_E2M1 ? kElemE2M1 : kElemE4M3);
  A.stat_exp = stat == MXN_STAT_SCALE_EXP;
  A.x = static_cast<const uint16_t*>(x);
  A.gamma = static_cast<const uint16_t*>(gamma);
  A.q = static_cast<uint8_t*>(q);
  A.scales = static_cast<uint8_t*>(scales);
  A.G_out = G_out;
  A.p = p;
  A.pmode = pmode_of(p);
  A.seed_lo = (uint32_t)seed;
  A.seed_hi = (uint32_t)(seed >> 32);
  A.scale_mma = scale_layout == MXN_SCALES_MMA;
  A.kp4 = (int)(((D / kBlock) + 3) / 4 * 4);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return launch_fwd(mode, rounding == MXN_ROUND_SR, A, T, (int)D, ld_x, s);
}

int mxnorm_fwd(const void* x, const void* gamma, void* q, void* scales, float* G_out, int64_t T,
               int64_t D, int64_t ld_x, float p, int rounding, uint64_t seed, int scale_layout,
               void* stream) {
  return fwd_like(kModeMXNorm, x, gamma, q, scales, G_out, T, D, ld_x, p, rounding, seed,
                  scale_layout, MXN_ELEM_E4M3, MXN_STAT_ABSMAX, stream);
}

int mxnorm_fwd_ex(const void* x, const void* gamma, void* q, void* scales, float* G_out, int64_t T,
                  int64_t D, int64_t ld_x, float p, int rounding, uint64_t seed, int scale_layout,
                  int elem_format, int statistic, void* stream) {
  return fwd_like(kModeMXNorm, x, gamma, q, scales, G_out, T, D, ld_x, p, rounding, seed,
                  scale_layout, elem_format, statistic, stream);
}

int mxfp8_cast(const void* x, void* q, void* scales, int64_t T, int64_t D, int64_t ld_x,
               int rounding, uint64_t seed, int scale_layout, void* stream) {
  return fwd_like(kModeCast, x, nullptr, q, scales, nullptr, T, D, ld_x, 1.0f, rounding, seed,
                  scale_layout, MXN_ELEM_E4M3, MXN_STAT_ABSMAX, stream);
}

int mx_cast_ex(const void* x, const void* gain, void* q, void* scales, int64_t T, int64_t D,
               int64_t ld_x, int rounding, uint64_t seed, int scale_layout, int elem_format,
               void* stream) {
  return fwd_like(kModeCast, x, gain, q, scales, nullptr, T, D, ld_x, 1.0f, rounding, seed,
                  scale_layout, elem_format, MXN_STAT_ABSMAX, stream);
}

int mxnorm_fold_weight(const void* w, const void* gamma, void* q, void* scales, int64_t N,
                       int64_t K, int64_t ld_w, int elem_format, int scale_layout, void* stream) {
  t_err.clear();
  if (!gamma && N != 0) return fail(MXN_ERR_ARG, "gamma is NULL (nothing to fold)");
  return fwd_like(kModeCast, w, gamma, q, scales, nullptr, N, K, ld_w, 1.0f, MXN_ROUND_RNE, 0,
                  scale_layout, elem_format, MXN_STAT_ABSMAX, stream);
}

size_t mxnorm_codes_bytes(int64_t T, int64_t D, int elem_format) {
  if (T < 0 || D <= 0 || D % kBlock != 0) return 0;
  if (elem_format == MXN_ELEM_E4M3) return (size_t)(T * D);
  if (elem_format == MXN_ELEM_E2M1 || elem_format == MXN_ELEM_NVFP4) return (size_t)(T * (D / 2));
  return 0;
}

int rmsnorm_bf16(const void* x, const void* gamma, void* y, int64_t T, int64_t D, int64_t ld_x,
                 float eps, void* stream) {
  t_err.clear();
  int rc = check_common(x, T, D, ld_x);
  if (!rc) rc = check_out(y, "y");
  if (!rc) rc = check_opt(gamma, "gamma");
  if (rc) return rc;
  if (!(eps >= 0.0f)) return fail(MXN_ERR_ARG, "eps = %g must be >= 0", (double)eps);
  if ((rc = injected())) return rc;
  if (T == 0) return MXN_OK;
  FwdArgs A{};
  A.x = static_cast<const uint16_t*>(x);
  A.gamma = static_cast<const uint16_t*>(gamma);
  A.y = static_cast<uint16_t*>(y);
  A.eps = eps;
  return launch_fwd(kModeRMSNorm, false, A, T, (int)D, ld_x, static_cast<cudaStream_t>(stream));
}

int rmsnorm_then_mxcast(const void* x, const void* gamma, float eps, void* y_tmp, void* q,
                        void* scales, int64_t T, int64_t D, int64_t ld_x, int scale_layout,
                        void* stream) {
  // Every argument of both passes is checked before the first launch.
  t_err.clear();
  int rc = check_common(x, T, D, ld_x);
  if (!rc) rc = check_out(y_tmp, "y_tmp");
  if (!rc) rc = check_out(q, "q");
  if (!rc) rc = check_out(scales, "scales");
  if (!rc) rc = check_opt(gamma, "gamma");
  if (rc) return rc;
  if (!(eps >= 0.0f)) return fail(MXN_ERR_ARG, "eps = %g must be >= 0", (double)eps);
  if (scale_layout != MXN_SCALES_ROWMAJOR && scale_layout != MXN_SCALES_MMA)
    return fail(MXN_ERR_ARG, "scale_layout = %d", scale_layout);
  rc = rmsnorm_bf16(x, gamma, y_tmp, T, D, ld_x, eps, stream);
  if (rc) return rc;
  return mxfp8_cast(y_tmp, q, scales, T, D, D, MXN_ROUND_RNE, 0, scale_layout, stream);
}

size_t mxnorm_bwd_workspace_size(int64_t T, int64_t D) {
  if (T <= 0 || D <= 0 || D % kBlock != 0 || D > kMaxBwdD) return 0;
  DeviceInfo dev;
  if (device_info(&dev)) return 0;
  BwdPlan P;
  if (plan_bwd(T, (int)D, dev.sms, &P)) return 0;
  return P.partial_rows() * (size_t)D * sizeof(float);
}

int mxnorm_bwd(const void* x, const void* dy, const void* gamma, const float* G, void* dx,
               void* dgamma, int64_t T, int64_t D, void* workspace, size_t workspace_bytes,
               void* stream) {
  t_err.clear();
  int rc = check_common(x, T, D, D);
  if (!rc) rc = check_out(dy, "dy");
  if (!rc) rc = check_out(G, "G");
  if (!rc) rc = check_out(dx, "dx");
  if (!rc) rc = check_opt(gamma, "gamma");
  if (!rc) rc = check_opt(dgamma, "dgamma");
  if (rc) return rc;
  if (D > kMaxBwdD) return fail(MXN_ERR_UNSUPPORTED, "mxnorm_bwd: D = %lld > %d", (long long)D, kMaxBwdD);
  if (dgamma && !gamma) return fail(MXN_ERR_ARG, "dgamma requested without gamma");
  if ((rc = injected())) return rc;
  if (T == 0) return MXN_OK;
  DeviceInfo dev;
  if ((rc = device_info(&dev))) return rc;
  BwdPlan P;
  if ((rc = plan_bwd(T, (int)D, dev.sms, &P))) return rc;
  const size_t need = P.partial_rows() * (size_t)D * sizeof(float);
  if (dgamma) {
    if (!workspace || !aligned16(workspace))
      return fail(MXN_ERR_ARG, "workspace is NULL or not 16-byte aligned");
    if (workspace_bytes < need)
      return fail(MXN_ERR_ARG, "workspace of %zu bytes, %zu needed", workspace_bytes, need);
  }
  BwdArgs A{};
  A.x = static_cast<const uint16_t*>(x);
  A.dy = static_cast<const uint16_t*>(dy);
  A.gamma = static_cast<const uint16_t*>(gamma);
  A.G = G;
  A.dx = static_cast<uint16_t*>(dx);
  A.partial = dgamma ? static_cast<float*>(workspace) : nullptr;
  A.status = dev.status;
  return launch_bwd(P, A, static_cast<uint16_t*>(dgamma), static_cast<cudaStream_t>(stream));
}

int mxnorm_bwd_noalloc(const void* x, const void* dy, const void* gamma, const float* G,
                       void* dx, void* dgamma, int64_t T, int64_t D, void* stream) {
  t_err.clear();
  int rc = check_common(x, T, D, D);
  if (!rc) rc = check_out(dy, "dy");
  if (!rc) rc = check_out(G, "G");
  if (!rc) rc = check_out(dx, "dx");
  if (!rc) rc = check_opt(gamma, "gamma");
  if (!rc) rc = check_opt(dgamma, "dgamma");
  if (rc) return rc;
  if (D > kMaxBwdD) return fail(MXN_ERR_UNSUPPORTED, "mxnorm_bwd_noalloc: D = %lld > %d", (long long)D, kMaxBwdD);
  if (dgamma && !gamma) return fail(MXN_ERR_ARG, "dgamma requested without gamma");
  if ((rc = injected())) return rc;
  if (T == 0) return MXN_OK;
  DeviceInfo dev;
  if ((rc = device_info(&dev))) return rc;
  // Each CTA writes one partial row of D floats: plan no more CTAs than the
  // scratch holds rows (the kernel is persistent, so fewer CTAs cover all
  // rows).
  BwdPlan P;
  if ((rc = plan_bwd(T, (int)D, dev.sms, &P, dgamma ? (int64_t)(kNoAllocScratchFloats / (size_t)D) : 0)))
    return rc;
  float* scratch = nullptr;
  if (dgamma && (rc = noalloc_scratch(&scratch))) return rc;
  BwdArgs A{};
  A.x = static_cast<const uint16_t*>(x);
  A.dy = static_cast<const uint16_t*>(dy);
  A.gamma = static_cast<const uint16_t*>(gamma);
  A.G = G;
  A.dx = static_cast<uint16_t*>(dx);
  A.partial = scratch;
  A.status = dev.status;
  return launch_bwd(P, A, static_cast<uint16_t*>(dgamma), static_cast<cudaStream_t>(stream));
}

int mxfp8_gemm(const void* a_q, const void* a_s, const void* b_q, const void* b_s, void* c, int64_t M,
               int64_t N, int64_t K, void* stream) {
  t_err.clear();
  if (M < 0 || N < 0 || K < 0) return fail(MXN_ERR_ARG, "negative GEMM shape");
  if (M == 0 || N == 0) return MXN_OK;
  if (K == 0) return fail(MXN_ERR_UNSUPPORTED, "mxfp8_gemm: K = 0");
  t_empty = false;  // every operand pointer is required from here on
  const void* ptrs[5] = {a_q, a_s, b_q, b_s, c};
  const char* names[5] = {"a_q", "a_s", "b_q", "b_s", "c"};
  for (int i = 0; i < 5; ++i) {
    int rc = check_out(ptrs[i], names[i]);
    if (rc) return rc;
  }
  if (M % gemm_mxfp8_tile_m() || N % gemm_mxfp8_tile_n() || K % gemm_mxfp8_tile_k())
    return fail(MXN_ERR_UNSUPPORTED, "mxfp8_gemm: M %% %d, N %% %d and K %% %d must be 0 (M=%lld N=%lld K=%lld)",
                gemm_mxfp8_tile_m(), gemm_mxfp8_tile_n(), gemm_mxfp8_tile_k(), (long long)M, (long long)N,
                (long long)K);
  if (M > (1 << 30) || N > (1 << 30) || K > (1 << 30)) return fail(MXN_ERR_UNSUPPORTED, "mxfp8_gemm: shape too large");
  int rc = injected();
  if (rc) return rc;
  DeviceInfo dev;
  if ((rc = device_info(&dev))) return rc;
  const char* why = "";
  const int e = gemm_mxfp8_launch(a_q, a_s, b_q, b_s, c, (int)M, (int)N, (int)K, dev.sms, dev.status,
                                  static_cast<cudaStream_t>(stream), &why);
  if (e) return fail(MXN_ERR_CUDA, "mxfp8_gemm: %s", why);
  return MXN_OK;
}

int mxnorm_debug_wait_timeout(uint64_t limit_ns, int* gave_up, void* stream) {
  t_err.clear();
  t_empty = false;
  int rc = check_out(gave_up, "gave_up");
  if (rc) return rc;
  if (limit_ns == 0 || limit_ns > 2000000000ull) return fail(MXN_ERR_ARG, "limit_ns = %llu", (unsigned long long)limit_ns);
  DeviceInfo dev;
  if ((rc = device_info(&dev))) return rc;
  wait_timeout_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, dev.status, gave_up);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "wait_timeout_probe_kernel launch");
  return MXN_OK;
}

const char* mxnorm_last_error(void) { return t_err.c_str(); }

int mxnorm_device_status(void* stream) {
  t_err.clear();
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned v = 0;
  e = cudaMemcpyFromSymbol(&v, g_mxn_status, sizeof v);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol(status)");
  if (v) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_mxn_status, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyToSymbol(status)");
    return fail(MXN_ERR_TIMEOUT, "a kernel gave up a bounded wait (status 0x%x)", v);
  }
  return MXN_OK;
}

int mxnorm_set_tuning(int consumer_threads, int stages, int ctas_per_sm) {
  t_err.clear();
  if (consumer_threads != 0 && (consumer_threads < 32 || consumer_threads > 512 || consumer_threads % 32))
    return fail(MXN_ERR_ARG, "consumer_threads = %d", consumer_threads);
  if (stages != 0 && (stages < 1 || stages > 16)) return fail(MXN_ERR_ARG, "stages = %d", stages);
  if (ctas_per_sm < 0 || ctas_per_sm > 8) return fail(MXN_ERR_ARG, "ctas_per_sm = %d", ctas_per_sm);
  g_tuning.consumer_threads = consumer_threads;
  g_tuning.stages = stages;
  g_tuning.ctas_per_sm = ctas_per_sm;
  return MXN_OK;
}

int mxnorm_set_gemm_tiles(int mode) {
  t_err.clear();
  if (mode < 0 || mode > 2) return fail(MXN_ERR_ARG, "gemm tile mode = %d", mode);
  gemm_mxfp8_set_tiles(mode);
  return MXN_OK;
}

void mxnorm_debug_fail_next(int count) { t_fail_next = count > 0 ? count : 0; }

}  // extern "C"
