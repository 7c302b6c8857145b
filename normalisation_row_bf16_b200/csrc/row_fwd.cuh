// row_fwd.cuh -- the single-input row kernels: MXNorm forward, MXCast and the
// RMSNorm pass of the two-pass comparator.
//
// MXNorm (gist.science, "MXNorm: Reusing MXFP block scales for efficient
// tensor normalisation", technical summary section 2.1) reads each row once:
// block absmax m_k -> generalised p-mean G -> y = x / G (* gamma) -> E8M0
// scale per block -> E4M3 codes.  The pages' own kernel ran through
// torch.compile on GB200 (section 3.2); this one is written for B200:
//
//  * persistent CTAs (grid = SMs x resident CTAs), each owning a strided set
//    of "row blocks" (rps consecutive rows);
//  * one producer thread streams whole rows into a ring of shared-memory
//    stages with 1-D bulk copies on the TMA engine (cp.async.bulk, no
//    multicast, L2 evict-first), so the bytes in flight do not depend on
//    register-file occupancy;
//  * consumer threads own one 32-element MX block each (bpt blocks when the
//    row has more than 512 blocks), so the block absmax, scale and cast are
//    thread-local; the row statistic is a K-input reduction (warp shuffles,
//    then one named barrier across the row's warps): K = D/32 inputs, the
//    32x smaller reduction the lay summary (section 3) points at;
//  * a thread reads its 64 bytes as four 16-byte chunks in a rotated order
//    (chunk (j + k/2) mod 4 at step j) so that the eight threads of a
//    shared-memory phase hit eight distinct 16-byte bank groups;
//  * each stage is released (mbarrier arrive) as soon as its data sit in
//    registers, before the arithmetic, so the next copy overlaps it.
#pragma once

#include "device_common.cuh"

namespace mxn {

enum RowMode { kModeMXNorm = 0, kModeCast = 1, kModeRMSNorm = 2 };
enum PMode { kP1 = 1, kP2 = 2, kP4 = 4, kPInf = 0, kPGeneral = 3 };

constexpr int kMaxConsumerThreads = 512;
constexpr int kRedSlots = 16;  // warps per row, at most

// Resident CTAs per SM the register budget is sized for, by consumer threads
// per CTA (each CTA adds one producer warp).
template <int NCT>
struct CtaShape {
  static constexpr int threads = NCT + 32;
  static constexpr int min_blocks = NCT <= 128 ? 4 : (NCT <= 256 ? 2 : 1);
};

struct RowCfg {
  int64_t T;             // rows
  int64_t ld_x;          // row stride of the input, elements
  int64_t n_row_blocks;  // ceil(T / rps)
  int D, K;              // row length, blocks per row
  int tpr, log2_tpr;     // consumer threads per row (power of two)
  int rps;               // rows per stage
  int stages;            // pipeline depth
  int n_cwarps;          // consumer warps
  uint32_t row_bytes;    // 2 * D
  uint32_t stage_bytes;  // rps * row_bytes
};

struct FwdArgs {
  const uint16_t* x;      // bf16 [T, ld_x]
  const uint16_t* gamma;  // bf16 [D] or null
  uint8_t* q;             // E4M3 [T, D]            (MXNorm, Cast)
  uint8_t* scales;        // E8M0                    (MXNorm, Cast)
  float* G_out;           // fp32 [T] or null        (MXNorm)
  uint16_t* y;            // bf16 [T, D]             (RMSNorm)
  unsigned* status;       // device status word
  float p, inv_p, eps;
  int pmode;
  int sr;
  uint32_t seed_lo, seed_hi;
  int scale_mma;          // scales in the tcgen05 128x4 layout
  int kp4;                // K rounded up to a multiple of 4 (MMA layout)
};

// Byte offset of scale (row, k) in the tcgen05 block-scale layout.
__device__ __forceinline__ int64_t mma_scale_offset(int64_t row, int k, int kp4) {
  return ((row >> 7) * (kp4 >> 2) + (k >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 +
         (k & 3);
}

// 2^n for integer n <= 0; 0 below the normal range (those terms are < 2^-126
// of the row's largest term and do not register in an fp32 sum).
__device__ __forceinline__ float exp2_int_or_zero(int n) { return n < -126 ? 0.0f : exp2_int(n); }

__device__ __forceinline__ float pow_p(float r, int pmode, float p) {
  switch (pmode) {
    case kP1: return r;
    case kP2: return r * r;
    case kP4: { const float s = r * r; return s * s; }
    default: return powf(r, p);
  }
}

// Factor 2^(p * d) that rescales a partial sum taken relative to 2^(E + d) to
// one taken relative to 2^E (d <= 0).
__device__ __forceinline__ float rescale_factor(int d, int pmode, float p) {
  switch (pmode) {
    case kP1: return exp2_int_or_zero(d);
    case kP2: return exp2_int_or_zero(2 * d);
    case kP4: return exp2_int_or_zero(4 * d);
    default: return exp2f(p * (float)d);
  }
}

// Unbiased exponent used to normalise the terms: that of M, at least -126.
__device__ __forceinline__ int norm_exponent(float M) {
  return max((int)((__float_as_uint(M) >> 23) & 0xFF) - 127, -126);
}

// 2^-E for E in [-126, 127] (2^-127 is an fp32 subnormal, still exact).
__device__ __forceinline__ float inv_pow2(int E) {
  return E == 127 ? __uint_as_float(0x00400000u) : exp2_int(-E);
}

template <typename T>
__device__ __forceinline__ T seg_max_u32(T v, int width) {
  for (int off = width >> 1; off > 0; off >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
  return v;
}
__device__ __forceinline__ float seg_sum(float v, int width) {
  for (int off = width >> 1; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
  return v;
}

// The row statistic G from this thread's block maxima (bf16 magnitude bits).
// Warp partials are taken relative to the warp maximum's power of two, so no
// term overflows or underflows; partials of different warps are combined by
// exact power-of-two factors (integer p) after one named barrier.
template <int BPT>
__device__ __forceinline__ float row_pmean(const uint32_t (&mb)[BPT], const FwdArgs& A,
                                           const RowCfg& C, float2* red, int grp, int tg,
                                           int lane, int par) {
  uint32_t mloc = 0;
#pragma unroll
  for (int b = 0; b < BPT; ++b) mloc = max(mloc, mb[b]);
  const int W = C.tpr < 32 ? C.tpr : 32;
  mloc = seg_max_u32(mloc, W);
  const float Mw = bf16bits_to_float(mloc);
  float sw = 0.0f;
  if (A.pmode != kPInf) {
    const float inv = inv_pow2(norm_exponent(Mw));
#pragma unroll
    for (int b = 0; b < BPT; ++b) sw += pow_p(bf16bits_to_float(mb[b]) * inv, A.pmode, A.p);
    sw = seg_sum(sw, W);
  }
  float M = Mw, S = sw;
  int E = norm_exponent(Mw);
  if (C.tpr > 32) {
    const int nw = C.tpr >> 5;
    float2* slot = red + (par * C.rps + grp) * kRedSlots;
    if (lane == 0) slot[tg >> 5] = make_float2(Mw, sw);
    named_barrier_sync(1 + grp, C.tpr);
    uint32_t mb_all = 0;
    for (int w = 0; w < nw; ++w) mb_all = max(mb_all, __float_as_uint(slot[w].x));
    M = __uint_as_float(mb_all);
    E = norm_exponent(M);
    S = 0.0f;
    if (A.pmode != kPInf)
      for (int w = 0; w < nw; ++w) {
        const float2 v = slot[w];
        S += v.y * rescale_factor(norm_exponent(v.x) - E, A.pmode, A.p);
      }
  }
  if (__float_as_uint(M) >= 0x7F800000u || A.pmode == kPInf) return M;  // inf / NaN / p = inf
  const float r = S / (float)C.K;
  float root;
  switch (A.pmode) {
    case kP1: root = r; break;
    case kP2: root = sqrtf(r); break;
    case kP4: root = sqrtf(sqrtf(r)); break;
    default: root = powf(r, A.inv_p); break;
  }
  return root * exp2_int(E);
}

__device__ __forceinline__ float row_sum(float v, const RowCfg& C, float2* red, int grp, int tg,
                                         int lane, int par) {
  const int W = C.tpr < 32 ? C.tpr : 32;
  v = seg_sum(v, W);
  if (C.tpr > 32) {
    const int nw = C.tpr >> 5;
    float2* slot = red + (par * C.rps + grp) * kRedSlots;
    if (lane == 0) slot[tg >> 5] = make_float2(v, 0.0f);
    named_barrier_sync(1 + grp, C.tpr);
    v = 0.0f;
    for (int w = 0; w < nw; ++w) v += slot[w].x;
  }
  return v;
}

// Producer: one thread streams row blocks into the stage ring.
__device__ __forceinline__ void produce_rows(const uint16_t* x, const RowCfg& C, uint8_t* stage0,
                                             uint64_t* full, uint64_t* empty, unsigned* status) {
  const uint64_t pol = policy_evict_first();
  int64_t it = 0;
  for (int64_t rb = blockIdx.x; rb < C.n_row_blocks; rb += gridDim.x, ++it) {
    const int s = (int)(it % C.stages);
    const uint32_t ph = (uint32_t)((it / C.stages) & 1);
    if (!mbar_wait_bounded(&empty[s], ph ^ 1u, status)) break;
    const int64_t r0 = rb * C.rps;
    const int nrows = (int)(C.T - r0 < (int64_t)C.rps ? C.T - r0 : (int64_t)C.rps);
    mbar_arrive_expect_tx(&full[s], (uint32_t)nrows * C.row_bytes);
    uint8_t* dst = stage0 + (size_t)s * C.stage_bytes;
    for (int r = 0; r < nrows; ++r)
      bulk_copy_g2s(dst + (size_t)r * C.row_bytes, x + (r0 + r) * C.ld_x, C.row_bytes, &full[s], pol);
  }
  // Leave no copy in flight: wait for the last issued phase of every stage.
  for (int64_t j = (it > C.stages ? it - C.stages : (int64_t)0); j < it; ++j)
    mbar_wait_bounded(&full[j % C.stages], (uint32_t)((j / C.stages) & 1), status);
}

template <int MODE, int BPT, int NCT, bool SR>
__global__ void __launch_bounds__(CtaShape<NCT>::threads, CtaShape<NCT>::min_blocks)
    row_fwd_kernel(const FwdArgs A, const RowCfg C) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* stage0 = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)C.stages * C.stage_bytes);
  uint64_t* empty = full + C.stages;
  float2* red = reinterpret_cast<float2*>(empty + C.stages);

  const int tid = threadIdx.x;
  constexpr int ncons = NCT;
  if (tid == 0) {
    for (int s = 0; s < C.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C.n_cwarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (tid >= ncons) {
    if (tid == ncons) produce_rows(A.x, C, stage0, full, empty, A.status);
    return;
  }

  const int lane = tid & 31;
  const int grp = tid >> C.log2_tpr;
  const int tg = tid & (C.tpr - 1);
  const bool has_gamma = (MODE != kModeCast) && (A.gamma != nullptr);

  // gamma for this thread's blocks, in the same rotated chunk order as x.
  uint32_t gw[BPT][16];
#pragma unroll
  for (int b = 0; b < BPT; ++b) {
    const int k = tg + b * C.tpr;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint4 v = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);  // 1.0
      if (has_gamma && k < C.K) {
        const int c = (j + (k >> 1)) & 3;
        v = ldg128_nc(A.gamma + (size_t)k * kBlock + c * 8);
      }
      gw[b][4 * j] = v.x; gw[b][4 * j + 1] = v.y; gw[b][4 * j + 2] = v.z; gw[b][4 * j + 3] = v.w;
    }
  }

  // A wait that gives up marks the kernel failed; the thread then keeps
  // running (without waiting again) so that every named barrier of its row
  // still completes, and its outputs are garbage but in bounds.
  bool ok = true;
  int par = 0;
  int64_t it = 0;
  for (int64_t rb = blockIdx.x; rb < C.n_row_blocks; rb += gridDim.x, ++it, par ^= 1) {
    const int s = (int)(it % C.stages);
    const uint32_t ph = (uint32_t)((it / C.stages) & 1);
    if (ok) ok = mbar_wait_bounded(&full[s], ph, A.status);

    const int64_t row = rb * C.rps + grp;
    const bool valid = row < C.T;
    const uint32_t srow = smem_u32(stage0 + (size_t)s * C.stage_bytes + (size_t)grp * C.row_bytes);

    uint32_t xw[BPT][16];
#pragma unroll
    for (int b = 0; b < BPT; ++b) {
      const int k = tg + b * C.tpr;
      const bool have = valid && k < C.K;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (have) v = lds128(srow + (uint32_t)k * 64u + (uint32_t)(((j + (k >> 1)) & 3) * 16));
        xw[b][4 * j] = v.x; xw[b][4 * j + 1] = v.y; xw[b][4 * j + 2] = v.z; xw[b][4 * j + 3] = v.w;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);

    if constexpr (MODE == kModeRMSNorm) {
      // ---------------------------------------------------------- RMSNorm
      float ss = 0.0f;
#pragma unroll
      for (int b = 0; b < BPT; ++b)
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float x0 = bf16lo(xw[b][j]), x1 = bf16hi(xw[b][j]);
          ss = fmaf(x0, x0, ss);
          ss = fmaf(x1, x1, ss);
        }
      ss = row_sum(ss, C, red, grp, tg, lane, par);
      const float rinv = 1.0f / sqrtf(ss / (float)C.D + A.eps);
#pragma unroll
      for (int b = 0; b < BPT; ++b) {
        const int k = tg + b * C.tpr;
        if (!valid || k >= C.K) continue;
        const int rot = (k >> 1) & 3;
        uint16_t* yrow = A.y + row * (int64_t)C.D + (int64_t)k * kBlock;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t w = xw[b][4 * j + i], g = gw[b][4 * j + i];
            float y0 = __fmul_rn(bf16lo(w), rinv), y1 = __fmul_rn(bf16hi(w), rinv);
            if (has_gamma) { y0 = __fmul_rn(y0, bf16lo(g)); y1 = __fmul_rn(y1, bf16hi(g)); }
            const __nv_bfloat162 h = __floats2bfloat162_rn(y0, y1);
            o[i] = *reinterpret_cast<const uint32_t*>(&h);
          }
          stg128_stream(yrow + ((j + rot) & 3) * 8, make_uint4(o[0], o[1], o[2], o[3]));
        }
      }
    } else {
      // ------------------------------------------------- MXNorm / MXCast
      uint32_t mb[BPT];
#pragma unroll
      for (int b = 0; b < BPT; ++b) mb[b] = absmax_bits_bf16x2(xw[b], 16);
      float sc = 1.0f, G = 0.0f;
      if constexpr (MODE == kModeMXNorm) {
        G = row_pmean<BPT>(mb, A, C, red, grp, tg, lane, par);
        sc = (G == 0.0f) ? 0.0f : __frcp_rn(G);
        if (valid && tg == 0 && A.G_out) A.G_out[row] = G;
      }
#pragma unroll
      for (int b = 0; b < BPT; ++b) {
        const int k = tg + b * C.tpr;
        if (!valid || k >= C.K) continue;
        const int rot = (k >> 1) & 3;
        float y[32];
        float a;
        if (MODE == kModeMXNorm && has_gamma) {
          a = 0.0f;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            y[2 * j] = __fmul_rn(__fmul_rn(bf16lo(xw[b][j]), sc), bf16lo(gw[b][j]));
            y[2 * j + 1] = __fmul_rn(__fmul_rn(bf16hi(xw[b][j]), sc), bf16hi(gw[b][j]));
            a = max_abs_nan(a, y[2 * j]);
            a = max_abs_nan(a, y[2 * j + 1]);
          }
        } else if (MODE == kModeMXNorm) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            y[2 * j] = __fmul_rn(bf16lo(xw[b][j]), sc);
            y[2 * j + 1] = __fmul_rn(bf16hi(xw[b][j]), sc);
          }
          a = __fmul_rn(bf16bits_to_float(mb[b]), sc);  // rounding is monotone
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            y[2 * j] = bf16lo(xw[b][j]);
            y[2 * j + 1] = bf16hi(xw[b][j]);
          }
          a = bf16bits_to_float(mb[b]);
        }
        const int e = e8m0_exponent_bits(__float_as_uint(a) & 0x7FFFFFFFu);  // a >= 0 or NaN
        uint32_t qw[8];
        uint8_t code;
        if (e == 128) {
          code = 0xFF;
#pragma unroll
          for (int i = 0; i < 8; ++i) qw[i] = 0x7F7F7F7Fu;
        } else {
          code = (uint8_t)(e + 127);
          const float inv = exp2_int(-e);
          if constexpr (!SR) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const uint32_t lo = cvt_e4m3x2_rn(__fmul_rn(y[4 * i], inv), __fmul_rn(y[4 * i + 1], inv));
              const uint32_t hi = cvt_e4m3x2_rn(__fmul_rn(y[4 * i + 2], inv), __fmul_rn(y[4 * i + 3], inv));
              qw[i] = lo | (hi << 16);
            }
          } else {
#pragma unroll
            for (int sl = 0; sl < 4; ++sl) {
              const int c = (sl + rot) & 3;  // chunk held in slot sl
              const uint64_t ctr = (uint64_t)(row * (int64_t)C.D + (int64_t)k * kBlock + c * 8) >> 2;
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const uint64_t cc = ctr + h;
                const uint4 r = philox4x32_10(make_uint4((uint32_t)cc, (uint32_t)(cc >> 32), 0u, 0u),
                                              A.seed_lo, A.seed_hi);
                const int i0 = sl * 8 + h * 4;
                const float v0 = sr_e4m3_grid(__fmul_rn(y[i0], inv), r.x);
                const float v1 = sr_e4m3_grid(__fmul_rn(y[i0 + 1], inv), r.y);
                const float v2 = sr_e4m3_grid(__fmul_rn(y[i0 + 2], inv), r.z);
                const float v3 = sr_e4m3_grid(__fmul_rn(y[i0 + 3], inv), r.w);
                qw[sl * 2 + h] = cvt_e4m3x2_rn(v0, v1) | (cvt_e4m3x2_rn(v2, v3) << 16);
              }
            }
          }
        }
        // Slot sl holds chunk (sl + rot) & 3; put chunk c at word pair 2c.
        // Two select stages rotate by (rot & 1) and then by (rot & 2) slots.
        uint32_t o[8];
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int h = 0; h < 2; ++h) o[2 * c + h] = (rot & 1) ? qw[2 * ((c + 3) & 3) + h] : qw[2 * c + h];
        uint32_t o2[8];
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int h = 0; h < 2; ++h) o2[2 * c + h] = (rot & 2) ? o[2 * ((c + 2) & 3) + h] : o[2 * c + h];
        uint8_t* qp = A.q + row * (int64_t)C.D + (int64_t)k * kBlock;
        stg128_stream(qp, make_uint4(o2[0], o2[1], o2[2], o2[3]));
        stg128_stream(qp + 16, make_uint4(o2[4], o2[5], o2[6], o2[7]));
        if (A.scale_mma) A.scales[mma_scale_offset(row, k, A.kp4)] = code;
        else A.scales[row * (int64_t)C.K + k] = code;
      }
    }
  }
}

}  // namespace mxn
