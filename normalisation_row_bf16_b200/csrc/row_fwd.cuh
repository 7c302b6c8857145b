// row_fwd.cuh -- the forward row kernels: MXNorm forward, MXCast and the
// RMSNorm pass of the two-pass comparator.
//
// MXNorm (gist.science, "MXNorm: Reusing MXFP block scales for efficient
// tensor normalisation", technical summary section 2.1) reads each row once:
// block absmax m_k -> generalised p-mean G -> y = x / G (* gamma) -> E8M0
// scale per block -> E4M3 codes.  The pages ran theirs through torch.compile
// on GB200 (section 3.2); this one is laid out for B200:
//
//  * A "row group" of tpr threads owns one row at a time (tpr = 32 up to
//    D = 4096, i.e. one warp per row; more warps per row beyond that; several
//    rows per warp below D = 1024).  Each thread owns BPT of the row's 32-element
//    MX blocks (k = tg + b * tpr), so the block absmax, scale and cast are
//    thread-local and the row statistic reduces K = D/32 numbers -- with warp
//    shuffles only when the row fits one warp (the lay summary's "32x less
//    reduction work", section 3).
//  * Each row group owns a ring of `stages` shared-memory row buffers filled by
//    1-D bulk copies (cp.async.bulk on the TMA engine, L2 evict-first, no
//    multicast) that its first thread issues, completing on the group's own
//    mbarriers: no group ever waits for another, and the bytes in flight do not
//    depend on register occupancy.
//  * A thread copies its blocks from the stage into registers and hands the
//    stage back after the block maxima (which use every register it read:
//    the reads are then complete) behind a proxy fence ordering its
//    shared-memory reads before the refill's bulk copy; the refill (row block
//    rb + stages * ngt) is issued before the rest of the row's arithmetic, so
//    each group keeps `stages` rows of compute as look-ahead whatever the
//    occupancy.  A thread reads its 64-byte block
//    as four 16-byte chunks in the order (j + k/2) mod 4, which puts the eight
//    threads of a shared-memory phase on eight distinct bank groups.
//  * gamma is converted once per CTA into shared memory in "slot order": the
//    16 bytes that match x chunk slot j of block k sit at (j * K + k) * 16, so
//    consecutive threads read consecutive 16-byte words.
//  * fp32 products run as packed f32x2 multiplies (two IEEE-rounded products
//    per instruction), the per-block maxima as 3-input max and bf16x2 max.
#pragma once

#include "device_common.cuh"

namespace mxn {

enum RowMode { kModeMXNorm = 0, kModeCast = 1, kModeRMSNorm = 2 };
// Element formats of the codes: E4M3 (MXFP8, a byte per code), E2M1 (MXFP4,
// two codes per byte, the even column in the low nibble), and NVFP4 (E2M1
// codes packed the same way, one E4M3 scale per 16 elements).
enum ElemFormat { kElemE4M3 = 0, kElemE2M1 = 1, kElemNVFP4 = 2 };
enum PMode { kP1 = 1, kP2 = 2, kP4 = 4, kPInf = 0, kPGeneral = 3 };

// Threads per CTA the register budget is sized for: a thread holding 4 blocks
// of its row needs ~120 registers (512 threads), 2 blocks ~96 (640), 1 block
// fits in 80 (768).
__host__ __device__ constexpr int fwd_max_threads(int bpt) { return bpt >= 4 ? 512 : (bpt == 2 ? 640 : 768); }
// Threads per CTA a kernel is compiled for (its __launch_bounds__).  One-warp
// rows of 65..128 blocks of E4M3 codes with nearest-even rounding launch 384
// threads, and are compiled for 384: up to 168 registers a thread.
// Stochastic rounding with two blocks a thread launches 512 (up to 128
// registers: the Philox rounds keep more in flight; measured on B200 at
// 8192 x 4096: 51.9 -> 50.0 us against 640, and 56.0 at 384).
__host__ __device__ constexpr int fwd_launch_threads(int bpt, int tpr, bool sr, int elem) {
  return (bpt >= 4 && tpr == 32 && !sr && elem == 0) ? 384 : ((sr && bpt == 2) ? 512 : fwd_max_threads(bpt));
}
constexpr int kRedSlots = 16;  // warps per row group, at most

struct FwdCfg {
  int64_t T;             // rows
  int64_t ld_x;          // row stride of x, elements
  int64_t n_row_blocks;  // ceil(T / rps)
  int64_t ngt;           // row groups that get rows (<= groups in the grid)
  int D, K;              // row length, MX blocks per row
  int tpr, log2_tpr;     // threads per row (power of two)
  int rps;               // rows per row group and stage (> 1 only when tpr < 32)
  int gthreads;          // threads per row group = max(tpr, 32)
  int ng;                // row groups per CTA
  int stages;            // ring depth per group
  uint32_t row_bytes;    // 2 * D
  uint32_t stage_bytes;  // rps * row_bytes
  uint32_t gamma_bytes;  // shared-memory gamma (0 when unused)
  uint32_t ring_off, bar_off, red_off;
  uint32_t code_row_bytes;  // code bytes per row (D for E4M3, D / 2 for E2M1 / NVFP4)
  uint32_t ostage_bytes;    // per-group code staging buffer (rps rows); 0: codes stored directly
  uint32_t out_off;         // offset of the staging buffers
  uint32_t rcp_off;         // NVFP4: offset of the 128-entry reciprocal table
};

struct FwdArgs {
  const uint16_t* x;      // bf16 [T, ld_x]
  const uint16_t* gamma;  // bf16 [D] or null
  uint8_t* q;             // E4M3 [T, D]            (MXNorm, Cast)
  uint8_t* scales;        // E8M0                    (MXNorm, Cast)
  float* G_out;           // fp32 [T] or null        (MXNorm)
  uint16_t* y;            // bf16 [T, D]             (RMSNorm)
  unsigned* status;       // device status word
  float p, eps;
  int n_stat;             // statistic terms per row (K; D / 16 for NVFP4)
  double inv_n_stat;      // 1 / n_stat, correctly rounded (host)
  float inv_k_pow2;       // 1 / n_stat when n_stat is a power of two, else 0
  int pmode;
  uint32_t seed_lo, seed_hi;
  int scale_mma;          // scales in the tcgen05 128x4 layout
  int kp4;                // K rounded up to a multiple of 4 (MMA layout)
  int elem;               // element format (kElemE4M3 / kElemE2M1; the kernel's template)
  int stat_exp;           // MXNorm statistic from the blocks' power-of-two scales
};

// Byte offset of scale (row, k) in the tcgen05 block-scale layout.
__device__ __forceinline__ int64_t mma_scale_offset(int64_t row, int k, int kp4) {
  return ((row >> 7) * (kp4 >> 2) + (k >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 +
         (k & 3);
}

// Unbiased exponent used to normalise the terms: that of M, at least -126.
__device__ __forceinline__ int norm_exponent(float M) {
  return max((int)((__float_as_uint(M) >> 23) & 0xFF) - 127, -126);
}

// 2^-E for E in [-126, 127] (2^-127 is an fp32 subnormal, still exact).
__device__ __forceinline__ float inv_pow2(int E) {
  return E == 127 ? __uint_as_float(0x00400000u) : exp2_int(-E);
}

__device__ __forceinline__ uint32_t seg_max(uint32_t v, int width) {
  for (int off = width >> 1; off > 0; off >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
  return v;
}
__device__ __forceinline__ float seg_sum(float v, int width) {
  for (int off = width >> 1; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
  return v;
}

__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
  uint32_t r;
  asm("redux.sync.max.u32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(v));
  return r;
}

// 2^n as a double for an integer n >= -1022 (0 below).
__device__ __forceinline__ double exp2_int_f64(int n) {
  return n < -1022 ? 0.0 : __longlong_as_double((long long)(n + 1023) << 52);
}

__device__ __forceinline__ double seg_sum_f64(double v, int width) {
  for (int off = width >> 1; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
  return v;
}

// Exact p-mean sums for p = 1, 2 in fp32 pairs.  A term t = (m / 2^Ew)^p has
// at most 16 significant bits and lies in [0, 4).  It splits exactly into hi,
// t rounded to a multiple of 2^-g (adding and subtracting 1.5 * 2^(23 - g)),
// and lo = t - hi, |lo| <= 2^-(g+1), with g = 13.  A warp adds at most 256
// terms: the hi parts are multiples of 2^-13 below 2^10 (23 bits), and the lo
// parts (below 2^-6 in all) stay exact while every term keeps its bits above
// 2^-29 -- for p = 2 while no nonzero block maximum is below 2^-7 of the warp
// maximum's power of two, for p = 1 below 2^-22.  The split flags a term
// outside that range (one unsigned compare on the bf16 bits); a warp holding
// one sums its terms in double instead (exact in double), a rare path.  Two
// fp32 shuffle sums then carry the exact total as hi + lo.
constexpr float kSplitMagic = 1536.0f;   // 1.5 * 2^10: rounds to multiples of 2^-13

__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;"
      : "=l"(d)
      : "l"(*reinterpret_cast<const uint64_t*>(&a)), "l"(*reinterpret_cast<const uint64_t*>(&b)));
  return *reinterpret_cast<const float2*>(&d);
}

template <int BPT>
__device__ __forceinline__ float2 pmean_split_sum(const uint32_t (&mb)[BPT], float inv, int pmode,
                                                  uint32_t tiny1, bool& inexact) {
  // r = m * inv is exact (a power-of-two scaling into [0, 2)); t = r^2 (p = 2)
  // or r * 1 (p = 1), which each fma forms exactly before its one rounding.
  // Two terms per packed f32x2 instruction; (hi, lo) sums kept per lane of
  // the pair, whose two hi (two lo) sums add exactly at the end.
  const float2 inv2 = make_float2(inv, inv), mg = make_float2(kSplitMagic, kSplitMagic);
  float2 hs = make_float2(0.0f, 0.0f), ls = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int b = 0; b < BPT; b += 2) {
    const float m0 = bf16bits_to_float(mb[b]), m1 = b + 1 < BPT ? bf16bits_to_float(mb[b + 1]) : 0.0f;
    const float2 r = mul2(make_float2(m0, m1), inv2);
    const float2 f = pmode == kP1 ? make_float2(1.0f, 1.0f) : r;
    const float2 hi = add2(fma2(r, f, mg), make_float2(-kSplitMagic, -kSplitMagic));
    hs = add2(hs, hi);
    ls = add2(ls, fma2(r, f, make_float2(-hi.x, -hi.y)));
  }
  // 0 < m < the range's lower bound, on the bits: (m - 1) < (bound - 1)
  // unsigned; zero maxima wrap to the top and never count
  uint32_t lowest = mb[0] - 1u;
#pragma unroll
  for (int b = 1; b < BPT; ++b) lowest = min(lowest, mb[b] - 1u);
  inexact = lowest < tiny1;
  return make_float2(__fadd_rn(hs.x, hs.y), __fadd_rn(ls.x, ls.y));
}

// sqrt(q) rounded to fp32 for q = s + e held exactly as an fp32 pair with
// |e| <= ulp(s) / 2, s in [2^-10, 4): g = the correctly rounded sqrt of s is
// at most one step from the answer, and which step follows from the exact
// residual s - g^2 (one fma: the residual of a correctly rounded square root
// is representable) plus e, against g * ulp(g) (half for the step below a
// power of two): sqrt(q) passes the midpoint g + ulp/2 iff q - g^2 exceeds
// g * ulp + ulp^2 / 4.  The fp32 sum of residual and e errs by ~2^-23 of
// g * ulp, so a decision within 2^-18 of a midpoint is left undecided
// (returns false) for the caller's double-precision path.
__device__ __forceinline__ bool sqrt_pair_rn(float s, float e, float& out) {
  const float g = __fsqrt_rn(s);
  const float d = __fadd_rn(__fmaf_rn(-g, g, s), e);        // q - g^2, rounded
  const uint32_t gb = __float_as_uint(g);
  const float u = __uint_as_float((gb & 0x7F800000u) - (23u << 23));   // ulp(g), g >= 2^-5
  const float t_up = __fmul_rn(g, u);                        // g * ulp, exact
  const bool pow2 = (gb & 0x7FFFFFu) == 0;
  const float t_dn = pow2 ? 0.5f * t_up : t_up;              // g * (ulp below g)
  const float band = t_up * 3.814697265625e-06f;            // 2^-18 * g * ulp
  const bool near = fabsf(d - t_up) <= band || fabsf(d + t_dn) <= band;
  out = d > t_up ? __fadd_rn(g, u) : (d < -t_dn ? __fsub_rn(g, pow2 ? 0.5f * u : u) : g);
  return !near;
}

__device__ __forceinline__ float2 seg_sum2(float2 v, int width) {
  for (int off = width >> 1; off > 0; off >>= 1)
    v = add2(v, make_float2(__shfl_xor_sync(0xFFFFFFFFu, v.x, off), __shfl_xor_sync(0xFFFFFFFFu, v.y, off)));
  return v;
}

// The p-mean's root in double from an exact (or double) sum S relative to
// 2^(p E): the correctly rounded S / K, a correctly rounded square root (two
// for p = 4), scaled and rounded once to fp32.  Kept out of line: rows of one
// warp reach it only for shapes and values the fp32 path leaves to it.
static __device__ __noinline__ float pmean_root_f64(double S, int pmode, int n_stat, double inv_n_stat, int E) {
  const double Kd = (double)n_stat;
  double q = S * inv_n_stat;
  q = fma(fma(-q, Kd, S), inv_n_stat, q);   // the correctly rounded S / K
  const double root = pmode == kP1 ? q : (pmode == kP2 ? sqrt(q) : sqrt(sqrt(q)));
  return __double2float_rn(root * exp2_int_f64(E));
}

// G from this thread's block maxima (bf16 magnitude bits).
//
// p = 1, 2: the terms relative to the warp maximum's power of two are summed
// exactly as fp32 pairs (pmean_split_sum, two shuffle sums); the warps of a
// longer row combine their pairs in double with exact power-of-two factors
// after one named barrier.  The exact sum is divided by K in double (correctly
// rounded), rooted with a correctly rounded double square root and rounded
// once to fp32.  p = 4: the terms (m / 2^E)^4 are exact in double (32-bit
// significands) and summed in double (exact unless they span more than
// ~2^11), then two double square roots.  Either way G is the definition's
// p-mean rounded to fp32 (unless the exact value lies within ~2^-45 of a
// rounding midpoint, or a row's maxima span more than the bounds above).
// p = infinity: the maximum.  Other p: fp32 powf terms relative to the
// maximum's power of two (within a few fp32 ulps).  M is combined on its bits
// (NaN wins).
template <int BPT, int TPR>
__device__ __forceinline__ float row_pmean(const uint32_t (&mb)[BPT], const FwdArgs& A,
                                           const FwdCfg& C, float2* red, int bar_id, int wig,
                                           int lane) {
  uint32_t mloc = mb[0];
#pragma unroll
  for (int b = 1; b < BPT; ++b) mloc = max(mloc, mb[b]);
  const int W = TPR ? 32 : C.tpr;
  mloc = TPR ? warp_max_u32(mloc) : seg_max(mloc, W);
  const bool split_p = A.pmode == kP1 || A.pmode == kP2;
  const int Ew = norm_exponent(bf16bits_to_float(mloc));
  const float inv = inv_pow2(Ew);
  float2 s2 = make_float2(0.0f, 0.0f);   // p = 1, 2: the warp's exact sum as hi + lo
  double sd = 0.0;                       // p = 4: the warp's double sum
  float sw = 0.0f;                       // other p: the warp's fp32 sum
  bool dp_sum = false;                   // p = 1, 2: the warp summed in double instead
  bool use_f64 = A.pmode == kP4;
  if (split_p) {
    // bf16 bits of the lower bound of the exact range: 2^(Ew - 7) for p = 2,
    // 2^(Ew - 22) for p = 1 (minus one, for the unsigned compare)
    const int eb = Ew + 127 - (A.pmode == kP2 ? 7 : 22);
    const uint32_t tiny1 = eb > 0 ? ((uint32_t)eb << 7) - 1u : 0u;
    bool inexact;
    s2 = seg_sum2(pmean_split_sum<BPT>(mb, inv, A.pmode, tiny1, inexact), W);
    dp_sum = use_f64 = __any_sync(0xFFFFFFFFu, inexact);
  }
  if (use_f64) {
    // p = 4, or p = 1, 2 with a term outside the fp32 pair's exact range:
    // (m / 2^E)^p in double (exact: at most 32 significant bits)
#pragma unroll
    for (int b = 0; b < BPT; ++b) {
      const double r = (double)(bf16bits_to_float(mb[b]) * inv), r2 = r * r;
      sd += A.pmode == kP1 ? r : (A.pmode == kP2 ? r2 : r2 * r2);
    }
    sd = seg_sum_f64(sd, W);
  } else if (!split_p && A.pmode != kPInf) {
#pragma unroll
    for (int b = 0; b < BPT; ++b) sw += powf(bf16bits_to_float(mb[b]) * inv, A.p);
    sw = seg_sum(sw, W);
  }
  uint32_t Mb = mloc;
  int Ef = Ew;
  double S = (split_p && !dp_sum) ? (double)s2.x + (double)s2.y : sd;
  float Sf = sw;
  if (TPR > 32) {
    // slots 0..7: the warps' maxima (bf16 bits) and fp32 sums; 8..15: their
    // exact sums as double, two 32-bit halves
    const int nw = TPR >> 5;
    if (lane == 0) {
      const uint64_t wide = (uint64_t)__double_as_longlong(S);
      red[wig] = make_float2(__uint_as_float(mloc), sw);
      red[8 + wig] = make_float2(__uint_as_float((uint32_t)wide), __uint_as_float((uint32_t)(wide >> 32)));
    }
    named_barrier_sync(bar_id, TPR);
    Mb = 0;
#pragma unroll
    for (int w = 0; w < nw; ++w) Mb = max(Mb, __float_as_uint(red[w].x));
    Ef = norm_exponent(bf16bits_to_float(Mb));
    S = 0.0;
    Sf = 0.0f;
#pragma unroll
    for (int w = 0; w < nw; ++w) {
      const int d = norm_exponent(__uint_as_float(__float_as_uint(red[w].x) << 16)) - Ef;
      const float2 v = red[8 + w];
      const double s_w = __longlong_as_double((long long)(((uint64_t)__float_as_uint(v.y) << 32) | __float_as_uint(v.x)));
      if (A.pmode == kP1 || A.pmode == kP2 || A.pmode == kP4) S += s_w * exp2_int_f64(A.pmode * d);
      else if (A.pmode != kPInf) Sf += red[w].y * exp2f(A.p * (float)d);
    }
  }
  const bool special = Mb >= 0x7F80u;       // inf / NaN: G is the maximum
  if (split_p && !(TPR <= 32 && dp_sum)) {
    // K a power of two: the sum as an fp32 pair sum + err, scaled by 1/K
    // exactly; p = 1 takes its rounded value, p = 2 the pair's square root
    // (sqrt_pair_rn); the result times 2^Ef is exact while it stays a normal
    // fp32 number.  A row of one warp forms the pair by Fast2Sum of its hi and
    // lo sums (hs >= 1, the warp maximum's own term, > |ls|: exact); a longer
    // row splits its double sum (the pair then carries it to ~2^-48, far
    // inside the band the root leaves undecided).  Anything else, and the rare
    // undecided root, take the double path below (each warp decides alike).
    float sum, err;
    if (TPR > 32) {
      sum = __double2float_rn(S);
      err = __double2float_rn(S - (double)sum);
    } else {
      sum = __fadd_rn(s2.x, s2.y);
      err = __fsub_rn(s2.y, __fsub_rn(sum, s2.x));
    }
    const float invK = A.inv_k_pow2;                          // 0 when K is not a power of two
    float gu = __fmul_rn(sum, invK);
    bool ok = invK != 0.0f && Ef >= -100;
    if (A.pmode == kP2) ok = sqrt_pair_rn(gu, __fmul_rn(err, invK), gu) && ok;
    if (__all_sync(0xFFFFFFFFu, ok || special))
      return special ? bf16bits_to_float(Mb) : __fmul_rn(gu, exp2_int(Ef));
  }
  if (special || A.pmode == kPInf) return bf16bits_to_float(Mb);  // inf / NaN / p = inf
  if (!split_p && A.pmode != kP4) return powf(Sf / (float)A.n_stat, 1.0f / A.p) * exp2_int(Ef);
  return pmean_root_f64(S, A.pmode, A.n_stat, A.inv_n_stat, Ef);
}

template <int TPR>
__device__ __forceinline__ float row_sum(float v, const FwdCfg& C, float2* red, int bar_id,
                                         int wig, int lane) {
  const int W = TPR ? 32 : C.tpr;
  v = seg_sum(v, W);
  if (TPR > 32) {
    const int nw = TPR >> 5;
    if (lane == 0) red[wig] = make_float2(v, 0.0f);
    named_barrier_sync(bar_id, TPR);
    v = 0.0f;
#pragma unroll
    for (int w = 0; w < nw; ++w) v += red[w].x;
  }
  return v;
}

// Issue the bulk copies of row block rb into `dst`, completing on `bar`.
__device__ __forceinline__ void issue_row_block(const uint16_t* x, const FwdCfg& C, int64_t rb,
                                                uint8_t* dst, uint64_t* bar, uint64_t pol) {
  const int64_t r0 = rb * C.rps;
  const int nrows = (int)(C.T - r0 < (int64_t)C.rps ? C.T - r0 : (int64_t)C.rps);
  mbar_arrive_expect_tx(bar, (uint32_t)nrows * C.row_bytes);
  for (int r = 0; r < nrows; ++r)
    bulk_copy_g2s(dst + (size_t)r * C.row_bytes, x + (r0 + r) * C.ld_x, C.row_bytes, bar, pol);
}

// The E4M3 codes of one block: 8 words, word 2j + h holding elements
// 8c + 4h .. 8c + 4h + 3 of the chunk c that slot j holds.  Returns the
// scale byte.  y are the block's 32 fp32 values in slot order, a their
// absmax (>= 0 or NaN).
template <bool SR, int ELEM>
__device__ __forceinline__ uint8_t quantise_block(const float (&y)[32], float a, int rot,
                                                  uint64_t idx0, const PhiloxKeys& pk,
                                                  uint32_t (&qw)[8]) {
  const uint32_t abits = __float_as_uint(a) & 0x7FFFFFFFu;
  const int e_raw = ELEM == kElemE2M1 ? e2m1_exponent_bits(abits) : e8m0_exponent_bits(abits);
  const bool nan_block = (e_raw == 128);     // NaN / inf in the block: fixed codes, scale 0xFF
  const int e = nan_block ? 0 : e_raw;
  const float inv = exp2_int(-e);
  const float2 inv2 = make_float2(inv, inv);
  if constexpr (ELEM == kElemE2M1) {
    // qw[j] holds slot j's eight codes
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
      float v[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 t = mul2(make_float2(y[8 * sl + 2 * i], y[8 * sl + 2 * i + 1]), inv2);
        v[2 * i] = t.x;
        v[2 * i + 1] = t.y;
      }
      if constexpr (SR) {
        const int c = (sl + rot) & 3;
        const uint64_t ctr = (idx0 + (uint64_t)(c * 8)) >> 2;
        uint4 rr[2] = {make_uint4((uint32_t)ctr, (uint32_t)(ctr >> 32), 0u, 0u),
                       make_uint4((uint32_t)(ctr + 1), (uint32_t)((ctr + 1) >> 32), 0u, 0u)};
        philox4x32_10_x2(rr[0], rr[1], pk);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          v[4 * h] = sr_e2m1_grid(v[4 * h], rr[h].x);
          v[4 * h + 1] = sr_e2m1_grid(v[4 * h + 1], rr[h].y);
          v[4 * h + 2] = sr_e2m1_grid(v[4 * h + 2], rr[h].z);
          v[4 * h + 3] = sr_e2m1_grid(v[4 * h + 3], rr[h].w);
        }
      }
      qw[sl] = nan_block ? 0x77777777u : cvt_e2m1x8_rn(v);
    }
  } else if constexpr (!SR) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 v0 = mul2(make_float2(y[4 * i], y[4 * i + 1]), inv2);
      const float2 v1 = mul2(make_float2(y[4 * i + 2], y[4 * i + 3]), inv2);
      qw[i] = cvt_e4m3x4_rn(v0.x, v0.y, v1.x, v1.y);
    }
  } else {
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
      const int c = (sl + rot) & 3;
      const uint64_t ctr = (idx0 + (uint64_t)(c * 8)) >> 2;
      // the slot's two counters (its 8 elements) in one interleaved Philox
      // (measured on B200: four counters at once ran 7% slower)
      uint4 rr[2] = {make_uint4((uint32_t)ctr, (uint32_t)(ctr >> 32), 0u, 0u),
                     make_uint4((uint32_t)(ctr + 1), (uint32_t)((ctr + 1) >> 32), 0u, 0u)};
      philox4x32_10_x2(rr[0], rr[1], pk);
      // the slot's 8 values onto the grid by the integer form; magnitudes
      // under 2^-6 are redone exactly, behind a warp vote on the minimum
      // magnitude of each half slot (zeros trip it too, and the key then picks
      // out the nonzero ones), so that only 4-element groups holding such a
      // value in some lane take that path.  In blocks of outlier channels the
      // scale is large and such values are common: halves measured 53.0 ->
      // 52.0 us at 8192 x 4096 against one vote per slot (quarters: 52.5).
      const uint32_t rw[8] = {rr[0].x, rr[0].y, rr[0].z, rr[0].w, rr[1].x, rr[1].y, rr[1].z, rr[1].w};
      float v[8], gv[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 t = mul2(make_float2(y[sl * 8 + 2 * i], y[sl * 8 + 2 * i + 1]), inv2);
        v[2 * i] = t.x;
        v[2 * i + 1] = t.y;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) gv[i] = sr_e4m3_grid_fast(__float_as_uint(v[i]), rw[i]);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        float vmin = min3_abs(fabsf(v[4 * q]), v[4 * q + 1], v[4 * q + 2]);
        vmin = min3_abs(vmin, v[4 * q + 3], v[4 * q + 3]);
        if (__any_sync(0xFFFFFFFFu, vmin < 0.015625f)) {
#pragma unroll
          for (int i = 4 * q; i < 4 * q + 4; ++i)
            if (sr_e4m3_small_key(__float_as_uint(v[i])) < kSrE4m3SmallKey) gv[i] = sr_e4m3_grid(v[i], rw[i]);
        }
      }
      qw[sl * 2] = cvt_e4m3x4_rn(gv[0], gv[1], gv[2], gv[3]);
      qw[sl * 2 + 1] = cvt_e4m3x4_rn(gv[4], gv[5], gv[6], gv[7]);
    }
  }
  if constexpr (ELEM == kElemE4M3) {
    // a block holding NaN or infinity is rare: one vote instead of a select
    // per word (every lane of the warp runs this together)
    if (__any_sync(0xFFFFFFFFu, nan_block)) {
#pragma unroll
      for (int i = 0; i < 8; ++i) qw[i] = nan_block ? 0x7F7F7F7Fu : qw[i];
    }
  }
  return nan_block ? (uint8_t)0xFF : (uint8_t)(e + 127);
}

// Store a block's codes: slot j holds chunk (j + rot) & 3, whose 8 codes go to
// bytes 8 * chunk .. 8 * chunk + 7 of the block (four 8-byte stores; the
// sectors fill up across the four).
__device__ __forceinline__ void store_codes(uint8_t* qp, const uint32_t (&qw)[8], int rot) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    asm volatile("st.global.cs.v2.b32 [%0], {%1, %2};" ::"l"(qp + ((j + rot) & 3) * 8),
                 "r"(qw[2 * j]), "r"(qw[2 * j + 1])
                 : "memory");
}

// The same 8-byte pieces into a shared-memory staging row (the block's 32
// bytes at `sa`), written out later by one bulk copy per row block.
__device__ __forceinline__ void stage_codes(uint32_t sa, const uint32_t (&qw)[8], int rot) {
#pragma unroll
  for (int j = 0; j < 4; ++j) sts64(sa + (uint32_t)(((j + rot) & 3) * 8), qw[2 * j], qw[2 * j + 1]);
}

// bf16 magnitude bits of the two 16-element halves of an NVFP4 block held in
// slot order (rotation 0 or 2: slots 0-1 hold one half, slots 2-3 the other;
// hA is the half in slots 0-1).  NaN magnitudes compare above infinity, so a
// NaN stays the maximum.
__device__ __forceinline__ void half_absmax_bits(const uint32_t (&w)[16], uint32_t& hA, uint32_t& hB) {
  uint32_t a[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t x = bf16x2_maxabs(bf16x2_maxabs(bf16x2_maxabs(w[8 * h], w[8 * h + 1]), bf16x2_maxabs(w[8 * h + 2], w[8 * h + 3])),
                                     bf16x2_maxabs(bf16x2_maxabs(w[8 * h + 4], w[8 * h + 5]), bf16x2_maxabs(w[8 * h + 6], w[8 * h + 7])));
    a[h] = max(x & 0x7FFFu, (x >> 16) & 0x7FFFu);
  }
  hA = a[0];
  hB = a[1];
}

// Absmax of each 8-element slot of a block's y (slot order), NaN-propagating.
__device__ __forceinline__ void slot_absmax(const float (&y)[32], float (&sm)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float m0 = max3_abs_nan(0.0f, y[8 * j], y[8 * j + 1]);
    float m1 = max3_abs_nan(0.0f, y[8 * j + 2], y[8 * j + 3]);
    m0 = max3_abs_nan(m0, y[8 * j + 4], y[8 * j + 5]);
    m1 = max3_abs_nan(m1, y[8 * j + 6], y[8 * j + 7]);
    sm[j] = max3_abs_nan(m0, m1, 0.0f);
  }
}

// fl32(1 / s) for every E4M3 scale code (0 for code 0 and for 0x7F, the code a
// NaN half gets), built once per CTA in shared memory with the correctly
// rounded reciprocal, so a block indexes it by the scale codes it already has.
__device__ __forceinline__ float e4m3_value_of_code(uint32_t c) {
  const uint32_t e = c >> 3, m = c & 7u;
  return e == 0 ? (float)m * (1.0f / 512.0f) : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// NVFP4 quantisation of one 32-element block (two 16-element NVFP4 blocks)
// held in slot order: per half, the E4M3 scale code (nvfp4_scale_codes2 of
// the half's absmax, 0x7F for a half holding NaN or infinity), then the E2M1
// codes of fl32(y * fl32(1/s)); a zero scale gives zero codes, a NaN half
// codes 0x7.  Returns the two scale codes (half 0 in bits 0..7).
template <bool SR>
__device__ __forceinline__ uint32_t quantise_nvfp4(const float (&y)[32], const float (&sm)[4], int rot,
                                                   uint64_t idx0, const PhiloxKeys& pk, const float* rtab,
                                                   uint32_t (&qw)[8]) {
  // Slot space (rotation 0 or 2): half A in slots 0-1, half B in slots 2-3;
  // half A is the block's first half when rot == 0, its second when rot == 2.
  float ah[2];
  ah[0] = max3_abs_nan(sm[0], sm[1], 0.0f);
  ah[1] = max3_abs_nan(sm[2], sm[3], 0.0f);
  uint32_t code[2], and_mask[2], or_mask[2];
  float inv[2];
  const bool bad2[2] = {!(ah[0] <= 3.402823466e38f), !(ah[1] <= 3.402823466e38f)};   // NaN or infinity
  const uint32_t cc = nvfp4_scale_codes2(bad2[0] ? 0.0f : ah[0], bad2[1] ? 0.0f : ah[1]);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const bool bad = bad2[h];
    code[h] = bad ? 0x7Fu : (h == 0 ? (cc & 0xFFu) : (cc >> 8));
    inv[h] = rtab[code[h]];                                        // 0 for codes 0 and 0x7F
    // a bad half's codes are all 0x7; a zero scale's are 0 (not -0)
    and_mask[h] = bad ? 0u : (code[h] == 0 ? 0u : 0xFFFFFFFFu);
    or_mask[h] = bad ? 0x77777777u : 0u;
  }
#pragma unroll
  for (int sl = 0; sl < 4; ++sl) {
    const int h = sl >> 1;
    const float2 inv2 = make_float2(inv[h], inv[h]);
    float v[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = mul2(make_float2(y[8 * sl + 2 * i], y[8 * sl + 2 * i + 1]), inv2);
      v[2 * i] = t.x;
      v[2 * i + 1] = t.y;
    }
    if constexpr (SR) {
      const int c = (sl + rot) & 3;
      const uint64_t ctr = (idx0 + (uint64_t)(c * 8)) >> 2;
      uint4 rr[2] = {make_uint4((uint32_t)ctr, (uint32_t)(ctr >> 32), 0u, 0u),
                     make_uint4((uint32_t)(ctr + 1), (uint32_t)((ctr + 1) >> 32), 0u, 0u)};
      philox4x32_10_x2(rr[0], rr[1], pk);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        v[4 * hh] = sr_e2m1_grid(v[4 * hh], rr[hh].x);
        v[4 * hh + 1] = sr_e2m1_grid(v[4 * hh + 1], rr[hh].y);
        v[4 * hh + 2] = sr_e2m1_grid(v[4 * hh + 2], rr[hh].z);
        v[4 * hh + 3] = sr_e2m1_grid(v[4 * hh + 3], rr[hh].w);
      }
    }
    qw[sl] = (cvt_e2m1x8_rn(v) & and_mask[h]) | or_mask[h];
  }
  // scale bytes in the block's order: half 0 in bits 0..7
  return rot == 0 ? (code[0] | (code[1] << 8)) : (code[1] | (code[0] << 8));
}

// E2M1 codes of a block (16 bytes): slot j's word goes to bytes
// 4 * ((j + rot) & 3) .. + 3.
__device__ __forceinline__ void store_codes_e2m1(uint8_t* qp, const uint32_t (&qw)[8], int rot) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    asm volatile("st.global.cs.b32 [%0], %1;" ::"l"(qp + ((j + rot) & 3) * 4), "r"(qw[j]) : "memory");
}

__device__ __forceinline__ void stage_codes_e2m1(uint32_t sa, const uint32_t (&qw)[8], int rot) {
#pragma unroll
  for (int j = 0; j < 4; ++j) sts32(sa + (uint32_t)(((j + rot) & 3) * 4), qw[j]);
}

// The power-of-two scale 2^e of a block whose absmax has bf16 bits m, as bf16
// bits (e by the rounded-up rule for the element format; 2^-127 is the bf16
// subnormal 0x0040).  Infinity and NaN pass through.
template <int ELEM>
__device__ __forceinline__ uint32_t scale_pow2_bf16(uint32_t m) {
  if (m >= 0x7F80u) return m;
  const int e = ELEM == kElemE2M1 ? e2m1_exponent_bits(m << 16) : e8m0_exponent_bits(m << 16);
  return e == -127 ? 0x0040u : (uint32_t)(e + 127) << 7;
}

// gamma for slot j of block k as 8 floats (in the order of the slot's words).
template <bool F32>
__device__ __forceinline__ void gamma_slot(const uint8_t* smem, int K, int j, int k, float2 (&g)[4]) {
  if constexpr (F32) {
    const float4 lo = *reinterpret_cast<const float4*>(smem + ((size_t)(2 * j) * K + k) * 16);
    const float4 hi = *reinterpret_cast<const float4*>(smem + ((size_t)(2 * j + 1) * K + k) * 16);
    g[0] = make_float2(lo.x, lo.y); g[1] = make_float2(lo.z, lo.w);
    g[2] = make_float2(hi.x, hi.y); g[3] = make_float2(hi.z, hi.w);
  } else {
    const uint4 v = *reinterpret_cast<const uint4*>(smem + ((size_t)j * K + k) * 16);
    g[0] = bf16x2_to_f2(v.x); g[1] = bf16x2_to_f2(v.y);
    g[2] = bf16x2_to_f2(v.z); g[3] = bf16x2_to_f2(v.w);
  }
}

template <int MODE, int TPR, bool SR>
constexpr bool kFwdBulkStores = (MODE != kModeRMSNorm) && (TPR > 32) && !SR;

// The chunk rotation of a thread's 64-byte blocks (slot j holds chunk
// (j + rot) & 3), from its thread index or, identically, a block index: all
// four rotations (eight threads of a shared-memory phase on eight distinct
// bank groups) for E4M3 and E2M1; for NVFP4 only 0 and 2, so slots 0-1 and
// 2-3 always hold the two 16-element halves and the per-half scale work needs
// no per-thread selects (at the price of two-way bank conflicts on the row
// loads).
template <int ELEM>
__device__ __forceinline__ int slot_rot(int x) {
  return ELEM == kElemNVFP4 ? ((x >> 1) & 1) << 1 : (x >> 1) & 3;
}

// gamma sits in shared memory as fp32 for rows of up to 8192 elements (up to
// 64 threads per row), as bf16 beyond.
__host__ __device__ constexpr bool gamma_fp32(int tpr) { return tpr == 0 || tpr <= 64; }

// TPR: threads per row as a compile-time constant (32, 64, 128, 256), or 0
// for rows of fewer than 32 blocks, where C.tpr (< 32) rows share a warp.
// HG: gamma given (MXNorm, RMSNorm); its shared-memory format follows TPR.
template <int MODE, int BPT, int TPR, bool SR, bool HG, int ELEM>
__global__ void __launch_bounds__(fwd_launch_threads(BPT, TPR, SR, ELEM), 1) row_fwd_kernel(const FwdArgs A, const FwdCfg C) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tpr = TPR ? TPR : C.tpr;
  const int gthreads = TPR ? TPR : 32;
  const int tid = threadIdx.x;
  const int g = tid / gthreads;             // row group within the CTA
  const int t = tid - g * gthreads;         // thread within the group
  const int rs = TPR ? 0 : (t >> C.log2_tpr);  // row slot within the stage (rps > 1 only)
  const int tg = t & (tpr - 1);             // thread within the row
  const int lane = tid & 31;
  const int wig = t >> 5;                   // warp within the group
  const int n_gwarps = gthreads >> 5;
  const bool issuer = (t == 0);

  uint8_t* ring = smem + C.ring_off + (size_t)g * C.stages * C.stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C.bar_off) + (size_t)g * 2 * C.stages;
  uint64_t* empty = full + C.stages;
  float2* red = reinterpret_cast<float2*>(smem + C.red_off) + (size_t)g * 2 * kRedSlots;
  // Rows of several warps (TPR > 32) stage their codes in the group's buffer
  // and write each row block with one bulk copy: full, contiguous lines for L2
  // and DRAM instead of each thread's 8-byte pieces (measured on B200 at
  // 16384 x 16384: 154 -> 137 us; rows of one warp or less, and stochastic
  // rounding, whose arithmetic the extra barrier stalls, measured faster with
  // direct stores).  The plan gives the buffer when it fits.
  const bool bulk_out = kFwdBulkStores<MODE, TPR, SR> && C.ostage_bytes != 0;
  const uint32_t ostage = smem_u32(smem + C.out_off + (size_t)g * C.ostage_bytes);
  constexpr bool has_gamma = HG;   // MXNorm's gain, RMSNorm's, or a cast's (folded weight)
  constexpr bool kGF32 = gamma_fp32(TPR);

  // Global row group, numbered group-major so that the groups of one row
  // window are spread over all SMs.  Groups at or past C.ngt have no rows (the
  // planner gives every active group the same number of row blocks, up to one).
  const int64_t gg = (int64_t)g * gridDim.x + blockIdx.x;
  const int64_t rb_end = gg < C.ngt ? C.n_row_blocks : 0;
  const uint64_t pol = policy_evict_first();
  // The first row copies go out before anything else, so their DRAM latency
  // overlaps the gamma set-up below.  Inputs are read only after the grids
  // this launch depends on have finished (programmatic dependent launch: the
  // barrier set-up above the wait overlaps the previous kernel's tail).
  if (issuer) {
    for (int s = 0; s < C.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], n_gwarps);
    }
    fence_barrier_init();
  }
  griddep_wait();
  griddep_launch_dependents();
  if (issuer) {
    for (int s = 0; s < C.stages; ++s) {
      const int64_t rb = gg + (int64_t)s * C.ngt;
      if (rb < rb_end) issue_row_block(A.x, C, rb, ring + (size_t)s * C.stage_bytes, &full[s], pol);
    }
  }
  // gamma -> shared memory in slot order, so that a warp's 16-byte reads of
  // slot j fall on consecutive words: as fp32, half h of slot j of block k
  // at ((2j + h) * K + k) * 16; as bf16 (long rows), slot j at (j * K + k) * 16.
  if constexpr (has_gamma) {
    for (int i = tid; i < C.K * 4; i += blockDim.x) {
      const int k = i >> 2, j = i & 3;
      const int c = (j + slot_rot<ELEM>(k)) & 3;
      const uint4 v = ldg128_nc(A.gamma + (size_t)k * kBlock + c * 8);
      if constexpr (kGF32) {
        const float4 lo = make_float4(bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y));
        const float4 hi = make_float4(bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w));
        *reinterpret_cast<float4*>(smem + ((size_t)(2 * j) * C.K + k) * 16) = lo;
        *reinterpret_cast<float4*>(smem + ((size_t)(2 * j + 1) * C.K + k) * 16) = hi;
      } else {
        *reinterpret_cast<uint4*>(smem + ((size_t)j * C.K + k) * 16) = v;
      }
    }
  }
  if constexpr (ELEM == kElemNVFP4) {
    float* rtab = reinterpret_cast<float*>(smem + C.rcp_off);
    for (int c = tid; c < 128; c += blockDim.x)
      rtab[c] = (c == 0 || c == 127) ? 0.0f : __frcp_rn(e4m3_value_of_code((uint32_t)c));
  }
  __syncthreads();

  // A wait that gives up marks the kernel failed; threads then keep going
  // without waiting so every named barrier still completes (outputs garbage,
  // accesses in bounds).
  const PhiloxKeys pkeys = philox_keys(A.seed_lo, A.seed_hi);   // used by stochastic rounding only
  bool ok = true;
  int par = 0;
  const int bar_id = 1 + g;
  const int rot = slot_rot<ELEM>(tg);      // the same for every block of the thread
  int64_t it = 0;
  for (int64_t rb = gg; rb < rb_end; rb += C.ngt, ++it, par ^= 1) {
    const int s = (int)(it % C.stages);
    const uint32_t ph = (uint32_t)((it / C.stages) & 1);
    if (ok) ok = mbar_wait_bounded(&full[s], ph, A.status);
    const int64_t row = rb * C.rps + rs;
    const bool valid = row < C.T;
    // scale byte offset of block k: row part once per row, then a few ops per
    // block (row-major: row * K + k; tcgen05 layout: mma_scale_offset split
    // into its row and k terms)
    const int64_t srow_off = A.scale_mma ? mma_scale_offset(row, 0, A.kp4) : row * (int64_t)C.K;
    const uint32_t srow = smem_u32(ring + (size_t)s * C.stage_bytes + (size_t)rs * C.row_bytes);

    // ---- the row into registers; after the block maxima the stage goes back
    // to the issuer, so the copy of row block rb + stages * ngt overlaps the
    // rest of this row's arithmetic.
    // (RMSNorm keeps the row in the stage instead: it reads it twice and hands
    // the stage back after its second pass, which needs far fewer registers.)
    constexpr bool kHold = (MODE != kModeRMSNorm);
    constexpr int kHoldB = kHold ? BPT : 1;
    uint32_t xr[kHoldB][16];
    // The staging buffer is free again once the previous row block's bulk
    // copy has read it; the group learns it at the barrier below (the
    // __syncwarp after the register copy, or a named barrier for longer rows).
    if (bulk_out && issuer) bulk_wait_read_all();
    if constexpr (kHold) {
#pragma unroll
      for (int b = 0; b < BPT; ++b) {
        const int k = tg + b * tpr;
        const bool have = valid && k < C.K;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (have) v = lds128(srow + (uint32_t)k * 64u + (uint32_t)(((j + rot) & 3) * 16));
          xr[b][4 * j] = v.x; xr[b][4 * j + 1] = v.y; xr[b][4 * j + 2] = v.z; xr[b][4 * j + 3] = v.w;
        }
      }
    }

    // ---- pass 1: block maxima (MXNorm, Cast) or sum of squares (RMSNorm)
    uint32_t mb[BPT];
    uint32_t mh[BPT][2];                      // NVFP4: the two 16-element halves
    float2 ss2 = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int b = 0; b < BPT; ++b) {
      if constexpr (MODE == kModeRMSNorm) {
        mb[b] = 0;
        const int k = tg + b * tpr;
        if (valid && k < C.K) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 v = lds128(srow + (uint32_t)k * 64u + (uint32_t)(((j + rot) & 3) * 16));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 xv = bf16x2_to_f2(w[i]);
              ss2 = fma2(xv, xv, ss2);
            }
          }
        }
      } else if constexpr (ELEM == kElemNVFP4) {
        half_absmax_bits(xr[b], mh[b][0], mh[b][1]);        // NVFP4 blocks are the halves
        mb[b] = max(mh[b][0], mh[b][1]);
      } else {
        mb[b] = block_absmax16(xr[b]);
      }
    }
    if constexpr (kHold) {
      // Hand the stage back once pass 1 has used every register read from it
      // (so those shared-memory reads are complete), behind a proxy fence that
      // orders them before the bulk copy that overwrites the stage: without
      // both, a refill could land before a slow ld.shared had read its data.
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (issuer) {
        const int64_t nrb = rb + (int64_t)C.stages * C.ngt;
        if (nrb < C.n_row_blocks) {
          if (ok) ok = mbar_wait_bounded(&empty[s], ph, A.status);
          if (ok) issue_row_block(A.x, C, nrb, ring + (size_t)s * C.stage_bytes, &full[s], pol);
        }
      }
      if (TPR > 32 && bulk_out) named_barrier_sync(bar_id, TPR);
    }

    float2* redp = red + par * kRedSlots;
    if constexpr (MODE == kModeRMSNorm) {
      // ---------------------------------------------------------- RMSNorm
      const float ss = row_sum<TPR>(ss2.x + ss2.y, C, redp, bar_id, wig, lane);
      const float rinv = 1.0f / sqrtf(ss / (float)C.D + A.eps);
      const float2 r2 = make_float2(rinv, rinv);
#pragma unroll
      for (int b = 0; b < BPT; ++b) {
        const int k = tg + b * tpr;
        const bool blk = valid && k < C.K;
        const int kk = k < C.K ? k : C.K - 1;          // in-range smem reads
        uint16_t* yrow = A.y + row * (int64_t)C.D + (int64_t)k * kBlock;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 v = lds128(srow + (uint32_t)kk * 64u + (uint32_t)(((j + rot) & 3) * 16));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
          float2 gf[4];
          if constexpr (has_gamma) gamma_slot<kGF32>(smem, C.K, j, kk, gf);
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float2 yv = mul2(bf16x2_to_f2(w[i]), r2);
            if constexpr (has_gamma) yv = mul2(yv, gf[i]);
            const __nv_bfloat162 h = __floats2bfloat162_rn(yv.x, yv.y);
            o[i] = *reinterpret_cast<const uint32_t*>(&h);
          }
          if (blk) stg128_stream(yrow + ((j + rot) & 3) * 8, make_uint4(o[0], o[1], o[2], o[3]));
        }
      }
      fence_proxy_async_smem();   // this thread's reads of the stage before its refill
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (issuer) {
        const int64_t nrb = rb + (int64_t)C.stages * C.ngt;
        if (nrb < C.n_row_blocks) {
          if (ok) ok = mbar_wait_bounded(&empty[s], ph, A.status);
          if (ok) issue_row_block(A.x, C, nrb, ring + (size_t)s * C.stage_bytes, &full[s], pol);
        }
      }
    } else {
      // ------------------------------------------------- MXNorm / MXCast
      float sc = 1.0f;
      if constexpr (MODE == kModeMXNorm) {
        float G;
        if constexpr (ELEM == kElemNVFP4) {
          // the statistic runs over the 16-element blocks; its scale-reuse form
          // uses the blocks' E4M3 scale values (exact in bf16)
          uint32_t mst[2 * BPT];
#pragma unroll
          for (int b = 0; b < BPT; ++b) {
            mst[2 * b] = mh[b][0];
            mst[2 * b + 1] = mh[b][1];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint32_t m = mst[2 * b + h];
              if (A.stat_exp && m < 0x7F80u)
                mst[2 * b + h] = __float_as_uint(nvfp4_scale_value(bf16bits_to_float(m))) >> 16;
            }
          }
          G = row_pmean<2 * BPT, TPR>(mst, A, C, redp, bar_id, wig, lane);
        } else {
          uint32_t mst[BPT];
#pragma unroll
          for (int b = 0; b < BPT; ++b) mst[b] = A.stat_exp ? scale_pow2_bf16<ELEM>(mb[b]) : mb[b];
          G = row_pmean<BPT, TPR>(mst, A, C, redp, bar_id, wig, lane);
        }
        sc = (G == 0.0f) ? 0.0f : __frcp_rn(G);
        if (valid && tg == 0 && A.G_out) A.G_out[row] = G;
      }
      const float2 s2 = make_float2(sc, sc);
#pragma unroll
      for (int b = 0; b < BPT; ++b) {
        const int k = tg + b * tpr;
        const bool blk = valid && k < C.K;             // blocks past K compute on zeros
        const int kk = k < C.K ? k : C.K - 1;          // in-range gamma reads
        float y[32];
        float a;
        float sm[4];                                   // NVFP4: per-slot maxima of y
        if constexpr (has_gamma) {
          float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float2 gf[4];
            gamma_slot<kGF32>(smem, C.K, j, kk, gf);
            float b0 = 0.0f, b1 = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 yv = mul2(mul2(bf16x2_to_f2(xr[b][4 * j + i]), s2), gf[i]);
              y[8 * j + 2 * i] = yv.x;
              y[8 * j + 2 * i + 1] = yv.y;
              if constexpr (ELEM == kElemNVFP4) {
                if (i & 1) b1 = max3_abs_nan(b1, yv.x, yv.y);
                else b0 = max3_abs_nan(b0, yv.x, yv.y);
              } else {
                if (i & 1) a1 = max3_abs_nan(a1, yv.x, yv.y);
                else a0 = max3_abs_nan(a0, yv.x, yv.y);
              }
            }
            if constexpr (ELEM == kElemNVFP4) sm[j] = max3_abs_nan(b0, b1, 0.0f);
          }
          a = max3_abs_nan(a0, a1, 0.0f);
        } else {
#pragma unroll
          for (int w = 0; w < 16; ++w) {
            float2 yv = bf16x2_to_f2(xr[b][w]);
            if (MODE == kModeMXNorm) yv = mul2(yv, s2);
            y[2 * w] = yv.x;
            y[2 * w + 1] = yv.y;
          }
          // fl(m * s) is the block max of fl(x * s): rounding is monotone.
          a = (MODE == kModeMXNorm) ? __fmul_rn(bf16bits_to_float(mb[b]), sc) : bf16bits_to_float(mb[b]);
        }
        uint32_t qw[8];
        const uint64_t idx0 = (uint64_t)(row * (int64_t)C.D + (int64_t)k * kBlock);
        if constexpr (ELEM == kElemNVFP4) {
          (void)a;
          if constexpr (!has_gamma) slot_absmax(y, sm);
          const uint32_t codes2 = quantise_nvfp4<SR>(y, sm, rot, idx0, pkeys,
                                                     reinterpret_cast<const float*>(smem + C.rcp_off), qw);
          if (blk) {
            if (bulk_out)
              stage_codes_e2m1(ostage + (uint32_t)rs * C.code_row_bytes + (uint32_t)k * (kBlock / 2), qw, rot);
            else
              store_codes_e2m1(A.q + row * (int64_t)(C.D / 2) + (int64_t)k * (kBlock / 2), qw, rot);
            *reinterpret_cast<uint16_t*>(A.scales + row * (int64_t)(2 * C.K) + 2 * k) = (uint16_t)codes2;
          }
        } else {
          const uint8_t code = quantise_block<SR, ELEM>(y, a, rot, idx0, pkeys, qw);
          if (blk) {
            if constexpr (ELEM == kElemE2M1) {
              if (bulk_out)
                stage_codes_e2m1(ostage + (uint32_t)rs * C.code_row_bytes + (uint32_t)k * (kBlock / 2), qw, rot);
              else
                store_codes_e2m1(A.q + row * (int64_t)(C.D / 2) + (int64_t)k * (kBlock / 2), qw, rot);
            } else {
              if (bulk_out)
                stage_codes(ostage + (uint32_t)rs * C.code_row_bytes + (uint32_t)k * kBlock, qw, rot);
              else
                store_codes(A.q + row * (int64_t)C.D + (int64_t)k * kBlock, qw, rot);
            }
            A.scales[srow_off + (A.scale_mma ? (int64_t)((k >> 2) * 512 + (k & 3)) : (int64_t)k)] = code;
          }
        }
      }
      // The row block's codes leave in one bulk copy once every thread of the
      // group has staged its blocks.
      if (bulk_out) {
        fence_proxy_async_smem();
        if (TPR > 32) named_barrier_sync(bar_id, TPR);
        else __syncwarp();
        if (issuer) {
          const int64_t r0 = rb * C.rps;
          const int64_t nrows = C.T - r0 < (int64_t)C.rps ? C.T - r0 : (int64_t)C.rps;
          bulk_copy_s2g(A.q + r0 * (int64_t)C.code_row_bytes, ostage, (uint32_t)nrows * C.code_row_bytes);
          bulk_commit();
        }
      }
    }

  }
  // Leave no copy in flight: the issuer waits for its bulk stores to have read
  // the staging buffer and for the last phase of every stage it filled
  // (already complete unless a wait gave up above).
  if (bulk_out && issuer) bulk_wait_read_all();   // staging buffers read before exit
  if (issuer && !ok) {
    for (int s = 0; s < C.stages; ++s) {
      const int64_t last_it = it - 1 - ((it - 1 - s) % C.stages + C.stages) % C.stages;
      if (last_it >= 0) mbar_wait_bounded(&full[s], (uint32_t)((last_it / C.stages) & 1), A.status);
    }
  }
}

// The instantiation for (blocks per thread, threads per row): 32 threads per
// row for up to 4 blocks each (rows of up to 128 blocks), 64..256 threads with
// 4 blocks each beyond, a runtime segment width for rows under 32 blocks.
// Each translation unit that calls this instantiates its own mode's kernels.
template <int MODE, bool SR, bool HG, int ELEM = kElemE4M3>
const void* pick_fwd_shape(int bpt, int tpr) {
  if (tpr < 32) return bpt == 1 ? (const void*)row_fwd_kernel<MODE, 1, 0, SR, HG, ELEM> : nullptr;
  if (tpr == 32) {
    switch (bpt) {
      case 1: return (const void*)row_fwd_kernel<MODE, 1, 32, SR, HG, ELEM>;
      case 2: return (const void*)row_fwd_kernel<MODE, 2, 32, SR, HG, ELEM>;
      case 4: return (const void*)row_fwd_kernel<MODE, 4, 32, SR, HG, ELEM>;
      default: return nullptr;
    }
  }
  if constexpr (SR) {
    // stochastic rounding: one or two blocks per thread (the Philox
    // arithmetic wants warps, not long unrolled bodies)
    if (bpt == 1) {
      switch (tpr) {
        case 64: return (const void*)row_fwd_kernel<MODE, 1, 64, SR, HG, ELEM>;
        case 128: return (const void*)row_fwd_kernel<MODE, 1, 128, SR, HG, ELEM>;
        case 256: return (const void*)row_fwd_kernel<MODE, 1, 256, SR, HG, ELEM>;
        default: return nullptr;
      }
    }
    if (bpt == 2) {
      switch (tpr) {
        case 64: return (const void*)row_fwd_kernel<MODE, 2, 64, SR, HG, ELEM>;
        case 128: return (const void*)row_fwd_kernel<MODE, 2, 128, SR, HG, ELEM>;
        case 256: return (const void*)row_fwd_kernel<MODE, 2, 256, SR, HG, ELEM>;
        default: return nullptr;
      }
    }
  }
  if (bpt != 4) return nullptr;
  switch (tpr) {
    case 64: return (const void*)row_fwd_kernel<MODE, 4, 64, SR, HG, ELEM>;
    case 128: return (const void*)row_fwd_kernel<MODE, 4, 128, SR, HG, ELEM>;
    case 256: return (const void*)row_fwd_kernel<MODE, 4, 256, SR, HG, ELEM>;
    default: return nullptr;
  }
}

}  // namespace mxn
