// device_common.cuh -- sm_100a device helpers for the MXNorm row kernels.
//
// Inline PTX for the bulk-copy (TMA engine) pipeline, bounded mbarrier waits,
// and the MX element arithmetic: E8M0 scale from a block absmax, the E4M3
// cast, Philox4x32-10 and stochastic rounding.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mxn {

constexpr int kBlock = 32;                       // MX block size B
constexpr uint64_t kWaitLimitNs = 1000000000ull; // bounded waits give up after ~1 s

// Status bits recorded in the device status word.
constexpr unsigned kStatusWaitTimeout = 1u;

// ----------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory counter add with acquire-release semantics at CTA scope:
// returns the old value.  The warp that brings a count to its total sees
// every earlier adder's prior accesses (here, its shared-memory reads of a
// stage) as complete.
__device__ __forceinline__ uint32_t smem_add_acq_rel(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;"
               : "=r"(old)
               : "r"(smem_u32(p)), "r"(v)
               : "memory");
  return old;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Make the initialised barriers visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: the warp sleeps until the phase
// completes or about `hint_ns` pass, instead of spinning on issue slots that
// the computing warps need.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// As mbar_wait_bounded below, with an explicit limit.
__device__ __forceinline__ bool mbar_wait_limit(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                                unsigned* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait_sleep(bar, parity, 20000u)) {
    if (global_timer_ns() - t0 > limit_ns) {
      atomicOr(status, kStatusWaitTimeout);
      return false;
    }
  }
  return true;
}

// Wait until the phase of `bar` with the given parity has completed, for at
// most kWaitLimitNs.  Returns false (and records the timeout in *status) if
// the wait gave up.  Sleeping waits: the clock is read once per ~20 us wake-up.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  unsigned* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait_sleep(bar, parity, 20000u)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      atomicOr(status, kStatusWaitTimeout);
      return false;
    }
  }
  return true;
}

// 1-D bulk copy global -> shared on the TMA engine, completing `bytes` of
// transaction count on `bar`.  Needs 16-byte aligned addresses and a size that
// is a multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_copy_g2s(void* smem_dst, const void* gmem_src,
                                              uint32_t bytes, uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// 1-D bulk copy shared -> global on the TMA engine, tracked by the issuing
// thread's bulk groups.  Needs 16-byte aligned addresses and a size that is a
// multiple of 16.
__device__ __forceinline__ void bulk_copy_s2g(void* gmem_dst, uint32_t smem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gmem_dst),
               "r"(smem_src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed shared -> global copy of this thread has read its
// source: the buffer may then be rewritten, or the CTA exit (the writes
// themselves complete with the grid, before any dependent grid runs).
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Order this thread's shared-memory writes before later bulk copies that read them.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void sts64(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void sts32(uint32_t addr, uint32_t a) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(a) : "memory");
}

// L2 policy for data read exactly once: evict first.
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Programmatic dependent launch: wait until the grids this one depends on in
// stream order have completed and their writes are visible (a no-op when the
// launch did not opt in), and let the next grid in the stream launch early
// (its CTAs run once SMs free up, and wait in their own griddep_wait).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// Streaming 16-byte global store (written once, not re-read here).
__device__ __forceinline__ void stg128_stream(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

// A 4-byte read-only global load that stays where it is written (volatile), so
// its latency overlaps what follows instead of being moved next to its use.
__device__ __forceinline__ float ldg_f32_early(const float* p) {
  float v;
  asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ldg128_nc(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// ------------------------------------------------------------- float helpers

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float bf16bits_to_float(uint32_t b16) { return __uint_as_float(b16 << 16); }

// 2^n for an integer n in [-126, 127], built from its exponent field.
__device__ __forceinline__ float exp2_int(int n) { return __uint_as_float((uint32_t)(n + 127) << 23); }

// Packed fp32 pairs (sm_100 f32x2 arithmetic): each call is one instruction
// doing two correctly rounded fp32 multiplies.
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;"
      : "=l"(d)
      : "l"(*reinterpret_cast<const uint64_t*>(&a)), "l"(*reinterpret_cast<const uint64_t*>(&b)));
  return *reinterpret_cast<const float2*>(&d);
}

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(d)
      : "l"(*reinterpret_cast<const uint64_t*>(&a)), "l"(*reinterpret_cast<const uint64_t*>(&b)),
        "l"(*reinterpret_cast<const uint64_t*>(&c)));
  return *reinterpret_cast<const float2*>(&d);
}

__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) { return make_float2(bf16lo(w), bf16hi(w)); }

// min(a, |b|, |c|) (a NaN operand is ignored).
__device__ __forceinline__ float min3_abs(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(fabsf(b)), "f"(fabsf(c)));
  return d;
}

// max(a, |b|, |c|), propagating NaN.
__device__ __forceinline__ float max3_abs_nan(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(fabsf(b)), "f"(fabsf(c)));
  return d;
}

// Packed bf16 pair whose halves are the larger magnitudes of a's and b's
// halves (signs are junk; NaN propagates).  Folding 16 words with it gives the
// block absmax in 15 instructions.
__device__ __forceinline__ uint32_t bf16x2_maxabs(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Magnitude bits (bf16, low 16 bits) of the absmax of 16 packed words.
__device__ __forceinline__ uint32_t block_absmax16(const uint32_t* w) {
  uint32_t a0 = bf16x2_maxabs(w[0], w[1]), a1 = bf16x2_maxabs(w[2], w[3]);
  uint32_t a2 = bf16x2_maxabs(w[4], w[5]), a3 = bf16x2_maxabs(w[6], w[7]);
  uint32_t a4 = bf16x2_maxabs(w[8], w[9]), a5 = bf16x2_maxabs(w[10], w[11]);
  uint32_t a6 = bf16x2_maxabs(w[12], w[13]), a7 = bf16x2_maxabs(w[14], w[15]);
  a0 = bf16x2_maxabs(a0, a1); a2 = bf16x2_maxabs(a2, a3);
  a4 = bf16x2_maxabs(a4, a5); a6 = bf16x2_maxabs(a6, a7);
  a0 = bf16x2_maxabs(a0, a2); a4 = bf16x2_maxabs(a4, a6);
  a0 = bf16x2_maxabs(a0, a4);
  return max(a0 & 0x7FFFu, (a0 >> 16) & 0x7FFFu);
}

// ------------------------------------------------------------------ E8M0 scale

// Scale exponent of a block whose absmax has fp32 bits `abits` (non-negative):
// the smallest e in [-127, 127] with a <= 448 * 2^e.  Writing a = m * 2^E with
// m in [1, 2), 448 = 1.75 * 2^8 gives e = E - 8 when m <= 1.75, else E - 7.
// Zero and fp32 subnormals give -127.  Returns 128 for NaN / infinity.
__device__ __forceinline__ int e8m0_exponent_bits(uint32_t abits) {
  if (abits >= 0x7F800000u) return 128;
  const int ef = (int)(abits >> 23);
  int e = ef - 127 - 8 + ((abits & 0x7FFFFFu) > 0x600000u ? 1 : 0);
  if (ef == 0) e = -127;
  return max(e, -127);  // finite fp32 keeps e <= 120
}

// The same rule for E2M1 elements (largest magnitude 6 = 1.5 * 2^2): the
// smallest e in [-127, 127] with a <= 6 * 2^e.
__device__ __forceinline__ int e2m1_exponent_bits(uint32_t abits) {
  if (abits >= 0x7F800000u) return 128;
  const int ef = (int)(abits >> 23);
  int e = ef - 127 - 2 + ((abits & 0x7FFFFFu) > 0x400000u ? 1 : 0);
  if (ef == 0) e = -127;
  return max(e, -127);
}

// ------------------------------------------------------------------ E4M3 cast

// Two fp32 -> two E4M3 codes, round to nearest even, saturating finite; the
// code of `lo` in bits 0..7, of `hi` in bits 8..15.
__device__ __forceinline__ uint32_t cvt_e4m3x2_rn(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return (uint32_t)r;
}

// Four fp32 -> four E4M3 codes (nearest even, saturating finite), packed with
// the code of `a` in bits 0..7 through `d` in bits 24..31.
__device__ __forceinline__ uint32_t cvt_e4m3x4_rn(float a, float b, float c, float d) {
  uint32_t r;
  asm("{\n\t.reg .b16 l, h;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 l, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 h, %4, %3;\n\t"
      "mov.b32 %0, {l, h};\n\t}"
      : "=r"(r)
      : "f"(a), "f"(b), "f"(c), "f"(d));
  return r;
}

// ------------------------------------------------------------------ NVFP4 scale

// The NVFP4 block scale: the smallest E4M3 value s with a <= 6 s (a >= 0
// finite), 448 when even that is too small, returned as its exact fp32 value.
// u = fl(a * c) with c the fp32 value just below 1/6 (6c = 1 - 2^-24, and a
// rounding adds at most 2^-24 relative: (1 - 2^-24)(1 + 2^-24) < 1) is below
// a / 6, so s is u rounded up onto the E4M3 grid -- 3 mantissa bits from 2^-6
// up (an integer add and mask on the bits), multiples of 2^-9 below -- or the
// next grid value when 6 s < a, which one exact comparison settles (6 s is
// exact in fp32).  For a > 6 * 448 the result is clamped to 448.
__device__ __forceinline__ float nvfp4_scale_value(float a) {
  const float u = a * 0.16666665673255920f;
  const uint32_t nb = (__float_as_uint(u) + 0xFFFFFu) & 0xFFF00000u;
  const float sub = ceilf(u * 512.0f) * (1.0f / 512.0f);
  const bool normal = u >= 0.015625f;
  float s = normal ? __uint_as_float(nb) : sub;
  const float next = normal ? __uint_as_float(nb + 0x100000u) : s + (1.0f / 512.0f);
  s = (6.0f * s < a) ? next : s;
  return fminf(s, 448.0f);
}

// Two E4M3 codes (bits 0..7 and 8..15) -> their exact values.
__device__ __forceinline__ float2 e4m3x2_to_f2(uint32_t cc) {
  float lo, hi;
  asm("{\n\t.reg .b16 c;\n\t.reg .b32 h2;\n\t.reg .f16 l, h;\n\t"
      "cvt.u16.u32 c, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 h2, c;\n\t"
      "mov.b32 {l, h}, h2;\n\t"
      "cvt.f32.f16 %0, l;\n\t"
      "cvt.f32.f16 %1, h;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(cc));
  return make_float2(lo, hi);
}

// The NVFP4 scale codes of two 16-element halves with absmax a0, a1 (>= 0
// finite): code 0 in bits 0..7, code 1 in bits 8..15 -- the codes of
// nvfp4_scale_value.  The wanted code is the smallest with 6 * value >= a
// (0x7E, 448, when none).  u = fl(a * c) is below a / 6 by under 2^-23 of it
// (see there; for a tiny a, by under 2^-150 absolute), far less than any E4M3
// step, so: with no grid value in [u, a / 6] the wanted code is u rounded up,
// which is u's nearest-even code or the next; with one, g, u's nearest code
// is g itself, and the wanted code is g (a = 6 g) or the next.  So take the
// nearest-even codes of both halves in one packed conversion (saturating at
// 448) and step each up once where 6 * value < a, never past 0x7E.  6 * value
// is exact in fp32.
__device__ __forceinline__ uint32_t nvfp4_scale_codes2(float a0, float a1) {
  constexpr float kC6 = 0.16666665673255920f;
  const float2 u = mul2(make_float2(a0, a1), make_float2(kC6, kC6));
  uint32_t cc = cvt_e4m3x2_rn(u.x, u.y);
  const float2 six = mul2(e4m3x2_to_f2(cc), make_float2(6.0f, 6.0f));
  const uint32_t up0 = (six.x < a0 && (cc & 0xFFu) != 0x7Eu) ? 1u : 0u;
  const uint32_t up1 = (six.y < a1 && (cc >> 8) != 0x7Eu) ? 0x100u : 0u;
  return cc + up0 + up1;
}

// ------------------------------------------------------------------ E2M1 cast

// Eight fp32 -> eight E2M1 codes (nearest even, saturating to +-6), packed
// four bits each with the code of v[0] in bits 0..3 through v[7] in bits
// 28..31 (cvt puts its first source in the high nibble of the byte).
__device__ __forceinline__ uint32_t cvt_e2m1x8_rn(const float (&v)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return r;
}

// ---------------------------------------------------------- Philox4x32-10

// Philox4x32 with 10 rounds (Salmon, Moraes, Dror, Shaw, SC'11): each round
// multiplies words 0 and 2 by fixed odd constants, swaps the halves and xors
// in the round key; the key advances by the Weyl constants between rounds.
//
// The round keys depend on the seed only, so a kernel builds them once
// (PhiloxKeys) and every call xors them in.
struct PhiloxKeys {
  uint32_t k0[10], k1[10];
};

__device__ __forceinline__ PhiloxKeys philox_keys(uint32_t seed_lo, uint32_t seed_hi) {
  PhiloxKeys K;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    K.k0[r] = seed_lo + (uint32_t)r * 0x9E3779B9u;
    K.k1[r] = seed_hi + (uint32_t)r * 0xBB67AE85u;
  }
  return K;
}

// Two independent counters in lock-step: the same rounds, interleaved, so each
// round's multiplies of one stream overlap the other's (two dependency chains).
__device__ __forceinline__ void philox4x32_10_x2(uint4& a, uint4& b, const PhiloxKeys& K) {
  constexpr uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t pa0 = (uint64_t)M0 * a.x, pa1 = (uint64_t)M1 * a.z;
    const uint64_t pb0 = (uint64_t)M0 * b.x, pb1 = (uint64_t)M1 * b.z;
    a = make_uint4((uint32_t)(pa1 >> 32) ^ a.y ^ K.k0[r], (uint32_t)pa1, (uint32_t)(pa0 >> 32) ^ a.w ^ K.k1[r],
                   (uint32_t)pa0);
    b = make_uint4((uint32_t)(pb1 >> 32) ^ b.y ^ K.k0[r], (uint32_t)pb1, (uint32_t)(pb0 >> 32) ^ b.w ^ K.k1[r],
                   (uint32_t)pb0);
  }
}

// Stochastic rounding of v (|v| <= 448, finite) onto the E4M3 grid, returned
// as the fp32 grid value (exact) with v's sign.  lo = the grid value at or
// below |v|, step = grid spacing there; up iff r < (|v| - lo) / step * 2^32.
// From 2^-6 up the grid keeps 3 fraction bits, so lo is |v| with its 20 low
// mantissa bits cleared and (|v| - lo) / step * 2^32 is exactly those 20 bits
// times 2^12: an integer comparison, and lo + step an integer add on the bits
// (a carry steps into the next binade).  Below 2^-6 (E4M3 subnormals, step
// 2^-9, rare after the block scale) the same quantities in fp32: lo a multiple
// of 2^-9, |v| - lo exact, the scaling by 2^41 a power of two; for an integer
// r, r < t holds iff r < ceil(t), and ceil(t) < 2^32.
//
// The comparison needs no compare: with L the 20 dropped bits and r' = r >> 12,
// r < L * 2^12 holds iff r' < L, iff L + (2^20 - 1 - r') >= 2^20, and
// 2^20 - 1 - r' is (~r) >> 12.  So adding (~r) >> 12 to the bits of v carries
// into the kept mantissa exactly when v rounds up (the carry may step into the
// next binade, which is lo + step; it cannot reach the sign, |v| <= 448), and
// clearing the 20 low bits leaves the grid value with v's sign.
//
// Split for speed: sr_e4m3_grid_fast is the integer form, exact for |v| >=
// 2^-6 and for zero; sr_e4m3_small_key(b) is below kSrE4m3SmallKey exactly
// when 0 < |v| < 2^-6 (zero and the sign map out of range).  A caller takes
// the integer form everywhere and redoes with sr_e4m3_grid only the elements
// the key flags, once a cheap test (the minimum magnitude) finds any.
__device__ __forceinline__ float sr_e4m3_grid_fast(uint32_t b, uint32_t r) {
  return __uint_as_float((b + ((~r) >> 12)) & 0xFFF00000u);
}
constexpr uint32_t kSrE4m3SmallKey = 2u * 0x3C800000u - 2u;
__device__ __forceinline__ uint32_t sr_e4m3_small_key(uint32_t b) { return b + b - 2u; }

__device__ __forceinline__ float sr_e4m3_grid(float v, uint32_t r) {
  const uint32_t b = __float_as_uint(v);
  const uint32_t ab = b & 0x7FFFFFFFu;
  if (ab >= 0x3C800000u) return sr_e4m3_grid_fast(b, r);
  const float a = __uint_as_float(ab);
  const float lo = truncf(a * 512.0f) * (1.0f / 512.0f);
  const uint32_t thr = __float2uint_ru((a - lo) * 2199023255552.0f);   // 2^41
  const float m = (r < thr) ? lo + (1.0f / 512.0f) : lo;
  return copysignf(m, v);
}

// The same on the E2M1 grid (|v| <= 6, which the rounded-up scale ensures):
// one fraction bit from 1 up, step 1/2 below 1.
__device__ __forceinline__ float sr_e2m1_grid(float v, uint32_t r) {
  const float a = fabsf(v);
  const uint32_t ab = __float_as_uint(a);
  float lo, step, inv_step_2_32;
  if (ab >= 0x3F800000u) {  // |v| >= 1: 1 fraction bit kept
    lo = __uint_as_float(ab & 0xFFC00000u);
    const uint32_t ebits = ab & 0x7F800000u;          // 2^E
    step = __uint_as_float(ebits - (1u << 23));       // 2^(E-1)
    inv_step_2_32 = __uint_as_float((uint32_t)(127 + 127 + 1 + 32) * (1u << 23) - ebits);  // 2^(33-E)
  } else {                  // below 1: step 1/2
    lo = truncf(a * 2.0f) * 0.5f;
    step = 0.5f;
    inv_step_2_32 = 8589934592.0f;                    // 2^33
  }
  const float t = (a - lo) * inv_step_2_32;
  const uint32_t thr = __float2uint_ru(t);
  const float m = (r < thr) ? lo + step : lo;
  return copysignf(m, v);
}

}  // namespace mxn
