// gemm_mxfp8.cu -- block-scaled MXFP8 GEMM on the sm_100a tensor cores.
//
// The consumer of MXNorm's output (gist.science, "MXNorm: Reusing MXFP block
// scales for efficient tensor normalisation", technical summary section 2.3:
// MXNormLinear feeds the MX-cast activations straight into an MX matmul):
//   C[m, n] = sum_k A(m, k) * B(n, k),  A(m,k) = e4m3(a_q[m,k]) * 2^(a_s[m,k/32] - 127),
//   B likewise, fp32 accumulation in tensor memory, bf16 output.
//
// Three tile shapes (gemm_mxfp8_set_tiles): 256 x 192 by default where the
// shape allows (described with its kernel below), 128 x 256 otherwise, and
// 256 x 256 on CTA pairs on request.  The 128 x 256 kernel: persistent CTAs,
// one per SM, walk the output tiles (tile t, then t + gridDim.x, ...; M-tiles
// fastest, so the CTAs in flight share B tiles):
//  * warp 0, one thread: the producer streams 128-element K stages of A
//    (128 x 128 B) and B (256 x 128 B) into a 4-stage shared-memory ring with
//    TMA tensor copies (128-byte swizzle, no multicast), and the stage's scale
//    atoms (the 128-row x 4-block, 512-byte tiles of the tcgen05 scale layout)
//    with 1-D bulk copies -- straight on into the next tile's stages;
//  * warp 1, one thread: copies each stage's scale atoms into tensor memory
//    (tcgen05.cp 32x128b, replicated to the four lane quarters), issues four
//    tcgen05.mma.kind::mxf8f6f4.block_scale (M = 128, N = 256, K = 32 each)
//    and frees the stage with tcgen05.commit; after a tile's last stage it
//    commits "accumulator full", and before a tile's first MMA it waits for
//    "accumulator empty";
//  * warps 2..9: each reads its lane quarter and column half of the fp32
//    accumulator (tcgen05.ld 32x32b, 128 columns) into registers, hands the
//    accumulator back, and only then converts to bf16 and stores -- so the
//    next tile's MMAs start after the tensor-memory read, not after the stores.
// Every mbarrier wait is bounded; a wait that gives up records itself in the
// device status word, every role stops, and the CTA waits (bounded) for its
// copies and MMAs in flight before it frees its tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "device_common.cuh"
#include "gemm_mxfp8.h"

namespace mxn {

// Process-wide switch of the tile shape (mxnorm_set_gemm_tiles): 0 (default)
// = 256 x 192 single-CTA tiles where M % 256 == 0 and N % 384 == 0, else 128 x
// 256; 1 = 256 x 256 tiles on CTA pairs where M % 256 == 0; 2 = 128 x 256
// single-CTA tiles.  Measured on B200 at 8192 x 6144 x 4096 (20-launch graphs,
// interleaved, median): 179 us for 256 x 192, 193 us for 128 x 256 and 216 us
// for the pairs, which move a third fewer operand bytes from L2 than 128 x 256
// but stall on the pair's coupling.
static int g_gemm_tiles = 0;
void gemm_mxfp8_set_tiles(int mode) { g_gemm_tiles = mode; }

namespace {

constexpr int kTileM = 128, kTileN = 256, kTileK = 128;  // K elements (= bytes) per stage
constexpr int kStages = 4;
constexpr int kEpiWarps = 8;                     // 4 lane quarters x 2 column halves
constexpr int kThreads = 64 + 32 * kEpiWarps;    // producer warp, MMA warp, epilogue warps
constexpr uint32_t kABytes = kTileM * kTileK;    // 16 KiB
constexpr uint32_t kBBytes = kTileN * kTileK;    // 32 KiB
constexpr uint32_t kSfaBytes = 512;              // one 128 x 4 scale atom
constexpr uint32_t kSfbBytes = 1024;             // two atoms (256 rows)
constexpr uint32_t kStageTx = kABytes + kBBytes + kSfaBytes + kSfbBytes;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;                  // accumulator: columns 0..255
constexpr uint32_t kSfCol0 = 256;                // scales: 12 columns per stage

struct Smem {
  uint8_t a[kStages][kABytes];                   // 1024-aligned (128B swizzle atoms)
  uint8_t b[kStages][kBBytes];
  uint8_t sfa[kStages][kSfaBytes];
  uint8_t sfb[kStages][kSfbBytes];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full;                             // MMA -> epilogue (tcgen05.commit)
  uint64_t acc_empty;                            // epilogue warps -> MMA
  uint64_t mma_done;                             // every MMA of this CTA retired
  uint32_t tmem_base;
  uint32_t failed;
  alignas(128) uint8_t cstage[kEpiWarps][32 * 64];            // per epilogue warp: 32 rows x 32 bf16 of C
};

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void bulk_g2s_plain(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Shared-memory matrix descriptor (tcgen05): start >> 4 in bits 0..13,
// leading byte offset >> 4 in 16..29, stride byte offset >> 4 in 32..45,
// version 1 in 46..47, layout type in 61..63 (2 = 128-byte swizzle, 0 = none).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}

// Instruction descriptor of kind::mxf8f6f4 with E8M0 block scales:
// A, B E4M3 (format 0), both K-major, N >> 3 in bits 17..22, scale format
// E8M0 in bit 23, M >> 4 in bits 24..28; scale-factor byte ids in 4..5 (B)
// and 29..30 (A); dense, K = 32.
__device__ __forceinline__ uint32_t instr_desc(uint32_t sf_id) {
  return (sf_id << 4) | ((uint32_t)(kTileN >> 3) << 17) | (1u << 23) | ((uint32_t)(kTileM >> 4) << 24) |
         (sf_id << 29);
}

__device__ __forceinline__ void mma_mxf8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

__device__ __forceinline__ void tmem_cp_sf(uint32_t tmem, uint64_t src_desc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(tmem), "l"(src_desc) : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 accumulator columns of this warp's 32 lanes (no wait).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// Orders every later use of r after the tensor-memory loads have landed: the
// first call carries the wait, and each call rewrites its registers, so the
// compiler cannot move a read of them above it.
__device__ __forceinline__ void tmem_ld_fence(uint32_t (&r)[32], bool wait) {
#define MXN_R32 "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), \
                "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),      \
                "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),     \
                "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),     \
                "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
  if (wait)
    asm volatile("tcgen05.wait::ld.sync.aligned;" : MXN_R32 :: "memory");
  else
    asm volatile("" : MXN_R32 :: "memory");
#undef MXN_R32
}

__device__ __forceinline__ bool failed_flag(const Smem& S) {
  return *reinterpret_cast<const volatile uint32_t*>(&S.failed) != 0;
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_mxfp8_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                      const uint8_t* __restrict__ a_s, const uint8_t* __restrict__ b_s,
                      uint16_t* __restrict__ c, int M, int N, int K, unsigned* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = M / kTileM;
  const int n_tiles_all = m_tiles * (N / kTileN);
  const int n_k = K / kTileK;
  const int kp4 = K / 32;                       // scale columns (K % 128 == 0, so already a multiple of 4)

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    mbar_init(&S.acc_full, 1);
    mbar_init(&S.acc_empty, kEpiWarps);
    mbar_init(&S.mma_done, 1);
    S.failed = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&S.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  // Programmatic dependent launch: the set-up above overlaps the previous
  // kernel's tail; operands are read and C written only after it completed.
  griddep_wait();
  griddep_launch_dependents();

  uint32_t n_issued = 0;                        // producer: stages issued
  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer
      uint32_t g = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles_all && ok; t += gridDim.x) {
        const int mt = t % m_tiles, nt = t / m_tiles;
        for (int kb = 0; kb < n_k; ++kb, ++g) {
          const int s = (int)(g % kStages);
          const uint32_t ph = (g / kStages) & 1u;
          if (!mbar_wait_bounded(&S.empty[s], ph ^ 1u, status) || failed_flag(S)) {
            atomicOr(&S.failed, 1u);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&S.full[s], kStageTx);
          tma_load_2d(S.a[s], &map_a, kb * kTileK, mt * kTileM, &S.full[s]);
          tma_load_2d(S.b[s], &map_b, kb * kTileK, nt * kTileN, &S.full[s]);
          // scale atoms: (row tile, 4-block group) -> 512 contiguous bytes
          bulk_g2s_plain(S.sfa[s], a_s + ((size_t)mt * (kp4 / 4) + kb) * 512, kSfaBytes, &S.full[s]);
          bulk_g2s_plain(S.sfb[s], b_s + ((size_t)(2 * nt) * (kp4 / 4) + kb) * 512, 512, &S.full[s]);
          bulk_g2s_plain(S.sfb[s] + 512, b_s + ((size_t)(2 * nt + 1) * (kp4 / 4) + kb) * 512, 512, &S.full[s]);
          n_issued = g + 1;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------- MMA
      uint32_t g = 0, it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles_all && ok; t += gridDim.x, ++it) {
        if (!mbar_wait_bounded(&S.acc_empty, (it & 1u) ^ 1u, status) || failed_flag(S)) {
          atomicOr(&S.failed, 1u);
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < n_k; ++kb, ++g) {
          const int s = (int)(g % kStages);
          const uint32_t ph = (g / kStages) & 1u;
          if (!mbar_wait_bounded(&S.full[s], ph, status) || failed_flag(S)) {
            atomicOr(&S.failed, 1u);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_col = kSfCol0 + (uint32_t)s * 12u, sfb_col = sfa_col + 4u;
          // scale atoms -> tensor memory: 32 rows x 16 B each, 8-row core matrices 128 B apart
          tmem_cp_sf(tmem + sfa_col, smem_desc(smem_u32(S.sfa[s]), 0, 128, 0));
          tmem_cp_sf(tmem + sfb_col, smem_desc(smem_u32(S.sfb[s]), 0, 128, 0));
          tmem_cp_sf(tmem + sfb_col + 4u, smem_desc(smem_u32(S.sfb[s] + 512), 0, 128, 0));
          const uint32_t a0 = smem_u32(S.a[s]), b0 = smem_u32(S.b[s]);
#pragma unroll
          for (int k = 0; k < kTileK / 32; ++k) {
            // 32 bytes further along the 128-byte swizzled rows; 8-row atoms 1024 B apart
            const uint64_t ad = smem_desc(a0 + 32u * k, 16, 1024, 2);
            const uint64_t bd = smem_desc(b0 + 32u * k, 16, 1024, 2);
            mma_mxf8(tmem + kAccCol, ad, bd, instr_desc((uint32_t)k),
                     (tmem + sfa_col) | ((uint32_t)k << 30), (tmem + sfb_col) | ((uint32_t)k << 30),
                     (kb > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit(&S.empty[s]);                // stage free once these MMAs retire
        }
        if (ok) tc_commit(&S.acc_full);          // the tile's accumulator is complete
      }
      tc_commit(&S.mma_done);                    // arrives once every MMA above has retired
      if (!ok) tc_commit(&S.acc_full);           // wake the epilogue; it sees the failure
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 2;
    const int quarter = warp & 3;                // tcgen05.ld reaches lanes 32 * (warp % 4) ..
    const int half = e >> 2;                     // columns 128 * half ..
    uint32_t it = 0;
    for (int t = blockIdx.x; t < n_tiles_all; t += gridDim.x, ++it) {
      const int mt = t % m_tiles, nt = t / m_tiles;
      const bool got = mbar_wait_bounded(&S.acc_full, it & 1u, status);
      tc_fence_after();
      if (!got || failed_flag(S)) {
        if (lane == 0) atomicOr(&S.failed, 1u);
        break;
      }
      uint32_t r[4][32];
      const uint32_t ta = tmem + kAccCol + (uint32_t)(half * 128) + ((uint32_t)(quarter * 32) << 16);
#pragma unroll
      for (int j = 0; j < 4; ++j) tmem_ld32(ta + 32u * j, r[j]);
      tmem_ld_fence(r[0], true);
#pragma unroll
      for (int j = 1; j < 4; ++j) tmem_ld_fence(r[j], false);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.acc_empty);  // the MMA thread may overwrite the accumulator
      // Each 32-column slice goes through the warp's staging buffer: lane l
      // writes its row (64 B, 16-byte chunk c at chunk c ^ ((l >> 1) & 3)), then
      // the warp writes 8 rows x 64 B per store instruction, whole sectors.
      uint8_t* stg = S.cstage[e];
      const uint32_t stg_u32 = smem_u32(stg);
      uint16_t* ctile = c + (size_t)(mt * kTileM + quarter * 32) * N + (size_t)nt * kTileN + half * 128;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t o[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[j][2 * i]), __uint_as_float(r[j][2 * i + 1]));
          o[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        __syncwarp();                              // the previous slice's reads are done
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint32_t off = (uint32_t)lane * 64u + (uint32_t)((v ^ ((lane >> 1) & 3)) * 16);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(stg_u32 + off), "r"(o[4 * v]),
                       "r"(o[4 * v + 1]), "r"(o[4 * v + 2]), "r"(o[4 * v + 3])
                       : "memory");
        }
        __syncwarp();
#pragma unroll
        for (int t2 = 0; t2 < 4; ++t2) {
          const int rr = t2 * 8 + (lane >> 2), cc = lane & 3;
          const uint4 v4 = lds128(stg_u32 + (uint32_t)rr * 64u + (uint32_t)((cc ^ ((rr >> 1) & 3)) * 16));
          *reinterpret_cast<uint4*>(ctile + (size_t)rr * N + 32 * j + 8 * cc) = v4;
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1 && lane == 0) mbar_wait_bounded(&S.mma_done, 0, status);
  // After a wait gave up, leave no copy in flight: the producer waits (bounded)
  // for the last issued phase of every stage.
  if (warp == 0 && lane == 0 && failed_flag(S))
    for (uint32_t j = (n_issued > (uint32_t)kStages ? n_issued - kStages : 0); j < n_issued; ++j)
      mbar_wait_bounded(&S.full[j % kStages], (j / kStages) & 1u, status);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

// ------------------------------------------------------------------ 2-SM tiles
//
// The same product on CTA pairs (a cluster of two CTAs on two SMs): each pair
// owns a 256 x 256 output tile.  CTA r of the pair loads A rows 128 r .. of the
// tile and B rows (output columns) 128 r .. of the tile into its own shared
// memory, with their scale atoms; one thread of CTA 0 issues
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 32), which reads A and B
// from both CTAs' shared memory at the same offsets and accumulates rows
// 128 r .. 128 r + 127 of the tile, all 256 columns, in CTA r's tensor memory.
// Per output element the pair moves half the B operand a single-CTA 128 x 256
// tile does: the L2 -> SM operand stream falls from (128 + 256) / (128 * 256)
// to (256 + 256) / (256 * 256) bytes per output per K step, a third less.
// Scales: CTA r holds the atom of its 128 A rows, and both B atoms of the tile
// (all 256 columns: each CTA's accumulator spans every column), measured on
// B200 -- with only its own B atom the other 128 columns came out wrong.
//  * Both CTAs' tensor copies complete on CTA 0's "full" barrier (.cta_group::2
//    copies; the barrier address is CTA 0's, found with mapa), which expects
//    both halves' bytes.
//  * CTA 0's MMA thread copies each CTA's scale atoms into that CTA's tensor
//    memory (tcgen05.cp.cta_group::2), issues the MMAs and frees the stage in
//    both CTAs with one tcgen05.commit per CTA (no multicast).
//  * The epilogue warps of both CTAs read their own accumulator half and
//    arrive on CTA 0's "accumulator empty" barrier (remote arrive from CTA 1).
// Tensor memory is allocated and freed as a pair (tcgen05.alloc/dealloc
// .cta_group::2 by warp 0 of both CTAs); a cluster barrier after set-up and
// another before the free order everything that crosses the pair.  Every
// mbarrier wait is bounded as in the single-CTA kernel.

constexpr int kStages2 = 6;
constexpr uint32_t kHalfBytes = 128 * kTileK;                // 16 KiB: 128 rows of A or of B
constexpr uint32_t kAtomBytes = 512;                         // one 128 x 4 scale atom
constexpr uint32_t kStageTx2 = 2u * (2u * kHalfBytes + 3u * kAtomBytes);   // both CTAs' bytes
constexpr uint32_t kSfCol2 = 256;                            // scales: 12 columns per stage

struct Smem2 {
  uint8_t a[kStages2][kHalfBytes];                           // 1024-aligned (128B swizzle atoms)
  uint8_t b[kStages2][kHalfBytes];
  uint8_t sfa[kStages2][kAtomBytes];                         // this CTA's 128 A rows
  uint8_t sfb[kStages2][2 * kAtomBytes];                     // all 256 B rows of the tile
  uint64_t full[kStages2];                                   // CTA 0's: both halves' bytes
  uint64_t empty[kStages2];                                  // each CTA's own
  uint64_t acc_full;                                         // each CTA's own
  uint64_t acc_empty;                                        // CTA 0's: both CTAs' epilogue warps
  uint64_t mma_done;                                         // CTA 0's
  uint32_t tmem_base;
  uint32_t failed;
  alignas(128) uint8_t cstage[kEpiWarps][32 * 64];
};

__device__ __forceinline__ bool failed_flag2(const Smem2& S) {
  return *reinterpret_cast<const volatile uint32_t*>(&S.failed) != 0;
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t n_clusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// Shared::cluster address of this CTA's shared-memory location `p` in CTA `rank`.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// 2-D tensor copy into this CTA's shared memory, completing on the mbarrier at
// shared::cluster address `bar` (CTA 0's).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void mma_mxf8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

__device__ __forceinline__ void tmem_cp_sf_pair(uint32_t tmem, uint64_t src_desc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(tmem), "l"(src_desc) : "memory");
}

// Arrive on the mbarrier at shared::cluster address `bar` once every prior
// tcgen05 operation of this thread has completed.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Instruction descriptor of the pair MMA: M = 256, N = 256, otherwise as instr_desc.
__device__ __forceinline__ uint32_t instr_desc_pair(uint32_t sf_id) {
  return (sf_id << 4) | ((uint32_t)(256 >> 3) << 17) | (1u << 23) | ((uint32_t)(256 >> 4) << 24) | (sf_id << 29);
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_mxfp8_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                           const __grid_constant__ CUtensorMap map_sa, const __grid_constant__ CUtensorMap map_sb,
                           uint16_t* __restrict__ c, int M, int N, int K, unsigned* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // A launch without a two-CTA cluster would make the paired allocation below
  // wait for a partner that does not exist: refuse it before anything else.
  if (cluster_size() != 2) {
    if (threadIdx.x == 0) atomicOr(status, kStatusWaitTimeout);
    return;
  }
  Smem2& S = *reinterpret_cast<Smem2*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int m_tiles = M / 256;
  const int n_tiles_all = m_tiles * (N / 256);
  const int n_k = K / kTileK;
  const int kp4 = K / 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages2; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    mbar_init(&S.acc_full, 1);
    mbar_init(&S.acc_empty, 2 * kEpiWarps);
    mbar_init(&S.mma_done, 1);
    S.failed = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&S.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();                           // both CTAs' barriers and allocation are in place
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  griddep_wait();
  griddep_launch_dependents();

  const uint32_t cid = cluster_id_x(), ncl = n_clusters_x();
  uint32_t n_issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      // ----------------------------------------------------- producer (both CTAs)
      uint32_t g = 0;
      bool ok = true;
      for (int t = (int)cid; t < n_tiles_all && ok; t += (int)ncl) {
        const int mt = t % m_tiles, nt = t / m_tiles;
        const int arow = mt * 256 + (int)rank * 128, brow = nt * 256 + (int)rank * 128;
        const int atile = 2 * mt + (int)rank;                                  // 128-row scale tiles
        for (int kb = 0; kb < n_k; ++kb, ++g) {
          const int s = (int)(g % kStages2);
          const uint32_t ph = (g / kStages2) & 1u;
          if (!mbar_wait_bounded(&S.empty[s], ph ^ 1u, status) || failed_flag2(S)) {
            atomicOr(&S.failed, 1u);
            ok = false;
            break;
          }
          const uint32_t bar0 = cluster_addr(&S.full[s], 0);
          if (rank == 0) mbar_arrive_expect_tx(&S.full[s], kStageTx2);
          tma_load_2d_pair(S.a[s], &map_a, kb * kTileK, arow, bar0);
          tma_load_2d_pair(S.b[s], &map_b, kb * kTileK, brow, bar0);
          // scale atoms: atom (tile, kb) is rows 4 * (tile * kp4 / 4 + kb) .. + 3 of the 128-byte-row view
          tma_load_2d_pair(S.sfa[s], &map_sa, 0, 4 * (atile * (kp4 / 4) + kb), bar0);
          tma_load_2d_pair(S.sfb[s], &map_sb, 0, 4 * ((2 * nt) * (kp4 / 4) + kb), bar0);
          tma_load_2d_pair(S.sfb[s] + kAtomBytes, &map_sb, 0, 4 * ((2 * nt + 1) * (kp4 / 4) + kb), bar0);
          n_issued = g + 1;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------- MMA (CTA 0)
      const uint32_t empty1_base = cluster_addr(&S.empty[0], 1);
      const uint32_t acc_full1 = cluster_addr(&S.acc_full, 1);
      uint32_t g = 0, it = 0;
      bool ok = true;
      for (int t = (int)cid; t < n_tiles_all && ok; t += (int)ncl, ++it) {
        if (!mbar_wait_bounded(&S.acc_empty, (it & 1u) ^ 1u, status) || failed_flag2(S)) {
          atomicOr(&S.failed, 1u);
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < n_k; ++kb, ++g) {
          const int s = (int)(g % kStages2);
          const uint32_t ph = (g / kStages2) & 1u;
          if (!mbar_wait_bounded(&S.full[s], ph, status) || failed_flag2(S)) {
            atomicOr(&S.failed, 1u);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_col = kSfCol2 + (uint32_t)s * 12u, sfb_col = sfa_col + 4u;
          tmem_cp_sf_pair(tmem + sfa_col, smem_desc(smem_u32(S.sfa[s]), 0, 128, 0));
          tmem_cp_sf_pair(tmem + sfb_col, smem_desc(smem_u32(S.sfb[s]), 0, 128, 0));
          tmem_cp_sf_pair(tmem + sfb_col + 4u, smem_desc(smem_u32(S.sfb[s] + kAtomBytes), 0, 128, 0));
          const uint32_t a0 = smem_u32(S.a[s]), b0 = smem_u32(S.b[s]);
#pragma unroll
          for (int k = 0; k < kTileK / 32; ++k) {
            const uint64_t ad = smem_desc(a0 + 32u * k, 16, 1024, 2);
            const uint64_t bd = smem_desc(b0 + 32u * k, 16, 1024, 2);
            mma_mxf8_pair(tmem + kAccCol, ad, bd, instr_desc_pair((uint32_t)k),
                          (tmem + sfa_col) | ((uint32_t)k << 30), (tmem + sfb_col) | ((uint32_t)k << 30),
                          (kb > 0 || k > 0) ? 1u : 0u);
          }
          // the stage is free in both CTAs once these MMAs retire
          tc_commit_pair(smem_u32(&S.empty[s]));
          tc_commit_pair(empty1_base + (uint32_t)s * 8u);
        }
        if (ok) {
          tc_commit_pair(smem_u32(&S.acc_full));
          tc_commit_pair(acc_full1);
        }
      }
      tc_commit_pair(smem_u32(&S.mma_done));
      if (!ok) {                                 // wake both epilogues; they see the failure or time out
        tc_commit_pair(smem_u32(&S.acc_full));
        tc_commit_pair(acc_full1);
      }
    }
  } else {
    // ------------------------------------------------------ epilogue (both CTAs)
    const int e = warp - 2;
    const int quarter = warp & 3;
    const int half = e >> 2;
    const uint32_t acc_empty0 = cluster_addr(&S.acc_empty, 0);
    uint32_t it = 0;
    for (int t = (int)cid; t < n_tiles_all; t += (int)ncl, ++it) {
      const int mt = t % m_tiles, nt = t / m_tiles;
      const bool got = mbar_wait_bounded(&S.acc_full, it & 1u, status);
      tc_fence_after();
      if (!got || failed_flag2(S)) {
        if (lane == 0) atomicOr(&S.failed, 1u);
        break;
      }
      uint32_t r[4][32];
      const uint32_t ta = tmem + kAccCol + (uint32_t)(half * 128) + ((uint32_t)(quarter * 32) << 16);
#pragma unroll
      for (int j = 0; j < 4; ++j) tmem_ld32(ta + 32u * j, r[j]);
      tmem_ld_fence(r[0], true);
#pragma unroll
      for (int j = 1; j < 4; ++j) tmem_ld_fence(r[j], false);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {                           // CTA 0's MMA thread may overwrite the accumulators
        if (rank == 0) mbar_arrive(&S.acc_empty);
        else mbar_arrive_remote(acc_empty0);
      }
      uint8_t* stg = S.cstage[e];
      const uint32_t stg_u32 = smem_u32(stg);
      uint16_t* ctile = c + (size_t)(mt * 256 + (int)rank * 128 + quarter * 32) * N + (size_t)nt * 256 + half * 128;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t o[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[j][2 * i]), __uint_as_float(r[j][2 * i + 1]));
          o[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        __syncwarp();
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint32_t off = (uint32_t)lane * 64u + (uint32_t)((v ^ ((lane >> 1) & 3)) * 16);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(stg_u32 + off), "r"(o[4 * v]),
                       "r"(o[4 * v + 1]), "r"(o[4 * v + 2]), "r"(o[4 * v + 3])
                       : "memory");
        }
        __syncwarp();
#pragma unroll
        for (int t2 = 0; t2 < 4; ++t2) {
          const int rr = t2 * 8 + (lane >> 2), cc = lane & 3;
          const uint4 v4 = lds128(stg_u32 + (uint32_t)rr * 64u + (uint32_t)((cc ^ ((rr >> 1) & 3)) * 16));
          *reinterpret_cast<uint4*>(ctile + (size_t)rr * N + 32 * j + 8 * cc) = v4;
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (rank == 0 && warp == 1 && lane == 0) mbar_wait_bounded(&S.mma_done, 0, status);
  // After a failure CTA 0 waits (bounded) for the last phase of every stage
  // its producer filled: both CTAs' copies of a stage complete there.
  if (rank == 0 && warp == 0 && lane == 0 && failed_flag2(S))
    for (uint32_t j = (n_issued > (uint32_t)kStages2 ? n_issued - kStages2 : 0); j < n_issued; ++j)
      mbar_wait_bounded(&S.full[j % kStages2], (j / kStages2) & 1u, status);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();                           // no MMA, copy or remote arrive into either CTA remains
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

// ------------------------------------------------------------------ 256 x 192 tiles
//
// One CTA per SM on 256 x 192 output tiles: two M = 128 accumulators of 192
// columns each (384 of the 512 tensor-memory columns; the scales of 3 stages
// take 48 more), so each K stage's operands -- A 256 x 128 B, B 192 x 128 B --
// feed twice the MMA work of a 128 x 256 tile's 48 KiB for 56 KiB: 22% fewer
// bytes per flop from L2, which bounds the 128 x 256 kernel, and 8192 x 6144
// splits into 1024 tiles (6.9 per SM) instead of 1536 (10.4).  Needs M % 256
// == 0 and N % 384 == 0 (every tile's B rows then lie in two whole 128-row
// scale atoms).
//  * warp 0, one thread: TMA tensor copies of A (box 128 B x 256 rows) and B
//    (128 B x 192 rows) and bulk copies of the two A scale atoms and of the two
//    B atoms that cover the tile's 192 rows;
//  * warp 2, running ahead of the MMA thread: rebuilds each stage's B scales
//    in tile order (an odd N-tile starts 64 rows into its first atom: lane l's
//    16 bytes hold its 4 row groups, so the tile's rows 0..127 are groups 2, 3
//    of the first atom and 0, 1 of the second) and signals the stage ready --
//    on the MMA thread's path this cost every stage a few hundred cycles;
//  * warp 1, one thread: copies the four scale atoms into tensor memory and
//    issues, for each 32-element K step, one MMA (M 128, N 192) per
//    accumulator;
//  * warps 3..14: lane quarter (warp % 4) x 128 of the 384 accumulator
//    columns each, read, handed back, converted and stored as in the
//    128 x 256 kernel.
constexpr int kWM = 256, kWN = 192;
constexpr int kWStages = 3;
constexpr int kWEpiWarps = 12;
constexpr int kWThreads = 96 + 32 * kWEpiWarps;  // producer, MMA, scale warp, epilogue warps
constexpr uint32_t kWABytes = kWM * kTileK;     // 32 KiB
constexpr uint32_t kWBBytes = kWN * kTileK;     // 24 KiB
constexpr uint32_t kWStageTx = kWABytes + kWBBytes + 4 * kSfaBytes;
constexpr uint32_t kWSfCol0 = 384;              // scales: 16 columns per stage

struct SmemW {
  uint8_t a[kWStages][kWABytes];                // 1024-aligned (128B swizzle atoms)
  uint8_t b[kWStages][kWBBytes];
  uint8_t sfa[kWStages][2 * kSfaBytes];         // A rows 0..127, 128..255 of the tile
  uint8_t sfb[kWStages][2 * kSfaBytes];         // the two B atoms covering the tile, as stored
  uint8_t sfb_t[kWStages][2 * kSfaBytes];       // B rows 0..127, 128..191 (+ zero groups) of the tile
  uint64_t full[kWStages];
  uint64_t empty[kWStages];
  uint64_t sf_ready[kWStages];                  // scale warp -> MMA: the stage's B scales rebuilt
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t mma_done;
  uint32_t tmem_base;
  uint32_t failed;
  alignas(128) uint8_t cstage[kWEpiWarps][32 * 64];
};

__device__ __forceinline__ uint32_t instr_desc_n(uint32_t sf_id, uint32_t n) {
  return (sf_id << 4) | ((n >> 3) << 17) | (1u << 23) | ((uint32_t)(kTileM >> 4) << 24) | (sf_id << 29);
}

__device__ __forceinline__ bool failed_flag_w(const SmemW& S) {
  return *reinterpret_cast<const volatile uint32_t*>(&S.failed) != 0;
}

__global__ void __launch_bounds__(kWThreads, 1)
    gemm_mxfp8_wide_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                           const uint8_t* __restrict__ a_s, const uint8_t* __restrict__ b_s,
                           uint16_t* __restrict__ c, int M, int N, int K, unsigned* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  SmemW& S = *reinterpret_cast<SmemW*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = M / kWM;
  const int n_tiles_all = m_tiles * (N / kWN);
  const int n_k = K / kTileK;
  const int kp4 = K / 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kWStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
      mbar_init(&S.sf_ready[s], 1);
    }
    mbar_init(&S.acc_full, 1);
    mbar_init(&S.acc_empty, kWEpiWarps);
    mbar_init(&S.mma_done, 1);
    S.failed = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&S.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  griddep_wait();
  griddep_launch_dependents();

  uint32_t n_issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer
      uint32_t g = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles_all && ok; t += gridDim.x) {
        const int mt = t % m_tiles, nt = t / m_tiles;
        const int fa = (3 * nt) >> 1;            // first B scale atom of the tile's rows
        for (int kb = 0; kb < n_k; ++kb, ++g) {
          const int s = (int)(g % kWStages);
          const uint32_t ph = (g / kWStages) & 1u;
          if (!mbar_wait_bounded(&S.empty[s], ph ^ 1u, status) || failed_flag_w(S)) {
            atomicOr(&S.failed, 1u);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&S.full[s], kWStageTx);
          tma_load_2d(S.a[s], &map_a, kb * kTileK, mt * kWM, &S.full[s]);
          tma_load_2d(S.b[s], &map_b, kb * kTileK, nt * kWN, &S.full[s]);
          bulk_g2s_plain(S.sfa[s], a_s + ((size_t)(2 * mt) * (kp4 / 4) + kb) * 512, 512, &S.full[s]);
          bulk_g2s_plain(S.sfa[s] + 512, a_s + ((size_t)(2 * mt + 1) * (kp4 / 4) + kb) * 512, 512, &S.full[s]);
          bulk_g2s_plain(S.sfb[s], b_s + ((size_t)fa * (kp4 / 4) + kb) * 512, 512, &S.full[s]);
          bulk_g2s_plain(S.sfb[s] + 512, b_s + ((size_t)(fa + 1) * (kp4 / 4) + kb) * 512, 512, &S.full[s]);
          n_issued = g + 1;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------- MMA
      uint32_t g = 0, it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles_all && ok; t += gridDim.x, ++it) {
        if (!mbar_wait_bounded(&S.acc_empty, (it & 1u) ^ 1u, status) || failed_flag_w(S)) {
          atomicOr(&S.failed, 1u);
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < n_k; ++kb, ++g) {
          const int s = (int)(g % kWStages);
          const uint32_t ph = (g / kWStages) & 1u;
          if (!mbar_wait_bounded(&S.full[s], ph, status) || !mbar_wait_bounded(&S.sf_ready[s], ph, status) ||
              failed_flag_w(S)) {
            atomicOr(&S.failed, 1u);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_col = kWSfCol0 + (uint32_t)s * 16u, sfb_col = sfa_col + 8u;
          tmem_cp_sf(tmem + sfa_col, smem_desc(smem_u32(S.sfa[s]), 0, 128, 0));
          tmem_cp_sf(tmem + sfa_col + 4u, smem_desc(smem_u32(S.sfa[s] + 512), 0, 128, 0));
          tmem_cp_sf(tmem + sfb_col, smem_desc(smem_u32(S.sfb_t[s]), 0, 128, 0));
          tmem_cp_sf(tmem + sfb_col + 4u, smem_desc(smem_u32(S.sfb_t[s] + 512), 0, 128, 0));
          const uint32_t a_base = smem_u32(S.a[s]), b_base = smem_u32(S.b[s]);
#pragma unroll
          for (int k = 0; k < kTileK / 32; ++k) {
            const uint64_t bd = smem_desc(b_base + 32u * k, 16, 1024, 2);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint64_t ad = smem_desc(a_base + (uint32_t)h * (kWABytes / 2) + 32u * k, 16, 1024, 2);
              mma_mxf8(tmem + (uint32_t)(h * kWN), ad, bd, instr_desc_n((uint32_t)k, kWN),
                       (tmem + sfa_col + 4u * h) | ((uint32_t)k << 30), (tmem + sfb_col) | ((uint32_t)k << 30),
                       (kb > 0 || k > 0) ? 1u : 0u);
            }
          }
          tc_commit(&S.empty[s]);
        }
        if (ok) tc_commit(&S.acc_full);
      }
      tc_commit(&S.mma_done);
      if (!ok) tc_commit(&S.acc_full);
    }
  } else if (warp == 2) {
    // ----------------------------------------------------- B scale rebuild
    // Runs ahead of the MMA thread (see above for the row-group order).
    uint32_t g = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles_all && ok; t += gridDim.x) {
      const bool odd = ((t / m_tiles) & 1) != 0;
      for (int kb = 0; kb < n_k; ++kb, ++g) {
        const int s = (int)(g % kWStages);
        const uint32_t ph = (g / kWStages) & 1u;
        const bool w = mbar_wait_bounded(&S.full[s], ph, status) && !failed_flag_w(S);
        if (!__all_sync(0xFFFFFFFFu, w)) {
          if (lane == 0) atomicOr(&S.failed, 1u);
          ok = false;
          break;
        }
        const uint4 a0 = reinterpret_cast<const uint4*>(S.sfb[s])[lane];
        const uint4 a1 = reinterpret_cast<const uint4*>(S.sfb[s] + 512)[lane];
        const uint4 t0 = odd ? make_uint4(a0.z, a0.w, a1.x, a1.y) : a0;
        const uint4 t1 = odd ? make_uint4(a1.z, a1.w, 0u, 0u) : make_uint4(a1.x, a1.y, 0u, 0u);
        reinterpret_cast<uint4*>(S.sfb_t[s])[lane] = t0;
        reinterpret_cast<uint4*>(S.sfb_t[s] + 512)[lane] = t1;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.sf_ready[s]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 3;
    const int quarter = warp & 3;
    const int third = e >> 2;                    // accumulator columns 128 * third ..
    uint32_t it = 0;
    for (int t = blockIdx.x; t < n_tiles_all; t += gridDim.x, ++it) {
      const int mt = t % m_tiles, nt = t / m_tiles;
      const bool got = mbar_wait_bounded(&S.acc_full, it & 1u, status);
      tc_fence_after();
      if (!got || failed_flag_w(S)) {
        if (lane == 0) atomicOr(&S.failed, 1u);
        break;
      }
      uint32_t r[4][32];
      const uint32_t ta = tmem + (uint32_t)(third * 128) + ((uint32_t)(quarter * 32) << 16);
#pragma unroll
      for (int j = 0; j < 4; ++j) tmem_ld32(ta + 32u * j, r[j]);
      tmem_ld_fence(r[0], true);
#pragma unroll
      for (int j = 1; j < 4; ++j) tmem_ld_fence(r[j], false);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.acc_empty);
      uint8_t* stg = S.cstage[e];
      const uint32_t stg_u32 = smem_u32(stg);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int col = third * 128 + 32 * j;    // of the 384: accumulator col / 192, column col % 192
        const int acc = col >= kWN ? 1 : 0;
        uint16_t* ctile = c + (size_t)(mt * kWM + acc * 128 + quarter * 32) * N + (size_t)nt * kWN + (col - acc * kWN);
        uint32_t o[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const __nv_bfloat162 hv = __floats2bfloat162_rn(__uint_as_float(r[j][2 * i]), __uint_as_float(r[j][2 * i + 1]));
          o[i] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        __syncwarp();
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint32_t off = (uint32_t)lane * 64u + (uint32_t)((v ^ ((lane >> 1) & 3)) * 16);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(stg_u32 + off), "r"(o[4 * v]),
                       "r"(o[4 * v + 1]), "r"(o[4 * v + 2]), "r"(o[4 * v + 3])
                       : "memory");
        }
        __syncwarp();
#pragma unroll
        for (int t2 = 0; t2 < 4; ++t2) {
          const int rr = t2 * 8 + (lane >> 2), cc = lane & 3;
          const uint4 v4 = lds128(stg_u32 + (uint32_t)rr * 64u + (uint32_t)((cc ^ ((rr >> 1) & 3)) * 16));
          *reinterpret_cast<uint4*>(ctile + (size_t)rr * N + 8 * cc) = v4;
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1 && lane == 0) mbar_wait_bounded(&S.mma_done, 0, status);
  if (warp == 0 && lane == 0 && failed_flag_w(S))
    for (uint32_t j = (n_issued > (uint32_t)kWStages ? n_issued - kWStages : 0); j < n_issued; ++j)
      mbar_wait_bounded(&S.full[j % kWStages], (j / kWStages) & 1u, status);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D map over a row-major uint8 [rows, cols] matrix, boxes of box_rows x 128 bytes, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, int rows, int cols, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols};
  const cuuint32_t box[2] = {(cuuint32_t)kTileK, (cuuint32_t)box_rows};
  const cuuint32_t elem[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, elem,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over a scale array in the tcgen05 layout viewed as rows of 128
// bytes: one 512-byte atom is a box of 4 rows (no swizzle).
bool make_sf_map(CUtensorMap* map, const void* base, size_t bytes) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {128, (cuuint64_t)(bytes / 128)};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {128, 4};
  const cuuint32_t elem[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, elem,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Clusters of two CTAs of the pair kernel that fit on the device at once
// (0 if none), looked up once per device.
int pair_clusters(int dev) {
  static int cached[64];
  static bool have[64];
  if (dev < 0 || dev >= 64) return 0;
  if (have[dev]) return cached[dev];
  int n = 0;
  const size_t smem = sizeof(Smem2);
  if (cudaFuncSetAttribute(gemm_mxfp8_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, (const void*)gemm_mxfp8_pair_kernel, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  cached[dev] = n;
  have[dev] = true;
  return n;
}

int launch_wide(const void* a_q, const void* a_s, const void* b_q, const void* b_s, void* c, int M, int N, int K,
                int sms, unsigned* status, cudaStream_t stream, const char** why) {
  CUtensorMap ma, mb;
  if (!make_map(&ma, a_q, M, K, kWM) || !make_map(&mb, b_q, N, K, kWN)) {
    *why = "cuTensorMapEncodeTiled failed";
    return -1;
  }
  const size_t smem = sizeof(SmemW);
  cudaError_t e = cudaFuncSetAttribute(gemm_mxfp8_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) { *why = cudaGetErrorString(e); return (int)e; }
  const int tiles = (M / kWM) * (N / kWN);
  const uint8_t* as = static_cast<const uint8_t*>(a_s);
  const uint8_t* bs = static_cast<const uint8_t*>(b_s);
  uint16_t* cp = static_cast<uint16_t*>(c);
  void* argv[] = {&ma, &mb, &as, &bs, &cp, &M, &N, &K, &status};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles < sms ? tiles : sms);
  cfg.blockDim = dim3(kWThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelExC(&cfg, (const void*)gemm_mxfp8_wide_kernel, argv);
  if (e != cudaSuccess) { *why = cudaGetErrorString(e); return (int)e; }
  return 0;
}

int launch_pair(const void* a_q, const void* a_s, const void* b_q, const void* b_s, void* c, int M, int N, int K,
                int clusters, unsigned* status, cudaStream_t stream, const char** why) {
  CUtensorMap ma, mb, msa, msb;
  if (!make_map(&ma, a_q, M, K, 128) || !make_map(&mb, b_q, N, K, 128) ||
      !make_sf_map(&msa, a_s, (size_t)M * (K / 32)) || !make_sf_map(&msb, b_s, (size_t)N * (K / 32))) {
    *why = "cuTensorMapEncodeTiled failed";
    return -1;
  }
  const int tiles = (M / 256) * (N / 256);
  const int ncl = tiles < clusters ? tiles : clusters;
  uint16_t* cp = static_cast<uint16_t*>(c);
  void* argv[] = {&ma, &mb, &msa, &msb, &cp, &M, &N, &K, &status};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * ncl);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = sizeof(Smem2);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelExC(&cfg, (const void*)gemm_mxfp8_pair_kernel, argv);
  if (e != cudaSuccess) { *why = cudaGetErrorString(e); return (int)e; }
  return 0;
}

}  // namespace

size_t gemm_mxfp8_smem_bytes() { return sizeof(Smem) + 1024; }

// Launch: returns 0, or -1 (tensor map could not be encoded) / cuda error code.
int gemm_mxfp8_launch(const void* a_q, const void* a_s, const void* b_q, const void* b_s, void* c, int M,
                      int N, int K, int sms, unsigned* status, cudaStream_t stream, const char** why) {
  // 256 x 192 tiles by default where the shape allows.
  if (g_gemm_tiles == 0 && M % kWM == 0 && N % (2 * kWN) == 0)
    return launch_wide(a_q, a_s, b_q, b_s, c, M, N, K, sms, status, stream, why);
  // 256 x 256 tiles on CTA pairs where the shape allows and the device has room.
  if (M % 256 == 0 && N % 256 == 0 && g_gemm_tiles == 1) {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) {
      const int ncl = pair_clusters(dev);
      const int cap = sms / 2;
      if (ncl > 0) return launch_pair(a_q, a_s, b_q, b_s, c, M, N, K, ncl < cap ? ncl : cap, status, stream, why);
    }
  }
  CUtensorMap ma, mb;
  if (!make_map(&ma, a_q, M, K, kTileM) || !make_map(&mb, b_q, N, K, kTileN)) {
    *why = "cuTensorMapEncodeTiled failed";
    return -1;
  }
  const size_t smem = sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(gemm_mxfp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) { *why = cudaGetErrorString(e); return (int)e; }
  const int tiles = (M / kTileM) * (N / kTileN);
  const uint8_t* as = static_cast<const uint8_t*>(a_s);
  const uint8_t* bs = static_cast<const uint8_t*>(b_s);
  uint16_t* cp = static_cast<uint16_t*>(c);
  void* argv[] = {&ma, &mb, &as, &bs, &cp, &M, &N, &K, &status};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles < sms ? tiles : sms);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelExC(&cfg, (const void*)gemm_mxfp8_kernel, argv);
  if (e != cudaSuccess) { *why = cudaGetErrorString(e); return (int)e; }
  return 0;
}

int gemm_mxfp8_tile_m() { return kTileM; }
int gemm_mxfp8_tile_n() { return kTileN; }
int gemm_mxfp8_tile_k() { return kTileK; }

}  // namespace mxn
