// row_bwd.cuh -- MXNorm backward.
//
// gist.science, "MXNorm: Reusing MXFP block scales for efficient tensor
// normalisation", technical summary section 2.3: the backward reuses the
// RMSNorm gradient as a straight-through estimator (the MX cast counts as the
// identity).  With g = gamma * dy and the forward's statistic G:
//     dx     = ( g - x * (x . g) / (x . x) ) / G
//     dgamma = sum over rows of dy * x / G
// which is the exact gradient of x -> x * gamma / (c * rms(x)) at G = c * rms(x).
//
// Laid out like the forward (row_fwd.cuh):
//  * a row group of tpr threads owns one row at a time (tpr = K up to 256
//    blocks, one 32-column block per thread; rows of 257..512 blocks take 256
//    threads with two blocks each; rows under 32 blocks share a warp), so a
//    thread's dgamma partial sums for its columns stay in registers across
//    every row the group sees;
//  * each group has its own ring of stages (x rows, then dy rows) filled by
//    1-D bulk copies that the group's first thread issues, completing on the
//    group's own mbarriers;
//  * a thread copies its x and dy blocks into registers and hands the stage
//    back after the first pass over them (in a row of several warps, the last
//    warp to get there issues the refill, so no warp waits for the others); G is fetched
//    before the row's wait; products run as packed fp32 pairs; the two row
//    sums (x . x, x . g) reduce with shuffles, plus shared memory and a named
//    barrier when a row spans several warps.
// At the end the CTA adds its groups' dgamma partial sums in shared memory
// (group order, fixed) and writes one partial row to the workspace;
// dgamma_reduce_kernel then adds the CTAs' rows in a fixed order
// (deterministic, no atomics on the sums).
#pragma once

#include "row_fwd.cuh"

namespace mxn {

// Threads per CTA the register budget is sized for: one block per thread
// (x, dy, gamma and 32 accumulators in registers) fits 512 threads, two
// blocks 256.
__host__ __device__ constexpr int bwd_max_threads(int bpt) { return bpt == 1 ? 512 : 256; }

struct BwdCfg {
  int64_t T;             // rows
  int64_t n_row_blocks;  // ceil(T / rps)
  int64_t ngt;           // row groups that get rows (<= groups in the grid)
  int D, K;              // row length, MX blocks per row
  int tpr, log2_tpr;     // threads per row (power of two)
  int rps;               // rows per group and stage (> 1 only when tpr < 32)
  int gthreads;          // threads per row group = max(tpr, 32)
  int ng;                // row groups per CTA
  int stages;            // ring depth per group
  uint32_t row_bytes;    // 2 * D
  uint32_t stage_bytes;  // 2 * rps * row_bytes: rps x rows, then rps dy rows
  uint32_t gamma_bytes;  // gamma (or ones) as fp32 in shared memory, slot order
  uint32_t ring_off, bar_off, red_off;
  uint32_t ostage_bytes;  // per-group dx staging buffer (rps rows); 0: dx stored directly
  uint32_t out_off;       // offset of the staging buffers
  uint32_t cnt_off;       // per group and stage: warps done with the stage (rows of several warps)
};

struct BwdArgs {
  const uint16_t* x;      // bf16 [T, D]
  const uint16_t* dy;     // bf16 [T, D]
  const uint16_t* gamma;  // bf16 [D] or null
  const float* G;         // fp32 [T]
  uint16_t* dx;           // bf16 [T, D]
  float* partial;         // fp32 [gridDim.x, D] or null (no dgamma): one partial row per CTA
  unsigned* status;
};

// bf16 pair -> fp32 pair, as an opaque instruction pair: the second pass
// converts its operands again instead of the compiler keeping the first
// pass's 96 converted floats live (which would not fit the register budget).
__device__ __forceinline__ float2 bf16x2_to_f2_again(uint32_t u) {
  uint32_t lo, hi;
  asm volatile("shl.b32 %0, %2, 16;\n\tand.b32 %1, %2, 0xFFFF0000;" : "=r"(lo), "=r"(hi) : "r"(u));
  return make_float2(__uint_as_float(lo), __uint_as_float(hi));
}

// Issue the bulk copies of row block rb (x rows, then dy rows) into `dst`.
__device__ __forceinline__ void issue_bwd_block(const BwdArgs& A, const BwdCfg& C, int64_t rb,
                                                uint8_t* dst, uint64_t* bar, uint64_t pol) {
  const int64_t r0 = rb * C.rps;
  const int nrows = (int)(C.T - r0 < (int64_t)C.rps ? C.T - r0 : (int64_t)C.rps);
  mbar_arrive_expect_tx(bar, 2u * (uint32_t)nrows * C.row_bytes);
  for (int r = 0; r < nrows; ++r) {
    bulk_copy_g2s(dst + (size_t)r * C.row_bytes, A.x + (r0 + r) * (int64_t)C.D, C.row_bytes, bar, pol);
    bulk_copy_g2s(dst + (size_t)(C.rps + r) * C.row_bytes, A.dy + (r0 + r) * (int64_t)C.D, C.row_bytes,
                  bar, pol);
  }
}

// The two row sums of a row group (segment of W lanes, then across warps).
template <int TPR>
__device__ __forceinline__ float2 row_sum2(float2 v, const BwdCfg& C, float2* red, int bar_id, int wig,
                                           int lane) {
  const int W = TPR ? (TPR < 32 ? TPR : 32) : C.tpr;
  v.x = seg_sum(v.x, W);
  v.y = seg_sum(v.y, W);
  if (TPR > 32) {
    constexpr int nw = TPR > 32 ? TPR / 32 : 1;
    if (lane == 0) red[wig] = v;
    named_barrier_sync(bar_id, TPR);
    v = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int w = 0; w < nw; ++w) {
      v.x += red[w].x;
      v.y += red[w].y;
    }
  }
  return v;
}

template <int BPT, int TPR>
__global__ void __launch_bounds__(bwd_max_threads(BPT), 1) row_bwd_kernel(const BwdArgs A, const BwdCfg C) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tpr = TPR ? TPR : C.tpr;
  const int gthreads = TPR ? (TPR < 32 ? 32 : TPR) : 32;
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
  uint32_t* done = reinterpret_cast<uint32_t*>(smem + C.cnt_off) + (size_t)g * C.stages;
  // dx goes through the group's staging buffer and out with one bulk copy per
  // row block (full, contiguous lines instead of each thread's 16-byte
  // pieces), when the plan gives one.
  const bool bulk_out = C.ostage_bytes != 0;
  const uint32_t ostage = smem_u32(smem + C.out_off + (size_t)g * C.ostage_bytes);

  const int64_t gg = (int64_t)g * gridDim.x + blockIdx.x;
  const int64_t rb_end = gg < C.ngt ? C.n_row_blocks : 0;
  const uint64_t pol = policy_evict_first();
  if (issuer) {
    for (int s = 0; s < C.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], n_gwarps);
      done[s] = 0u;
    }
    fence_barrier_init();
  }
  griddep_wait();
  griddep_launch_dependents();
  if (issuer) {
    for (int s = 0; s < C.stages; ++s) {
      const int64_t rb = gg + (int64_t)s * C.ngt;
      if (rb < rb_end) issue_bwd_block(A, C, rb, ring + (size_t)s * C.stage_bytes, &full[s], pol);
    }
  }

  // gamma (ones when NULL) into shared memory once per CTA, as fp32 in slot
  // order: the first and second halves of x chunk slot j of block k at
  // ((2j + h) * K + k) * 16, so a warp's reads of one slot fall on
  // consecutive words and no thread converts gamma per row (registers stay
  // free for x, dy and the dgamma sums).
  const int rot = (tg >> 1) & 3;
  for (int i = tid; i < C.K * 4; i += blockDim.x) {
    const int k = i >> 2, j = i & 3;
    const int c = (j + (k >> 1)) & 3;
    uint4 v = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    if (A.gamma != nullptr) v = ldg128_nc(A.gamma + (size_t)k * kBlock + c * 8);
    *reinterpret_cast<float4*>(smem + ((size_t)(2 * j) * C.K + k) * 16) =
        make_float4(bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y));
    *reinterpret_cast<float4*>(smem + ((size_t)(2 * j + 1) * C.K + k) * 16) =
        make_float4(bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w));
  }
  float acc[BPT][32];
#pragma unroll
  for (int b = 0; b < BPT; ++b)
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[b][i] = 0.0f;
  __syncthreads();                          // barrier set-up visible to every thread

  bool ok = true;
  int par = 0;
  const int bar_id = 1 + g;
  int64_t it = 0;
  // G of the group's next row is loaded one row ahead.
  float G_next = (gg < rb_end && gg * C.rps + rs < C.T) ? ldg_f32_early(A.G + gg * C.rps + rs) : 0.0f;
  for (int64_t rb = gg; rb < rb_end; rb += C.ngt, ++it, par ^= 1) {
    const int s = (int)(it % C.stages);
    const uint32_t ph = (uint32_t)((it / C.stages) & 1);
    const int64_t row = rb * C.rps + rs;
    const bool valid = row < C.T;
    const float G = G_next;
    const int64_t row_n = (rb + C.ngt) * C.rps + rs;
    G_next = (rb + C.ngt < rb_end && row_n < C.T) ? ldg_f32_early(A.G + row_n) : 0.0f;
    if (ok) ok = mbar_wait_bounded(&full[s], ph, A.status);
    const uint8_t* st = ring + (size_t)s * C.stage_bytes;
    const uint32_t sx = smem_u32(st + (size_t)rs * C.row_bytes);
    const uint32_t sd = smem_u32(st + (size_t)(C.rps + rs) * C.row_bytes);

    // The staging buffer is free again once the previous row block's bulk
    // copy has read it; the group learns it at the __syncwarp below, or at
    // the row sum's named barrier for rows of several warps.
    if (bulk_out && issuer) bulk_wait_read_all();
    // ---- x and dy into registers
    uint32_t xr[BPT][16], dr[BPT][16];
#pragma unroll
    for (int b = 0; b < BPT; ++b) {
      const int k = tg + b * tpr;
      const bool have = valid && k < C.K;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t off = (uint32_t)k * 64u + (uint32_t)(((j + rot) & 3) * 16);
        uint4 a = make_uint4(0u, 0u, 0u, 0u), d = make_uint4(0u, 0u, 0u, 0u);
        if (have) { a = lds128(sx + off); d = lds128(sd + off); }
        xr[b][4 * j] = a.x; xr[b][4 * j + 1] = a.y; xr[b][4 * j + 2] = a.z; xr[b][4 * j + 3] = a.w;
        dr[b][4 * j] = d.x; dr[b][4 * j + 1] = d.y; dr[b][4 * j + 2] = d.z; dr[b][4 * j + 3] = d.w;
      }
    }
    const int64_t nrb = rb + (int64_t)C.stages * C.ngt;

    // ---- pass 1: x . x and x . g (g = gamma * dy), and the dgamma partials
    // dy * x / G (they need only G, which is known before the row arrives).
    // dy * x is exact in fp32 (two 8-bit significands), so x . g adds the
    // same exact terms x * gamma * dy as a sum over x * (gamma * dy) would.
    const float invG = (G != 0.0f) ? __frcp_rn(G) : 0.0f;
    const float2 invG2 = make_float2(invG, invG);
    float2 xx = make_float2(0.0f, 0.0f), xg = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int b = 0; b < BPT; ++b) {
      const int kk = (tg + b * tpr) < C.K ? tg + b * tpr : C.K - 1;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float2 gf[4];
        gamma_slot<true>(smem, C.K, j, kk, gf);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int w = 4 * j + i;
          const float2 x2 = bf16x2_to_f2(xr[b][w]);
          const float2 p2 = mul2(bf16x2_to_f2(dr[b][w]), x2);
          xx = fma2(x2, x2, xx);
          xg = fma2(p2, gf[i], xg);
          const float2 a2 = fma2(p2, invG2, make_float2(acc[b][2 * w], acc[b][2 * w + 1]));
          acc[b][2 * w] = a2.x;
          acc[b][2 * w + 1] = a2.y;
        }
      }
    }
    // Refill, once pass 1 has used every register read from the stage (so
    // those shared-memory reads are complete) and behind a proxy fence that
    // orders them before the bulk copy overwriting the stage.  A one-warp row
    // refills at once; in a row of several warps each warp counts itself done,
    // and the one that completes the count issues the refill (the
    // acquire-release add orders every warp's reads before it).
    fence_proxy_async_smem();
    __syncwarp();
    if constexpr (TPR > 32) {
      if (lane == 0 && smem_add_acq_rel(&done[s], 1u) == (uint32_t)(n_gwarps - 1)) {
        done[s] = 0u;   // next added to after this stage's next fill completes
        if (ok && nrb < C.n_row_blocks) issue_bwd_block(A, C, nrb, ring + (size_t)s * C.stage_bytes, &full[s], pol);
      }
    } else {
      if (lane == 0) mbar_arrive(&empty[s]);
      if (issuer && nrb < C.n_row_blocks) {
        if (ok) ok = mbar_wait_bounded(&empty[s], ph, A.status);
        if (ok) issue_bwd_block(A, C, nrb, ring + (size_t)s * C.stage_bytes, &full[s], pol);
      }
    }
    const float2 tot = row_sum2<TPR>(make_float2(xx.x + xx.y, xg.x + xg.y), C, red + par * kRedSlots,
                                     bar_id, wig, lane);

    // ---- pass 2: dx (zero for a row with G = 0 or x = 0)
    const bool live = valid && (G != 0.0f) && (tot.x != 0.0f);
    const float coef = live ? tot.y / tot.x : 0.0f;
    const float sdx = live ? invG : 0.0f;
    const float2 ncoef2 = make_float2(-coef, -coef), sdx2 = make_float2(sdx, sdx);
#pragma unroll
    for (int b = 0; b < BPT; ++b) {
      const int k = tg + b * tpr;
      const bool blk = valid && k < C.K;
      uint16_t* dxrow = A.dx + row * (int64_t)C.D + (int64_t)k * kBlock;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int kk = k < C.K ? k : C.K - 1;
        float2 gf[4];
        gamma_slot<true>(smem, C.K, j, kk, gf);
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int w = 4 * j + i;
          const float2 x2 = bf16x2_to_f2_again(xr[b][w]);
          const float2 g2 = mul2(gf[i], bf16x2_to_f2_again(dr[b][w]));
          const float2 r = mul2(fma2(x2, ncoef2, g2), sdx2);
          const __nv_bfloat162 h = __floats2bfloat162_rn(r.x, r.y);
          o[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        if (blk) {
          if (bulk_out)
            sts128(ostage + (uint32_t)(rs * C.D + k * kBlock + ((j + rot) & 3) * 8) * 2u,
                   make_uint4(o[0], o[1], o[2], o[3]));
          else
            stg128_stream(dxrow + ((j + rot) & 3) * 8, make_uint4(o[0], o[1], o[2], o[3]));
        }
      }
    }
    if (bulk_out) {
      fence_proxy_async_smem();
      if (TPR > 32) named_barrier_sync(bar_id, TPR);
      else __syncwarp();
      if (issuer) {
        const int64_t r0 = rb * C.rps;
        const int64_t nrows = C.T - r0 < (int64_t)C.rps ? C.T - r0 : (int64_t)C.rps;
        bulk_copy_s2g(A.dx + r0 * (int64_t)C.D, ostage, (uint32_t)nrows * C.row_bytes);
        bulk_commit();
      }
    }
  }
  if (bulk_out && issuer) bulk_wait_read_all();   // staging buffers read before exit
  // Leave no copy in flight: the issuer waits for the last phase of every stage
  // filled (already complete unless a wait gave up above).
  if (issuer && !ok) {
    for (int s = 0; s < C.stages; ++s) {
      const int64_t last_it = it - 1 - ((it - 1 - s) % C.stages + C.stages) % C.stages;
      if (last_it >= 0) mbar_wait_bounded(&full[s], (uint32_t)((last_it / C.stages) & 1), A.status);
    }
  }
  if (A.partial == nullptr) return;

  // ---- the CTA's partial dgamma row.  Rows sharing a warp first fold their
  // row slots together (xor butterfly over the slot bits of the lane); each
  // group then puts its sums into its own idle ring (D floats fit in one
  // stage), and the CTA adds the groups in group order.
  if (TPR == 0) {
    for (int m = tpr; m < 32; m <<= 1) {
#pragma unroll
      for (int b = 0; b < BPT; ++b)
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[b][i] += __shfl_xor_sync(0xFFFFFFFFu, acc[b][i], m);
    }
  }
  __syncthreads();                          // every group is past its last row
  float* gsum = reinterpret_cast<float*>(smem + C.ring_off);   // row g at g * stages * stage_bytes
  const size_t gstride = (size_t)C.stages * C.stage_bytes / sizeof(float);
  if (rs == 0) {
#pragma unroll
    for (int b = 0; b < BPT; ++b) {
      const int k = tg + b * tpr;
      if (k < C.K) {
        float* prow = gsum + (size_t)g * gstride + (size_t)k * kBlock;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float* p = prow + ((j + rot) & 3) * 8;
          reinterpret_cast<float4*>(p)[0] = make_float4(acc[b][8 * j], acc[b][8 * j + 1], acc[b][8 * j + 2],
                                                        acc[b][8 * j + 3]);
          reinterpret_cast<float4*>(p)[1] = make_float4(acc[b][8 * j + 4], acc[b][8 * j + 5],
                                                        acc[b][8 * j + 6], acc[b][8 * j + 7]);
        }
      }
    }
  }
  __syncthreads();
  float4* out = reinterpret_cast<float4*>(A.partial + (int64_t)blockIdx.x * C.D);
  for (int c = tid; c < C.D / 4; c += blockDim.x) {
    float4 v = reinterpret_cast<const float4*>(gsum)[c];
    for (int q = 1; q < C.ng; ++q) {
      const float4 w = reinterpret_cast<const float4*>(gsum + (size_t)q * gstride)[c];
      v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
    }
    out[c] = v;
  }
}

// dgamma[j] = sum over the n_part partial rows, in a fixed order: thread
// (tx, ty) of a 32 x 32 CTA adds rows ty, ty + 32, ... of column j = 32 *
// blockIdx.x + tx (eight rows' loads in flight at a time, added in row
// order); the 32 lane sums are then added in ty order.
__global__ void __launch_bounds__(1024) dgamma_reduce_kernel(const float* partial, int64_t n_part,
                                                             int D, uint16_t* dgamma) {
  __shared__ float sh[32][33];
  griddep_wait();                  // the backward kernel's partial rows are complete
  griddep_launch_dependents();     // the next kernel may start its set-up
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int j = blockIdx.x * 32 + tx;
  float s = 0.0f;
  if (j < D) {
    for (int64_t r0 = ty; r0 < n_part; r0 += 8 * 32) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t r = r0 + 32 * u;
        v[u] = r < n_part ? partial[r * D + j] : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) s += v[u];
    }
  }
  sh[ty][tx] = s;
  __syncthreads();
  if (ty == 0 && j < D) {
    float t = 0.0f;
    for (int i = 0; i < 32; ++i) t += sh[i][tx];
    const __nv_bfloat16 h = __float2bfloat16_rn(t);
    dgamma[j] = *reinterpret_cast<const uint16_t*>(&h);
  }
}

// The instantiation for (blocks per thread, threads per row).
inline const void* pick_bwd_shape(int bpt, int tpr) {
  if (bpt == 2) return tpr == 256 ? (const void*)row_bwd_kernel<2, 256> : nullptr;
  if (bpt != 1) return nullptr;
  if (tpr < 32) return (const void*)row_bwd_kernel<1, 0>;
  switch (tpr) {
    case 32: return (const void*)row_bwd_kernel<1, 32>;
    case 64: return (const void*)row_bwd_kernel<1, 64>;
    case 128: return (const void*)row_bwd_kernel<1, 128>;
    case 256: return (const void*)row_bwd_kernel<1, 256>;
    default: return nullptr;
  }
}

}  // namespace mxn
