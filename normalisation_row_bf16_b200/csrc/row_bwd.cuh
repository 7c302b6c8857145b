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
// Same pipeline as the forward (row_fwd.cuh): a producer thread streams the x
// row and the dy row of each row block into a shared-memory stage with 1-D
// bulk copies; a consumer thread owns one 32-column block of every row it
// sees, so its dgamma partial sums stay in registers across rows.  At the end
// every row group writes its partial row to the workspace; a second kernel adds
// the partial rows in a fixed order (deterministic, no atomics).
#pragma once

#include "row_fwd.cuh"

namespace mxn {

constexpr int kMaxConsumerThreads = 512;

// Launch shape of the backward: one consumer thread per 32-column block, rows
// grouped rps per stage, one producer warp per CTA.
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
  uint32_t stage_bytes;  // rps * row_bytes * 2 (x and dy)
};

// Resident CTAs per SM the register budget is sized for, by consumer threads
// per CTA (each CTA adds one producer warp).
template <int NCT>
struct CtaShape {
  static constexpr int threads = NCT + 32;
};

struct BwdArgs {
  const uint16_t* x;      // bf16 [T, D]
  const uint16_t* dy;     // bf16 [T, D]
  const uint16_t* gamma;  // bf16 [D] or null
  const float* G;         // fp32 [T]
  uint16_t* dx;           // bf16 [T, D]
  float* partial;         // fp32 [gridDim.x * rps, D] or null (no dgamma)
  unsigned* status;
};

__device__ __forceinline__ void produce_rows2(const uint16_t* x, const uint16_t* dy,
                                              const RowCfg& C, uint8_t* stage0, uint64_t* full,
                                              uint64_t* empty, unsigned* status) {
  const uint64_t pol = policy_evict_first();
  int64_t it = 0;
  for (int64_t rb = blockIdx.x; rb < C.n_row_blocks; rb += gridDim.x, ++it) {
    const int s = (int)(it % C.stages);
    const uint32_t ph = (uint32_t)((it / C.stages) & 1);
    if (!mbar_wait_bounded(&empty[s], ph ^ 1u, status)) break;
    const int64_t r0 = rb * C.rps;
    const int nrows = (int)(C.T - r0 < (int64_t)C.rps ? C.T - r0 : (int64_t)C.rps);
    mbar_arrive_expect_tx(&full[s], 2u * (uint32_t)nrows * C.row_bytes);
    uint8_t* dst = stage0 + (size_t)s * C.stage_bytes;
    for (int r = 0; r < nrows; ++r) {
      bulk_copy_g2s(dst + (size_t)r * C.row_bytes, x + (r0 + r) * C.ld_x, C.row_bytes, &full[s], pol);
      bulk_copy_g2s(dst + (size_t)(C.rps + r) * C.row_bytes, dy + (r0 + r) * C.ld_x, C.row_bytes,
                    &full[s], pol);
    }
  }
  for (int64_t j = (it > C.stages ? it - C.stages : (int64_t)0); j < it; ++j)
    mbar_wait_bounded(&full[j % C.stages], (uint32_t)((j / C.stages) & 1), status);
}

// Row sums of two quantities at once.
__device__ __forceinline__ float2 row_sum2(float2 v, const RowCfg& C, float2* red, int grp, int tg,
                                           int lane, int par) {
  const int W = C.tpr < 32 ? C.tpr : 32;
  v.x = seg_sum(v.x, W);
  v.y = seg_sum(v.y, W);
  if (C.tpr > 32) {
    const int nw = C.tpr >> 5;
    float2* slot = red + (par * C.rps + grp) * kRedSlots;
    if (lane == 0) slot[tg >> 5] = v;
    named_barrier_sync(1 + grp, C.tpr);
    v = make_float2(0.0f, 0.0f);
    for (int w = 0; w < nw; ++w) {
      v.x += slot[w].x;
      v.y += slot[w].y;
    }
  }
  return v;
}

template <int NCT>
__global__ void __launch_bounds__(CtaShape<NCT>::threads, NCT <= 128 ? 2 : 1)
    row_bwd_kernel(const BwdArgs A, const RowCfg C) {
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
    if (tid == ncons) produce_rows2(A.x, A.dy, C, stage0, full, empty, A.status);
    return;
  }

  const int lane = tid & 31;
  const int grp = tid >> C.log2_tpr;
  const int tg = tid & (C.tpr - 1);
  const int k = tg;                       // one 32-column block per thread
  const bool mine = k < C.K;
  const int rot = (k >> 1) & 3;

  uint32_t gw[16];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint4 v = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    if (A.gamma != nullptr && mine) v = ldg128_nc(A.gamma + (size_t)k * kBlock + ((j + rot) & 3) * 8);
    gw[4 * j] = v.x; gw[4 * j + 1] = v.y; gw[4 * j + 2] = v.z; gw[4 * j + 3] = v.w;
  }
  float acc[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) acc[i] = 0.0f;

  // Each thread copies its x and dy blocks from the stage into registers and
  // hands the stage back before any arithmetic, so the producer refills it
  // while the row is reduced; G is fetched before the row's wait.  Products
  // run as packed fp32 pairs.
  bool ok = true;
  int par = 0;
  int64_t it = 0;
  for (int64_t rb = blockIdx.x; rb < C.n_row_blocks; rb += gridDim.x, ++it, par ^= 1) {
    const int s = (int)(it % C.stages);
    const uint32_t ph = (uint32_t)((it / C.stages) & 1);
    const int64_t row = rb * C.rps + grp;
    const bool valid = row < C.T;
    const bool have = valid && mine;
    const float G = have ? __ldg(A.G + row) : 0.0f;
    if (ok) ok = mbar_wait_bounded(&full[s], ph, A.status);
    const uint8_t* sbase = stage0 + (size_t)s * C.stage_bytes;
    const uint32_t sx = smem_u32(sbase + (size_t)grp * C.row_bytes) + (uint32_t)k * 64u;
    const uint32_t sd = smem_u32(sbase + (size_t)(C.rps + grp) * C.row_bytes) + (uint32_t)k * 64u;
    uint32_t xa[16], da[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t off = (uint32_t)(((j + rot) & 3) * 16);
      uint4 a = make_uint4(0u, 0u, 0u, 0u), d = make_uint4(0u, 0u, 0u, 0u);
      if (have) { a = lds128(sx + off); d = lds128(sd + off); }
      xa[4 * j] = a.x; xa[4 * j + 1] = a.y; xa[4 * j + 2] = a.z; xa[4 * j + 3] = a.w;
      da[4 * j] = d.x; da[4 * j + 1] = d.y; da[4 * j + 2] = d.z; da[4 * j + 3] = d.w;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);

    float2 xx = make_float2(0.0f, 0.0f), xg = make_float2(0.0f, 0.0f);  // (x . x, x . g) halves
#pragma unroll
    for (int w = 0; w < 16; ++w) {
      const float2 x2 = bf16x2_to_f2(xa[w]);
      const float2 g2 = mul2(bf16x2_to_f2(gw[w]), bf16x2_to_f2(da[w]));
      xx = fma2(x2, x2, xx);
      xg = fma2(x2, g2, xg);
    }
    const float2 tot = row_sum2(make_float2(xx.x + xx.y, xg.x + xg.y), C, red, grp, tg, lane, par);
    if (have) {
      const bool live = (G != 0.0f) && (tot.x != 0.0f);
      const float invG = live ? __frcp_rn(G) : 0.0f;
      const float coef = live ? tot.y / tot.x : 0.0f;
      const float2 ncoef2 = make_float2(-coef, -coef), invG2 = make_float2(invG, invG);
      uint16_t* dxrow = A.dx + row * (int64_t)C.D + (int64_t)k * kBlock;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int w = 4 * j + i;
          const float2 x2 = bf16x2_to_f2(xa[w]);
          const float2 d2 = bf16x2_to_f2(da[w]);
          const float2 g2 = mul2(bf16x2_to_f2(gw[w]), d2);
          const float2 r = mul2(fma2(x2, ncoef2, g2), invG2);
          const __nv_bfloat162 h = __floats2bfloat162_rn(r.x, r.y);
          o[i] = *reinterpret_cast<const uint32_t*>(&h);
          const float2 a2 = fma2(mul2(d2, x2), invG2, make_float2(acc[2 * w], acc[2 * w + 1]));
          acc[2 * w] = a2.x;
          acc[2 * w + 1] = a2.y;
        }
        stg128_stream(dxrow + ((j + rot) & 3) * 8, make_uint4(o[0], o[1], o[2], o[3]));
      }
    }
  }

  if (A.partial != nullptr && mine) {
    float* prow = A.partial + ((int64_t)blockIdx.x * C.rps + grp) * C.D + (int64_t)k * kBlock;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float* p = prow + ((j + rot) & 3) * 8;
      reinterpret_cast<float4*>(p)[0] = make_float4(acc[8 * j], acc[8 * j + 1], acc[8 * j + 2], acc[8 * j + 3]);
      reinterpret_cast<float4*>(p)[1] = make_float4(acc[8 * j + 4], acc[8 * j + 5], acc[8 * j + 6], acc[8 * j + 7]);
    }
  }
}

// dgamma[j] = sum over the n_part partial rows, in a fixed order: thread
// (tx, ty) of a 32 x 32 CTA adds rows ty, ty + 32, ... of column j = 32 *
// blockIdx.x + tx; the 32 lane sums are then added in ty order.
__global__ void __launch_bounds__(1024) dgamma_reduce_kernel(const float* partial, int64_t n_part,
                                                             int D, uint16_t* dgamma) {
  __shared__ float sh[32][33];
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int j = blockIdx.x * 32 + tx;
  float s = 0.0f;
  if (j < D)
    for (int64_t r = ty; r < n_part; r += 32) s += partial[r * D + j];
  sh[ty][tx] = s;
  __syncthreads();
  if (ty == 0 && j < D) {
    float t = 0.0f;
    for (int i = 0; i < 32; ++i) t += sh[i][tx];
    const __nv_bfloat16 h = __float2bfloat16_rn(t);
    dgamma[j] = *reinterpret_cast<const uint16_t*>(&h);
  }
}

}  // namespace mxn
