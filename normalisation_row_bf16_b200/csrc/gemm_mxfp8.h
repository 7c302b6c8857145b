// gemm_mxfp8.h -- launcher of the block-scaled MXFP8 GEMM (gemm_mxfp8.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace mxn {

// C[M, N] (bf16, row-major) = A[M, K] x B[N, K]^T with E4M3 codes and E8M0
// scales in the tcgen05 128 x 4 scale layout.  M % 128 == 0, N % 256 == 0,
// K % 128 == 0, 16-byte aligned pointers (checked by the caller).  Persistent
// CTAs, one per SM (at most `sms`), on the tiles gemm_mxfp8_set_tiles selects.
// Returns 0, or non-zero with *why set.
int gemm_mxfp8_launch(const void* a_q, const void* a_s, const void* b_q, const void* b_s, void* c, int M,
                      int N, int K, int sms, unsigned* status, cudaStream_t stream, const char** why);
// Tile shape: 0 (default) = 256 x 192 tiles on single CTAs where M % 256 == 0
// and N % 384 == 0, 128 x 256 otherwise; 1 = 256 x 256 tiles on CTA pairs
// where M % 256 == 0; 2 = 128 x 256 tiles on single CTAs.
void gemm_mxfp8_set_tiles(int mode);
size_t gemm_mxfp8_smem_bytes();
int gemm_mxfp8_tile_m();
int gemm_mxfp8_tile_n();
int gemm_mxfp8_tile_k();

}  // namespace mxn
