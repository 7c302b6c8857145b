/*
 * mxnorm.h -- C ABI of the B200 (sm_100a) MXNorm library, libmxnorm_b200.so.
 *
 * MXNorm (gist.science, "MXNorm: Reusing MXFP block scales for efficient
 * tensor normalisation", technical summary section 2.1) replaces RMSNorm ahead
 * of an MX-quantised linear layer.  For each row of a bf16 activation it takes
 * the absolute maximum m_k of every block of B = 32 consecutive elements,
 * estimates the row's RMS as their generalised p-mean
 *     G = ((1/K) sum_k m_k^p)^(1/p),   K = D / 32,
 * normalises the row by 1/G (and a gain gamma), and writes the result as
 * MXFP8: one E4M3 code per element plus one E8M0 power-of-two scale per block
 * of 32, in a single pass over HBM.
 *
 * Conventions shared by every entry point
 *  - Device pointers unless stated.  The caller owns all memory; the library
 *    never allocates device memory and keeps no pointer after returning.
 *  - Calls are asynchronous and ordered on the CUDA stream `stream`
 *    (a cudaStream_t; NULL means the legacy default stream).  They launch on
 *    the device that is current on the calling thread.
 *  - Tensors are row-major.  T = rows (tokens), D = row length (hidden size),
 *    D a multiple of 32, 32 <= D <= MXN_MAX_D.  ld_x = distance in elements
 *    between consecutive rows of x (ld_x >= D, a multiple of 8).  Every other
 *    tensor is dense (its row stride is its row length).
 *  - Every device pointer must be 16-byte aligned.
 *  - Return value: MXN_OK (0) on success, a negative mxn_status otherwise.  On
 *    error nothing is launched (MXN_ERR_ARG / MXN_ERR_UNSUPPORTED) or the launch
 *    failed (MXN_ERR_CUDA); mxnorm_last_error() then describes the cause.
 *    No entry point traps or aborts.
 *  - E4M3 codes follow the OCP FP8 E4M3 encoding (bias 7, no infinities, NaN =
 *    S.1111.111, largest finite 448), as "FP8 Formats for Deep Learning" (cited
 *    on the "Recipes for Pre-training LLMs with MXFP8" page) defines it.  E8M0
 *    scale codes c stand for 2^(c - 127); 0xFF is NaN.
 *  - Scale rule ("Recipes for Pre-training LLMs with MXFP8", abstract, read as
 *    "round the scale up so that no element saturates"): for a block whose
 *    absmax is a, the scale is 2^e with e the smallest integer in [-127, 127]
 *    such that a <= 448 * 2^e.  A block holding NaN or infinity gets scale
 *    0xFF and code 0x7F for every element.
 */
#ifndef MXNORM_B200_H
#define MXNORM_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Largest supported row length. */
#define MXN_MAX_D 32768

/* Status codes. */
enum mxn_status {
    MXN_OK = 0,
    MXN_ERR_ARG = -1,          /* invalid argument: shape, alignment, null, p */
    MXN_ERR_UNSUPPORTED = -2,  /* valid but not supported here (D > MXN_MAX_D, ...) */
    MXN_ERR_CUDA = -3,         /* a CUDA call or kernel launch failed */
    MXN_ERR_TIMEOUT = -4       /* a kernel gave up a bounded wait (see mxnorm_device_status) */
};

/* Rounding of the E4M3 element cast. */
enum mxn_rounding {
    MXN_ROUND_RNE = 0,  /* nearest, ties to even, saturating to +-448 */
    /* Stochastic rounding (aibr.jp article on stochastic rounding with BF16 and
       Adam, section 3): a value between two neighbouring E4M3 values lo < hi
       becomes hi with probability (|v| - lo) / (hi - lo), so its expectation is
       v.  The draw is word (idx & 3) of Philox4x32-10 (Salmon et al., SC'11)
       with key = (seed low 32 bits, seed high 32 bits) and counter =
       (idx >> 2 low 32 bits, idx >> 2 high 32 bits, 0, 0), idx = row * D + col
       (independent of ld_x); hi is taken iff word < frac * 2^32, exactly. */
    MXN_ROUND_SR = 1
};

/* Layout of the E8M0 scales. */
enum mxn_scale_layout {
    /* scales[row * K + k], K = D / 32: one byte per block, row-major. */
    MXN_SCALES_ROWMAJOR = 0,
    /* The layout tcgen05 block-scaled MMA consumes (128 x 4 tiles, K-major):
       rows padded to a multiple of 128 and K to a multiple of 4; the byte of
       (row, k) is at ((row / 128) * (Kp / 4) + k / 4) * 512 + (row % 32) * 16
       + ((row % 128) / 32) * 4 + (k % 4), Kp = K rounded up to 4.  Padding
       bytes are not written. */
    MXN_SCALES_MMA = 1
};

/* Bytes the MX scales (one per 32 elements) of a [T, D] tensor occupy in the
   given layout; 0 if the arguments are invalid.  NVFP4 scales are T * D / 16
   bytes, row-major (MXN_ELEM_NVFP4 below). */
size_t mxnorm_scales_bytes(int64_t T, int64_t D, int layout);

/* Element format of the MX codes. */
enum mxn_elem_format {
    MXN_ELEM_E4M3 = 0,  /* MXFP8: one E4M3 code per byte, codes [T, D] */
    /* MXFP4: E2M1 elements (the FP4 variant the MXNorm summary reports a
       layer speedup for, section 3; element format as in the OCP
       Microscaling v1.0 format, which the pages do not spell out): sign,
       2 exponent bits (bias 1), 1 mantissa bit, magnitudes 0, 0.5, 1, 1.5,
       2, 3, 4, 6, no infinity or NaN.  Two codes per byte, the even column
       in bits 0..3: codes [T, D / 2].  Scale rule as for E4M3 with 6 in
       place of 448; nearest-even saturates to +-6; a block holding NaN or
       infinity gets scale 0xFF and element code 0x7. */
    MXN_ELEM_E2M1 = 1,
    /* NVFP4 (the FP4 format the MXNorm summary's section 3 quotes its layer
       speedup with; the pages do not define it): E2M1 codes packed as for
       MXN_ELEM_E2M1, codes [T, D / 2], in blocks of 16 elements, each with an
       E4M3 scale s, the smallest E4M3 value with amax <= 6 * s; codes are
       E2M1(fl32(y * fl32(1 / s))).  No tensor-wide scale: MXNorm's output is
       bounded by K^(1/p) * max|gamma|, which keeps every s inside E4M3.
       Scales: uint8 [T, D / 16] row-major (MXN_SCALES_ROWMAJOR only).  An
       all-zero block gets scale 0 and codes 0; a block holding NaN or
       infinity scale 0x7F and codes 0x7.  MXNorm's statistic runs over the
       16-element blocks (K = D / 16). */
    MXN_ELEM_NVFP4 = 2
};

/* Block statistic of the MXNorm p-mean. */
enum mxn_statistic {
    MXN_STAT_ABSMAX = 0,     /* m_k = block absmax of x (section 2.1) */
    /* Scale reuse (the MXNorm title: reusing the MX block scales): m_k is
       replaced by 2^e_k, e_k the scale exponent of block k of x by the rule
       above for the element format (a zero block gives 2^-127); for NVFP4 by
       the block's E4M3 scale value; infinities and NaN pass through. */
    MXN_STAT_SCALE_EXP = 1
};

/* Bytes the codes of a [T, D] tensor occupy in the given element format; 0 if
   the arguments are invalid. */
size_t mxnorm_codes_bytes(int64_t T, int64_t D, int elem_format);

/*
 * MXNorm forward (MXNorm page, technical summary section 2.1; gain as in
 * section 2.3).  For every row r of x:
 *   m_k   = max over block k of |x|                          (exact)
 *   G_r   = ((1/K) sum_k m_k^p)^(1/p) in fp32; p = +inf gives max_k m_k
 *   s     = fl32(1 / G_r)  (s = 0 when G_r = 0)
 *   y_j   = fl32(x_j * s), then y_j = fl32(y_j * gamma_j) if gamma != NULL
 *   per block: scale 2^e from max |y| (rule above); code_j = E4M3(fl32(y_j * 2^-e))
 * x       bf16 [T, ld_x] (first D columns used)
 * gamma   bf16 [D] or NULL (NULL when the gain is folded into the next
 *         layer's weight, section 2.3)
 * q       uint8 [T, D] E4M3 codes (written)
 * scales  uint8, mxnorm_scales_bytes(T, D, scale_layout) bytes (written)
 * G_out   fp32 [T] (written) or NULL; the backward pass takes it.
 * p       > 0 (INFINITY allowed); 2 is the default the page settles on
 *         (section 3.1: p = 1 was unstable at 8B parameters).
 * rounding  enum mxn_rounding; seed is used only by MXN_ROUND_SR.
 * G_out agrees with the exact p-mean to about 1e-6 relative (fp32 reduction).
 */
int mxnorm_fwd(const void* x, const void* gamma, void* q, void* scales, float* G_out,
               int64_t T, int64_t D, int64_t ld_x, float p, int rounding, uint64_t seed,
               int scale_layout, void* stream);

/*
 * mxnorm_fwd with a choice of element format (enum mxn_elem_format; q holds
 * mxnorm_codes_bytes(T, D, elem_format) bytes) and of block statistic (enum
 * mxn_statistic).  Every other argument as in mxnorm_fwd; with MXN_ELEM_E4M3
 * and MXN_STAT_ABSMAX it is mxnorm_fwd.  Stochastic rounding draws its words
 * as for E4M3 and rounds between neighbouring E2M1 values.
 */
int mxnorm_fwd_ex(const void* x, const void* gamma, void* q, void* scales, float* G_out,
                  int64_t T, int64_t D, int64_t ld_x, float p, int rounding, uint64_t seed,
                  int scale_layout, int elem_format, int statistic, void* stream);

/*
 * MX quantisation of x itself (MXCast; MXNorm page, technical summary section
 * 1.2): y = x, then the per-block scale and code of mxnorm_fwd.
 * Same argument meanings as mxnorm_fwd.
 */
int mxfp8_cast(const void* x, void* q, void* scales, int64_t T, int64_t D, int64_t ld_x,
               int rounding, uint64_t seed, int scale_layout, void* stream);

/*
 * MXCast with an optional gain along each row and a choice of element format:
 * y_j = fl32(x_j * gain_j) (exact: a bf16 product fits fp32), or y = x when
 * gain is NULL; then scales and codes as in mxnorm_fwd_ex.  gain bf16 [D].
 */
int mx_cast_ex(const void* x, const void* gain, void* q, void* scales, int64_t T, int64_t D,
               int64_t ld_x, int rounding, uint64_t seed, int scale_layout, int elem_format,
               void* stream);

/*
 * MXNormLinear weight folding (MXNorm page, technical summary section 2.3: the
 * gain gamma moves into the next layer's weight, W' = diag(gamma) W, and
 * MXNorm then runs with gamma = NULL).  w is that weight stored the way
 * mxfp8_gemm reads its B operand: one output feature per row, bf16 [N, ld_w],
 * K = input features contiguous.  Writes the MX codes and scales of
 * w[n, k] * gamma[k] (nearest-even): q mxnorm_codes_bytes(N, K, elem_format)
 * bytes, scales in scale_layout.  gamma bf16 [K], required.  Same as
 * mx_cast_ex(w, gamma, ..., MXN_ROUND_RNE, 0, ...).
 */
int mxnorm_fold_weight(const void* w, const void* gamma, void* q, void* scales, int64_t N,
                       int64_t K, int64_t ld_w, int elem_format, int scale_layout, void* stream);

/*
 * RMSNorm (MXNorm page, sections 1.1-1.2, the layer MXNorm replaces):
 *   y = bf16( fl32(x * 1/sqrt(mean(x^2) + eps)) * gamma ), fp32 arithmetic.
 * x bf16 [T, ld_x]; gamma bf16 [D] or NULL; y bf16 [T, D] (written).
 */
int rmsnorm_bf16(const void* x, const void* gamma, void* y, int64_t T, int64_t D, int64_t ld_x,
                 float eps, void* stream);

/*
 * The two-pass comparator of MXNorm (section 1.2, RMSNorm and MXCast as
 * separate steps): rmsnorm_bf16 into y_tmp, then mxfp8_cast of y_tmp with
 * nearest-even rounding.  y_tmp bf16 [T, D] is caller-owned scratch and holds
 * the RMSNorm output afterwards.  scales in scale_layout.
 */
int rmsnorm_then_mxcast(const void* x, const void* gamma, float eps, void* y_tmp, void* q,
                        void* scales, int64_t T, int64_t D, int64_t ld_x, int scale_layout,
                        void* stream);

/*
 * MXNorm backward (MXNorm page, technical summary section 2.3: the RMSNorm
 * gradient reused as a straight-through estimator; the cast is taken as the
 * identity).  With g = gamma * dy (gamma = 1 when NULL), per row:
 *   dx     = ( g - x * (x . g) / (x . x) ) / G
 *   dgamma = sum over rows of dy * x / G
 * (the exact gradient of x -> x * gamma / (c * rms(x)) when G = c * rms(x)).
 * A row with G = 0 or x = 0 gets dx = 0 and adds nothing to dgamma.
 * x, dy   bf16 [T, D] dense; gamma bf16 [D] or NULL; G fp32 [T] from mxnorm_fwd.
 * dx      bf16 [T, D] (written; fp32 arithmetic, one rounding).
 * dgamma  bf16 [D] (written) or NULL; must be NULL when gamma is NULL.
 *         Deterministic: partial sums in a fixed order, no atomics.
 * workspace  device scratch of at least mxnorm_bwd_workspace_size(T, D)
 *         bytes (fp32 partial sums, one row of D per CTA of the launch),
 *         16-byte aligned; may be NULL when dgamma is NULL.  Contents on
 *         entry are ignored.
 */
int mxnorm_bwd(const void* x, const void* dy, const void* gamma, const float* G, void* dx,
               void* dgamma, int64_t T, int64_t D, void* workspace, size_t workspace_bytes,
               void* stream);

/* Scratch bytes mxnorm_bwd needs for (T, D) on the current device. */
size_t mxnorm_bwd_workspace_size(int64_t T, int64_t D);

/*
 * Block-scaled MXFP8 GEMM on the tcgen05 tensor cores (MXNorm page, technical
 * summary section 2.3: MXNormLinear feeds the MX-cast activations into an MX
 * matmul; "Recipes for Pre-training LLMs with MXFP8": MXFP8-E4M3 operands):
 *   C[m, n] = sum_k A(m, k) * B(n, k),
 *   A(m, k) = E4M3(a_q[m, k]) * 2^(scale(m, k/32) - 127), B likewise,
 * accumulated in fp32, written as bf16.
 * a_q   uint8 [M, K] E4M3 codes, row-major (K contiguous) -- mxnorm_fwd's q
 * a_s   uint8 scales of A in the MXN_SCALES_MMA layout (M x K/32 bytes)
 * b_q   uint8 [N, K] E4M3 codes, K contiguous (the weight transposed) --
 *       mxfp8_cast of W^T
 * b_s   uint8 scales of B in the MXN_SCALES_MMA layout (N x K/32 bytes)
 * c     bf16 [M, N] row-major (written)
 * Requires M % 128 == 0, N % 256 == 0, K % 128 == 0 (MXN_ERR_UNSUPPORTED
 * otherwise); M = 0 or N = 0 is a no-op.  Persistent CTAs, one per SM,
 * walk the 128 x 256 output tiles.
 */
int mxfp8_gemm(const void* a_q, const void* a_s, const void* b_q, const void* b_s, void* c, int64_t M,
               int64_t N, int64_t K, void* stream);

/*
 * mxnorm_bwd without a workspace argument, for callers that cannot allocate
 * device memory when they call: plugins inside an engine that owns every
 * allocation, and real-time loops that must not call cudaMalloc.  The paper
 * has no counterpart; this is a deployment convenience.
 *
 * Same arguments, results and limits as mxnorm_bwd (D <= 16384), except that
 * the dgamma partial sums live in one 8 MiB scratch array inside this library
 * (2^21 fp32).  The CUDA runtime reserves it on a device when the library's
 * kernels are first used there (lazy module loading: not necessarily when the
 * library is loaded), whether or not this entry point is ever called, and it
 * stays until the process exits -- so every process that uses the library,
 * each rank of a multi-GPU job included, holds 8 MiB on each device it uses.
 * The call allocates nothing.  To fit the scratch it may launch fewer CTAs
 * than mxnorm_bwd (every CTA writes one partial row of D fp32, at most
 * 2^21 / D rows in all, which is at least 128 at D <= 16384).
 * The first call on a device looks up the scratch array's device address
 * (cudaGetSymbolAddress); make that first call outside any stream capture.
 * Every call on a device shares the one scratch array: calls that may overlap
 * on the GPU (different streams, or different host threads) race and must be
 * serialised by the caller.  Each call overwrites every partial it reads, so
 * nothing has to be cleared between calls.
 */
int mxnorm_bwd_noalloc(const void* x, const void* dy, const void* gamma, const float* G,
                       void* dx, void* dgamma, int64_t T, int64_t D, void* stream);

/* Message for the last error on the calling thread ("" if none).  The string
   stays valid until the thread's next call into the library. */
const char* mxnorm_last_error(void);

/*
 * Waits for `stream`, then reads and clears the current device's status word.
 * Kernels that wait on a barrier bound each wait (about a second); a wait that
 * gives up records itself there and the kernel returns early, its outputs then
 * being incomplete.  Returns MXN_OK, MXN_ERR_TIMEOUT, or MXN_ERR_CUDA.
 */
int mxnorm_device_status(void* stream);

/*
 * Launch tuning for the row kernels: threads per CTA (a multiple of 32 up to
 * 512, split into row groups; capped at what the kernel's register budget
 * allows -- 512 for most shapes, 256 for the backward's two-block rows),
 * shared-memory stages per row group (1..16) and CTAs per SM (1..8); 0 keeps
 * the library's choice.
 * Process-wide; not thread-safe against concurrent launches.  Returns
 * MXN_ERR_ARG for out-of-range values; a shape that does not fit an SM makes
 * the next launch return MXN_ERR_UNSUPPORTED.
 */
int mxnorm_set_tuning(int consumer_threads, int stages, int ctas_per_sm);

/*
 * Tile shape of mxfp8_gemm.  0 (default) runs 256 x 192 output tiles on single
 * CTAs (two M = 128 tcgen05 accumulators, 22% fewer operand bytes per flop
 * than 128 x 256) whenever M % 256 == 0 and N % 384 == 0, and 128 x 256 tiles
 * otherwise; 1 runs 256 x 256 tiles on pairs of CTAs on two SMs (a two-CTA
 * cluster, tcgen05.mma.cta_group::2; each CTA loads half of the tile's A and
 * B rows) whenever M % 256 == 0, and 128 x 256 tiles otherwise; 2 runs 128 x
 * 256 tiles on single CTAs.  The results are identical (same products, same
 * fp32 accumulation order per output).  Process-wide; returns MXN_ERR_ARG for
 * any other value.
 */
int mxnorm_set_gemm_tiles(int mode);

/*
 * Test hook: the next `count` entry-point calls on this thread fail with
 * MXN_ERR_CUDA before launching (host-side fault injection; nothing runs on
 * the GPU).  count = 0 clears it.
 */
void mxnorm_debug_fail_next(int count);

/*
 * Test hook for the bounded waits: launches one thread that waits on an
 * mbarrier nothing ever arrives on, for at most limit_ns (0 < limit_ns <= 2 s).
 * The wait gives up, sets the device status word (mxnorm_device_status then
 * returns MXN_ERR_TIMEOUT) and writes 1 to the device int *gave_up; the
 * context stays usable.  No trap, no fault.
 */
int mxnorm_debug_wait_timeout(uint64_t limit_ns, int* gave_up, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MXNORM_B200_H */
