/*
 * fp8bs.h -- C ABI of libfp8bs: FP8 (e4m3) dynamic quantization and scaled
 * GEMM for NVIDIA B200 (sm_100a).
 *
 * The operations (see each function for the passage that defines it):
 *
 *   quantize     a group G of inputs (1x128 slice, 128x128 tile, row, tensor):
 *                amax = max|x| over G, s = 448 / max(amax, 1e-12) in fp32
 *                (IEEE), q = e4m3(x * s) rounded to nearest even and saturated
 *                to +-448, and the reciprocal r = 1/s is stored as the scale.
 *   scaled GEMM  C[m,n] = sum_kb  rA(m,kb) * rB(n,kb) * sum_{k in block kb} qA[m,k] qB[n,k]
 *                with K blocks of 128, fp32 accumulation on the tensor cores,
 *                per-K-block promotion of the partial sums in fp32 registers,
 *                bf16 or fp32 output.
 *
 * e4m3 is the OCP 8-bit E4M3 format (bias 7, no infinities, max 448).
 *
 * Conventions for every entry point:
 *   - All pointers are DEVICE pointers owned by the caller.  The library
 *     allocates no device memory.  Its only device state is compiled in: one
 *     int of device-side error flag (see fp8bs_check_device_error) and the
 *     16 KB scratch array of fp8_quant_tensor_noalloc, both held by every GPU
 *     that loads the library until the process exits.
 *   - Every call is asynchronous on `stream` (0 = legacy default stream) and
 *     never synchronizes, except fp8bs_check_device_error.
 *   - Arguments are validated before anything is launched; on an error status
 *     nothing has been launched and no output was touched.
 *   - Matrices are row-major with an explicit leading dimension in ELEMENTS.
 *     Scale grids are column-major fp32 with an explicit leading dimension:
 *     the scale of (row i, block j) lives at scale[i + j*ld].
 *   - Inputs must be finite (NaN/Inf inputs are outside the contract).
 *   - Only compute capability 10.x devices (B200, sm_100a) are supported;
 *     anything else returns FP8BS_ERR_NO_SM100.  There is no fallback path.
 */
#ifndef FP8BS_H
#define FP8BS_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP8BS_OK = 0,
    FP8BS_ERR_INVALID_ARG = 1,   /* null pointer, size < 1, ld too small, bad flag      */
    FP8BS_ERR_UNSUPPORTED = 2,   /* unknown enum value                                  */
    FP8BS_ERR_ALIGNMENT = 3,     /* pointer / leading dimension / size alignment rule   */
    FP8BS_ERR_WORKSPACE = 4,     /* workspace given but smaller than required           */
    FP8BS_ERR_CUDA = 5,          /* a CUDA runtime/driver call or launch failed         */
    FP8BS_ERR_TIMEOUT = 6,       /* a device-side wait ran past its limit (see below)   */
    FP8BS_ERR_NO_SM100 = 7,      /* current device is not compute capability 10.x     */
    FP8BS_ERR_SCALE = 8          /* a power-of-two GEMM recipe met a scale that is not an
                                    exact power of two (device-side, see below)          */
} fp8bs_status;

typedef enum { FP8BS_BF16 = 0, FP8BS_F32 = 1 } fp8bs_dtype;

typedef enum {
    FP8BS_SCALE_TENSOR = 0,              /* rA = scale_a[0],              rB = scale_b[0]               */
    FP8BS_SCALE_ROWWISE = 1,             /* rA = scale_a[m],              rB = scale_b[n]               */
    FP8BS_SCALE_BLOCK_1x128_128x128 = 2, /* rA = scale_a[m + kb*ld_sa],   rB = scale_b[n/128 + kb*ld_sb] */
    FP8BS_SCALE_BLOCK_1x128_1x128 = 3,   /* rA = scale_a[m + kb*ld_sa],   rB = scale_b[n + kb*ld_sb]     */
    /* The same two block recipes with power-of-two scales, applied by the
     * tensor cores' block-scaled MMA (see fp8_scaled_gemm). */
    FP8BS_SCALE_BLOCK_1x128_128x128_POW2 = 4,
    FP8BS_SCALE_BLOCK_1x128_1x128_POW2 = 5
} fp8bs_scale_mode;

typedef enum { FP8BS_SCALE_COL_MAJOR = 0 } fp8bs_scale_layout;

/* The scale rule of the group quantizations (the *_ex entry points).
 * FP32: s = 448 / max(amax, 1e-12) in fp32, the rule of every other entry point.
 * POW2: s = the largest power of two not above that fp32 value, so that the
 *       stored reciprocal 1/s is an exact power of two: the form a UE8M0 scale
 *       factor (8-bit biased exponent) holds, which the POW2 GEMM recipes
 *       take.  q = e4m3(x * s) and the stored 1/s as for FP32. */
typedef enum { FP8BS_SCALE_RULE_FP32 = 0, FP8BS_SCALE_RULE_POW2 = 1 } fp8bs_scale_rule;

/*
 * fp8_quant_1x128 -- dynamic quantization with one scale per 1x128 group.
 *
 * Defined by: pytorch/ao PR #2592 "add more generic kernel for fp8 blockwise
 * scaling" (Performance table, block shape (1,128)); pytorch/ao PR #2785
 * "integrate torch._scaled_mm into Float8BlockwiseLinear and add bench
 * script" (Summary: column-major scales, reciprocal scales written directly
 * by the quant kernel).
 *
 * x          rows x cols, dtype xt (bf16 or fp32), leading dim ldx elements.
 * transpose_out = 0: groups run along the contiguous dim (cols).
 *            q:          rows x cols e4m3 bytes, leading dim ldq.
 *            scale_inv:  grid rows x ceil(cols/128), scale_inv[r + g*ld_scale],
 *                        ld_scale >= rows.
 * transpose_out = 1: groups run along the rows of x ("scaled along tokens"),
 *            and the quantized TRANSPOSE is written:
 *            q:          cols x rows e4m3 bytes, q[c*ldq + r], leading dim ldq >= rows.
 *            scale_inv:  grid cols x ceil(rows/128), scale_inv[c + g*ld_scale],
 *                        ld_scale >= cols.
 * A ragged last group (size not a multiple of 128) is quantized over its valid
 * elements only.
 * Alignment: x, q, scale_inv 16-byte aligned; ldx*sizeof(xt) and ldq multiples
 * of 16 bytes; cols % 16 == 0 (and rows % 16 == 0 when transpose_out);
 * ld_scale % 4 == 0.  Otherwise FP8BS_ERR_ALIGNMENT.
 */
fp8bs_status fp8_quant_1x128(const void* x, fp8bs_dtype xt, int64_t rows, int64_t cols, int64_t ldx,
                             uint8_t* q, int64_t ldq, float* scale_inv, int64_t ld_scale,
                             int transpose_out, cudaStream_t stream);

/*
 * fp8_quant_1x128_dual -- both 1x128 quantizations of one tensor from a
 * single read of it.
 *
 * Defined by: the two operand recipes of the FP8 blockwise linear layer in
 * pytorch/ao PR #2785 "integrate torch._scaled_mm into Float8BlockwiseLinear
 * and add bench script" (Summary): the activation is quantized 1x128 along
 * its contiguous dimension for the forward GEMM and 1x128 along tokens (the
 * rows) for the weight-gradient GEMM; likewise the output gradient for the
 * input-gradient and weight-gradient GEMMs.  The group rule is that of
 * fp8_quant_1x128 (pytorch/ao PR #2592, block shape (1,128)).
 *
 * The results are byte-identical to the two calls
 *     fp8_quant_1x128(x, ..., q,   ldq,   scale_inv,   ld_scale,   0, stream)
 *     fp8_quant_1x128(x, ..., q_t, ldq_t, scale_inv_t, ld_scale_t, 1, stream)
 * with the layouts documented there:
 *     q:           rows x cols, leading dim ldq >= cols;
 *     scale_inv:   scale_inv[r + g*ld_scale], g < ceil(cols/128), ld_scale >= rows;
 *     q_t:         cols x rows (the transpose), leading dim ldq_t >= rows;
 *     scale_inv_t: scale_inv_t[c + g*ld_scale_t], g < ceil(rows/128), ld_scale_t >= cols.
 * All four outputs are written; none may be null and none may overlap x or
 * one another.  The caller owns every buffer.
 * Alignment: x and the four outputs 16-byte aligned; ldx*sizeof(xt), ldq and
 * ldq_t multiples of 16 bytes; rows % 16 == 0 and cols % 16 == 0; ld_scale and
 * ld_scale_t % 4 == 0.  Otherwise FP8BS_ERR_ALIGNMENT.  Other argument errors:
 * FP8BS_ERR_INVALID_ARG (null pointer, size < 1, leading dimension too small),
 * FP8BS_ERR_UNSUPPORTED (unknown dtype).  Nothing is launched when a check
 * fails.  Asynchronous on `stream`.
 */
fp8bs_status fp8_quant_1x128_dual(const void* x, fp8bs_dtype xt, int64_t rows, int64_t cols, int64_t ldx,
                                  uint8_t* q, int64_t ldq, float* scale_inv, int64_t ld_scale,
                                  uint8_t* q_t, int64_t ldq_t, float* scale_inv_t, int64_t ld_scale_t,
                                  cudaStream_t stream);

/*
 * fp8_quant_128x128 -- dynamic quantization with one scale per 128x128 tile.
 *
 * Defined by: pytorch/ao PR #2592 (Performance table, block shape (128,128));
 * the weight side of the (BlockWise1x128, BlockWise128x128) recipe in
 * pytorch/ao PR #4209 "[codex] add repro for blockwise _scaled_mm
 * investigation" (Findings So Far); 2-D tile loads as in PR #2785's stack
 * ("load 2d chunks for groupwise quant to enable coalesced gmem accesses").
 *
 * x            rows x cols, dtype xt, leading dim ldx.
 * q            (nullable) rows x cols e4m3, leading dim ldq.
 * scale_inv    grid ceil(rows/128) x ceil(cols/128), scale_inv[bi + bj*ld_scale],
 *              ld_scale >= ceil(rows/128).  Required when q != NULL.
 * q_t          (nullable) the same quantized tile bytes transposed: cols x rows,
 *              q_t[c*ldq_t + r], leading dim ldq_t >= rows.
 * scale_inv_t  the transposed grid ceil(cols/128) x ceil(rows/128),
 *              scale_inv_t[bj + bi*ld_scale_t], ld_scale_t >= ceil(cols/128).
 *              Required when q_t != NULL.
 * At least one of q, q_t must be non-NULL.  Edge tiles are quantized over
 * their valid elements only.
 * Alignment: pointers 16-byte aligned; ldx*sizeof(xt), ldq, ldq_t multiples of
 * 16 bytes; rows % 16 == 0 and cols % 16 == 0; ld_scale, ld_scale_t % 4 == 0.
 */
fp8bs_status fp8_quant_128x128(const void* x, fp8bs_dtype xt, int64_t rows, int64_t cols, int64_t ldx,
                               uint8_t* q, int64_t ldq, float* scale_inv, int64_t ld_scale,
                               uint8_t* q_t, int64_t ldq_t, float* scale_inv_t, int64_t ld_scale_t,
                               cudaStream_t stream);

/*
 * fp8_quant_1x128_ex, fp8_quant_1x128_dual_ex, fp8_quant_128x128_ex -- the
 * three group quantizations above with a selectable scale rule.
 *
 * Defined by: the entry points without the suffix (same arguments, layouts,
 * alignment rules and errors) and the scale rule `rule` (fp8bs_scale_rule):
 * FP8BS_SCALE_RULE_FP32 gives byte-identical results to them;
 * FP8BS_SCALE_RULE_POW2 rounds each group's fp32 scale down to a power of two
 * before quantizing, for the power-of-two GEMM recipes (the fast-accumulation
 * variant of pytorch/pytorch issue #159940, Describe the bug: USE_FAST_ACCUM,
 * in its B200 form).  An unknown rule gives FP8BS_ERR_UNSUPPORTED.
 */
fp8bs_status fp8_quant_1x128_ex(const void* x, fp8bs_dtype xt, int64_t rows, int64_t cols, int64_t ldx,
                                uint8_t* q, int64_t ldq, float* scale_inv, int64_t ld_scale,
                                int transpose_out, fp8bs_scale_rule rule, cudaStream_t stream);
fp8bs_status fp8_quant_1x128_dual_ex(const void* x, fp8bs_dtype xt, int64_t rows, int64_t cols, int64_t ldx,
                                     uint8_t* q, int64_t ldq, float* scale_inv, int64_t ld_scale,
                                     uint8_t* q_t, int64_t ldq_t, float* scale_inv_t, int64_t ld_scale_t,
                                     fp8bs_scale_rule rule, cudaStream_t stream);
fp8bs_status fp8_quant_128x128_ex(const void* x, fp8bs_dtype xt, int64_t rows, int64_t cols, int64_t ldx,
                                  uint8_t* q, int64_t ldq, float* scale_inv, int64_t ld_scale,
                                  uint8_t* q_t, int64_t ldq_t, float* scale_inv_t, int64_t ld_scale_t,
                                  fp8bs_scale_rule rule, cudaStream_t stream);

/*
 * fp8_quant_tensor -- dynamic quantization with one scale for the whole tensor.
 *
 * Defined by: ROCm/aiter issue #1765 "[Issue]: Does gemm_a8w8 support
 * per-tensor quant?" (Steps to Reproduce: per_tensor_quant returns the
 * quantized tensor and a single dequantization scale, dequant = q * scale).
 *
 * x          n contiguous elements of dtype xt.
 * q          n e4m3 bytes.
 * scale_inv  one float (the dequantization scale 1/s).
 * workspace  device scratch of at least fp8_quant_tensor_workspace_size(n)
 *            bytes, 16-byte aligned; no initial contents needed.  Two launches
 *            (amax partials, then quantize) share it on `stream`.
 * Alignment: x, q 16-byte aligned; n % 16 == 0.
 */
size_t fp8_quant_tensor_workspace_size(int64_t n);
fp8bs_status fp8_quant_tensor(const void* x, fp8bs_dtype xt, int64_t n, uint8_t* q, float* scale_inv,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * fp8_quant_tensor_noalloc -- fp8_quant_tensor for callers that cannot
 * allocate device memory.
 *
 * The paper has no counterpart to this entry point; it exists for callers
 * that cannot call cudaMalloc (or any allocator) where they quantize -- for
 * example a plugin whose host framework hands it no workspace, or code that
 * must not trigger an allocation's implicit device synchronization or grow
 * its memory footprint.  Same arguments, result and alignment rules as
 * fp8_quant_tensor, minus the workspace: its amax scratch is a fixed 16 KB
 * array compiled into the library, which every GPU that loads the library
 * holds until the process exits.  This entry point allocates nothing.
 *
 * Limit: n <= 268435456 (2^28) elements; larger n returns FP8BS_ERR_WORKSPACE
 * without launching anything.
 * Set-up: the first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.
 * Sharing: all calls on a device share the one array.  Calls whose kernels
 * overlap on the GPU (e.g. issued on different streams without ordering)
 * race on it and may return wrong scales; order them on one stream or with
 * events.  Nothing needs clearing between calls: every scratch slot a call
 * reads was written earlier in the same call.
 */
fp8bs_status fp8_quant_tensor_noalloc(const void* x, fp8bs_dtype xt, int64_t n, uint8_t* q, float* scale_inv,
                                      cudaStream_t stream);

/*
 * fp8_quant_rowwise -- dynamic quantization with one scale per row.
 *
 * Defined by: the rowwise variant of scaled_mm (pytorch/pytorch issue #159940,
 * Describe the bug: the scaled_mm template's SCALING_ROWWISE flag); applied to
 * x (per row) and to W (per row of W = per output column).
 *
 * x          rows x cols, dtype xt, leading dim ldx.
 * q          rows x cols e4m3, leading dim ldq.
 * scale_inv  rows floats.
 * Alignment: x, q 16-byte aligned; ldx*sizeof(xt), ldq multiples of 16 bytes;
 * cols % 16 == 0; scale_inv 4-byte aligned.
 */
fp8bs_status fp8_quant_rowwise(const void* x, fp8bs_dtype xt, int64_t rows, int64_t cols, int64_t ldx,
                               uint8_t* q, int64_t ldq, float* scale_inv, cudaStream_t stream);

/*
 * fp8_scaled_gemm -- D = scaled (A . Bt^T), the "TN" layout of F.linear.
 *
 * Defined by: the explicit dequantized matmul of pytorch/ao PR #4209 (What
 * Changed: FP32 reference, dequantized matmul and kernels on the same
 * quantized inputs and reciprocal scales) and of ROCm/aiter issue #1765 (Steps
 * to Reproduce: F.linear(q_x*s_x, q_w*s_w)); recipes (1x128, 128x128) and
 * (1x128, 1x128) from PR #4209 (Findings So Far and its review thread),
 * per-tensor from issue #1765, rowwise from pytorch/pytorch issue #159940.
 *
 * A          M x K e4m3, leading dim lda (bytes).
 * Bt         N x K e4m3, leading dim ldb (bytes): row n holds column n of B.
 * scale_a    TENSOR: 1 float.  ROWWISE: M floats.  BLOCK_*: grid M x ceil(K/128),
 *            scale_a[m + kb*ld_sa], ld_sa >= M.
 * scale_b    TENSOR: 1 float.  ROWWISE: N floats.
 *            BLOCK_1x128_128x128: grid ceil(N/128) x ceil(K/128), scale_b[nb + kb*ld_sb],
 *            ld_sb >= ceil(N/128) (as written by fp8_quant_128x128 on Bt).
 *            BLOCK_1x128_1x128: grid N x ceil(K/128), scale_b[n + kb*ld_sb], ld_sb >= N.
 * D          M x N, dtype out_dtype (bf16 rounded to nearest even, or fp32),
 *            leading dim ldd elements.
 * workspace  optional fp32 scratch for split-K (used when the output has too few
 *            256x128 tiles to keep the GPU's CTA pairs busy).  Pass NULL/0 to disable split-K, or
 *            at least fp8_scaled_gemm_workspace_size(M, N, K, mode) bytes.  The
 *            split partial sums are added in a fixed order: results are
 *            deterministic.
 * Any M, N >= 1 and any K >= 16 with K % 16 == 0 (any number of K blocks;
 * a ragged last K block contributes its valid columns only).
 * Alignment: A, Bt, scale_a, scale_b, workspace 16-byte aligned; lda, ldb
 * multiples of 16; ld_sa, ld_sb % 4 == 0 for the block modes; D aligned to its
 * element size.  Any ldd >= N works; when D is 16-byte aligned and
 * ldd*sizeof(out) is a multiple of 16 the output is written in 16-byte
 * chunks, otherwise element by element.
 *
 * The power-of-two recipes BLOCK_1x128_128x128_POW2 and BLOCK_1x128_1x128_POW2
 * compute the same sum with the scale grids of their plain counterparts, but
 * every scale must be an exact power of two in [2^-126, 2^127] (what
 * fp8_quant_*_ex with FP8BS_SCALE_RULE_POW2 writes).  The tensor cores apply
 * the scales (block-scaled MMA with UE8M0 scale factors, each 128-wide K block
 * given as four identical 32-wide blocks) and accumulate every K block of a
 * tile (of a split, with split-K) in one fp32 accumulator, without the
 * per-K-block promotion in registers: the fast-accumulation variant of
 * pytorch/pytorch issue #159940 (Describe the bug: USE_FAST_ACCUM), in its
 * B200 form.  A scale that is not such a power of two sets the device error
 * flag (fp8bs_check_device_error returns FP8BS_ERR_SCALE) and the output is
 * unspecified.
 */
size_t fp8_scaled_gemm_workspace_size(int64_t M, int64_t N, int64_t K, fp8bs_scale_mode mode);
fp8bs_status fp8_scaled_gemm(int64_t M, int64_t N, int64_t K,
                             const uint8_t* A, int64_t lda, const uint8_t* Bt, int64_t ldb,
                             const float* scale_a, int64_t ld_sa, const float* scale_b, int64_t ld_sb,
                             fp8bs_scale_mode mode, fp8bs_scale_layout layout,
                             void* D, int64_t ldd, fp8bs_dtype out_dtype,
                             void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Storage order of the B operand of fp8_scaled_gemm_ex. */
typedef enum {
    FP8BS_MAJOR_K = 0,    /* B^T stored N x K row-major (K contiguous), as fp8_scaled_gemm takes it */
    FP8BS_MAJOR_MN = 1    /* B stored K x N row-major (N contiguous)                               */
} fp8bs_major;

/*
 * fp8_scaled_gemm_ex -- fp8_scaled_gemm with the storage order of B chosen by
 * the caller: B^T (N x K, K-major, b_major = FP8BS_MAJOR_K, exactly
 * fp8_scaled_gemm) or B itself (K x N, MN-major, b_major = FP8BS_MAJOR_MN).
 *
 * Defined by: the same dequantized matmul as fp8_scaled_gemm.  The MN-major
 * form lets the backward GEMMs of the blockwise linear read an operand in the
 * orientation it is stored in, as the blockwise linear of pytorch/ao PR #2785
 * "integrate torch._scaled_mm into Float8BlockwiseLinear and add bench
 * script" (Summary) consumes W and grad_out: dgrad dX = dY . W reads the
 * forward's W_q (N_w x K_w) as B = W_q, K = N_w, N = K_w, with the forward's
 * 128x128 scale grid, so no transposed copy of W_q is needed.
 *
 * With b_major = FP8BS_MAJOR_MN:
 * B          K x N e4m3, leading dim ldb >= N (bytes), ldb % 16 == 0.
 * scale_b    TENSOR: 1 float.  ROWWISE: N floats.
 *            BLOCK_1x128_128x128: the grid of B's 128x128 tiles in B's storage
 *            order, ceil(K/128) x ceil(N/128): rB(n, kb) = scale_b[kb + (n/128)*ld_sb],
 *            ld_sb >= ceil(K/128) (as fp8_quant_128x128 writes it for the K x N
 *            matrix).
 *            BLOCK_1x128_1x128 and the POW2 recipes with B_MN: FP8BS_ERR_UNSUPPORTED
 *            (with FP8BS_MAJOR_K every recipe is fp8_scaled_gemm's).
 * Everything else (A, scale_a, D, workspace, alignment, errors) as
 * fp8_scaled_gemm.  Asynchronous on `stream`.
 */
fp8bs_status fp8_scaled_gemm_ex(int64_t M, int64_t N, int64_t K,
                                const uint8_t* A, int64_t lda, const uint8_t* B, int64_t ldb, fp8bs_major b_major,
                                const float* scale_a, int64_t ld_sa, const float* scale_b, int64_t ld_sb,
                                fp8bs_scale_mode mode, fp8bs_scale_layout layout,
                                void* D, int64_t ldd, fp8bs_dtype out_dtype,
                                void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * fp8_scaled_gemm_quant -- the scaled GEMM with its bf16 output quantized
 * 1x128 along N in the epilogue, for a consumer that needs the output in FP8
 * (the next layer's GEMM), so that the output is not read back from memory
 * to be quantized.
 *
 * Defined by: fp8_scaled_gemm followed by fp8_quant_1x128 on its bf16 output;
 * pytorch/ao PR #2785 "integrate torch._scaled_mm into Float8BlockwiseLinear
 * and add bench script" (Benchmarks: the quantization launches are the gap to
 * the bf16 linear).  The quantized bytes and scales are identical to those of
 * fp8_quant_1x128 applied to D (the epilogue rounds to bf16 first and applies
 * the same group rule to the rounded values).
 *
 * Arguments as fp8_scaled_gemm (output dtype bf16, no split-K workspace), plus:
 * D          optional (NULL: the bf16 output is not stored; its quantization is
 *            still that of the values D would hold), leading dim ldd >= N.
 * q_out      M x N e4m3 bytes, leading dim ldq_out >= N, ldq_out % 16 == 0.
 * scale_out  grid M x ceil(N/128) of reciprocal scales, scale_out[m + g*ld_scale_out],
 *            ld_scale_out >= M, ld_scale_out % 4 == 0.
 * q_out and scale_out 16-byte aligned.  The caller owns every buffer.
 * Recipes: TENSOR, ROWWISE and BLOCK_1x128_128x128; the others return
 * FP8BS_ERR_UNSUPPORTED.  Errors as fp8_scaled_gemm; nothing is launched when
 * a check fails.  Asynchronous on `stream`.
 */
fp8bs_status fp8_scaled_gemm_quant(int64_t M, int64_t N, int64_t K,
                                   const uint8_t* A, int64_t lda, const uint8_t* Bt, int64_t ldb,
                                   const float* scale_a, int64_t ld_sa, const float* scale_b, int64_t ld_sb,
                                   fp8bs_scale_mode mode, fp8bs_scale_layout layout,
                                   void* D, int64_t ldd, uint8_t* q_out, int64_t ldq_out,
                                   float* scale_out, int64_t ld_scale_out, cudaStream_t stream);

/*
 * fp8_scaled_gemm_grouped -- G independent blockwise GEMMs in one launch (a
 * grouped / mixture-of-experts GEMM): D_g = scaled(A_g . B_g^T), g = 0..G-1,
 * each with the 1x128 x 128x128 recipe and its own B_g.
 *
 * Defined by: the grouped blockwise GEMM pytorch/ao PR #2785 "integrate
 * torch._scaled_mm into Float8BlockwiseLinear and add bench script" mentions
 * beside the blockwise linear (review thread: ScaledGroupedMMTensor); each
 * group is exactly fp8_scaled_gemm with BLOCK_1x128_128x128.
 *
 * groups       G, 1 .. 64.
 * group_rows   HOST array of G row counts M_g >= 0 (tokens per group; 0 allowed).
 * A            the groups' rows packed: (sum M_g) x K e4m3, group g's first row
 *              at sum_{h<g} M_h; leading dim lda.
 * Bt           the groups' B^T stacked: (G*N) x K e4m3, group g at rows g*N ..
 *              g*N+N-1; leading dim ldb.
 * scale_a      1x128 grid over A's packed rows, scale_a[m + kb*ld_sa], ld_sa >= sum M_g.
 * scale_b      G grids of ceil(N/128) x ceil(K/128), group g's at scale_b +
 *              g*sb_group_stride, element [nb + kb*ld_sb]; sb_group_stride >=
 *              ld_sb * ceil(K/128).
 * D            (sum M_g) x N packed like A, dtype out_dtype, leading dim ldd.
 * Recipe BLOCK_1x128_128x128 only (others: FP8BS_ERR_UNSUPPORTED).  No split-K.
 * Alignment as fp8_scaled_gemm.  All groups empty: returns FP8BS_OK at once
 * (the matrix pointers may then be NULL).
 * Asynchronous on `stream`; group_rows is read before the call returns.
 */
fp8bs_status fp8_scaled_gemm_grouped(int64_t groups, const int64_t* group_rows, int64_t N, int64_t K,
                                     const uint8_t* A, int64_t lda, const uint8_t* Bt, int64_t ldb,
                                     const float* scale_a, int64_t ld_sa, const float* scale_b, int64_t ld_sb,
                                     int64_t sb_group_stride, fp8bs_scale_mode mode, fp8bs_scale_layout layout,
                                     void* D, int64_t ldd, fp8bs_dtype out_dtype, cudaStream_t stream);

/* Human-readable name of a status code (static string). */
const char* fp8bs_status_string(fp8bs_status s);

/*
 * fp8bs_check_device_error -- synchronizes `stream`, then reads and clears the
 * library's device-side error flag.  The GEMM kernel bounds every wait on its
 * internal pipeline barriers (a few seconds); a wait that runs out sets the
 * flag, the kernel drains its copies in flight, frees its tensor memory and
 * returns, so the CUDA context stays usable.  Returns FP8BS_ERR_TIMEOUT if the
 * flag was set by a wait, FP8BS_ERR_SCALE if it was set only by a power-of-two
 * GEMM recipe that met a scale which is not a power of two, FP8BS_ERR_CUDA if
 * the stream reports an error, else FP8BS_OK.
 */
fp8bs_status fp8bs_check_device_error(cudaStream_t stream);

/*
 * fp8bs_selftest_wait_timeout -- exercises the device-side failure detection.
 *
 * Not part of the method: a self-test of the library's bounded device waits.
 * Launches one thread that waits, with the same bounded wait the GEMM
 * pipeline uses, on an mbarrier phase nothing completes.  After `limit_ns`
 * (1 .. 10^10 ns) it sets the device error flag and returns; nothing faults or
 * hangs, and the CUDA context stays usable.  A following
 * fp8bs_check_device_error(stream) returns FP8BS_ERR_TIMEOUT (and clears it).
 */
fp8bs_status fp8bs_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8BS_H */
