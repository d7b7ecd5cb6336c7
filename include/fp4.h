/*
 * fp4.h -- C ABI of the B200 (sm_100a) block-scaled FP4 library.
 *
 * Block-scaled FP4 stores every element as a four-bit E2M1 code (1 sign,
 * 2 exponent, 1 mantissa bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) and
 * shares one scale per block of consecutive elements along the last
 * dimension:
 *   NVFP4  16-element blocks, E4M3 (FN) block scale s_b, FP32 global scale g;
 *          x_hat = q * s_b * g.
 *   MXFP4  32-element blocks, E8M0 power-of-two scale 2^e; x_hat = q * 2^e.
 * Definitions: "NVFP4 与 MXFP4 格式" (charlestar.github.io, nvfp4-mxfp4-
 * format) sections 1-5 and 8; "FP4 / NVFP4 数学总结" (devpress.csdn.net)
 * sections 3, 9 and 10; "FP4、FP8 与 INT8/INT4" (tom-jerr.github.io)
 * section 3.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers.  Every pointer is a DEVICE pointer owned by the caller.  x and
 * y must be 32-byte aligned and packed 16-byte aligned (else FP4_ERR_ALIGN:
 * the kernels move whole blocks with 256-bit vector loads and stores); scales,
 * global_scale, block_loss, status and workspace need only the alignment of
 * their element type (workspace: 4 bytes).  The library never
 * allocates, frees or synchronises; all work is queued on `stream`
 * (a cudaStream_t; NULL = the legacy default stream) and the call returns
 * as soon as it is queued.
 *
 * Layout.  x is a contiguous row-major [rows, cols] tensor of fp32 or bf16.
 * Blocks run along a row: cols must be a multiple of 16 (NVFP4, scale
 * search) or 32 (MXFP4), else FP4_ERR_SHAPE -- incomplete blocks are
 * rejected, as the pages' reference programs do.  rows * cols may be zero
 * (nothing is launched; a quantiser still writes g = 1 and no error).
 *   packed  uint8 [rows, cols/2]: element 2i in the low nibble, 2i+1 in the
 *           high nibble of byte i ("NVFP4 与 MXFP4 格式" section 1).
 *   scales  uint8 [rows, cols/16] E4M3 (NVFP4) or [rows, cols/32] E8M0
 *           (MXFP4), plain row-major, one byte per block.
 *   global_scale  one fp32 in device memory holding g = fl32(A / (6*448)),
 *           A = max|x| over the tensor: the DEQUANT multiplier (the page's
 *           `a`, not the reciprocal some GEMM interfaces call global_scale).
 *
 * Errors.  Argument errors (NULL pointer, bad shape, misalignment, unknown
 * dtype, workspace too small) are returned at once and nothing is queued.
 * Launch failures return FP4_ERR_CUDA.  Data errors are found on the GPU
 * and reported through `status`, a caller-owned device int32: a kernel
 * that finds one stores its code there only if the word still holds FP4_OK,
 * so the first error sticks until the CALLER clears the word (the library
 * never does).  When *status != FP4_OK after a call, that call's outputs are
 * unspecified.  Data errors: FP4_ERR_NONFINITE (a NaN or Inf in x) and
 * FP4_ERR_RANGE (NVFP4 global scale below the smallest normal fp32 for a
 * nonzero tensor, i.e. 0 < A < 2688 * 2^-126).
 *
 * Concurrency.  Calls on one stream are ordered.  Two calls that share a
 * workspace must not run concurrently on different streams.
 */
#ifndef FP4_B200_H
#define FP4_B200_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fp4_status {
    FP4_OK = 0,
    FP4_ERR_INVALID_ARG = 1, /* NULL pointer, unknown enum, negative size */
    FP4_ERR_SHAPE = 2,       /* cols not a multiple of the block size; overflow */
    FP4_ERR_ALIGN = 3,       /* x / y not 32-byte or packed not 16-byte aligned */
    FP4_ERR_NONFINITE = 4,   /* (device status) NaN or Inf in the input */
    FP4_ERR_RANGE = 5,       /* (device status) NVFP4 global scale out of range */
    FP4_ERR_WORKSPACE = 6,   /* workspace NULL or smaller than required */
    FP4_ERR_CUDA = 7,        /* a CUDA launch or query failed */
    FP4_ERR_TIMEOUT = 8      /* (device status) a bounded wait on a copy ran out */
} fp4_status;

typedef enum fp4_dtype { FP4_F32 = 0, FP4_BF16 = 1 } fp4_dtype;
typedef enum fp4_format { FP4_NVFP4 = 0, FP4_MXFP4 = 1 } fp4_format;

/* MXFP4 scale rule: the OCP rounding-down rule e = floor(log2 A_b) - 2, or
 * the ceil rule 2^ceil(log2(A_b / 6)) ("NVFP4 与 MXFP4 格式" section 5). */
typedef enum fp4_mx_rule { FP4_MX_FLOOR = 0, FP4_MX_CEIL = 1 } fp4_mx_rule;

/* Human-readable name of a status value (static string). */
const char *fp4_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int fp4_version(void);

/* Bytes of device workspace the NVFP4 quantiser, the scale search and the
 * tensor amax need for a [rows, cols] input: per-CTA partial maxima, a CTA
 * counter and the amax word.  Any caller-owned device buffer of at least
 * this size, 4-byte aligned, works.  It must be zero-filled once before its
 * first use (e.g. cudaMemset after allocation); every call leaves the counter
 * at zero again, and the rest of the buffer is scratch. */
size_t fp4_workspace_bytes(fp4_format fmt, int64_t rows, int64_t cols);

/* Tensor amax A = max |x| over n elements ("NVFP4 与 MXFP4 格式" section 3,
 * A is the tensor absolute maximum; section 4 reference program, first
 * step).  Writes A as one fp32 to device `amax`.  A NaN or Inf in x sets
 * FP4_ERR_NONFINITE in *status (and *amax then holds a non-finite value).
 * One launch: per-CTA maxima into `workspace`, folded by the last CTA. */
fp4_status fp4_tensor_amax(const void *x, fp4_dtype dtype, int64_t n, float *amax,
                           void *workspace, size_t workspace_bytes, int32_t *status,
                           cudaStream_t stream);

/* NVFP4 quantise + pack ("NVFP4 与 MXFP4 格式" section 3, the two-scale
 * quantiser; section 4 reference program; "FP4 / NVFP4 数学总结" section 10).
 *   g   = fl32(A / 2688); A = 0 gives g = 1.
 *   s_b = E4M3 code nearest (ties to even code) to the exact rational
 *         A_b / (6 g), saturated at 448; A_b = block max |x|.
 *   codes: zero scale -> all sixteen codes 0; else v = fl32(x / fl32(s_b*g))
 *         (IEEE single division) rounded to the nearest E2M1 value, ties to
 *         the even code, |v| > 6 saturating, the sign bit of x kept.
 * Outputs packed [rows, cols/2], scales [rows, cols/16] (E4M3 codes) and
 * *global_scale = g.  Two kernels: tensor amax into the workspace, then the
 * fused block-amax / scale / divide / round / pack pass.  Data errors:
 * NONFINITE, RANGE.
 *
 * Every kernel of the library is launched with programmatic stream
 * serialisation: it is launched as the previous kernel on the stream retires
 * its CTAs and waits for that kernel's memory operations before touching
 * memory. */
fp4_status fp4_nvfp4_quantize(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                              uint8_t *packed, uint8_t *scales, float *global_scale,
                              void *workspace, size_t workspace_bytes, int32_t *status,
                              cudaStream_t stream);

/* NVFP4 quantise + pack given a tensor amax already in device memory (for a
 * tensor split across calls or devices whose amax was combined by the
 * caller, e.g. a max all-reduce).  Same outputs and rules as
 * fp4_nvfp4_quantize with A = *amax; a non-finite *amax sets NONFINITE. */
fp4_status fp4_nvfp4_quantize_with_amax(const void *x, fp4_dtype dtype, int64_t rows,
                                        int64_t cols, const float *amax, uint8_t *packed,
                                        uint8_t *scales, float *global_scale, int32_t *status,
                                        cudaStream_t stream);

/* MXFP4 quantise + pack ("NVFP4 与 MXFP4 格式" section 2, E8M0 32-blocks;
 * section 5, the OCP rounding-down scale rule).  Per 32-block:
 * e = floor(log2 A_b) - 2 clamped to [-127, 127] (an all-zero block clamps
 * to -127), scale byte e + 127, codes of v = x * 2^-e (exact) rounded as
 * for NVFP4 (block maxima in [6, 8) * 2^e saturate to 6).  One kernel, one
 * pass.  Data error: NONFINITE. */
fp4_status fp4_mxfp4_quantize(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                              uint8_t *packed, uint8_t *scales, int32_t *status,
                              cudaStream_t stream);

/* MXFP4 quantise + pack with the ceil scale rule of "NVFP4 与 MXFP4 格式"
 * section 5 and its section 6 helper (ModelOpt-style 2^ceil(log2(A_b/6))):
 * e = max(E - 3, -127) with A_b = m 2^E (m in [0.5, 1)), plus 1 when
 * A_b > 6 * 2^e; an all-zero block gets scale 1 (byte 127).  No element
 * clips.  Otherwise as fp4_mxfp4_quantize; dequantise with FP4_MXFP4. */
fp4_status fp4_mxfp4_quantize_ceil(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                                   uint8_t *packed, uint8_t *scales, int32_t *status,
                                   cudaStream_t stream);

/* NVFP4 quantise + pack with the "four over six" block scale
 * ("FP4、FP8 与 INT8/INT4" section 4: mapping the block maximum to 4 rather
 * than 6 can place the other values on better grid points).  g as for
 * fp4_nvfp4_quantize; per block the E4M3 codes nearest to A_b/(6g) and to
 * A_b/(4g) are compared on the loss of the emitted artefact (as in
 * fp4_scale_search, summed in double); the max-to-4 scale is taken only
 * when strictly better.  block_loss (nullable) gets the chosen loss in
 * fp32.  Dequantise with FP4_NVFP4.  Data errors: NONFINITE, RANGE. */
fp4_status fp4_nvfp4_quantize_four_over_six(const void *x, fp4_dtype dtype, int64_t rows,
                                            int64_t cols, uint8_t *packed, uint8_t *scales,
                                            float *global_scale, float *block_loss,
                                            void *workspace, size_t workspace_bytes,
                                            int32_t *status, cudaStream_t stream);

/* Dequantise ("FP4 / NVFP4 数学总结" section 3, x_hat = q * s_b * g;
 * "FP4、FP8 与 INT8/INT4" section 3.2, x_hat = 2^e q).
 *   NVFP4: y = fl32(fl32(p * s_b) * g), p the E2M1 value of the code
 *          (code 8 = -0), s_b the E4M3 value of the scale byte (0x7F/0xFF
 *          -> NaN), g = *global_scale.
 *   MXFP4: y = p * 2^(byte - 127) (exact; byte 255 -> NaN); global_scale
 *          is ignored and may be NULL.
 * y is [rows, cols] of out_dtype: fp32 as computed, or bf16 rounded to
 * nearest even.  No data errors (foreign NaN scale bytes give NaN). */
fp4_status fp4_dequantize(fp4_format fmt, const uint8_t *packed, const uint8_t *scales,
                          const float *global_scale, int64_t rows, int64_t cols, void *y,
                          fp4_dtype out_dtype, cudaStream_t stream);

/* MSE-minimising NVFP4 block-scale search ("FP4 / NVFP4 数学总结" section 9,
 * Loss(s) = sum_i (x_i - s Round(x_i / s))^2; "NVFP4 与 MXFP4 格式" section 4,
 * the max-based E4M3 scale need not minimise the block MSE).
 * g as for fp4_nvfp4_quantize.  Candidates per 16-block: the E4M3 codes
 * nearest to m_k * A_b / (6 g), m_k = (147 + k) / 210, k = 0..63 (64 points
 * evenly spaced over [0.70, 1.00], each an exact rational rounded once).
 * Each candidate's loss is that of the artefact the quantiser would emit at
 * that scale (codes as in fp4_nvfp4_quantize, x_hat as in fp4_dequantize),
 * summed in double; the smallest loss wins, exact ties go to the larger
 * scale.  Emits the winner's packed codes, scale byte and g; block_loss
 * (fp32 [rows, cols/16], may be NULL) receives the winning loss rounded to
 * fp32.  Data errors: NONFINITE, RANGE. */
fp4_status fp4_scale_search(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                            uint8_t *packed, uint8_t *scales, float *global_scale,
                            float *block_loss, void *workspace, size_t workspace_bytes,
                            int32_t *status, cudaStream_t stream);

/* fp4_scale_search over a caller's candidate grid: m_k = (p + k) / q for
 * k = 0..n_cand-1 (fp4_scale_search is n_cand = 64, p = 147, q = 210); each
 * candidate the E4M3 code nearest to (p + k) A_b / (6 q g), the quotient
 * rounded once to double, exactly as the fixed grid.  Requires n_cand >= 1,
 * p >= 16 (then consecutive candidates lie within a factor 17/16, so every
 * E4M3 code between the smallest and the largest candidate is one of
 * them), p + n_cand - 1 <= 2^20 and 1 <= q <= 2^20; otherwise
 * FP4_ERR_INVALID_ARG.  m_k may exceed 1 (scales above the max-based one,
 * saturating at 448).  Everything else as fp4_scale_search. */
fp4_status fp4_scale_search_grid(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols, int n_cand, int p,
                                 int q, uint8_t *packed, uint8_t *scales, float *global_scale, float *block_loss,
                                 void *workspace, size_t workspace_bytes, int32_t *status, cudaStream_t stream);

/* Scale search given a tensor amax already in device memory (e.g. from
 * fp4_tensor_amax, shared with fp4_nvfp4_quantize_with_amax so the tensor
 * is read once for both).  Same outputs and rules as fp4_scale_search with
 * A = *amax; a non-finite *amax sets NONFINITE.  One kernel. */
fp4_status fp4_scale_search_with_amax(const void *x, fp4_dtype dtype, int64_t rows,
                                      int64_t cols, const float *amax, uint8_t *packed,
                                      uint8_t *scales, float *global_scale, float *block_loss,
                                      int32_t *status, cudaStream_t stream);

/* NVFP4 quantise + pack without a caller workspace.  No counterpart in the
 * pages: it exists for callers that cannot allocate device memory -- code
 * running where cudaMalloc is off limits (an inference-engine plugin's
 * execute callback, a serving loop that must not allocate once requests
 * flow) or whose device memory was all reserved up front and handed out as
 * tensors.  Same arguments, outputs, rules and errors as fp4_nvfp4_quantize
 * minus the workspace, which lives instead in a 4128-byte __device__ array
 * inside the library (held on every GPU that loads it until exit; enough
 * for every shape -- a shape needing more would get FP4_ERR_WORKSPACE).
 * All calls on a device share that array: calls whose kernels overlap on
 * the GPU race and must be ordered by the caller.  Each call clears the
 * array's counter word on `stream` before its kernels.  Every call looks up
 * the array's address in the current context (a non-primary context, or a
 * context created again after cudaDeviceReset, gets its own copy); the first
 * call in a context also loads the library's device code there, so make it
 * before any stream capture begins. */
fp4_status fp4_nvfp4_quantize_noalloc(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                                      uint8_t *packed, uint8_t *scales, float *global_scale,
                                      int32_t *status, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Ragged rows and column-wise grouping ("NVFP4 与 MXFP4 格式" sections 6-8).
 *
 * Padded layout.  A [rows, cols] matrix whose cols is not a multiple of the
 * block size G (16 NVFP4, 32 MXFP4) is quantised as if every row were
 * padded with +0 to Kp = ceil(cols / G) * G elements (section 8: rows *
 * ceil(cols/G) blocks, not ceil(rows*cols/G); the pad value is not given on
 * the page, and +0 changes no block maximum).  The outputs are the plain
 * layout of the padded [rows, Kp] matrix: packed uint8 [rows, Kp/2], scales
 * uint8 [rows, Kp/G]; NVFP4 g is that of the logical elements.  For cols a
 * multiple of G the padded layout is the plain one, and the calls below are
 * the plain calls.  Dequantisation of a padded layout (section 7: decode as
 * padded, then cut each row back) writes only the logical [rows, cols].
 * x must be 32-byte aligned as everywhere; y of fp4_dequantize_padded needs
 * only its element alignment.
 *
 * Column-wise grouping.  Section 6: blocks taken down the columns of W are
 * other blocks than those along its rows (Q(W)^T != Q(W^T)).  The
 * _columns calls quantise W^T, the [cols, rows] transpose of the row-major
 * x [rows, cols], without materialising it: the outputs are the padded
 * layout of W^T (packed [cols, ceil(rows/G)*G/2], scales [cols,
 * ceil(rows/G)]); decode them with fp4_dequantize_padded(rows = cols of x,
 * cols = rows of x).  x is read in 4-byte words down its columns: rows,
 * cols below 2^31 (else FP4_ERR_SHAPE) and a row pitch (cols * element
 * size) that is a multiple of 4 bytes, i.e. an even cols for bf16 (else
 * FP4_ERR_ALIGN).
 * ------------------------------------------------------------------------ */

/* NVFP4 quantise + pack of x [rows, cols], any cols >= 0, padded layout.
 * Workspace, outputs and errors as fp4_nvfp4_quantize. */
fp4_status fp4_nvfp4_quantize_padded(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                                     uint8_t *packed, uint8_t *scales, float *global_scale,
                                     void *workspace, size_t workspace_bytes, int32_t *status,
                                     cudaStream_t stream);

/* fp4_nvfp4_quantize_padded given the tensor amax already in device memory
 * (e.g. from fp4_tensor_amax, or a max all-reduce of per-rank amaxes), as
 * fp4_nvfp4_quantize_with_amax is to fp4_nvfp4_quantize: A = *amax (4-byte
 * aligned), one kernel, no workspace.  Outputs and data errors as
 * fp4_nvfp4_quantize_padded. */
fp4_status fp4_nvfp4_quantize_padded_with_amax(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                                               const float *amax, uint8_t *packed, uint8_t *scales,
                                               float *global_scale, int32_t *status, cudaStream_t stream);

/* MXFP4 quantise + pack of x [rows, cols], any cols >= 0, padded layout,
 * with scale rule `rule`.  Errors as fp4_mxfp4_quantize. */
fp4_status fp4_mxfp4_quantize_padded(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                                     fp4_mx_rule rule, uint8_t *packed, uint8_t *scales,
                                     int32_t *status, cudaStream_t stream);

/* Dequantise a padded layout of the logical [rows, cols] matrix into y
 * [rows, cols] (fp32 or bf16), as fp4_dequantize on the padded matrix
 * followed by cutting every row to cols. */
fp4_status fp4_dequantize_padded(fp4_format fmt, const uint8_t *packed, const uint8_t *scales,
                                 const float *global_scale, int64_t rows, int64_t cols, void *y,
                                 fp4_dtype out_dtype, cudaStream_t stream);

/* NVFP4 quantise + pack of W^T for x = W [rows, cols] (column-wise blocks),
 * padded layout of the [cols, rows] transpose; g from the amax of W.
 * Workspace as fp4_nvfp4_quantize.  Data errors NONFINITE, RANGE. */
fp4_status fp4_nvfp4_quantize_columns(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                                      uint8_t *packed, uint8_t *scales, float *global_scale,
                                      void *workspace, size_t workspace_bytes, int32_t *status,
                                      cudaStream_t stream);

/* fp4_nvfp4_quantize_columns given the amax of W already in device memory
 * (4-byte aligned): one kernel, no workspace.  Outputs and data errors as
 * fp4_nvfp4_quantize_columns. */
fp4_status fp4_nvfp4_quantize_columns_with_amax(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                                                const float *amax, uint8_t *packed, uint8_t *scales,
                                                float *global_scale, int32_t *status, cudaStream_t stream);

/* MXFP4 quantise + pack of W^T for x = W [rows, cols], padded layout of the
 * transpose, scale rule `rule`.  Data error NONFINITE. */
fp4_status fp4_mxfp4_quantize_columns(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                                      fp4_mx_rule rule, uint8_t *packed, uint8_t *scales,
                                      int32_t *status, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * The consumer on the tensor cores ("NVFP4 与 MXFP4 格式" section 6: with
 * both operands of Y = X W blocked along K, an output is g_X g_W times the
 * sum over blocks of s_X s_W times the block's payload dot product).
 * ------------------------------------------------------------------------ */

/* Bytes of the MMA scale layout of a [rows, blocks] scale matrix:
 * ceil(rows/128) * 128 * ceil(blocks/4) * 4. */
size_t fp4_mma_scales_bytes(int64_t rows, int64_t blocks);

/* Block scales [rows, blocks] (one byte per 16-block, row-major, as the
 * quantisers write them) -> the tiled layout the sm100 block-scaled MMA
 * reads (not on the pages): 128-row x 4-block tiles of 512 bytes, row-band
 * major with the block tiles of a band contiguous; inside a tile row r = r0
 * + 32 r1 (r0 < 32) and block j (< 4) at byte 16 r0 + 4 r1 + j; rows and
 * blocks past the matrix are 0.  out: fp4_mma_scales_bytes bytes, 4-byte
 * aligned.  One kernel. */
fp4_status fp4_scales_to_mma_layout(const uint8_t *scales, int64_t rows, int64_t blocks, uint8_t *out,
                                    cudaStream_t stream);

/* D [M, N] fp32 row-major = g_a g_b A B^T on the tensor cores (tcgen05.mma
 * kind::mxf4nvf4, 16-element blocks, E4M3 scales, fp32 accumulation in
 * tensor memory).  A: packed [M, K/2] with scales_a_mma = the MMA layout of
 * its [M, K/16] scales; B: packed [N, K/2] (the K-grouping of a K x N
 * weight stored N x K) with scales_b_mma; global scales as the quantisers
 * write them.  M and N multiples of 128, K a multiple of 256 (else
 * FP4_ERR_SHAPE); packed, scales and d 16-byte aligned.  One kernel: the
 * CTA-pair kernel (below) when M and N are multiples of 256 and its
 * 256 x 256 tiles number at least half the SMs, else one CTA per 128 x
 * 128 tile.
 * A copy that never completes ends the kernel with FP4_ERR_TIMEOUT in
 * *status.  The accumulation order inside the tensor core is the
 * hardware's: D agrees with the exact product to fp32 accumulation
 * accuracy, not bit for bit. */
fp4_status fp4_nvfp4_gemm(const uint8_t *packed_a, const uint8_t *scales_a_mma, const float *global_scale_a,
                          const uint8_t *packed_b, const uint8_t *scales_b_mma, const float *global_scale_b,
                          int64_t M, int64_t N, int64_t K, float *d, int32_t *status, cudaStream_t stream);

/* Which GEMM kernel fp4_nvfp4_gemm_ex runs. */
typedef enum fp4_gemm_kernel {
    FP4_GEMM_AUTO = 0,    /* the choice fp4_nvfp4_gemm makes */
    FP4_GEMM_CTA = 1,     /* one CTA per 128 x 128 tile of D (cta_group::1) */
    FP4_GEMM_CTA_PAIR = 2 /* persistent, one cluster of two CTAs per 256 x 256
                             tile at a time (cta_group::2, M = N = 256 MMAs);
                             M and N multiples of 256, else FP4_ERR_SHAPE */
} fp4_gemm_kernel;

/* fp4_nvfp4_gemm with the kernel named (FP4_ERR_INVALID_ARG for an unknown
 * value).  Both kernels compute the same sums; the order of the fp32
 * accumulation inside the tensor core may differ between them. */
fp4_status fp4_nvfp4_gemm_ex(const uint8_t *packed_a, const uint8_t *scales_a_mma, const float *global_scale_a,
                             const uint8_t *packed_b, const uint8_t *scales_b_mma, const float *global_scale_b,
                             int64_t M, int64_t N, int64_t K, float *d, fp4_gemm_kernel kernel, int32_t *status,
                             cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Grouped calls: many matrices per call, each with its own scales.
 *
 * The global scale is a per-tensor quantity ("NVFP4 与 MXFP4 格式" section 3:
 * A is the absolute maximum of the tensor being quantised), so a weight set
 * of many matrices is quantised matrix by matrix, each with its own A and g.
 * The grouped entry points do exactly what one single-matrix call per item
 * would do -- bit for bit the same packed codes, scale bytes, g and
 * dequantised values -- in a few launches for the whole set instead of one
 * or two per matrix.  `items` is a HOST array read during the call only;
 * every pointer inside it is a device pointer with the alignment and layout
 * rules above.  Items may be empty (rows * cols == 0).  All argument checks
 * run on every item before anything is queued.
 * ------------------------------------------------------------------------ */

/* One matrix of a grouped quantisation. */
typedef struct fp4_quant_item {
    const void *x;       /* input [rows, cols], fp32 or bf16 (the call's dtype) */
    int64_t rows, cols;  /* cols % 16 == 0 (NVFP4) or % 32 == 0 (MXFP4) */
    uint8_t *packed;     /* uint8 [rows, cols/2] */
    uint8_t *scales;     /* uint8 [rows, cols/16] E4M3 or [rows, cols/32] E8M0 */
    float *global_scale; /* NVFP4: receives this matrix's g; MXFP4: unused */
} fp4_quant_item;

/* One matrix of a grouped dequantisation. */
typedef struct fp4_dequant_item {
    const uint8_t *packed;     /* uint8 [rows, cols/2] */
    const uint8_t *scales;     /* as produced by the quantisers */
    const float *global_scale; /* NVFP4: this matrix's g; MXFP4: unused */
    void *y;                   /* output [rows, cols], fp32 or bf16 (out_dtype) */
    int64_t rows, cols;
} fp4_dequant_item;

/* Workspace of fp4_nvfp4_quantize_grouped: one 32-bit word per item,
 * rounded up to 256 bytes.  Any contents on entry (the call clears it on
 * `stream` first); after the call, in stream order, word i holds the fp32
 * bit pattern of max|x| of item i. */
size_t fp4_grouped_workspace_bytes(int n_items);

/* Tensor amax of every item: after the call, in stream order, workspace
 * word i holds max|x_i| as an fp32 (bit pattern), as fp4_tensor_amax gives
 * for item i (NVFP4 item rules: cols % 16 == 0; global_scale unused).  The
 * call clears the words on `stream` first.  A NaN or Inf in any item sets
 * NONFINITE.  One clear and one kernel per 256 items or 2^30 x 64 KB. */
fp4_status fp4_tensor_amax_grouped(const fp4_quant_item *items, int n_items, fp4_dtype dtype,
                                   void *workspace, size_t workspace_bytes, int32_t *status,
                                   cudaStream_t stream);

/* NVFP4 quantise + pack of every item given the amax words of
 * fp4_tensor_amax_grouped (`amax_words`, device, word i = item i), as
 * fp4_nvfp4_quantize_with_amax per item.  One kernel per 256 items or 2^30
 * blocks. */
fp4_status fp4_nvfp4_quantize_grouped_with_amax(const fp4_quant_item *items, int n_items,
                                                fp4_dtype dtype, const void *amax_words,
                                                int32_t *status, cudaStream_t stream);

/* NVFP4 quantise + pack of every item, each with its own tensor amax and
 * global scale g_i = fl32(A_i / 2688), exactly as fp4_nvfp4_quantize per
 * item.  A NaN or Inf in any item sets NONFINITE; an item whose g underflows
 * sets RANGE; the outputs of such an item are unspecified, the others are
 * still correct.  fp4_tensor_amax_grouped followed by
 * fp4_nvfp4_quantize_grouped_with_amax on the workspace. */
fp4_status fp4_nvfp4_quantize_grouped(const fp4_quant_item *items, int n_items, fp4_dtype dtype,
                                      void *workspace, size_t workspace_bytes, int32_t *status,
                                      cudaStream_t stream);

/* MXFP4 quantise + pack of every item, as fp4_mxfp4_quantize per item
 * (OCP rounding-down scale rule); _ceil: as fp4_mxfp4_quantize_ceil.  One
 * kernel per 256 items or 2^30 blocks. */
fp4_status fp4_mxfp4_quantize_grouped(const fp4_quant_item *items, int n_items, fp4_dtype dtype,
                                      int32_t *status, cudaStream_t stream);
fp4_status fp4_mxfp4_quantize_ceil_grouped(const fp4_quant_item *items, int n_items,
                                           fp4_dtype dtype, int32_t *status, cudaStream_t stream);

/* Dequantise every item, as fp4_dequantize per item.  One kernel per 256
 * items or 2^30 units of 16 codes. */
fp4_status fp4_dequantize_grouped(fp4_format fmt, const fp4_dequant_item *items, int n_items,
                                  fp4_dtype out_dtype, cudaStream_t stream);

/* Tests only: the largest number of work units one launch takes (default
 * 2^30, restored by units = 0; else a multiple of 64 from 64 up).  Every
 * call above splits larger problems into several launches at this limit;
 * lowering it makes small tensors cross those split points.  Process-wide,
 * not thread-safe; set it only while no other call is being made.
 * FP4_ERR_INVALID_ARG for other values. */
fp4_status fp4_set_launch_unit_limit(int64_t units);

/* Launch planner of the grouped calls alone, for tests (host only, no GPU
 * work).  Splits items of units[i] work units into launches of at most
 * max_units units (64 .. 2^30) and max_entries entries (1 .. 256), as the
 * grouped calls do with the largest limits: piece k covers units
 * [first_of[k], first_of[k] + count_of[k]) of item item_of[k] in launch
 * launch_of[k].  Returns the number of pieces (the arrays hold the first
 * max_pieces of them), or -1 for invalid arguments. */
int fp4_grouped_plan(const int64_t *units, int n_items, int64_t max_units, int max_entries,
                     int32_t *launch_of, int32_t *item_of, int64_t *first_of, int64_t *count_of,
                     int max_pieces);

/* Element encoder alone, for tests: codes[i] = E2M1 code of the fp32 value
 * v[i] (nearest, ties to even code, saturating, sign bit kept).  A NaN or
 * Inf in v gives an unspecified code.  codes is uint8 [n] (one code per
 * byte, unpacked). */
fp4_status fp4_e2m1_round(const float *v, uint8_t *codes, int64_t n, cudaStream_t stream);

/* E2M1 round trip alone, for tests: out[2i] = value of the code of v[i]
 * decoded from the packed codes the encoder returns in registers, and
 * out[2i+1] = the same value from the fused quantise-dequantise routine the
 * scale search uses.  out is fp32 [2n]. */
fp4_status fp4_e2m1_roundtrip(const float *v, float *out, int64_t n, cudaStream_t stream);

/* NVFP4 element quotient + encoder alone, for tests: codes[i] = E2M1 code
 * of fl32(x[i] / d[i]) computed by the same device routine the NVFP4
 * quantiser uses for one element (d[i] > 0 finite, x[i] finite). */
fp4_status fp4_nv_encode_quotient(const float *x, const float *d, uint8_t *codes, int64_t n,
                                  cudaStream_t stream);

/* Bounded wait alone, for tests: one warp waits on a shared-memory barrier
 * that nothing arrives on, for `tries` polls (1 .. 2^18; every wait of the
 * kernels that copy with TMA is bounded the same way, at 2^18 polls of about
 * 4 us each, i.e. about a second).  When the
 * wait runs out the kernel records FP4_ERR_TIMEOUT in *status (first error
 * sticks) and returns, leaving the context usable; *elapsed_ns (device
 * int64) receives the wait's duration on the GPU's global timer.
 * FP4_ERR_INVALID_ARG for other tries or NULL pointers. */
fp4_status fp4_test_bounded_wait(uint32_t tries, int32_t *status, int64_t *elapsed_ns, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FP4_B200_H */
