/*
 * jetfire.h - C ABI of the per-block (32x32) INT8 data-flow library for B200 (sm_100a).
 *
 * What is computed (source: "Jetfire: Efficient and Accurate Transformer Pretraining with INT8
 * Data Flow and Per-Block Quantization", atlas.scime.ai summary page, section "Approach"):
 * every linear and non-linear operator of a transformer layer reads and writes INT8 tensors that
 * carry one scale factor per block, with block size B = 32; quantization is applied on-chip, and
 * the weight gradient, too, is an INT8 product with per-block scales. The "Fp8 vs int8" page gives
 * the signed INT8 range and the dequantization x = FP(q) * s.
 *
 * Readings taken where the pages are silent (each is stated once here and applies to every call):
 *   - blocks are 32 x 32; block (I, J) covers rows 32I..32I+31 and columns 32J..32J+31;
 *   - the scale of a block is s = absmax / 127 in fp32 (IEEE division, no zero point);
 *   - a code is q = clamp(rint(x / s), -127, 127): IEEE fp32 quotient, round half to even;
 *     -128 is never produced (it is accepted on input); an all-zero block, or one whose s
 *     underflows to 0, gets s = 0 and codes 0; subnormals are honoured (no flush to zero);
 *   - the GEMMs rescale the exact int32 partial of every 32-wide block of the contraction axis by
 *     fp32(s_A * s_B) and accumulate in fp32 (block order unspecified), then re-quantize the fp32
 *     result per 32x32 block on-chip;
 *   - GELU is 0.5 x (1 + erf(x / sqrt 2)); LayerNorm uses the biased variance over the full row.
 *
 * Data layout (all device memory, all row-major and contiguous, all owned by the caller):
 *   a quantized tensor T of shape [rows, cols] is a pair
 *     T.q  int8  [rows, cols]          codes, 16-byte aligned
 *     T.s  fp32  [rows/32, cols/32]    one scale per block, 4-byte aligned
 *   rows and cols must be multiples of 32 (0 is allowed: the call does nothing).
 *
 * Execution: every call validates its arguments on the host, returns an error code without
 * enqueuing anything if they are invalid, otherwise enqueues its kernel(s) on `stream` (a
 * cudaStream_t passed as void*; NULL = the legacy default stream) and returns without waiting.
 * The library allocates, frees and retains no device memory of its own per call: every buffer is
 * the caller's. The one exception is a 16 MiB static scratch array that the library's module holds
 * on each device where it is loaded, used only by jf_layernorm_i8_bwd_noalloc. Resetting a device
 * (cudaDeviceReset) while the library is loaded is not supported. Outputs must not overlap inputs.
 * Inputs must be finite. Kernel-side failures (a bounded wait that timed out) are reported by
 * jf_device_status(). Calls are thread-safe; calls on different streams may run concurrently.
 * There is no CPU fallback: on a machine without an sm_100 GPU every compute call returns
 * JF_ERR_DEVICE.
 */
#ifndef JETFIRE_H
#define JETFIRE_H

#include <stdint.h>

#if defined(__GNUC__)
#define JF_API __attribute__((visibility("default")))
#else
#define JF_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Read-only quantized tensor (device pointers). */
typedef struct {
  const int8_t* q;
  const float* s;
  int64_t rows, cols;
} jf_cqtensor;

/* Writable quantized tensor (device pointers). */
typedef struct {
  int8_t* q;
  float* s;
  int64_t rows, cols;
} jf_qtensor;

/* Element types of unquantized tensors. */
typedef enum { JF_F32 = 0, JF_BF16 = 1, JF_F16 = 2 } jf_dtype;

/* Status codes. */
typedef enum {
  JF_OK = 0,
  JF_ERR_NULL = -1,    /* a required pointer is NULL */
  JF_ERR_SHAPE = -2,   /* a dimension is negative, not a multiple of 32, or shapes disagree */
  JF_ERR_ALIGN = -3,   /* a pointer is not aligned as documented */
  JF_ERR_DTYPE = -4,   /* unknown jf_dtype */
  JF_ERR_ALIAS = -5,   /* an output overlaps an input */
  JF_ERR_CUDA = -6,    /* a CUDA runtime or driver call failed (launch, tensor-map encode) */
  JF_ERR_TIMEOUT = -7, /* reported by jf_device_status: a kernel's bounded wait ran out */
  JF_ERR_DEVICE = -8,  /* no usable sm_100 device is current */
  JF_ERR_WORKSPACE = -9, /* the caller's workspace is NULL, misaligned or smaller than required */
  JF_ERR_ARG = -10       /* an enumerated argument (jf_granularity) is unknown */
} jf_status;

/* Scale granularity of the quantizer variants (f3): one fp32 scale per 32x32 block ([rows/32,
 * cols/32], the Jetfire rule), per row / token ([rows]), per column / channel ([cols]), or one for
 * the whole tensor ([1]). */
typedef enum { JF_GRAN_BLOCK = 0, JF_GRAN_TOKEN = 1, JF_GRAN_CHANNEL = 2, JF_GRAN_TENSOR = 3 } jf_granularity;

/*
 * a1. Per-block quantization (summary, "Approach": per-block scale factors, B = 32).
 *   x     device, [rows, cols] row-major of dtype `dt` (fp32, bf16 or fp16), 16-byte aligned
 *   q     device, int8 [rows, cols], 16-byte aligned (output)
 *   s     device, fp32 [rows/32, cols/32], 4-byte aligned (output)
 * Codes and scales are bit-exact with the rule above (bf16/fp16 are widened exactly first).
 * The kernel stages x through shared memory with TMA tile loads and waits on them with bounded
 * waits: if one runs out, the kernel gives up and jf_device_status reports JF_ERR_TIMEOUT. With
 * JF_PLAIN_LOADS=1 in the environment when the library is loaded (read once, at load time) a kernel
 * with plain loads runs instead (the path for inputs the driver cannot describe with a tensor map);
 * its results are identical.
 */
JF_API int jf_quantize_block(const void* x, jf_dtype dt, int64_t rows, int64_t cols, int8_t* q, float* s,
                      void* stream);

/*
 * f1 (second half). jf_quantize_block that also writes the row statistics LayerNorm_i8 needs of
 * its input (summary, "Approach": quantization on-chip; here the LayerNorm's row sums move into the
 * op that produces its input, so the LayerNorm needs no pass of its own to find them).
 *   stats  device int32 [rows][cols/32][2], 8-byte aligned (output): for row r and block column J,
 *          (sum of q[r, j], sum of q[r, j]^2) over the block's 32 columns (exact integers).
 * q and s are identical to jf_quantize_block's. Errors as jf_quantize_block, plus JF_ERR_NULL /
 * JF_ERR_ALIGN / JF_ERR_ALIAS for stats.
 */
JF_API int jf_quantize_block_rowstats(const void* x, jf_dtype dt, int64_t rows, int64_t cols, int8_t* q, float* s,
                                      int32_t* stats, void* stream);

/*
 * a2. Dequantization y = fp32(q) * s, rounded to nearest even into `dt` ("Fp8 vs int8" page).
 *   q, s  the quantized tensor (device, layout as above)
 *   y     device, [rows, cols] of dtype `dt`, 16-byte aligned (output); bit-exact.
 */
JF_API int jf_dequantize_block(const int8_t* q, const float* s, int64_t rows, int64_t cols, void* y, jf_dtype dt,
                        void* stream);

/*
 * a3. Linear forward Y = X W^T (summary, "Approach": INT8 linear operator with per-block scales).
 *   X  [M, K] quantized activations, W [N, K] quantized weights, Y [M, N] (output).
 *   Y(m, n) = sum_kb fp32(sX(m/32, kb) sW(n/32, kb)) * sum_{k in kb} Xq(m, k) Wq(n, k),
 *   re-quantized per 32x32 block into Y.q / Y.s.
 *   y_f32  optional device fp32 [M, N] (16-byte aligned) that receives the fp32 result before
 *          re-quantization. Y.q may be NULL (then Y.s is ignored) when y_f32 is given; at least
 *          one of the two outputs is required.
 */
JF_API int jf_linear_fwd(jf_cqtensor X, jf_cqtensor W, jf_qtensor Y, float* y_f32, void* stream);

/*
 * f1. Linear forward with GELU fused into the re-quantization epilogue (summary, "Approach":
 *     quantization happens on-chip; here the activation that follows fc1 happens there too).
 *   X [M, K], W [N, K] as in jf_linear_fwd. With P the fp32 pre-activation that jf_linear_fwd
 *   computes, Y = requant(GELU(P)) per 32x32 block, GELU in its exact erf form applied to the fp32
 *   P (not to its INT8 re-quantization), so the result differs from jf_linear_fwd followed by
 *   jf_gelu_i8 by that one rounding step.
 *   Y     [M, N] output; Y.q and Y.s are required.
 *   Ypre  optional [M, N] output: requant(P), identical to jf_linear_fwd's Y. Pass Ypre.q = NULL to
 *         skip it; it is what the backward of GELU needs.
 *   Errors as jf_linear_fwd; JF_ERR_NULL when Y.q is NULL; JF_ERR_ALIAS when any two of the
 *   outputs, or an output and an input, overlap.
 */
JF_API int jf_linear_fwd_gelu(jf_cqtensor X, jf_cqtensor W, jf_qtensor Y, jf_qtensor Ypre, void* stream);

/*
 * a4. Input gradient dX = dY W (the INT8 backward of the linear layer).
 *   dY [M, N], W [N, K] (read re-blocked along N, no transpose pass), dX [M, K] (output).
 *   dX(m, k) = sum_nb fp32(sdY(m/32, nb) sW(nb, k/32)) * sum_{n in nb} dYq(m, n) Wq(n, k).
 *   dx_f32 as y_f32 above.
 */
JF_API int jf_linear_dgrad(jf_cqtensor dY, jf_cqtensor W, jf_qtensor dX, float* dx_f32, void* stream);

/*
 * a5. Weight gradient dW = dY^T X (summary, "Approach": the weight gradient, too, is an INT8
 *     product with one scale per block).
 *   dY [M, N], X [M, K] (both read re-blocked along M), dW [N, K] (output).
 *   dW(n, k) = sum_mb fp32(sdY(mb, n/32) sX(mb, k/32)) * sum_{m in mb} dYq(m, n) Xq(m, k).
 *   dw_f32 as y_f32 above (an optimizer, or a data-parallel gradient reduction, wants fp32).
 */
JF_API int jf_linear_wgrad(jf_cqtensor dY, jf_cqtensor X, jf_qtensor dW, float* dw_f32, void* stream);

/*
 * a6. GELU on INT8 blocks (summary, "Approach" and "Problem": non-linear operators read and write
 *     INT8 with per-block scales). Y = requant(GELU(fp32(X.q) * X.s)), same shape as X.
 */
JF_API int jf_gelu_i8(jf_cqtensor X, jf_qtensor Y, void* stream);

/*
 * a7. LayerNorm on INT8 blocks. Per row r of X [M, H]: x = fp32(q) * s, mean and biased variance
 *     over the H columns, y = (x - mean) / sqrt(var + eps) * gamma + beta, re-quantized per block.
 *   gamma, beta  device fp32 [H], 16-byte aligned.
 */
JF_API int jf_layernorm_i8(jf_cqtensor X, const float* gamma, const float* beta, float eps, jf_qtensor Y,
                    void* stream);

/*
 * f1 (second half). jf_layernorm_i8 with each row's mean and biased variance formed from `stats`,
 * the row statistics jf_quantize_block_rowstats wrote for X (mean = sum_J s * S1 / H, mean square
 * = sum_J s^2 * S2 / H, in fp64), so X is read once. The caller passes the stats of this X; the
 * result is then LayerNorm_i8 of X (the row sums are the same numbers, added in another order).
 *   stats  device int32 [rows][cols/32][2], 8-byte aligned.
 * Errors as jf_layernorm_i8, plus JF_ERR_NULL / JF_ERR_ALIGN / JF_ERR_ALIAS for stats.
 */
JF_API int jf_layernorm_i8_rowstats(jf_cqtensor X, const int32_t* stats, const float* gamma, const float* beta,
                                    float eps, jf_qtensor Y, void* stream);

/*
 * f2. Backward of GELU_i8 (summary, "Approach": the backward pass keeps the INT8 data flow too).
 *   X   [M, N] the saved pre-activation (the forward's input), dY [M, N] the upstream gradient,
 *   dX  [M, N] output: requant(fp32(dY.q) dY.s * GELU'(fp32(X.q) X.s)) per 32x32 block, where
 *       GELU'(x) = Phi(x) + x phi(x) (Phi, phi: the standard normal CDF and density).
 *   Errors: JF_ERR_SHAPE if the three shapes differ; JF_ERR_ALIAS if dX overlaps an input.
 */
JF_API int jf_gelu_i8_bwd(jf_cqtensor X, jf_cqtensor dY, jf_qtensor dX, void* stream);

/*
 * f2. Backward of LayerNorm_i8 (same layer as jf_layernorm_i8, same eps).
 *   X      [M, H] the forward's input; dY [M, H] the upstream gradient; gamma fp32 [H] (16-byte
 *          aligned). Per row, with x = fp32(q) s, xhat = (x - mean) rstd, rstd = 1 / sqrt(var + eps)
 *          and g = dy gamma:
 *            dX = requant(rstd (g - mean(g) - xhat mean(g xhat))) per 32x32 block,
 *          and over all rows dgamma = sum dy xhat, dbeta = sum dy (fp32 [H], deterministic).
 *   dgamma, dbeta  nullable device fp32 [H]; when either is given, `workspace` must hold at least
 *          jf_layernorm_i8_bwd_workspace_bytes(M, H) bytes of caller-owned device memory, 16-byte
 *          aligned (per-CTA column sums; its contents on entry do not matter). Otherwise the
 *          workspace is not used and may be NULL.
 *   H is at most 24576 (the column sums of a CTA live in shared memory).
 *   Errors: JF_ERR_NULL if gamma or dX.q is NULL; JF_ERR_SHAPE for H > 24576; JF_ERR_WORKSPACE as
 *          above; JF_ERR_ALIAS if any output (workspace included) overlaps an input or another output.
 */
JF_API int jf_layernorm_i8_bwd(jf_cqtensor X, jf_cqtensor dY, const float* gamma, float eps, jf_qtensor dX,
                               float* dgamma, float* dbeta, void* workspace, int64_t workspace_bytes,
                               void* stream);

/* Bytes of workspace jf_layernorm_i8_bwd needs for X of [rows, cols]:
 * min(rows / 32, 296) * 2 * cols * 4, or -1 for an invalid shape (cols > 24576 included). */
JF_API int64_t jf_layernorm_i8_bwd_workspace_bytes(int64_t rows, int64_t cols);

/*
 * Allocation-free variant of jf_layernorm_i8_bwd (no counterpart on the pages: an engineering entry
 * point for callers that cannot provide a workspace). Same arguments, results and errors, checked in
 * the same order, but the per-CTA column sums go to a 16 MiB scratch array that the library holds in
 * device memory for its whole lifetime, so neither the caller nor the library allocates anything per
 * call. After every other argument check has passed, shapes whose workspace
 * (jf_layernorm_i8_bwd_workspace_bytes) exceeds 16 MiB are rejected with JF_ERR_WORKSPACE before
 * anything is enqueued. The scratch is shared by every call on a device: calls of this function that
 * ask for dgamma or dbeta must not run concurrently with each other (issue them on one stream).
 * Without dgamma and dbeta it is jf_layernorm_i8_bwd with no workspace.
 */
JF_API int jf_layernorm_i8_bwd_noalloc(jf_cqtensor X, jf_cqtensor dY, const float* gamma, float eps,
                                       jf_qtensor dX, float* dgamma, float* dbeta, void* stream);

/*
 * The plain INT8 tensor-core product C = A B^T with an int32 result and no scales (no counterpart
 * on the pages: it measures the tensor core's INT8 rate, the ceiling the block-scaled GEMMs above
 * are reported against, with the same TMA / tcgen05 machinery and no per-block rescale).
 *   A  device int8 [M, K] row-major, B device int8 [N, K] row-major (both 16-byte aligned)
 *   C  device int32 [M, N] row-major, 16-byte aligned (output), exact.
 *   M a multiple of 128, N of 256, K of 128 and at most 65536 (no int32 overflow); else JF_ERR_SHAPE.
 *   Errors: JF_ERR_NULL, JF_ERR_ALIGN, JF_ERR_ALIAS (C overlaps A or B) as elsewhere.
 */
JF_API int jf_gemm_i8_s32(const int8_t* A, const int8_t* B, int32_t* C, int64_t M, int64_t N, int64_t K,
                          void* stream);

/*
 * f3. Quantization at another granularity: the baselines of the summary's ablation ("Measured
 *     effects table": per-block scales quantize activations with channel outliers more accurately
 *     than per-token ones). The rule is that of jf_quantize_block (s = absmax / 127, IEEE quotient,
 *     round half to even, clamp to +-127, s = 0 and codes 0 for an all-zero group), with one scale
 *     per group of the granularity `g`. x as in jf_quantize_block; q int8 [rows, cols] (16-byte
 *     aligned); s fp32 with jf_granular_scale_count(rows, cols, g) entries (4-byte aligned).
 *     Codes and scales are bit-exact. JF_GRAN_BLOCK is jf_quantize_block.
 */
JF_API int jf_quantize_granular(const void* x, jf_dtype dt, int64_t rows, int64_t cols, jf_granularity g, int8_t* q,
                                float* s, void* stream);

/* Number of scales of a [rows, cols] tensor at granularity g, or -1 for an invalid shape or g. */
JF_API int64_t jf_granular_scale_count(int64_t rows, int64_t cols, jf_granularity g);

/* f3. y = fp32(q) * s of the element's group, rounded to nearest even into dt (bit-exact). */
JF_API int jf_dequantize_granular(const int8_t* q, const float* s, int64_t rows, int64_t cols, jf_granularity g,
                                  void* y, jf_dtype dt, void* stream);

/*
 * f3. The error of a quantization (the summary's accuracy metric behind the ablation): writes
 *     sums[0] = sum over elements of (x - q s)^2, sums[1] = sum of x^2 and
 *     sums[2] = sums[0] / (rows * cols), the mean squared error, in fp64 to the device array `sums`
 *     (3 doubles, 8-byte aligned); x, q and s as above, all exact in fp64, so only the order of the
 *     fp64 additions (unspecified) affects the sums. An empty tensor gives three zeros.
 */
JF_API int jf_quantization_error(const void* x, jf_dtype dt, const int8_t* q, const float* s, int64_t rows,
                                 int64_t cols, jf_granularity g, double* sums, void* stream);

/*
 * f4. MXFP8 comparison (OCP Microscaling Formats v1.0; not on the pages: the B200's hardware block
 *     scaling, measured beside the per-block INT8 path). Quantization of x [rows, cols] (dtype dt,
 *     16-byte aligned) in blocks of 32 consecutive elements of a row: e = floor(log2(max |x|)) - 8
 *     clamped to [-127, 127] (-127 for an all-zero block), scale byte e + 127 (E8M0), codes = E4M3
 *     of x * 2^-e, round to nearest even, saturating at +-448.
 *   codes   uint8 [rows, cols], 16-byte aligned; scales uint8 [rows, cols / 32]. Bit-exact.
 */
JF_API int jf_mx_quantize(const void* x, jf_dtype dt, int64_t rows, int64_t cols, uint8_t* codes, uint8_t* scales,
                          void* stream);

/*
 * f4. Y = A B^T with A [M, K] and B [N, K] in MXFP8 (codes and scale bytes as jf_mx_quantize
 *     writes them), on tcgen05.mma kind::mxf8f6f4.block_scale: the tensor core applies the scales
 *     and accumulates in fp32. y fp32 [M, N] (16-byte aligned). K must be a positive multiple of 128
 *     and the scale arrays 4-byte aligned (JF_ERR_SHAPE / JF_ERR_ALIGN otherwise).
 */
JF_API int jf_mx_linear_fwd(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* b_codes,
                            const uint8_t* b_scales, int64_t M, int64_t N, int64_t K, float* y, void* stream);

/*
 * Self-test of the failure path (no counterpart on the pages): enqueues a kernel whose bounded wait
 * on a barrier that nothing arrives on gives up after limit_ns nanoseconds (1 ms .. 10 s, else
 * JF_ERR_ARG), the same way any kernel of the library gives up a wait. The next jf_device_status
 * then returns JF_ERR_TIMEOUT and clears the status; the context stays usable.
 */
JF_API int jf_selftest_wait_timeout(int64_t limit_ns, void* stream);

/* Static description of a status code (never NULL). */
JF_API const char* jf_strerror(int status);

/*
 * Synchronizes `stream`, then returns and clears the device-side status of the library on the
 * current device: JF_OK, or JF_ERR_TIMEOUT if a kernel gave up a bounded wait since the last
 * call (its outputs are then undefined), or JF_ERR_CUDA if the synchronization failed.
 */
JF_API int jf_device_status(void* stream);

/* Number of SMs of the current device, as the kernels size their grids (0 if none). */
JF_API int jf_sm_count(void);

#ifdef __cplusplus
}
#endif

#endif /* JETFIRE_H */
