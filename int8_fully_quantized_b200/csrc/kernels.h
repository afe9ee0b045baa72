// Internal launch functions (called by the C ABI in api.cu after argument validation).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

namespace jf {

// The driver's cuTensorMapEncodeTiled (null if the driver does not provide it).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// `status`: the device status word, raised when a bounded wait in the kernel runs out; null selects
// the plain-load kernel (no TMA staging, no waits). `stats` (optional, int32 [R][C/32][2]): per row
// and block, the sums of q and q^2 (what LayerNorm_i8 needs of its input rows).
cudaError_t launch_quantize(const void* x, int dtype, int64_t R, int64_t C, int8_t* q, float* s, int32_t* stats,
                            unsigned int* status, int sm_count, cudaStream_t st);
cudaError_t launch_dequantize(const int8_t* q, const float* s, int64_t R, int64_t C, void* y, int dtype,
                              int sm_count, cudaStream_t st);
cudaError_t launch_gelu_i8(const int8_t* q, const float* s, int64_t R, int64_t C, int8_t* qo, float* so,
                           int sm_count, cudaStream_t st);
// Failure-path self-test (selftest.cu): a bounded wait that runs out after limit_ns and raises the
// timeout bit of *status.
cudaError_t launch_wait_selftest(unsigned int* status, unsigned long long limit_ns, cudaStream_t st);

// MXFP8 comparison path (mxfp8.cu): MX quantization (E4M3 codes, E8M0 scale bytes per 1x32 block of
// a row) and Y = A B^T with the tensor core's block scaling (K a multiple of 128).
cudaError_t launch_mx_quantize(const void* x, int dtype, int64_t R, int64_t K, uint8_t* codes, uint8_t* scales,
                               int sm_count, cudaStream_t st);
cudaError_t launch_mx_gemm(const uint8_t* a_q, const uint8_t* a_s, const uint8_t* b_q, const uint8_t* b_s, int64_t M,
                           int64_t N, int64_t K, float* y, unsigned int* status, int sm_count, cudaStream_t st);

// Granularity variants of the quantizer and the quantization-error sums (granular.cu). Scales:
// block [R/32, C/32], token [R], channel [C], tensor [1].
enum Granularity { kGranBlock = 0, kGranToken = 1, kGranChannel = 2, kGranTensor = 3 };
cudaError_t launch_quantize_granular(const void* x, int dtype, int64_t R, int64_t C, int g, int8_t* q, float* s,
                                     unsigned int* status, int sm_count, cudaStream_t st);
cudaError_t launch_dequantize_granular(const int8_t* q, const float* s, int64_t R, int64_t C, int g, void* y,
                                       int dtype, int sm_count, cudaStream_t st);
cudaError_t launch_quant_error(const void* x, int dtype, const int8_t* q, const float* s, int64_t R, int64_t C, int g,
                               double* sums, int sm_count, cudaStream_t st);

// INT8 backward of GELU_i8 and LayerNorm_i8 (backward.cu). `part` is the fp32 workspace of
// per-CTA column sums, [ln_bwd_ctas(R)][2][H]; null when neither dgamma nor dbeta is wanted.
constexpr int64_t kLnBwdMaxCtas = 296;   // two resident CTAs on each of 148 SMs
constexpr int64_t kLnBwdMaxCols = 24576; // the [2][H] fp32 accumulators fit in one SM's shared memory
int64_t ln_bwd_ctas(int64_t R);
// Size of the static scratch the allocation-free LayerNorm backward uses in place of a workspace,
// and its device address on the current device (looked up once per device; null on failure).
constexpr int64_t kLnBwdScratchBytes = int64_t(16) << 20;
float* ln_bwd_static_scratch();
cudaError_t launch_gelu_i8_bwd(const int8_t* xq, const float* xs, const int8_t* dq, const float* ds, int64_t R,
                               int64_t C, int8_t* qo, float* so, int sm_count, cudaStream_t st);
cudaError_t launch_layernorm_i8_bwd(const int8_t* xq, const float* xs, const int8_t* dq, const float* ds, int64_t R,
                                    int64_t H, const float* gamma, float eps, int8_t* qo, float* so, float* part,
                                    float* dgamma, float* dbeta, cudaStream_t st);
cudaError_t launch_layernorm_i8(const int8_t* q, const float* s, int64_t R, int64_t H, const float* gamma,
                                const float* beta, float eps, int8_t* qo, float* so, const int32_t* stats,
                                cudaStream_t st);

// Block-scaled INT8 GEMM: out[r, c] = sum over 32-blocks kb of the contraction axis of
// fp32(sA(r/32, kb) * sB(c/32, kb)) * sum_{k in kb} A(r, k) B(c, k), re-quantized per 32x32 block.
// The operand views differ per mode (see gemm.cu).
enum GemmMode { kFwd = 0, kDgrad = 1, kWgrad = 2 };
enum GemmAct { kActNone = 0, kActGelu = 1 };

struct GemmArgs {
  int mode;
  const int8_t* a_q;  // A codes (X for fwd, dY for dgrad and wgrad)
  const float* a_s;
  const int8_t* b_q;  // B codes (W for fwd and dgrad, X for wgrad)
  const float* b_s;
  int64_t rows, cols, depth;  // output rows, output cols, contraction length
  int64_t a_ld, b_ld;         // row pitch (elements) of the stored A and B matrices
  int8_t* y_q;                // nullable
  float* y_s;                 // non-null when y_q is
  float* y_f32;               // nullable
  int act;                    // GemmAct: activation applied to the fp32 result before y is written
  int8_t* pre_q;              // nullable (kActGelu only): the re-quantized pre-activation
  float* pre_s;               // non-null when pre_q is
  unsigned int* status;       // device status word (bit flags of ptx.cuh)
};

cudaError_t launch_gemm(const GemmArgs& g, int sm_count, cudaStream_t st);

// Plain INT8 GEMM C = A B^T (int32), A [M, K] and B [N, K] row-major: the tensor core's INT8 rate with
// no per-block rescale. M % 128 == 0, N % 256 == 0, K % 128 == 0.
cudaError_t launch_gemm_s32(const int8_t* a, const int8_t* b, int32_t* c, int64_t M, int64_t N, int64_t K,
                            unsigned int* status, int sm_count, cudaStream_t st);

}  // namespace jf
