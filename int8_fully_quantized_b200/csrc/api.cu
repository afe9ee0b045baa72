// C ABI of the library: argument validation, then the kernel launch (see include/jetfire.h).
#include <cstdint>
#include <cstdlib>
#include <mutex>
#include <cuda_runtime.h>

// NVTX ranges around the compute entry points, compiled in only with -DJF_NVTX (the separate
// instrumented build of build_lib.py --nvtx): header-only NVTX 3, no library to link.
#ifdef JF_NVTX
#include <nvtx3/nvToolsExt.h>
namespace {
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};
}  // namespace
#define JF_RANGE(name) const NvtxRange jf_nvtx_range_(name)
#else
#define JF_RANGE(name) ((void)0)
#endif

#include "jetfire.h"
#include "kernels.h"
#include "ptx.cuh"

namespace jf {
__device__ unsigned int g_status = 0u;
}

namespace {

struct DevInfo {
  int sm_count = 0;
  bool ok = false;
  unsigned int* status = nullptr;  // device address of jf::g_status on this device
};

// Per-device SM count and capability check (cached per device ordinal; the first call on a device
// fills its entry under a lock, so concurrent first calls from several threads are safe). The
// cached status-word address belongs to the device's primary context: resetting the device
// (cudaDeviceReset) while the library is loaded is not supported.
DevInfo device_info() {
  static std::mutex mu;
  static DevInfo cache[64];
  static bool probed[64] = {false};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return DevInfo{};
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!probed[dev]) {
    DevInfo d;
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess) {
      d.ok = (major == 10);
      d.sm_count = sms;
      void* addr = nullptr;
      if (cudaGetSymbolAddress(&addr, jf::g_status) == cudaSuccess) {
        d.status = static_cast<unsigned int*>(addr);
      } else {
        cudaGetLastError();
        d.ok = false;
      }
    } else {
      cudaGetLastError();
    }
    cache[dev] = d;
    probed[dev] = true;
  }
  return cache[dev];
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
inline bool dims_ok(int64_t r, int64_t c) {
  return r >= 0 && c >= 0 && (r % 32) == 0 && (c % 32) == 0 && r < (int64_t(1) << 31) && c < (int64_t(1) << 31);
}
inline bool overlap(const void* a, int64_t na, const void* b, int64_t nb) {
  if (a == nullptr || b == nullptr || na <= 0 || nb <= 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + uintptr_t(nb) && b0 < a0 + uintptr_t(na);
}
inline int64_t elem_size(jf_dtype dt) { return dt == JF_F32 ? 4 : 2; }
inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? JF_OK : JF_ERR_CUDA; }

// JF_PLAIN_LOADS=1 in the environment when the library is loaded selects the quantizer's plain-load
// kernel, which otherwise serves only inputs the driver will not describe with a TMA tensor map. The
// variable is read once, at load time, so no call reads the environment.
const bool g_plain_loads = [] {
  const char* v = std::getenv("JF_PLAIN_LOADS");
  return v != nullptr && v[0] == '1';
}();
inline bool plain_loads_forced() { return g_plain_loads; }

int check_cq(const jf_cqtensor& t) {
  if (!dims_ok(t.rows, t.cols)) return JF_ERR_SHAPE;
  if (t.rows == 0 || t.cols == 0) return JF_OK;
  if (t.q == nullptr || t.s == nullptr) return JF_ERR_NULL;
  if (!aligned(t.q, 16) || !aligned(t.s, 4)) return JF_ERR_ALIGN;
  return JF_OK;
}

// Output quantized tensor; `need_q` false allows q == NULL (fp32-only output).
int check_q(const jf_qtensor& t, bool need_q) {
  if (!dims_ok(t.rows, t.cols)) return JF_ERR_SHAPE;
  if (t.rows == 0 || t.cols == 0) return JF_OK;
  if (t.q == nullptr) return need_q ? JF_ERR_NULL : JF_OK;
  if (t.s == nullptr) return JF_ERR_NULL;
  if (!aligned(t.q, 16) || !aligned(t.s, 4)) return JF_ERR_ALIGN;
  return JF_OK;
}

int64_t qbytes(const jf_cqtensor& t) { return t.rows * t.cols; }
int64_t sbytes(int64_t r, int64_t c) { return (r / 32) * (c / 32) * 4; }

// Shared validation + launch of the three GEMMs. A/B are the stored operands.
// `pre` (activation kActGelu only; q may be NULL) receives the re-quantized pre-activation.
int gemm_call(int mode, const jf_cqtensor& A, const jf_cqtensor& B, const jf_qtensor& Y, float* y_f32,
              int64_t rows, int64_t cols, int64_t depth, void* stream, int act = jf::kActNone,
              jf_qtensor pre = jf_qtensor{nullptr, nullptr, 0, 0}) {
  int st;
  if ((st = check_cq(A)) != JF_OK) return st;
  if ((st = check_cq(B)) != JF_OK) return st;
  if ((st = check_q(Y, false)) != JF_OK) return st;
  if (Y.rows != rows || Y.cols != cols) return JF_ERR_SHAPE;
  if (pre.q != nullptr) {
    if ((st = check_q(pre, true)) != JF_OK) return st;
    if (pre.rows != rows || pre.cols != cols) return JF_ERR_SHAPE;
  }
  if (rows == 0 || cols == 0) return JF_OK;
  if (Y.q == nullptr && y_f32 == nullptr) return JF_ERR_NULL;
  if (y_f32 != nullptr && !aligned(y_f32, 16)) return JF_ERR_ALIGN;
  // outputs must not overlap inputs (nor each other)
  const void* ins[4] = {A.q, A.s, B.q, B.s};
  const int64_t in_n[4] = {qbytes(A), sbytes(A.rows, A.cols), qbytes(B), sbytes(B.rows, B.cols)};
  const void* outs[5] = {Y.q, Y.q ? Y.s : nullptr, y_f32, pre.q, pre.q ? pre.s : nullptr};
  const int64_t out_n[5] = {rows * cols, sbytes(rows, cols), rows * cols * 4, rows * cols, sbytes(rows, cols)};
  for (int o = 0; o < 5; ++o) {
    for (int i = 0; i < 4; ++i)
      if (overlap(outs[o], out_n[o], ins[i], in_n[i])) return JF_ERR_ALIAS;
    for (int o2 = o + 1; o2 < 5; ++o2)
      if (overlap(outs[o], out_n[o], outs[o2], out_n[o2])) return JF_ERR_ALIAS;
  }
  const DevInfo d = device_info();
  if (!d.ok) return JF_ERR_DEVICE;
  jf::GemmArgs g;
  g.mode = mode;
  g.a_q = A.q;
  g.a_s = A.s;
  g.b_q = B.q;
  g.b_s = B.s;
  g.rows = rows;
  g.cols = cols;
  g.depth = depth;
  g.a_ld = A.cols;
  g.b_ld = B.cols;
  g.y_q = Y.q;
  g.y_s = Y.q ? Y.s : nullptr;
  g.y_f32 = y_f32;
  g.act = act;
  g.pre_q = pre.q;
  g.pre_s = pre.q ? pre.s : nullptr;
  g.status = d.status;
  if (depth == 0) {
    // empty contraction: the result is exactly zero (codes 0, scales 0)
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    if (Y.q) {
      e = cudaMemsetAsync(Y.q, 0, size_t(rows * cols), s);
      if (e == cudaSuccess) e = cudaMemsetAsync(Y.s, 0, size_t(sbytes(rows, cols)), s);
    }
    if (e == cudaSuccess && y_f32) e = cudaMemsetAsync(y_f32, 0, size_t(rows * cols * 4), s);
    // GELU(0) = 0: the fused output and the pre-activation are zero as well
    if (e == cudaSuccess && pre.q) {
      e = cudaMemsetAsync(pre.q, 0, size_t(rows * cols), s);
      if (e == cudaSuccess) e = cudaMemsetAsync(pre.s, 0, size_t(sbytes(rows, cols)), s);
    }
    return cuda_status(e);
  }
  return cuda_status(jf::launch_gemm(g, d.sm_count, static_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

// Bytes of the row statistics of a [rows, cols] tensor: int32 [rows][cols/32][2].
inline int64_t statbytes(int64_t rows, int64_t cols) { return rows * (cols / 32) * 2 * 4; }

static int quantize_impl(const void* x, jf_dtype dt, int64_t rows, int64_t cols, int8_t* q, float* s,
                         int32_t* stats, bool want_stats, void* stream) {
  if (dt != JF_F32 && dt != JF_BF16 && dt != JF_F16) return JF_ERR_DTYPE;
  if (!dims_ok(rows, cols)) return JF_ERR_SHAPE;
  if (rows == 0 || cols == 0) return JF_OK;
  if (x == nullptr || q == nullptr || s == nullptr || (want_stats && stats == nullptr)) return JF_ERR_NULL;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(s, 4) || (want_stats && !aligned(stats, 8))) return JF_ERR_ALIGN;
  const int64_t nx = rows * cols * elem_size(dt);
  if (overlap(q, rows * cols, x, nx) || overlap(s, sbytes(rows, cols), x, nx) ||
      overlap(q, rows * cols, s, sbytes(rows, cols)))
    return JF_ERR_ALIAS;
  if (want_stats) {
    const int64_t nst = statbytes(rows, cols);
    if (overlap(stats, nst, x, nx) || overlap(stats, nst, q, rows * cols) || overlap(stats, nst, s, sbytes(rows, cols)))
      return JF_ERR_ALIAS;
  }
  const DevInfo d = device_info();
  if (!d.ok) return JF_ERR_DEVICE;
  return cuda_status(jf::launch_quantize(x, int(dt), rows, cols, q, s, want_stats ? stats : nullptr,
                                          plain_loads_forced() ? nullptr : d.status, d.sm_count,
                                          static_cast<cudaStream_t>(stream)));
}

int jf_quantize_block(const void* x, jf_dtype dt, int64_t rows, int64_t cols, int8_t* q, float* s,
                      void* stream) {
  JF_RANGE(__func__);
  return quantize_impl(x, dt, rows, cols, q, s, nullptr, false, stream);
}

int jf_quantize_block_rowstats(const void* x, jf_dtype dt, int64_t rows, int64_t cols, int8_t* q, float* s,
                               int32_t* stats, void* stream) {
  JF_RANGE(__func__);
  return quantize_impl(x, dt, rows, cols, q, s, stats, true, stream);
}

int jf_dequantize_block(const int8_t* q, const float* s, int64_t rows, int64_t cols, void* y, jf_dtype dt,
                        void* stream) {
  JF_RANGE(__func__);
  if (dt != JF_F32 && dt != JF_BF16 && dt != JF_F16) return JF_ERR_DTYPE;
  if (!dims_ok(rows, cols)) return JF_ERR_SHAPE;
  if (rows == 0 || cols == 0) return JF_OK;
  if (q == nullptr || s == nullptr || y == nullptr) return JF_ERR_NULL;
  if (!aligned(q, 16) || !aligned(s, 4) || !aligned(y, 16)) return JF_ERR_ALIGN;
  const int64_t ny = rows * cols * elem_size(dt);
  if (overlap(y, ny, q, rows * cols) || overlap(y, ny, s, sbytes(rows, cols))) return JF_ERR_ALIAS;
  const DevInfo d = device_info();
  if (!d.ok) return JF_ERR_DEVICE;
  return cuda_status(jf::launch_dequantize(q, s, rows, cols, y, int(dt), d.sm_count, static_cast<cudaStream_t>(stream)));
}

int jf_linear_fwd(jf_cqtensor X, jf_cqtensor W, jf_qtensor Y, float* y_f32, void* stream) {
  JF_RANGE(__func__);
  if (!dims_ok(X.rows, X.cols) || !dims_ok(W.rows, W.cols)) return JF_ERR_SHAPE;
  if (X.cols != W.cols) return JF_ERR_SHAPE;
  return gemm_call(jf::kFwd, X, W, Y, y_f32, X.rows, W.rows, X.cols, stream);
}

int jf_linear_fwd_gelu(jf_cqtensor X, jf_cqtensor W, jf_qtensor Y, jf_qtensor Ypre, void* stream) {
  JF_RANGE(__func__);
  if (!dims_ok(X.rows, X.cols) || !dims_ok(W.rows, W.cols)) return JF_ERR_SHAPE;
  if (X.cols != W.cols) return JF_ERR_SHAPE;
  if (Y.q == nullptr && X.rows != 0 && W.rows != 0) return JF_ERR_NULL;
  return gemm_call(jf::kFwd, X, W, Y, nullptr, X.rows, W.rows, X.cols, stream, jf::kActGelu, Ypre);
}

int jf_linear_dgrad(jf_cqtensor dY, jf_cqtensor W, jf_qtensor dX, float* dx_f32, void* stream) {
  JF_RANGE(__func__);
  if (!dims_ok(dY.rows, dY.cols) || !dims_ok(W.rows, W.cols)) return JF_ERR_SHAPE;
  if (dY.cols != W.rows) return JF_ERR_SHAPE;
  return gemm_call(jf::kDgrad, dY, W, dX, dx_f32, dY.rows, W.cols, dY.cols, stream);
}

int jf_linear_wgrad(jf_cqtensor dY, jf_cqtensor X, jf_qtensor dW, float* dw_f32, void* stream) {
  JF_RANGE(__func__);
  if (!dims_ok(dY.rows, dY.cols) || !dims_ok(X.rows, X.cols)) return JF_ERR_SHAPE;
  if (dY.rows != X.rows) return JF_ERR_SHAPE;
  return gemm_call(jf::kWgrad, dY, X, dW, dw_f32, dY.cols, X.cols, dY.rows, stream);
}

int jf_gelu_i8(jf_cqtensor X, jf_qtensor Y, void* stream) {
  JF_RANGE(__func__);
  int st;
  if ((st = check_cq(X)) != JF_OK) return st;
  if ((st = check_q(Y, true)) != JF_OK) return st;
  if (X.rows != Y.rows || X.cols != Y.cols) return JF_ERR_SHAPE;
  if (X.rows == 0 || X.cols == 0) return JF_OK;
  const int64_t nq = qbytes(X), ns = sbytes(X.rows, X.cols);
  if (overlap(Y.q, nq, X.q, nq) || overlap(Y.q, nq, X.s, ns) || overlap(Y.s, ns, X.q, nq) ||
      overlap(Y.s, ns, X.s, ns) || overlap(Y.q, nq, Y.s, ns))
    return JF_ERR_ALIAS;
  const DevInfo d = device_info();
  if (!d.ok) return JF_ERR_DEVICE;
  return cuda_status(jf::launch_gelu_i8(X.q, X.s, X.rows, X.cols, Y.q, Y.s, d.sm_count, static_cast<cudaStream_t>(stream)));
}

static int layernorm_impl(jf_cqtensor X, const int32_t* stats, bool want_stats, const float* gamma,
                          const float* beta, float eps, jf_qtensor Y, void* stream) {
  int st;
  if ((st = check_cq(X)) != JF_OK) return st;
  if ((st = check_q(Y, true)) != JF_OK) return st;
  if (X.rows != Y.rows || X.cols != Y.cols) return JF_ERR_SHAPE;
  if (X.rows == 0 || X.cols == 0) return JF_OK;
  if (gamma == nullptr || beta == nullptr || (want_stats && stats == nullptr)) return JF_ERR_NULL;
  if (!aligned(gamma, 16) || !aligned(beta, 16) || (want_stats && !aligned(stats, 8))) return JF_ERR_ALIGN;
  const int64_t nq = qbytes(X), ns = sbytes(X.rows, X.cols);
  if (overlap(Y.q, nq, X.q, nq) || overlap(Y.q, nq, X.s, ns) || overlap(Y.s, ns, X.q, nq) ||
      overlap(Y.s, ns, X.s, ns) || overlap(Y.q, nq, Y.s, ns) || overlap(Y.q, nq, gamma, X.cols * 4) ||
      overlap(Y.q, nq, beta, X.cols * 4) || overlap(Y.s, ns, gamma, X.cols * 4) || overlap(Y.s, ns, beta, X.cols * 4))
    return JF_ERR_ALIAS;
  if (want_stats) {
    const int64_t nst = statbytes(X.rows, X.cols);
    if (overlap(Y.q, nq, stats, nst) || overlap(Y.s, ns, stats, nst)) return JF_ERR_ALIAS;
  }
  const DevInfo d = device_info();
  if (!d.ok) return JF_ERR_DEVICE;
  return cuda_status(jf::launch_layernorm_i8(X.q, X.s, X.rows, X.cols, gamma, beta, eps, Y.q, Y.s,
                                             want_stats ? stats : nullptr, static_cast<cudaStream_t>(stream)));
}

int jf_layernorm_i8(jf_cqtensor X, const float* gamma, const float* beta, float eps, jf_qtensor Y,
                    void* stream) {
  JF_RANGE(__func__);
  return layernorm_impl(X, nullptr, false, gamma, beta, eps, Y, stream);
}

int jf_layernorm_i8_rowstats(jf_cqtensor X, const int32_t* stats, const float* gamma, const float* beta, float eps,
                             jf_qtensor Y, void* stream) {
  JF_RANGE(__func__);
  return layernorm_impl(X, stats, true, gamma, beta, eps, Y, stream);
}

int jf_gelu_i8_bwd(jf_cqtensor X, jf_cqtensor dY, jf_qtensor dX, void* stream) {
  JF_RANGE(__func__);
  int st;
  if ((st = check_cq(X)) != JF_OK) return st;
  if ((st = check_cq(dY)) != JF_OK) return st;
  if ((st = check_q(dX, true)) != JF_OK) return st;
  if (X.rows != dY.rows || X.cols != dY.cols || X.rows != dX.rows || X.cols != dX.cols) return JF_ERR_SHAPE;
  if (X.rows == 0 || X.cols == 0) return JF_OK;
  const int64_t nq = qbytes(X), ns = sbytes(X.rows, X.cols);
  const void* ins[4] = {X.q, X.s, dY.q, dY.s};
  const int64_t in_n[4] = {nq, ns, nq, ns};
  for (int i = 0; i < 4; ++i)
    if (overlap(dX.q, nq, ins[i], in_n[i]) || overlap(dX.s, ns, ins[i], in_n[i])) return JF_ERR_ALIAS;
  if (overlap(dX.q, nq, dX.s, ns)) return JF_ERR_ALIAS;
  const DevInfo d = device_info();
  if (!d.ok) return JF_ERR_DEVICE;
  return cuda_status(jf::launch_gelu_i8_bwd(X.q, X.s, dY.q, dY.s, X.rows, X.cols, dX.q, dX.s, d.sm_count,
                                            static_cast<cudaStream_t>(stream)));
}

int64_t jf_layernorm_i8_bwd_workspace_bytes(int64_t rows, int64_t cols) {
  if (!dims_ok(rows, cols) || cols > jf::kLnBwdMaxCols) return -1;
  return jf::ln_bwd_ctas(rows) * 2 * cols * 4;
}

}  // extern "C"

namespace {
// Every check of the LayerNorm backward that does not involve the workspace, in the order both
// entry points apply them: tensors, shapes, NULL gamma, alignment, then overlaps among the
// inputs and outputs (the workspace is checked by the caller of this function).
int ln_bwd_validate(const jf_cqtensor& X, const jf_cqtensor& dY, const float* gamma, const jf_qtensor& dX,
                    const float* dgamma, const float* dbeta) {
  int st;
  if ((st = check_cq(X)) != JF_OK) return st;
  if ((st = check_cq(dY)) != JF_OK) return st;
  if ((st = check_q(dX, true)) != JF_OK) return st;
  if (X.rows != dY.rows || X.cols != dY.cols || X.rows != dX.rows || X.cols != dX.cols) return JF_ERR_SHAPE;
  if (X.cols > jf::kLnBwdMaxCols) return JF_ERR_SHAPE;
  if (X.rows == 0 || X.cols == 0) return JF_OK;
  if (gamma == nullptr) return JF_ERR_NULL;
  if (!aligned(gamma, 16) || !aligned(dgamma, 4) || !aligned(dbeta, 4)) return JF_ERR_ALIGN;
  const int64_t nq = qbytes(X), ns = sbytes(X.rows, X.cols), H = X.cols;
  const void* ins[5] = {X.q, X.s, dY.q, dY.s, gamma};
  const int64_t in_n[5] = {nq, ns, nq, ns, H * 4};
  const void* outs[4] = {dX.q, dX.s, dgamma, dbeta};
  const int64_t out_n[4] = {nq, ns, H * 4, H * 4};
  for (int o = 0; o < 4; ++o) {
    for (int i = 0; i < 5; ++i)
      if (overlap(outs[o], out_n[o], ins[i], in_n[i])) return JF_ERR_ALIAS;
    for (int o2 = o + 1; o2 < 4; ++o2)
      if (overlap(outs[o], out_n[o], outs[o2], out_n[o2])) return JF_ERR_ALIAS;
  }
  return JF_OK;
}

// The launch shared by both entry points, after validation. `part` is the column-sum workspace
// (NULL when neither dgamma nor dbeta is wanted).
int ln_bwd_launch(const jf_cqtensor& X, const jf_cqtensor& dY, const float* gamma, float eps, const jf_qtensor& dX,
                  float* dgamma, float* dbeta, float* part, void* stream) {
  const DevInfo d = device_info();
  if (!d.ok) return JF_ERR_DEVICE;
  return cuda_status(jf::launch_layernorm_i8_bwd(X.q, X.s, dY.q, dY.s, X.rows, X.cols, gamma, eps, dX.q, dX.s, part,
                                                 dgamma, dbeta, static_cast<cudaStream_t>(stream)));
}
}  // namespace

extern "C" {

int jf_layernorm_i8_bwd(jf_cqtensor X, jf_cqtensor dY, const float* gamma, float eps, jf_qtensor dX, float* dgamma,
                        float* dbeta, void* workspace, int64_t workspace_bytes, void* stream) {
  JF_RANGE(__func__);
  int st;
  if ((st = ln_bwd_validate(X, dY, gamma, dX, dgamma, dbeta)) != JF_OK) return st;
  if (X.rows == 0 || X.cols == 0) return JF_OK;
  const bool want_param_grads = dgamma != nullptr || dbeta != nullptr;
  if (!want_param_grads) return ln_bwd_launch(X, dY, gamma, eps, dX, nullptr, nullptr, nullptr, stream);
  const int64_t nw = jf_layernorm_i8_bwd_workspace_bytes(X.rows, X.cols);
  if (workspace == nullptr || !aligned(workspace, 16) || workspace_bytes < nw) return JF_ERR_WORKSPACE;
  const int64_t nq = qbytes(X), ns = sbytes(X.rows, X.cols), H = X.cols;
  const void* others[7] = {X.q, X.s, dY.q, dY.s, gamma, dX.q, dX.s};
  const int64_t other_n[7] = {nq, ns, nq, ns, H * 4, nq, ns};
  for (int i = 0; i < 7; ++i)
    if (overlap(workspace, nw, others[i], other_n[i])) return JF_ERR_ALIAS;
  if (overlap(workspace, nw, dgamma, H * 4) || overlap(workspace, nw, dbeta, H * 4)) return JF_ERR_ALIAS;
  return ln_bwd_launch(X, dY, gamma, eps, dX, dgamma, dbeta, static_cast<float*>(workspace), stream);
}

int jf_layernorm_i8_bwd_noalloc(jf_cqtensor X, jf_cqtensor dY, const float* gamma, float eps, jf_qtensor dX,
                                float* dgamma, float* dbeta, void* stream) {
  JF_RANGE(__func__);
  // the same argument checks, in the same order, as jf_layernorm_i8_bwd; only then the scratch size
  int st;
  if ((st = ln_bwd_validate(X, dY, gamma, dX, dgamma, dbeta)) != JF_OK) return st;
  if (X.rows == 0 || X.cols == 0) return JF_OK;
  if (dgamma == nullptr && dbeta == nullptr) return ln_bwd_launch(X, dY, gamma, eps, dX, nullptr, nullptr, nullptr, stream);
  if (jf_layernorm_i8_bwd_workspace_bytes(X.rows, X.cols) > jf::kLnBwdScratchBytes) return JF_ERR_WORKSPACE;
  const DevInfo d = device_info();
  if (!d.ok) return JF_ERR_DEVICE;
  float* scratch = jf::ln_bwd_static_scratch();
  if (scratch == nullptr) return JF_ERR_CUDA;
  return ln_bwd_launch(X, dY, gamma, eps, dX, dgamma, dbeta, scratch, stream);
}

int64_t jf_granular_scale_count(int64_t rows, int64_t cols, jf_granularity g) {
  if (!dims_ok(rows, cols)) return -1;
  switch (g) {
    case JF_GRAN_BLOCK: return (rows / 32) * (cols / 32);
    case JF_GRAN_TOKEN: return rows;
    case JF_GRAN_CHANNEL: return cols;
    case JF_GRAN_TENSOR: return 1;
    default: return -1;
  }
}

namespace {
bool gran_ok(jf_granularity g) { return g == JF_GRAN_BLOCK || g == JF_GRAN_TOKEN || g == JF_GRAN_CHANNEL || g == JF_GRAN_TENSOR; }
}  // namespace

int jf_quantize_granular(const void* x, jf_dtype dt, int64_t rows, int64_t cols, jf_granularity g, int8_t* q,
                         float* s, void* stream) {
  JF_RANGE(__func__);
  if (dt != JF_F32 && dt != JF_BF16 && dt != JF_F16) return JF_ERR_DTYPE;
  if (!gran_ok(g)) return JF_ERR_ARG;
  if (!dims_ok(rows, cols)) return JF_ERR_SHAPE;
  if (rows == 0 || cols == 0) return JF_OK;
  if (x == nullptr || q == nullptr || s == nullptr) return JF_ERR_NULL;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(s, 4)) return JF_ERR_ALIGN;
  const int64_t nx = rows * cols * elem_size(dt), ns = jf_granular_scale_count(rows, cols, g) * 4;
  if (overlap(q, rows * cols, x, nx) || overlap(s, ns, x, nx) || overlap(q, rows * cols, s, ns)) return JF_ERR_ALIAS;
  const DevInfo d = device_info();
  if (!d.ok) return JF_ERR_DEVICE;
  return cuda_status(jf::launch_quantize_granular(x, int(dt), rows, cols, int(g), q, s,
                                                   plain_loads_forced() ? nullptr : d.status, d.sm_count,
                                                  static_cast<cudaStream_t>(stream)));
}

int jf_dequantize_granular(const int8_t* q, const float* s, int64_t rows, int64_t cols, jf_granularity g, void* y,
                           jf_dtype dt, void* stream) {
  JF_RANGE(__func__);
  if (dt != JF_F32 && dt != JF_BF16 && dt != JF_F16) return JF_ERR_DTYPE;
  if (!gran_ok(g)) return JF_ERR_ARG;
  if (!dims_ok(rows, cols)) return JF_ERR_SHAPE;
  if (rows == 0 || cols == 0) return JF_OK;
  if (q == nullptr || s == nullptr || y == nullptr) return JF_ERR_NULL;
  if (!aligned(q, 16) || !aligned(s, 4) || !aligned(y, 16)) return JF_ERR_ALIGN;
  const int64_t ny = rows * cols * elem_size(dt), ns = jf_granular_scale_count(rows, cols, g) * 4;
  if (overlap(y, ny, q, rows * cols) || overlap(y, ny, s, ns)) return JF_ERR_ALIAS;
  const DevInfo d = device_info();
  if (!d.ok) return JF_ERR_DEVICE;
  return cuda_status(jf::launch_dequantize_granular(q, s, rows, cols, int(g), y, int(dt), d.sm_count,
                                                    static_cast<cudaStream_t>(stream)));
}

int jf_quantization_error(const void* x, jf_dtype dt, const int8_t* q, const float* s, int64_t rows, int64_t cols,
                          jf_granularity g, double* sums, void* stream) {
  JF_RANGE(__func__);
  if (dt != JF_F32 && dt != JF_BF16 && dt != JF_F16) return JF_ERR_DTYPE;
  if (!gran_ok(g)) return JF_ERR_ARG;
  if (!dims_ok(rows, cols)) return JF_ERR_SHAPE;
  if (sums == nullptr) return JF_ERR_NULL;
  if (!aligned(sums, 8)) return JF_ERR_ALIGN;
  const int64_t nx = rows * cols * elem_size(dt), ns = jf_granular_scale_count(rows, cols, g) * 4;
  if (rows != 0 && cols != 0) {
    if (x == nullptr || q == nullptr || s == nullptr) return JF_ERR_NULL;
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(s, 4)) return JF_ERR_ALIGN;
    if (overlap(sums, 24, x, nx) || overlap(sums, 24, q, rows * cols) || overlap(sums, 24, s, ns)) return JF_ERR_ALIAS;
  }
  const DevInfo d = device_info();
  if (!d.ok) return JF_ERR_DEVICE;
  if (rows == 0 || cols == 0)
    return cuda_status(cudaMemsetAsync(sums, 0, 3 * sizeof(double), static_cast<cudaStream_t>(stream)));
  return cuda_status(jf::launch_quant_error(x, int(dt), q, s, rows, cols, int(g), sums, d.sm_count,
                                            static_cast<cudaStream_t>(stream)));
}

int jf_mx_quantize(const void* x, jf_dtype dt, int64_t rows, int64_t cols, uint8_t* codes, uint8_t* scales,
                   void* stream) {
  JF_RANGE(__func__);
  if (dt != JF_F32 && dt != JF_BF16 && dt != JF_F16) return JF_ERR_DTYPE;
  if (!dims_ok(rows, cols)) return JF_ERR_SHAPE;
  if (rows == 0 || cols == 0) return JF_OK;
  if (x == nullptr || codes == nullptr || scales == nullptr) return JF_ERR_NULL;
  if (!aligned(x, 16) || !aligned(codes, 16)) return JF_ERR_ALIGN;
  const int64_t nx = rows * cols * elem_size(dt), nc = rows * cols, ns = rows * (cols / 32);
  if (overlap(codes, nc, x, nx) || overlap(scales, ns, x, nx) || overlap(codes, nc, scales, ns)) return JF_ERR_ALIAS;
  const DevInfo d = device_info();
  if (!d.ok) return JF_ERR_DEVICE;
  return cuda_status(jf::launch_mx_quantize(x, int(dt), rows, cols, codes, scales, d.sm_count,
                                            static_cast<cudaStream_t>(stream)));
}

int jf_mx_linear_fwd(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* b_codes, const uint8_t* b_scales,
                     int64_t M, int64_t N, int64_t K, float* y, void* stream) {
  JF_RANGE(__func__);
  if (!dims_ok(M, K) || !dims_ok(N, K) || K % 128 != 0) return JF_ERR_SHAPE;
  if (M == 0 || N == 0) return JF_OK;
  if (K == 0) return JF_ERR_SHAPE;
  if (a_codes == nullptr || a_scales == nullptr || b_codes == nullptr || b_scales == nullptr || y == nullptr)
    return JF_ERR_NULL;
  if (!aligned(a_codes, 16) || !aligned(b_codes, 16) || !aligned(a_scales, 4) || !aligned(b_scales, 4) ||
      !aligned(y, 16))
    return JF_ERR_ALIGN;
  const void* ins[4] = {a_codes, a_scales, b_codes, b_scales};
  const int64_t in_n[4] = {M * K, M * (K / 32), N * K, N * (K / 32)};
  for (int i = 0; i < 4; ++i)
    if (overlap(y, M * N * 4, ins[i], in_n[i])) return JF_ERR_ALIAS;
  const DevInfo d = device_info();
  if (!d.ok) return JF_ERR_DEVICE;
  return cuda_status(jf::launch_mx_gemm(a_codes, a_scales, b_codes, b_scales, M, N, K, y, d.status, d.sm_count,
                                        static_cast<cudaStream_t>(stream)));
}

int jf_gemm_i8_s32(const int8_t* A, const int8_t* B, int32_t* C, int64_t M, int64_t N, int64_t K, void* stream) {
  JF_RANGE(__func__);
  if (M < 0 || N < 0 || K < 0 || M % 128 != 0 || N % 256 != 0 || K % 128 != 0 || K > 65536 ||
      M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31))
    return JF_ERR_SHAPE;
  if (M == 0 || N == 0) return JF_OK;
  if (C == nullptr) return JF_ERR_NULL;
  if (!aligned(C, 16)) return JF_ERR_ALIGN;
  if (K == 0) return cuda_status(cudaMemsetAsync(C, 0, size_t(M * N * 4), static_cast<cudaStream_t>(stream)));
  if (A == nullptr || B == nullptr) return JF_ERR_NULL;
  if (!aligned(A, 16) || !aligned(B, 16)) return JF_ERR_ALIGN;
  if (overlap(C, M * N * 4, A, M * K) || overlap(C, M * N * 4, B, N * K)) return JF_ERR_ALIAS;
  const DevInfo d = device_info();
  if (!d.ok) return JF_ERR_DEVICE;
  return cuda_status(jf::launch_gemm_s32(A, B, C, M, N, K, d.status, d.sm_count, static_cast<cudaStream_t>(stream)));
}

int jf_selftest_wait_timeout(int64_t limit_ns, void* stream) {
  JF_RANGE(__func__);
  if (limit_ns < 1000000 || limit_ns > 10000000000ll) return JF_ERR_ARG;
  const DevInfo d = device_info();
  if (!d.ok) return JF_ERR_DEVICE;
  return cuda_status(jf::launch_wait_selftest(d.status, static_cast<unsigned long long>(limit_ns),
                                              static_cast<cudaStream_t>(stream)));
}

const char* jf_strerror(int status) {
  switch (status) {
    case JF_OK: return "ok";
    case JF_ERR_NULL: return "a required pointer is NULL";
    case JF_ERR_SHAPE: return "bad shape: dimensions must be non-negative multiples of 32 and agree";
    case JF_ERR_ALIGN: return "misaligned pointer (codes and fp32/bf16/fp16 data: 16 bytes; scales: 4 bytes)";
    case JF_ERR_DTYPE: return "unknown dtype";
    case JF_ERR_ALIAS: return "an output overlaps an input or another output";
    case JF_ERR_CUDA: return "a CUDA runtime/driver call failed";
    case JF_ERR_TIMEOUT: return "a kernel's bounded wait timed out; outputs are undefined";
    case JF_ERR_DEVICE: return "no usable sm_100 (B200) device is current";
    case JF_ERR_WORKSPACE: return "workspace is NULL, not 16-byte aligned or smaller than the size asked for";
    case JF_ERR_ARG: return "unknown granularity (or other enumerated argument)";
    default: return "unknown status";
  }
}

int jf_device_status(void* stream) {
  JF_RANGE(__func__);
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return JF_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, jf::g_status, sizeof(v)) != cudaSuccess) return JF_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(jf::g_status, &zero, sizeof(zero)) != cudaSuccess) return JF_ERR_CUDA;
  if (v & jf::kStatusTimeout) return JF_ERR_TIMEOUT;
  return v ? JF_ERR_CUDA : JF_OK;
}

int jf_sm_count(void) {
  const DevInfo d = device_info();
  return d.sm_count;
}

}  // extern "C"
