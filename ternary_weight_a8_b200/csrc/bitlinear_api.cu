// C ABI of the BitLinear W1.58A8 forward: argument checks, workspace layout,
// dispatch to the kernels, and the layer chain.  The declarations and their
// contracts are in include/bitlinear.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <mutex>
#include <string>

#include "bitlinear.h"
#include "common.cuh"
#include "kernels.h"

namespace {

thread_local std::string g_last_error;
thread_local int g_path = 0;  // 0 auto, 1 GEMV, 2 GEMM

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(BL_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

constexpr size_t kStatusBytes = 256;

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Device-accessible pointer with the given alignment?  Returns BL_OK or an error code.
int check_ptr(const void* p, const char* name, size_t align, bool nullable = false) {
  if (p == nullptr) {
    if (nullable) return BL_OK;
    return fail(BL_ERR_INVALID_ARG, "%s is NULL", name);
  }
  if (reinterpret_cast<uintptr_t>(p) % align != 0) {
    return fail(BL_ERR_MISALIGNED, "%s (%p) is not %zu-byte aligned", name, p, align);
  }
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(BL_ERR_INVALID_ARG, "%s (%p): cudaPointerGetAttributes failed: %s", name, p,
                cudaGetErrorString(e));
  }
  if (attr.type == cudaMemoryTypeUnregistered ||
      (attr.type == cudaMemoryTypeHost && attr.devicePointer == nullptr)) {
    return fail(BL_ERR_INVALID_ARG, "%s (%p) is not device-accessible memory", name, p);
  }
  return BL_OK;
}

int check_dtype(int t, const char* name) {
  if (t != BL_F32 && t != BL_BF16) return fail(BL_ERR_INVALID_ARG, "%s: unknown dtype %d", name, t);
  return BL_OK;
}

int check_nk(int N, int K) {
  if (N < 1) return fail(BL_ERR_UNSUPPORTED_SHAPE, "N = %d: need N >= 1", N);
  if (N > (1 << 24)) return fail(BL_ERR_UNSUPPORTED_SHAPE, "N = %d: need N <= 2^24", N);
  if (K < 64 || K % 64 != 0) return fail(BL_ERR_UNSUPPORTED_SHAPE, "K = %d: need K >= 64 and K %% 64 == 0", K);
  return BL_OK;
}

// Workspace layout: [0, 256) status block (status word, decode ticket
// counters), then the quantised activations of the call: q [M][ldq] with
// ldq = K rounded up to 128 (zero padding), s [M], rowsum [M]; every region
// 256-byte aligned.
int code_pitch(int K) { return (K + 127) / 128 * 128; }

struct FwdLayout {
  size_t xq, scale, rowsum, total;
};

FwdLayout forward_layout(int M, int K) {
  FwdLayout l;
  l.xq = kStatusBytes;
  l.scale = l.xq + round_up(static_cast<size_t>(M) * code_pitch(K), 256);
  l.rowsum = l.scale + round_up(static_cast<size_t>(M) * 4, 256);
  l.total = l.rowsum + round_up(static_cast<size_t>(M) * 4, 256);
  return l;
}

#define BL_TRY(expr)            \
  do {                          \
    int _rc = (expr);           \
    if (_rc != BL_OK) return _rc; \
  } while (0)

// Bytes [16, 24) of the status block: the decode kernel's ticket counters.
uint32_t* tickets_of(void* ws) { return reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + 16); }

// The product kernel for M tokens: the decode GEMV for M <= 16 (when its
// activations fit on chip), else the tensor-core GEMM; bitlinear_set_path
// overrides the choice on the calling thread.
int choose_gemv(int M, int K, bool* gemv) {
  bool v = M <= 16;
  if (g_path == 1) {
    if (M > 16) return fail(BL_ERR_UNSUPPORTED_SHAPE, "GEMV path forced with M = %d > 16", M);
    v = true;
  } else if (g_path == 2) {
    v = false;
  }
  (void)K;
  *gemv = v;
  return BL_OK;
}

int gemv_fail(cudaError_t e) { return cuda_fail(e, "GEMV launch"); }

int launch_gemm_q(const uint8_t* packed, const float* gamma, int N, int K, int M, const int8_t* xq, int ldx,
                  const float* scale, const int32_t* rowsum, void* y, int y_dtype, int32_t* acc_out,
                  uint32_t* status, cudaStream_t s) {
  bl::ProductArgs a{packed, gamma, N, K, M, xq, ldx, scale, rowsum, y,
                    y_dtype == BL_BF16 ? bl::kOutBF16 : bl::kOutF32, acc_out, status};
  cudaError_t e = bl::launch_gemm(a, s, true);
  if (e != cudaSuccess) return cuda_fail(e, "GEMM launch");
  return BL_OK;
}

}  // namespace

namespace bl {
int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

__global__ void wait_timeout_selftest_kernel(uint32_t* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const WaitCtl ctl{status, &abort_flag, limit_ns};
  if (threadIdx.x == 0) {
    // Nothing ever arrives on this barrier: the wait must give up by itself.
    mbar_wait(smem_u32(&bar), 0, ctl);
  }
  __syncthreads();
}

cudaError_t launch_wait_timeout_selftest(uint32_t* status, int limit_us, cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(status, static_cast<unsigned long long>(limit_us) * 1000ull);
  return cudaGetLastError();
}
}  // namespace bl

extern "C" {

const char* bitlinear_last_error(void) { return g_last_error.c_str(); }

int bitlinear_version(void) { return 100; }

int bitlinear_set_path(int path) {
  if (path < 0 || path > 2) return fail(BL_ERR_INVALID_ARG, "path %d not in {0, 1, 2}", path);
  g_path = path;
  return BL_OK;
}

size_t bitlinear_pack_workspace_bytes(int N, int K) {
  (void)K;
  if (N < 0) return 0;
  return kStatusBytes + round_up(static_cast<size_t>(N) * sizeof(double), 256);
}

int bitlinear_pack_weights(const float* W, int N, int K, uint8_t* packed, float* gamma,
                           void* workspace, size_t workspace_bytes, void* stream) {
  BL_TRY(check_nk(N, K));
  BL_TRY(check_ptr(W, "W", 16));
  BL_TRY(check_ptr(packed, "packed", 16));
  BL_TRY(check_ptr(gamma, "gamma", 4));
  BL_TRY(check_ptr(workspace, "workspace", 256));
  const size_t need = bitlinear_pack_workspace_bytes(N, K);
  if (workspace_bytes < need)
    return fail(BL_ERR_WORKSPACE_TOO_SMALL, "pack workspace %zu < %zu bytes", workspace_bytes, need);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  double* row_sums = reinterpret_cast<double*>(static_cast<uint8_t*>(workspace) + kStatusBytes);
  cudaError_t e = bl::launch_gamma(W, N, K, row_sums, gamma, s);
  if (e != cudaSuccess) return cuda_fail(e, "gamma launch");
  e = bl::launch_ternary_pack(W, N, K, gamma, packed, s);
  if (e != cudaSuccess) return cuda_fail(e, "pack launch");
  // The forward kernels start loading packed weights before waiting for the
  // kernel before them (programmatic dependent launch), which makes only that
  // kernel's writes visible after the wait.  A stream operation that is not a
  // kernel ends the pack (rewriting the status word's zero), so the next
  // kernel on the stream starts only once the packed weights are complete.
  e = cudaMemsetAsync(workspace, 0, sizeof(uint32_t), s);
  if (e != cudaSuccess) return cuda_fail(e, "pack completion");
  return BL_OK;
}

int bitlinear_quant_act(const void* x, int x_dtype, int M, int K, int8_t* xq, float* scale,
                        int32_t* rowsum, void* stream) {
  BL_TRY(check_dtype(x_dtype, "x_dtype"));
  if (M < 0) return fail(BL_ERR_INVALID_ARG, "M = %d < 0", M);
  if (K < 64 || K % 64 != 0) return fail(BL_ERR_UNSUPPORTED_SHAPE, "K = %d: need K >= 64 and K %% 64 == 0", K);
  if (M == 0) return BL_OK;
  BL_TRY(check_ptr(x, "x", 16));
  BL_TRY(check_ptr(xq, "xq", 16));
  BL_TRY(check_ptr(scale, "scale", 4));
  BL_TRY(check_ptr(rowsum, "rowsum", 4, true));
  cudaError_t e = bl::launch_act_quant(x, x_dtype == BL_BF16, M, K, K, xq, scale, rowsum,
                                       static_cast<cudaStream_t>(stream), true);
  if (e != cudaSuccess) return cuda_fail(e, "act_quant launch");
  return BL_OK;
}

size_t bitlinear_ste_workspace_bytes(int M, int N, int K) {
  if (M < 0 || N < 0 || K < 0) return 0;
  return kStatusBytes + bl::ste_scratch_bytes(M, N, K);
}

int bitlinear_ste_backward(const uint8_t* packed, const float* gamma, int N, int K, const void* dy,
                           const int8_t* xq, const float* scale, int M, void* dx, int dx_dtype, float* dw,
                           void* workspace, size_t workspace_bytes, void* stream) {
  BL_TRY(check_nk(N, K));
  if (N % 64 != 0) return fail(BL_ERR_UNSUPPORTED_SHAPE, "N = %d: the backward needs N %% 64 == 0", N);
  if (M < 0) return fail(BL_ERR_INVALID_ARG, "M = %d < 0", M);
  if (M % 8 != 0) return fail(BL_ERR_UNSUPPORTED_SHAPE, "M = %d: the backward needs M %% 8 == 0", M);
  BL_TRY(check_dtype(dx_dtype, "dx_dtype"));
  if (M == 0 || (!dx && !dw)) return BL_OK;
  BL_TRY(check_ptr(packed, "packed", 16));
  BL_TRY(check_ptr(gamma, "gamma", 4));
  BL_TRY(check_ptr(dy, "dy", 16));
  BL_TRY(check_ptr(xq, "xq", 16));
  BL_TRY(check_ptr(scale, "scale", 4));
  BL_TRY(check_ptr(dx, "dx", 16, true));
  BL_TRY(check_ptr(dw, "dw", 16, true));
  BL_TRY(check_ptr(workspace, "workspace", 256));
  const size_t need = bitlinear_ste_workspace_bytes(M, N, K);
  if (workspace_bytes < need)
    return fail(BL_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", workspace_bytes, need);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaError_t e = bl::launch_ste_backward(packed, gamma, N, K, dy, xq, scale, M, dx, dx_dtype == BL_BF16, dw,
                                          ws + kStatusBytes, reinterpret_cast<uint32_t*>(ws),
                                          static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "straight-through backward launch");
  return BL_OK;
}

int bitlinear_forward_lut(const uint8_t* packed, const float* gamma, int N, int K, const int8_t* xq,
                          const float* scale, const int32_t* rowsum, int M, void* y, int y_dtype, int32_t* acc_out,
                          void* stream) {
  BL_TRY(check_nk(N, K));
  BL_TRY(check_dtype(y_dtype, "y_dtype"));
  if (M != 1) return fail(BL_ERR_UNSUPPORTED_SHAPE, "M = %d: the lookup-table product takes one token", M);
  if (K > bl::kLutMaxK)
    return fail(BL_ERR_UNSUPPORTED_SHAPE, "K = %d: the lookup tables need K <= %d", K, bl::kLutMaxK);
  BL_TRY(check_ptr(packed, "packed", 16));
  BL_TRY(check_ptr(gamma, "gamma", 4));
  BL_TRY(check_ptr(xq, "xq", 16));
  BL_TRY(check_ptr(scale, "scale", 4));
  BL_TRY(check_ptr(rowsum, "rowsum", 4));
  BL_TRY(check_ptr(y, "y", 4));
  BL_TRY(check_ptr(acc_out, "acc_out", 4, true));
  cudaError_t e = bl::launch_lut_gemv(packed, gamma, N, K, xq, scale, rowsum, y,
                                      y_dtype == BL_BF16 ? bl::kOutBF16 : bl::kOutF32, acc_out,
                                      static_cast<cudaStream_t>(stream), true);
  if (e != cudaSuccess) return cuda_fail(e, "lookup-table product launch");
  return BL_OK;
}

int bitlinear_glu_quant(const void* gate, const void* up, int x_dtype, int M, int N, int act, void* h,
                        int8_t* xq, float* scale, int32_t* rowsum, void* stream) {
  BL_TRY(check_dtype(x_dtype, "x_dtype"));
  if (M < 0) return fail(BL_ERR_INVALID_ARG, "M = %d < 0", M);
  if (N < 64 || N % 64 != 0) return fail(BL_ERR_UNSUPPORTED_SHAPE, "N = %d: need N >= 64 and N %% 64 == 0", N);
  if (act != BL_GLU_RELU2 && act != BL_GLU_SILU) return fail(BL_ERR_INVALID_ARG, "act = %d: unknown", act);
  if (M == 0) return BL_OK;
  BL_TRY(check_ptr(gate, "gate", 16));
  BL_TRY(check_ptr(up, "up", 16));
  BL_TRY(check_ptr(h, "h", 16, true));
  BL_TRY(check_ptr(xq, "xq", 16));
  BL_TRY(check_ptr(scale, "scale", 4));
  BL_TRY(check_ptr(rowsum, "rowsum", 4, true));
  cudaError_t e = bl::launch_glu_quant(gate, up, x_dtype == BL_BF16, M, N, act == BL_GLU_RELU2 ? bl::kGluRelu2
                                                                                             : bl::kGluSilu,
                                       h, xq, scale, rowsum, static_cast<cudaStream_t>(stream), true);
  if (e != cudaSuccess) return cuda_fail(e, "glu_quant launch");
  return BL_OK;
}

int bitlinear_rmsnorm_quant(const void* x, int x_dtype, int M, int K, const float* gain, float eps, void* x_norm,
                            int8_t* xq, float* scale, int32_t* rowsum, void* stream) {
  BL_TRY(check_dtype(x_dtype, "x_dtype"));
  if (M < 0) return fail(BL_ERR_INVALID_ARG, "M = %d < 0", M);
  if (K < 64 || K % 64 != 0) return fail(BL_ERR_UNSUPPORTED_SHAPE, "K = %d: need K >= 64 and K %% 64 == 0", K);
  if (!(eps >= 0.0f) || !(eps < INFINITY)) return fail(BL_ERR_INVALID_ARG, "eps = %g: need a finite eps >= 0", eps);
  if (M == 0) return BL_OK;
  BL_TRY(check_ptr(x, "x", 16));
  BL_TRY(check_ptr(gain, "gain", 16, true));
  BL_TRY(check_ptr(x_norm, "x_norm", 16, true));
  BL_TRY(check_ptr(xq, "xq", 16));
  BL_TRY(check_ptr(scale, "scale", 4));
  BL_TRY(check_ptr(rowsum, "rowsum", 4, true));
  cudaError_t e = bl::launch_rmsnorm_quant(x, x_dtype == BL_BF16, M, K, gain, eps, x_norm, xq, scale, rowsum,
                                           static_cast<cudaStream_t>(stream), true);
  if (e != cudaSuccess) return cuda_fail(e, "rmsnorm_quant launch");
  return BL_OK;
}

size_t bitlinear_workspace_bytes(int M, int N, int K) {
  (void)N;
  if (M < 0 || K < 0) return 0;
  return forward_layout(M, K).total;
}

int bitlinear_set_decode_split(int ctas) {
  if (ctas < 0 || ctas > 8) return fail(BL_ERR_INVALID_ARG, "ctas = %d not in [0, 8]", ctas);
  bl::gemv_force_ksplit(ctas);
  return BL_OK;
}

int bitlinear_set_decode_form(int form) {
  if (form < 0 || form > 2) return fail(BL_ERR_INVALID_ARG, "form = %d not in [0, 2]", form);
  bl::gemv_force_form(form);
  return BL_OK;
}

int bitlinear_forward_quantized(const uint8_t* packed, const float* gamma, int N, int K,
                                const int8_t* xq, const float* scale, const int32_t* rowsum,
                                int M, void* y, int y_dtype, int32_t* acc_out, void* workspace,
                                size_t workspace_bytes, void* stream) {
  BL_TRY(check_nk(N, K));
  BL_TRY(check_dtype(y_dtype, "y_dtype"));
  if (M < 0) return fail(BL_ERR_INVALID_ARG, "M = %d < 0", M);
  if (M == 0) return BL_OK;
  BL_TRY(check_ptr(packed, "packed", 16));
  BL_TRY(check_ptr(gamma, "gamma", 4));
  BL_TRY(check_ptr(xq, "xq", 16));
  BL_TRY(check_ptr(scale, "scale", 4));
  BL_TRY(check_ptr(rowsum, "rowsum", 4));
  BL_TRY(check_ptr(y, "y", 16));
  BL_TRY(check_ptr(acc_out, "acc_out", 16, true));
  BL_TRY(check_ptr(workspace, "workspace", 256));
  if (workspace_bytes < kStatusBytes)
    return fail(BL_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", workspace_bytes, kStatusBytes);
  bool gemv = false;
  BL_TRY(choose_gemv(M, K, &gemv));
  if (gemv && K % 128 != 0) {
    // The decode kernel reads codes in 128-byte blocks; a [M][K] buffer with K % 128 != 0 has none.
    if (g_path == 1) return fail(BL_ERR_UNSUPPORTED_SHAPE, "GEMV on caller codes needs K %% 128 == 0 (K = %d)", K);
    gemv = false;
  }
  uint32_t* status = static_cast<uint32_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (gemv) {
    const bl::GemvLayerArgs L{packed, gamma, N, K, xq, scale, rowsum, K, y, acc_out};
    cudaError_t e = bl::launch_gemv_group(&L, 1, M, bl::kInInt8, y_dtype == BL_BF16 ? bl::kOutBF16 : bl::kOutF32,
                                          status, tickets_of(workspace), s, true);
    return e == cudaSuccess ? BL_OK : gemv_fail(e);
  }
  return launch_gemm_q(packed, gamma, N, K, M, xq, K, scale, rowsum, y, y_dtype, acc_out, status, s);
}

// The forward on a caller-supplied scratch laid out as forward_layout(M, K)
// (the status block included).
static int forward_on(const uint8_t* packed, const float* gamma, int N, int K, const void* x, int x_dtype, int M,
                      void* y, int y_dtype, int32_t* acc_out, uint8_t* ws, cudaStream_t s) {
  const FwdLayout l = forward_layout(M, K);
  bool gemv = false;
  BL_TRY(choose_gemv(M, K, &gemv));
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  const int yt = y_dtype == BL_BF16 ? bl::kOutBF16 : bl::kOutF32;
  if (gemv && bl::gemv_fuses_quant(M, K, x_dtype == BL_BF16, true)) {
    // Small activations: the decode kernel quantises them itself (one launch).
    const bl::GemvLayerArgs L{packed, gamma, N, K, x, nullptr, nullptr, 0, y, acc_out};
    cudaError_t e = bl::launch_gemv_group(&L, 1, M, x_dtype == BL_BF16 ? bl::kInBF16 : bl::kInF32, yt, status,
                                          tickets_of(ws), s, true);
    return e == cudaSuccess ? BL_OK : gemv_fail(e);
  }
  int8_t* xq = reinterpret_cast<int8_t*>(ws + l.xq);
  float* scale = reinterpret_cast<float*>(ws + l.scale);
  int32_t* rowsum = reinterpret_cast<int32_t*>(ws + l.rowsum);
  const int ldq = code_pitch(K);
  cudaError_t e = bl::launch_act_quant(x, x_dtype == BL_BF16, M, K, ldq, xq, scale, rowsum, s, true);
  if (e != cudaSuccess) return cuda_fail(e, "act_quant launch");
  if (gemv) {
    const bl::GemvLayerArgs L{packed, gamma, N, K, xq, scale, rowsum, ldq, y, acc_out};
    e = bl::launch_gemv_group(&L, 1, M, bl::kInInt8, yt, status, tickets_of(ws), s, true);
    return e == cudaSuccess ? BL_OK : gemv_fail(e);
  }
  return launch_gemm_q(packed, gamma, N, K, M, xq, ldq, scale, rowsum, y, y_dtype, acc_out, status, s);
}

int bitlinear_forward(const uint8_t* packed, const float* gamma, int N, int K, const void* x,
                      int x_dtype, int M, void* y, int y_dtype, int32_t* acc_out, void* workspace,
                      size_t workspace_bytes, void* stream) {
  BL_TRY(check_nk(N, K));
  BL_TRY(check_dtype(x_dtype, "x_dtype"));
  BL_TRY(check_dtype(y_dtype, "y_dtype"));
  if (M < 0) return fail(BL_ERR_INVALID_ARG, "M = %d < 0", M);
  if (M == 0) return BL_OK;
  BL_TRY(check_ptr(packed, "packed", 16));
  BL_TRY(check_ptr(gamma, "gamma", 4));
  BL_TRY(check_ptr(x, "x", 16));
  BL_TRY(check_ptr(y, "y", 16));
  BL_TRY(check_ptr(acc_out, "acc_out", 16, true));
  BL_TRY(check_ptr(workspace, "workspace", 256));
  const FwdLayout l = forward_layout(M, K);
  if (workspace_bytes < l.total)
    return fail(BL_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", workspace_bytes, l.total);
  return forward_on(packed, gamma, N, K, x, x_dtype, M, y, y_dtype, acc_out, static_cast<uint8_t*>(workspace),
                    static_cast<cudaStream_t>(stream));
}

// Every layer of a chain has its own region of codes (the layers of one
// decode group are live together): status block, then per layer q, s, rowsum.
static size_t chain_region_bytes(int M, int K) { return forward_layout(M, K).total - kStatusBytes; }

size_t bitlinear_chain_workspace_bytes(const bl_layer* layers, int n_layers, int M) {
  if (!layers || n_layers <= 0 || M < 0) return 0;
  size_t total = kStatusBytes;
  for (int i = 0; i < n_layers; ++i) total += chain_region_bytes(M, layers[i].K);
  return total;
}

static bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

int bitlinear_layer_chain(const bl_layer* layers, int n_layers, int M, int x_dtype, int y_dtype,
                          void* workspace, size_t workspace_bytes, void* stream) {
  if (!layers) return fail(BL_ERR_INVALID_ARG, "layers is NULL");
  if (n_layers < 0) return fail(BL_ERR_INVALID_ARG, "n_layers = %d < 0", n_layers);
  BL_TRY(check_dtype(x_dtype, "x_dtype"));
  BL_TRY(check_dtype(y_dtype, "y_dtype"));
  if (M < 0) return fail(BL_ERR_INVALID_ARG, "M = %d < 0", M);
  if (M == 0 || n_layers == 0) return BL_OK;
  if (n_layers > 64) return fail(BL_ERR_INVALID_ARG, "n_layers = %d > 64", n_layers);
  BL_TRY(check_ptr(workspace, "workspace", 256));
  for (int i = 0; i < n_layers; ++i) {
    const bl_layer& L = layers[i];
    BL_TRY(check_nk(L.N, L.K));
    BL_TRY(check_ptr(L.packed, "layer.packed", 16));
    BL_TRY(check_ptr(L.gamma, "layer.gamma", 4));
    if (L.xq) {
      BL_TRY(check_ptr(L.xq, "layer.xq", 16));
      BL_TRY(check_ptr(L.scale, "layer.scale", 4));
      BL_TRY(check_ptr(L.rowsum, "layer.rowsum", 4));
    } else {
      BL_TRY(check_ptr(L.x, "layer.x", 16));
    }
    BL_TRY(check_ptr(L.y, "layer.y", 16));
    BL_TRY(check_ptr(L.acc_out, "layer.acc_out", 16, true));
  }
  const size_t need = bitlinear_chain_workspace_bytes(layers, n_layers, M);
  if (workspace_bytes < need)
    return fail(BL_ERR_WORKSPACE_TOO_SMALL, "chain workspace %zu < %zu bytes", workspace_bytes, need);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool x_bf16 = x_dtype == BL_BF16;
  const size_t xsz = x_bf16 ? 2 : 4, ysz = y_dtype == BL_BF16 ? 2 : 4;
  const int yt = y_dtype == BL_BF16 ? bl::kOutBF16 : bl::kOutF32;

  // Region of each layer.
  size_t off[64];
  {
    size_t o = kStatusBytes;
    for (int i = 0; i < n_layers; ++i) {
      off[i] = o;
      o += chain_region_bytes(M, layers[i].K);
    }
  }
  auto region = [&](int i, int8_t** xq, float** sc, int32_t** rs) {
    const FwdLayout l = forward_layout(M, layers[i].K);
    *xq = reinterpret_cast<int8_t*>(ws + off[i] + (l.xq - kStatusBytes));
    *sc = reinterpret_cast<float*>(ws + off[i] + (l.scale - kStatusBytes));
    *rs = reinterpret_cast<int32_t*>(ws + off[i] + (l.rowsum - kStatusBytes));
  };
  // The codes of layer i: the caller's, or those quantised into a region.
  // quant_src[i]: the layer whose region holds layer i's quantised input (-1: the caller's codes).
  int quant_src[64];
  for (int i = 0; i < n_layers; ++i) quant_src[i] = -2;
  auto codes_of = [&](int i, const int8_t** xq, const float** sc, const int32_t** rs, int* ld) {
    if (layers[i].xq) {
      *xq = layers[i].xq;
      *sc = layers[i].scale;
      *rs = layers[i].rowsum;
      *ld = layers[i].K;
      return;
    }
    int8_t* q;
    float* c;
    int32_t* r;
    region(quant_src[i], &q, &c, &r);
    *xq = q;
    *sc = c;
    *rs = r;
    *ld = code_pitch(layers[i].K);
  };
  // Same input already quantised earlier in this call?
  auto shared_src = [&](int i) -> int {
    for (int j = 0; j < i; ++j)
      if (quant_src[j] == j && !layers[j].xq && layers[j].x == layers[i].x && layers[j].K == layers[i].K) return j;
    return i;
  };

  int i = 0;
  while (i < n_layers) {
    bool gemv = false;
    BL_TRY(choose_gemv(M, layers[i].K, &gemv));
    // Caller codes reach the decode kernel only in 128-byte blocks.
    if (gemv && layers[i].xq && layers[i].K % 128 != 0) gemv = false;
    if (!gemv) {
      if (!layers[i].xq) {
        quant_src[i] = shared_src(i);
        if (quant_src[i] == i) {
          int8_t* xq;
          float* sc;
          int32_t* rsum;
          region(i, &xq, &sc, &rsum);
          cudaError_t e = bl::launch_act_quant(layers[i].x, x_bf16, M, layers[i].K, code_pitch(layers[i].K), xq, sc,
                                               rsum, s, true);
          if (e != cudaSuccess) return cuda_fail(e, "act_quant launch");
        }
      }
      const int8_t* xq;
      const float* sc;
      const int32_t* rsum;
      int ld;
      codes_of(i, &xq, &sc, &rsum, &ld);
      BL_TRY(launch_gemm_q(layers[i].packed, layers[i].gamma, layers[i].N, layers[i].K, M, xq, ld, sc, rsum,
                           layers[i].y, y_dtype, layers[i].acc_out, status, s));
      ++i;
      continue;
    }
    // A decode group: following layers that also take the GEMV path the same way
    // and neither read what the group writes nor write what it reads.
    auto fused_of = [&](int k) { return !layers[k].xq && bl::gemv_fuses_quant(M, layers[k].K, x_bf16); };
    const bool fused = fused_of(i);
    int j = i + 1;
    while (j < n_layers && j - i < bl::kGvMaxLayers) {
      bool gj = false;
      if (choose_gemv(M, layers[j].K, &gj) != BL_OK || !gj) break;
      if (layers[j].xq && layers[j].K % 128 != 0) break;
      if (fused_of(j) != fused) break;
      // Input (activations or caller codes) and output byte ranges of a layer.
      auto in_of = [&](int k, const void** p, size_t* n) {
        *p = layers[k].xq ? static_cast<const void*>(layers[k].xq) : layers[k].x;
        *n = static_cast<size_t>(M) * layers[k].K * (layers[k].xq ? 1 : xsz);
      };
      bool independent = true;
      const void* xj;
      size_t nxj;
      in_of(j, &xj, &nxj);
      const size_t yj = static_cast<size_t>(M) * layers[j].N * ysz;
      for (int k = i; k < j && independent; ++k) {
        const void* xk;
        size_t nxk;
        in_of(k, &xk, &nxk);
        const size_t yk = static_cast<size_t>(M) * layers[k].N * ysz;
        if (ranges_overlap(xj, nxj, layers[k].y, yk) || ranges_overlap(layers[j].y, yj, xk, nxk) ||
            ranges_overlap(layers[j].y, yj, layers[k].y, yk))
          independent = false;
      }
      if (!independent) break;
      ++j;
    }
    bl::GemvLayerArgs args[bl::kGvMaxLayers];
    for (int k = i; k < j; ++k) {
      const bl_layer& L = layers[k];
      if (fused) {
        args[k - i] = bl::GemvLayerArgs{L.packed, L.gamma, L.N, L.K, L.x, nullptr, nullptr, 0, L.y, L.acc_out};
      } else {
        if (!L.xq) quant_src[k] = shared_src(k);
        const int8_t* xq;
        const float* sc;
        const int32_t* rsum;
        int ld;
        codes_of(k, &xq, &sc, &rsum, &ld);
        args[k - i] = bl::GemvLayerArgs{L.packed, L.gamma, L.N, L.K, xq, sc, rsum, ld, L.y, L.acc_out};
      }
    }
    if (!fused) {
      // Quantise the group's distinct raw inputs once, in one launch.
      bl::QuantArgs qa[bl::kGvMaxLayers];
      int nq = 0;
      for (int k = i; k < j; ++k) {
        if (layers[k].xq || quant_src[k] != k) continue;
        int8_t* xq;
        float* sc;
        int32_t* rsum;
        region(k, &xq, &sc, &rsum);
        qa[nq++] = bl::QuantArgs{layers[k].x, xq, sc, rsum, layers[k].K, code_pitch(layers[k].K)};
      }
      if (nq > 0) {
        cudaError_t e = bl::launch_act_quant_group(qa, nq, M, x_bf16, s, true);
        if (e != cudaSuccess) return cuda_fail(e, "act_quant launch");
      }
    }
    const int xt = fused ? (x_bf16 ? bl::kInBF16 : bl::kInF32) : bl::kInInt8;
    cudaError_t e = bl::launch_gemv_group(args, j - i, M, xt, yt, status, tickets_of(workspace), s, true);
    if (e != cudaSuccess) return gemv_fail(e);
    i = j;
  }
  return BL_OK;
}

// ---------------------------------------------------------------------------
// The FFN's gate and up BitLinears with the gated activation and the down
// BitLinear's input quantisation.  Workspace: status block, the codes of x,
// h [M][N] (for callers that do not want h; elements of 4 bytes at most,
// 256-rounded), then (1 to 8 tokens) the fused launch's counters, zeroed
// before it, or (9 to 16 tokens) the gate and up outputs [2][M][N].
//
// Up to 8 tokens one decode launch forms h and its codes; for 9 to 16 the
// launch's grid-wide step costs more than it saves (measured at the 70B FFN
// width, 16 tokens: 51.9 us fused against 45.4 us for the products, then the
// gated activation kernel), so the call runs those two launches instead,
// with the same results bit for bit.
// ---------------------------------------------------------------------------
constexpr int kGluFusedMaxTokens = 8;

struct GluLayout {
  size_t h, zero, gu, total;
};

static GluLayout glu_layout(int M, int N, int K) {
  GluLayout g;
  g.h = forward_layout(M, K).total;
  g.zero = g.h + round_up(static_cast<size_t>(M) * N * 4, 256);
  g.gu = g.zero;
  g.total = g.zero;
  if (M >= 1 && M <= kGluFusedMaxTokens) g.total = g.zero + bl::gemv_glu_scratch_bytes(N);
  if (M > kGluFusedMaxTokens && M <= 16) g.total = g.gu + round_up(2 * static_cast<size_t>(M) * N * 4, 256);
  return g;
}

size_t bitlinear_gate_up_glu_workspace_bytes(int M, int N, int K) {
  if (M < 0 || N < 0 || K < 0) return 0;
  return glu_layout(M, N, K).total;
}

int bitlinear_gate_up_glu(const uint8_t* packed_gate, const float* gamma_gate, const uint8_t* packed_up,
                          const float* gamma_up, int N, int K, const void* x, int x_dtype, int M, int act, void* h,
                          int8_t* xq, float* scale, int32_t* rowsum, void* workspace, size_t workspace_bytes,
                          void* stream) {
  BL_TRY(check_nk(N, K));
  if (N % 64 != 0) return fail(BL_ERR_UNSUPPORTED_SHAPE, "N = %d: h is the down BitLinear's input, N %% 64 == 0", N);
  BL_TRY(check_dtype(x_dtype, "x_dtype"));
  if (act != BL_GLU_RELU2 && act != BL_GLU_SILU) return fail(BL_ERR_INVALID_ARG, "act = %d: unknown", act);
  if (M < 0) return fail(BL_ERR_INVALID_ARG, "M = %d < 0", M);
  if (M == 0) return BL_OK;
  BL_TRY(check_ptr(packed_gate, "packed_gate", 16));
  BL_TRY(check_ptr(gamma_gate, "gamma_gate", 4));
  BL_TRY(check_ptr(packed_up, "packed_up", 16));
  BL_TRY(check_ptr(gamma_up, "gamma_up", 4));
  BL_TRY(check_ptr(x, "x", 16));
  BL_TRY(check_ptr(h, "h", 16, true));
  BL_TRY(check_ptr(xq, "xq", 16));
  BL_TRY(check_ptr(scale, "scale", 4));
  BL_TRY(check_ptr(rowsum, "rowsum", 4));
  BL_TRY(check_ptr(workspace, "workspace", 256));
  const GluLayout g = glu_layout(M, N, K);
  if (workspace_bytes < g.total)
    return fail(BL_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", workspace_bytes, g.total);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool x_bf16 = x_dtype == BL_BF16;
  const int at = x_bf16 ? bl::kOutBF16 : bl::kOutF32;  // gate/up outputs and h in the activation type
  void* hh = h ? h : static_cast<void*>(ws + g.h);
  const FwdLayout f = forward_layout(M, K);
  int8_t* cq = reinterpret_cast<int8_t*>(ws + f.xq);
  float* cs = reinterpret_cast<float*>(ws + f.scale);
  int32_t* cr = reinterpret_cast<int32_t*>(ws + f.rowsum);
  const int ldq = code_pitch(K);
  bool gemv = false;
  BL_TRY(choose_gemv(M, K, &gemv));
  if (gemv && M > kGluFusedMaxTokens) {
    // 9 to 16 tokens: the gate and up products into the workspace (one decode
    // launch after the quantisation of x), then the gated activation kernel.
    const size_t xsz = x_bf16 ? 2 : 4;
    void* yg = ws + g.gu;
    void* yu = ws + g.gu + static_cast<size_t>(M) * N * xsz;
    const bool fused = bl::gemv_fuses_quant(M, K, x_bf16);
    bl::GemvLayerArgs L[2];
    cudaError_t e;
    if (fused) {
      L[0] = bl::GemvLayerArgs{packed_gate, gamma_gate, N, K, x, nullptr, nullptr, 0, yg, nullptr};
      L[1] = bl::GemvLayerArgs{packed_up, gamma_up, N, K, x, nullptr, nullptr, 0, yu, nullptr};
    } else {
      L[0] = bl::GemvLayerArgs{packed_gate, gamma_gate, N, K, cq, cs, cr, ldq, yg, nullptr};
      L[1] = bl::GemvLayerArgs{packed_up, gamma_up, N, K, cq, cs, cr, ldq, yu, nullptr};
      e = bl::launch_act_quant(x, x_bf16, M, K, ldq, cq, cs, cr, s, true);
      if (e != cudaSuccess) return cuda_fail(e, "act_quant launch");
    }
    e = bl::launch_gemv_group(L, 2, M, fused ? (x_bf16 ? bl::kInBF16 : bl::kInF32) : bl::kInInt8, at, status,
                              tickets_of(ws), s, true);
    if (e != cudaSuccess) return gemv_fail(e);
    e = bl::launch_glu_quant(yg, yu, x_bf16, M, N, act == BL_GLU_RELU2 ? bl::kGluRelu2 : bl::kGluSilu, h, xq, scale,
                             rowsum, s, true);
    return e == cudaSuccess ? BL_OK : cuda_fail(e, "glu_quant launch");
  }
  if (gemv) {
    // One decode launch: gate, up, h and its codes (after the quantisation of x,
    // which also clears the launch's counters).
    const bool fused = bl::gemv_fuses_quant(M, K, x_bf16);
    bl::GemvLayerArgs L[2];
    if (fused) {
      L[0] = bl::GemvLayerArgs{packed_gate, gamma_gate, N, K, x, nullptr, nullptr, 0, nullptr, nullptr};
      L[1] = bl::GemvLayerArgs{packed_up, gamma_up, N, K, x, nullptr, nullptr, 0, nullptr, nullptr};
    } else {
      L[0] = bl::GemvLayerArgs{packed_gate, gamma_gate, N, K, cq, cs, cr, ldq, nullptr, nullptr};
      L[1] = bl::GemvLayerArgs{packed_up, gamma_up, N, K, cq, cs, cr, ldq, nullptr, nullptr};
    }
    cudaError_t e;
    if (fused) {
      e = cudaMemsetAsync(ws + g.zero, 0, g.total - g.zero, s);
      if (e != cudaSuccess) return cuda_fail(e, "clearing the fused launch's counters");
    } else {
      e = bl::launch_act_quant(x, x_bf16, M, K, ldq, cq, cs, cr, s, true, ws + g.zero, g.total - g.zero);
      if (e != cudaSuccess) return cuda_fail(e, "act_quant launch");
    }
    const bl::GemvGluArgs G{act == BL_GLU_RELU2 ? bl::kGluRelu2 : bl::kGluSilu, hh, xq, scale, rowsum,
                            reinterpret_cast<uint32_t*>(ws + g.zero)};
    e = bl::launch_gemv_group(L, 2, M, fused ? (x_bf16 ? bl::kInBF16 : bl::kInF32) : bl::kInInt8, at, status,
                              tickets_of(ws), s, true, &G);
    return e == cudaSuccess ? BL_OK : gemv_fail(e);
  }
  // Many tokens: the quantisation of x, one tensor-core GEMM over the gate and
  // up weights whose epilogue writes h, then the quantisation of h.
  cudaError_t e = bl::launch_act_quant(x, x_bf16, M, K, ldq, cq, cs, cr, s, true);
  if (e != cudaSuccess) return cuda_fail(e, "act_quant launch");
  bl::ProductArgs a{packed_gate, gamma_gate, N, K, M, cq, ldq, cs, cr, hh, at, nullptr, status};
  a.packed2 = packed_up;
  a.gamma2 = gamma_up;
  a.glu_act = act == BL_GLU_RELU2 ? bl::kGluRelu2 : bl::kGluSilu;
  e = bl::launch_gemm(a, s, true);
  if (e != cudaSuccess) return cuda_fail(e, "GEMM launch (gate and up with the gated activation)");
  e = bl::launch_act_quant(hh, x_bf16, M, N, N, xq, scale, rowsum, s, true);
  if (e != cudaSuccess) return cuda_fail(e, "act_quant launch (h)");
  return BL_OK;
}

int bitlinear_device_status(void* workspace, void* stream) {
  BL_TRY(check_ptr(workspace, "workspace", 256));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  uint32_t word = 0;
  e = cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (word != 0) {
    e = cudaMemset(workspace, 0, sizeof(word));
    if (e != cudaSuccess) return cuda_fail(e, "status clear");
    return fail(BL_ERR_DEVICE_TIMEOUT, "a device-side wait ran out of time (status 0x%x)", word);
  }
  return BL_OK;
}

int bitlinear_selftest_wait_timeout(void* workspace, size_t workspace_bytes, int limit_us, void* stream) {
  BL_TRY(check_ptr(workspace, "workspace", 256));
  if (workspace_bytes < kStatusBytes)
    return fail(BL_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", workspace_bytes, kStatusBytes);
  if (limit_us < 1 || limit_us > 1000000) return fail(BL_ERR_INVALID_ARG, "limit_us = %d not in [1, 1e6]", limit_us);
  cudaError_t e = bl::launch_wait_timeout_selftest(static_cast<uint32_t*>(workspace), limit_us,
                                                   static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
  return BL_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// bitlinear_forward_noalloc: the forward for callers that cannot allocate.
//
// Some callers have no way to hand the library a workspace: code that runs
// where cudaMalloc is off limits (it can synchronise the whole device, so a
// latency-critical decode loop or a real-time thread avoids it), plug-ins
// hosted by an engine that owns every device allocation through its own
// pool and exposes no allocator to them, and callers holding a device-wide
// lock they must not block under.  This entry point gives them the same
// forward as bitlinear_forward, with the scratch in a fixed array that this
// file declares in device memory, so nothing is allocated per call.
//
// The array costs every GPU that loads the library kNoAllocScratchBytes of
// memory until the process exits.  Every call uses the same array, so calls
// whose work overlaps on the GPU (two streams, or two host threads issuing
// at once) race on it; calls in one stream are fine.  Each call clears the
// array's 256-byte control block first, so nothing left by an earlier call
// carries over.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB

// The scratch.  On the host this name is only a shadow of the device symbol,
// never an address to give a kernel; noalloc_scratch() looks the address up.
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Identity of the current context (0 if the driver cannot tell): the cached
// address is valid only in the context it was looked up in, and a device
// reset or a released primary context gives the device a new one.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
    looked_up = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx && get_id(ctx, &id) == CUDA_SUCCESS) return id;
  return 0;
}

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[64] = {nullptr};
unsigned long long g_noalloc_ctx[64] = {0};

// Device address of the scratch on the current device: looked up once per
// device and context, with that device current, then cached.  (Before the
// first CUDA call of the process no context is current yet; the lookup then
// creates it and is repeated once on the next call, under its identity.)
int noalloc_scratch(uint8_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(BL_ERR_CUDA, "device index %d out of range", dev);
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev] || ctx == 0 || g_noalloc_ctx[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
    if (p == nullptr) return fail(BL_ERR_CUDA, "cudaGetSymbolAddress(scratch) returned NULL");
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = ctx;
  }
  *out = static_cast<uint8_t*>(g_noalloc_ptr[dev]);
  return BL_OK;
}

}  // namespace

extern "C" int bitlinear_forward_noalloc(const uint8_t* packed, const float* gamma, int N, int K, const void* x,
                                         int x_dtype, int M, void* y, int y_dtype, int32_t* acc_out,
                                         void* stream) {
  BL_TRY(check_nk(N, K));
  BL_TRY(check_dtype(x_dtype, "x_dtype"));
  BL_TRY(check_dtype(y_dtype, "y_dtype"));
  if (M < 0) return fail(BL_ERR_INVALID_ARG, "M = %d < 0", M);
  if (M == 0) return BL_OK;
  BL_TRY(check_ptr(packed, "packed", 16));
  BL_TRY(check_ptr(gamma, "gamma", 4));
  BL_TRY(check_ptr(x, "x", 16));
  BL_TRY(check_ptr(y, "y", 16));
  BL_TRY(check_ptr(acc_out, "acc_out", 16, true));
  // Same layout as a bitlinear_forward workspace: control block, then q, s,
  // rowsum.  What the call needs depends on its path: the decode kernel
  // quantising in-kernel needs only the control block, the others the codes too.
  const FwdLayout l = forward_layout(M, K);
  bool gemv = false;
  BL_TRY(choose_gemv(M, K, &gemv));
  const bool fused = gemv && bl::gemv_fuses_quant(M, K, x_dtype == BL_BF16, true);
  const size_t need = fused ? kStatusBytes : l.total;
  if (need > kNoAllocScratchBytes)
    return fail(BL_ERR_WORKSPACE_TOO_SMALL,
                "M = %d, K = %d needs %zu bytes of scratch but the fixed scratch holds %zu; "
                "use bitlinear_forward with a workspace",
                M, K, need, kNoAllocScratchBytes);
  uint8_t* scratch = nullptr;
  BL_TRY(noalloc_scratch(&scratch));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(scratch, 0, kStatusBytes, s);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the scratch control block");
  return forward_on(packed, gamma, N, K, x, x_dtype, M, y, y_dtype, acc_out, scratch, s);
}

extern "C" int bitlinear_noalloc_status(void* stream) {
  uint8_t* scratch = nullptr;
  BL_TRY(noalloc_scratch(&scratch));
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  uint32_t word = 0;
  e = cudaMemcpy(&word, scratch, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (word != 0) {
    e = cudaMemset(scratch, 0, sizeof(word));
    if (e != cudaSuccess) return cuda_fail(e, "status clear");
    return fail(BL_ERR_DEVICE_TIMEOUT, "a device-side wait of a no-allocation call ran out of time (status 0x%x)",
                word);
  }
  return BL_OK;
}
