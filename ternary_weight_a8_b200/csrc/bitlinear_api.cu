// C ABI of the BitLinear W1.58A8 forward: argument checks, workspace layout,
// dispatch to the kernels, and the layer chain.  The declarations and their
// contracts are in include/bitlinear.h.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>

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

// Workspace layout: [0, 256) status word, then the quantised activations of
// the call (q [M][K], s [M], rowsum [M]), each region 256-byte aligned.
struct FwdLayout {
  size_t xq, scale, rowsum, total;
};

FwdLayout forward_layout(int M, int K) {
  FwdLayout l;
  l.xq = kStatusBytes;
  l.scale = l.xq + round_up(static_cast<size_t>(M) * K, 256);
  l.rowsum = l.scale + round_up(static_cast<size_t>(M) * 4, 256);
  l.total = l.rowsum + round_up(static_cast<size_t>(M) * 4, 256);
  return l;
}

#define BL_TRY(expr)            \
  do {                          \
    int _rc = (expr);           \
    if (_rc != BL_OK) return _rc; \
  } while (0)

// The product kernel for this call: the decode GEMV for M <= 16 (unless its
// activations do not fit on chip), else the tensor-core GEMM; bitlinear_set_path
// overrides the choice on the calling thread.
int choose_gemv(int M, int N, int K, bool* gemv) {
  bool v = M <= 16;
  if (g_path == 1) {
    if (M > 16) return fail(BL_ERR_UNSUPPORTED_SHAPE, "GEMV path forced with M = %d > 16", M);
    v = true;
  } else if (g_path == 2) {
    v = false;
  }
  if (v && bl::plan_gemv(M, N, K).splits == 0) {
    if (g_path == 1)
      return fail(BL_ERR_UNSUPPORTED_SHAPE, "GEMV path forced but M*K = %lld does not fit on chip",
                  static_cast<long long>(M) * K);
    v = false;
  }
  *gemv = v;
  return BL_OK;
}

int launch_product(bool gemv, const uint8_t* packed, const float* gamma, int N, int K, int M, const int8_t* xq,
                   const float* scale, const int32_t* rowsum, void* y, int y_dtype, int32_t* acc_out,
                   uint32_t* status, cudaStream_t s) {
  const int yt = y_dtype == BL_BF16 ? bl::kOutBF16 : bl::kOutF32;
  cudaError_t e;
  if (gemv) {
    bl::GemvArgs a{packed, gamma, N, K, M, xq, bl::kInInt8, scale, y, yt, acc_out, status};
    e = bl::launch_gemv(a, s, true);
  } else {
    bl::ProductArgs a{packed, gamma, N, K, M, xq, scale, rowsum, y, yt, acc_out, status};
    e = bl::launch_gemm(a, s, true);
  }
  if (e != cudaSuccess) return cuda_fail(e, gemv ? "GEMV launch" : "GEMM launch");
  return BL_OK;
}

// One forward on raw activations.  *xq_valid tells whether the workspace
// already holds this x quantised (a chain's layers that share their input);
// it is updated when this call quantises x into the workspace.
int forward_one(const uint8_t* packed, const float* gamma, int N, int K, const void* x, int x_dtype, int M,
                void* y, int y_dtype, int32_t* acc_out, uint8_t* ws, const FwdLayout& l, bool* xq_valid,
                cudaStream_t s) {
  bool gemv = false;
  BL_TRY(choose_gemv(M, N, K, &gemv));
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  if (gemv && bl::gemv_fuses_quant(M, K)) {
    // Small activations: the GEMV blocks quantise them on chip (one launch, no round trip).
    bl::GemvArgs a{packed, gamma, N, K, M, x, x_dtype == BL_BF16 ? bl::kInBF16 : bl::kInF32, nullptr, y,
                   y_dtype == BL_BF16 ? bl::kOutBF16 : bl::kOutF32, acc_out, status};
    cudaError_t e = bl::launch_gemv(a, s, true);
    if (e != cudaSuccess) return cuda_fail(e, "GEMV launch");
    return BL_OK;
  }
  int8_t* xq = reinterpret_cast<int8_t*>(ws + l.xq);
  float* scale = reinterpret_cast<float*>(ws + l.scale);
  int32_t* rowsum = reinterpret_cast<int32_t*>(ws + l.rowsum);
  if (!*xq_valid) {
    cudaError_t e = bl::launch_act_quant(x, x_dtype == BL_BF16, M, K, xq, scale, rowsum, s, true);
    if (e != cudaSuccess) return cuda_fail(e, "act_quant launch");
    *xq_valid = true;
  }
  return launch_product(gemv, packed, gamma, N, K, M, xq, scale, rowsum, y, y_dtype, acc_out, status, s);
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
  cudaError_t e = bl::launch_act_quant(x, x_dtype == BL_BF16, M, K, xq, scale, rowsum,
                                       static_cast<cudaStream_t>(stream), true);
  if (e != cudaSuccess) return cuda_fail(e, "act_quant launch");
  return BL_OK;
}

size_t bitlinear_workspace_bytes(int M, int N, int K) {
  (void)N;
  if (M < 0 || K < 0) return 0;
  return forward_layout(M, K).total;
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
  BL_TRY(choose_gemv(M, N, K, &gemv));
  return launch_product(gemv, packed, gamma, N, K, M, xq, scale, rowsum, y, y_dtype, acc_out,
                        static_cast<uint32_t*>(workspace), static_cast<cudaStream_t>(stream));
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
  bool xq_valid = false;
  return forward_one(packed, gamma, N, K, x, x_dtype, M, y, y_dtype, acc_out, static_cast<uint8_t*>(workspace),
                     l, &xq_valid, static_cast<cudaStream_t>(stream));
}

size_t bitlinear_chain_workspace_bytes(const bl_layer* layers, int n_layers, int M) {
  if (!layers || n_layers <= 0 || M < 0) return 0;
  int k_max = 64;
  for (int i = 0; i < n_layers; ++i)
    if (layers[i].K > k_max) k_max = layers[i].K;
  return forward_layout(M, k_max).total;
}

int bitlinear_layer_chain(const bl_layer* layers, int n_layers, int M, int x_dtype, int y_dtype,
                          void* workspace, size_t workspace_bytes, void* stream) {
  if (!layers) return fail(BL_ERR_INVALID_ARG, "layers is NULL");
  if (n_layers < 0) return fail(BL_ERR_INVALID_ARG, "n_layers = %d < 0", n_layers);
  BL_TRY(check_dtype(x_dtype, "x_dtype"));
  BL_TRY(check_dtype(y_dtype, "y_dtype"));
  if (M < 0) return fail(BL_ERR_INVALID_ARG, "M = %d < 0", M);
  if (M == 0 || n_layers == 0) return BL_OK;
  BL_TRY(check_ptr(workspace, "workspace", 256));
  for (int i = 0; i < n_layers; ++i) {
    const bl_layer& L = layers[i];
    BL_TRY(check_nk(L.N, L.K));
    BL_TRY(check_ptr(L.packed, "layer.packed", 16));
    BL_TRY(check_ptr(L.gamma, "layer.gamma", 4));
    BL_TRY(check_ptr(L.x, "layer.x", 16));
    BL_TRY(check_ptr(L.y, "layer.y", 16));
  }
  const size_t need = bitlinear_chain_workspace_bytes(layers, n_layers, M);
  if (workspace_bytes < need)
    return fail(BL_ERR_WORKSPACE_TOO_SMALL, "chain workspace %zu < %zu bytes", workspace_bytes, need);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  bool xq_valid = false;
  for (int i = 0; i < n_layers; ++i) {
    const bl_layer& L = layers[i];
    const bool shared_input = i > 0 && layers[i - 1].x == L.x && layers[i - 1].K == L.K;
    if (!shared_input) xq_valid = false;
    BL_TRY(forward_one(L.packed, L.gamma, L.N, L.K, L.x, x_dtype, M, L.y, y_dtype, nullptr, ws,
                       forward_layout(M, L.K), &xq_valid, s));
  }
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
