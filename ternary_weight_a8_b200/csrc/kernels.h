// Internal launchers of the BitLinear kernels (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

namespace bl {

enum OutType { kOutF32 = 0, kOutBF16 = 1 };

// Launch helper: cudaLaunchKernelEx, optionally as a programmatic dependent
// of the preceding kernel on the stream.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                   bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

int num_sms();

// Runs `set` (a function attribute, which belongs to the current device's
// context) unless it already succeeded on the calling thread's current
// device: one bit per device, up to 64 devices (beyond that, every call).
template <typename F>
cudaError_t once_per_device(std::atomic<uint64_t>& done, F&& set) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 64;
  const uint64_t bit = dev < 64 ? (uint64_t{1} << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  const cudaError_t e = set();
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
  return e;
}

// Offline weight path.
cudaError_t launch_gamma(const float* W, int N, int K, double* row_sums, float* gamma,
                         cudaStream_t stream);
cudaError_t launch_ternary_pack(const float* W, int N, int K, const float* gamma, uint8_t* packed,
                                cudaStream_t stream);

// Per-token activation quantisation: one input, or several inputs in one launch.
struct QuantArgs {
  const void* x;
  int8_t* xq;       // [M][ldq], zero past K
  float* scale;
  int32_t* rowsum;  // may be null
  int K, ldq;
};
constexpr int kQuantMaxItems = 8;
// zero / zero_bytes (16-byte aligned, a multiple of 16; may be null / 0): a
// region the launch also clears, once the preceding kernel has finished
// (the split scratch of the decode launch that follows).
cudaError_t launch_act_quant(const void* x, int x_bf16, int M, int K, int ldq, int8_t* xq, float* scale,
                             int32_t* rowsum, cudaStream_t stream, bool pdl, void* zero = nullptr,
                             size_t zero_bytes = 0);
cudaError_t launch_act_quant_group(const QuantArgs* items, int n_items, int M, int x_bf16, cudaStream_t stream,
                                   bool pdl, void* zero = nullptr, size_t zero_bytes = 0);

// RMSNorm (gain optional) fused with the per-token quantisation; x_norm
// (optional) receives the normalised activations in the input type.
cudaError_t launch_rmsnorm_quant(const void* x, int x_bf16, int M, int K, const float* gain, float eps, void* x_norm,
                                 int8_t* xq, float* scale, int32_t* rowsum, cudaStream_t stream, bool pdl);

// The FFN's gated activation h = act(gate) * up fused with the per-token
// quantisation of h (the down BitLinear's input); h (optional) written in the
// activation type.
enum GluAct { kGluRelu2 = 0, kGluSilu = 1 };
cudaError_t launch_glu_quant(const void* gate, const void* up, int x_bf16, int M, int N, int act, void* h,
                             int8_t* xq, float* scale, int32_t* rowsum, cudaStream_t stream, bool pdl);

enum InType { kInInt8 = 0, kInBF16 = 1, kInF32 = 2 };

// Tensor-core GEMM on quantised activations (many tokens).
struct ProductArgs {
  const uint8_t* packed;
  const float* gamma;
  int N, K, M;
  const int8_t* xq;
  int ldx;  // row pitch of xq (>= K, multiple of 16)
  const float* scale;
  const int32_t* rowsum;
  void* y;
  int y_type;  // OutType
  int32_t* acc_out;
  uint32_t* status;
  // The FFN's gate and up products in one launch (glu_act >= 0): packed /
  // gamma are the gate BitLinear's, packed2 / gamma2 the up BitLinear's (same
  // N and K), and y receives h = act(gate) * up [M][N] in y_type; acc_out
  // must be null.  glu_act = -1: a plain product.
  const uint8_t* packed2 = nullptr;
  const float* gamma2 = nullptr;
  int glu_act = -1;
};

// Decode GEMV (M <= 16) over a group of independent layers in one launch.
// Each layer's activations are raw (fp32 / bf16, quantised in the kernel) or
// int8 codes with their token scales; x_type is the same for the whole group.
struct GemvLayerArgs {
  const uint8_t* packed;
  const float* gamma;
  int N, K;
  const void* x;          // raw activations [M][K], or int8 codes [M][ldx]
  const float* scale;     // token scales of the codes
  const int32_t* rowsum;  // code sums of the codes
  int ldx;                // row pitch of the codes: a multiple of 128 >= K, zero past K
  void* y;
  int32_t* acc_out;
};
constexpr int kGvMaxLayers = 8;
bool gemv_fuses_quant(int M, int K, int x_bf16, bool single = false);
// CTAs per unit of the decode kernel's K-split (a cluster): 0 lets the kernel
// choose (by the unit count), else forced (1 .. 8, capped by the stages).  Per thread.
void gemv_force_ksplit(int ks);
// Form of the decode product for 2 to 16 tokens on int8 codes: 0 (default)
// and 1 the CUDA-core kernel, 2 the tensor-core kernel whenever eligible.  Per thread.
void gemv_force_form(int form);
bool gemv_tc_eligible(const GemvLayerArgs* layers, int n_layers, int M);
cudaError_t launch_gemv_tc(const GemvLayerArgs* layers, int n_layers, int M, int y_type, uint32_t* status,
                           uint32_t* tickets, cudaStream_t stream, bool pdl);

// The FFN's gated activation fused into the launch of its gate and up
// BitLinears (layers[0] = gate, layers[1] = up, same N and K; their y are
// not written): h = act(gate) * up [M][N] in the activation type (y_type),
// and its per-token quantisation (codes [M][N], scales, code sums) for the
// down BitLinear.  `zeroed`: gemv_glu_scratch_bytes(N) bytes, zero at launch.
struct GemvGluArgs {
  int act;  // GluAct
  void* h;
  int8_t* xq;
  float* scale;
  int32_t* rowsum;
  uint32_t* zeroed;
};
size_t gemv_glu_scratch_bytes(int N);

// tickets: two zero-initialised uint32 in device memory (reset by the kernel after use).
cudaError_t launch_gemv_group(const GemvLayerArgs* layers, int n_layers, int M, int x_type, int y_type,
                              uint32_t* status, uint32_t* tickets, cudaStream_t stream, bool pdl,
                              const GemvGluArgs* glu = nullptr);

// cuTensorMapEncodeTiled from the driver (no link-time dependency on libcuda).
#ifdef CUDA_VERSION
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
#endif
void* tensor_map_encoder();
cudaError_t launch_gemm(const ProductArgs& a, cudaStream_t stream, bool pdl);

// Lookup-table decode product for one token (the T-MAC-style alternative):
// codes of one token [K], K % 64 == 0 and K <= kLutMaxK (its tables fill
// shared memory: 8 bytes per input).
constexpr int kLutMaxK = 24576;
cudaError_t launch_lut_gemv(const uint8_t* packed, const float* gamma, int N, int K, const int8_t* xq,
                            const float* scale, const int32_t* rowsum, void* y, int y_type, int32_t* acc_out,
                            cudaStream_t stream, bool pdl);

// The straight-through backward: dx = gamma (dy . t) [M][K] (fp32 or bf16,
// null to skip) and dW = dy^T . bf16(q / s) [N][K] fp32 (null to skip), from
// the packed weights, bf16 dy [M][N] and the forward's codes and scales.
// scratch: ste_scratch_bytes(M, N, K) bytes, 256-byte aligned.
size_t ste_scratch_bytes(int M, int N, int K);
cudaError_t launch_ste_backward(const uint8_t* packed, const float* gamma, int N, int K, const void* dy, const int8_t* xq,
                                const float* scale, int M, void* dx, bool dx_bf16, float* dw, uint8_t* scratch,
                                uint32_t* status, cudaStream_t stream);

// Self-test of the bounded device wait.
cudaError_t launch_wait_timeout_selftest(uint32_t* status, int limit_us, cudaStream_t stream);

}  // namespace bl
