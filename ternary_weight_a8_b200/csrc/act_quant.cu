// Per-token 8-bit activation quantisation.
//
// "BitNet's Real Bet: Designing the Whole Inference Stack", section "A
// low-bit model is a whole-stack design": activations take a separate
// per-token 8-bit path.  "A Two-Billion Ternary Bet": activations are
// quantised dynamically.  Reading (the pages print no formula): symmetric
// absmax, s = 127 / max(amax, 1e-5), q = clamp(rint(x * s), -128, 127), in
// fp32 with round-half-to-even.  The kernel also writes sum_k q[m][k], which
// the product kernels use to turn sums over the stored codes c = t + 1 into
// sums over t.
//
// One block per token; the token is read twice (absmax, then quantise), the
// second time from L1/L2.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace bl {

constexpr int kQuantThreads = 256;

struct Vec8 {
  float v[8];
};

__device__ __forceinline__ Vec8 load8(const float* p) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  return Vec8{{a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w}};
}

__device__ __forceinline__ Vec8 load8(const __nv_bfloat16* p) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  Vec8 r;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    r.v[2 * i] = __uint_as_float(w[i] << 16);            // low half: element 2i
    r.v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);  // high half: element 2i+1
  }
  return r;
}

template <typename T, typename Op>
__device__ __forceinline__ T block_reduce(T v, Op op, T* smem) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) smem[warp] = v;
  __syncthreads();
  T r = smem[0];
  for (int i = 1; i < kQuantThreads / 32; ++i) r = op(r, smem[i]);
  __syncthreads();
  return r;
}

template <typename TX>
__global__ void __launch_bounds__(kQuantThreads) act_quant_kernel(const TX* __restrict__ x, int K,
                                                                  int8_t* __restrict__ xq,
                                                                  float* __restrict__ scale,
                                                                  int32_t* __restrict__ rowsum) {
  __shared__ float red_f[kQuantThreads / 32];
  __shared__ int red_i[kQuantThreads / 32];
  griddep_launch_dependents();
  griddep_wait();  // x may be the preceding kernel's output

  const int m = blockIdx.x;
  const TX* xr = x + static_cast<size_t>(m) * K;
  int8_t* qr = xq + static_cast<size_t>(m) * K;

  float amax = 0.0f;
  for (int k = threadIdx.x * 8; k < K; k += kQuantThreads * 8) {
    const Vec8 v = load8(xr + k);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v.v[i]));
  }
  amax = block_reduce(amax, [](float a, float b) { return fmaxf(a, b); }, red_f);
  const float s = __fdiv_rn(127.0f, fmaxf(amax, 1e-5f));

  int sum = 0;
  for (int k = threadIdx.x * 8; k < K; k += kQuantThreads * 8) {
    const Vec8 v = load8(xr + k);
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int q = __float2int_rn(__fmul_rn(v.v[i], s));
      q = min(max(q, -128), 127);
      sum += q;
      packed[i >> 2] |= (static_cast<uint32_t>(q) & 0xffu) << (8 * (i & 3));
    }
    *reinterpret_cast<uint2*>(qr + k) = make_uint2(packed[0], packed[1]);
  }
  sum = block_reduce(sum, [](int a, int b) { return a + b; }, red_i);
  if (threadIdx.x == 0) {
    scale[m] = s;
    if (rowsum) rowsum[m] = sum;
  }
}

cudaError_t launch_act_quant(const void* x, int x_bf16, int M, int K, int8_t* xq, float* scale,
                             int32_t* rowsum, cudaStream_t stream, bool pdl) {
  if (M <= 0) return cudaSuccess;
  if (x_bf16) {
    return launch(act_quant_kernel<__nv_bfloat16>, dim3(M), dim3(kQuantThreads), 0, stream, pdl,
                  static_cast<const __nv_bfloat16*>(x), K, xq, scale, rowsum);
  }
  return launch(act_quant_kernel<float>, dim3(M), dim3(kQuantThreads), 0, stream, pdl,
                static_cast<const float*>(x), K, xq, scale, rowsum);
}

}  // namespace bl
