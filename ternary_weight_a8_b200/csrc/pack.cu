// Offline weight path: absmean gamma, ternarisation and 2-bit packing.
//
// "BitNet b1.58 and the 1-Bit AI Architecture Revolution", section "The
// BitLinear Layer and AbsMean Quantization": gamma = mean |W| over the whole
// matrix; t = clamp(round(W / (gamma + 1e-5)), -1, 1).
// "BitNet's Real Bet: Designing the Whole Inference Stack", section "A
// low-bit model is a whole-stack design": four ternary values per int8.
//
// gamma's double sum runs in a fixed order (each row over k ascending, then
// the row sums over n ascending), so its fp32 value, and every tie decision
// of the ternarisation that depends on it, is reproducible bit for bit.
#include "common.cuh"
#include "kernels.h"

namespace bl {

// Row sums sum_k |W[n][k]| in double, each in the fixed order k = 0, 1, ...
// A warp takes 32 rows: it reads them kGroup x 32 columns at a time, lane l
// loading column l of each row of each 32-column chunk (one 128-byte line
// per load, 32 * kGroup of them in flight, which is what keeps the few warps
// of a matrix fed), and after a transpose of each chunk through shared
// memory lane r adds row r's values in column order.
constexpr int kRowWarps = 4;
constexpr int kGroup = 4;  // 32-column chunks loaded at once

__global__ void __launch_bounds__(32 * kRowWarps) gamma_row_sums_kernel(const float* __restrict__ W, int N,
                                                                       int K, double* __restrict__ row_sums) {
  __shared__ float tile[kRowWarps][32][33];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = (blockIdx.x * kRowWarps + warp) * 32;
  if (row0 >= N) return;  // warp-uniform
  float (*t)[33] = tile[warp];
  double acc = 0.0;
  for (int k0 = 0; k0 < K; k0 += 32 * kGroup) {  // K % 64 == 0: whole 32-column chunks
    float v[kGroup][32];
#pragma unroll
    for (int c = 0; c < kGroup; ++c)
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        const int n = row0 + r, k = k0 + 32 * c + lane;
        v[c][r] = (n < N && k < K) ? __ldg(W + static_cast<size_t>(n) * K + k) : 0.0f;
      }
#pragma unroll
    for (int c = 0; c < kGroup; ++c) {
      if (k0 + 32 * c >= K) break;  // uniform
#pragma unroll
      for (int r = 0; r < 32; ++r) t[r][lane] = v[c][r];
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 32; ++i) acc = __dadd_rn(acc, fabs(static_cast<double>(t[lane][i])));
      __syncwarp();
    }
  }
  if (row0 + lane < N) row_sums[row0 + lane] = acc;
}

// One block: the row sums are staged through shared memory a chunk at a
// time and added by one thread in ascending n; gamma = fp32(sum / (N*K)).
__global__ void __launch_bounds__(256) gamma_finalize_kernel(const double* __restrict__ row_sums,
                                                             int N, long long count,
                                                             float* __restrict__ gamma) {
  __shared__ double chunk[2048];
  double total = 0.0;
  for (int base = 0; base < N; base += 2048) {
    const int len = min(2048, N - base);
    for (int i = threadIdx.x; i < len; i += blockDim.x) chunk[i] = row_sums[base + i];
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int i = 0; i < len; ++i) total = __dadd_rn(total, chunk[i]);
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    *gamma = (count > 0) ? __double2float_rn(__ddiv_rn(total, static_cast<double>(count))) : 0.0f;
  }
}

__device__ __forceinline__ uint32_t ternary_code(float w, float d) {
  float t = rintf(__fdiv_rn(w, d));  // IEEE divide, round half to even
  t = fminf(fmaxf(t, -1.0f), 1.0f);
  return static_cast<uint32_t>(static_cast<int>(t) + 1);  // code c = t + 1
}

// One thread per 16-element group: reads 64 bytes of W, writes one 32-bit
// packed word (element 4j+b of the group -> byte b, bits [2j, 2j+1]).
__global__ void __launch_bounds__(256) ternary_pack_kernel(const float* __restrict__ W,
                                                           long long groups,
                                                           const float* __restrict__ gamma,
                                                           uint32_t* __restrict__ packed) {
  const float d = __fadd_rn(*gamma, 1e-5f);
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; g < groups;
       g += stride) {
    const float4* src = reinterpret_cast<const float4*>(W) + g * 4;
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 v = __ldg(src + j);  // elements 4j .. 4j+3 of the group
      word |= ternary_code(v.x, d) << (0 + 2 * j);
      word |= ternary_code(v.y, d) << (8 + 2 * j);
      word |= ternary_code(v.z, d) << (16 + 2 * j);
      word |= ternary_code(v.w, d) << (24 + 2 * j);
    }
    packed[g] = word;
  }
}

cudaError_t launch_gamma(const float* W, int N, int K, double* row_sums, float* gamma,
                         cudaStream_t stream) {
  gamma_row_sums_kernel<<<(N + 32 * kRowWarps - 1) / (32 * kRowWarps), 32 * kRowWarps, 0, stream>>>(W, N, K,
                                                                                                 row_sums);
  gamma_finalize_kernel<<<1, 256, 0, stream>>>(row_sums, N, static_cast<long long>(N) * K, gamma);
  return cudaGetLastError();
}

cudaError_t launch_ternary_pack(const float* W, int N, int K, const float* gamma, uint8_t* packed,
                                cudaStream_t stream) {
  const long long groups = static_cast<long long>(N) * (K / 16);
  long long blocks = (groups + 255) / 256;
  const long long cap = static_cast<long long>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  ternary_pack_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      W, groups, gamma, reinterpret_cast<uint32_t*>(packed));
  return cudaGetLastError();
}

}  // namespace bl
