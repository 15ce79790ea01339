// Lookup-table decode product (one token): the T-MAC-style alternative to
// the tensor-core decode kernel, kept to compare the two on B200.
//
// "BitNet b1.58 and the 1-Bit AI Architecture Revolution", section "The CPU
// Revival: bitnet.cpp and T-MAC": with four ternary weights per group only a
// few partial sums of the activations are possible, so they are precomputed
// and looked up instead of multiplied; the sign structure cuts the table to
// 16 binary combinations.  Here a stored code is c = t + 1 = lo + 2 hi (two
// bits), so for the four inputs that share a packed byte
//   sum_j c_j q_j = T[lo bits] + 2 T[hi bits],  T[mask] = sum_{j in mask} q_j,
// one 16-entry table per four inputs serving both bit planes; y then follows
// as in the other kernels: acc = sum c q - sum q, y = acc * (gamma / s).
//
// Every block builds the token's tables for all of K in shared memory (int16
// entries, entry-major so that consecutive lanes, which read consecutive
// tables, fall in different banks), then each warp takes whole rows: lanes
// read consecutive 32-bit words of the packed row (coalesced), split each
// byte into its two 4-bit planes and add two table entries, and the warp
// sums its lanes at the end of the row.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace bl {

constexpr int kLutWarps = 8;
constexpr int kLutThreads = 32 * kLutWarps;

// Tables of `nt` groups, entry-major: entry e of table t at [e * pitch + t].
__device__ __forceinline__ int lut_pitch(int nt) { return (nt + 63) / 64 * 64; }

// The 4-bit mask of bits 0, 2, 4, 6 of a byte (its low bit plane).
__device__ __forceinline__ uint32_t even_bits4(uint32_t x) {
  x &= 0x55u;
  x = (x | (x >> 1)) & 0x33u;
  x = (x | (x >> 2)) & 0x0Fu;
  return x;
}

template <typename TY>
__global__ void __launch_bounds__(kLutThreads) lut_gemv_kernel(const uint32_t* __restrict__ packed, const float* gamma_p,
                                                               int N, int K, const int8_t* __restrict__ xq,
                                                               const float* scale, const int32_t* rowsum,
                                                               TY* __restrict__ y, int32_t* __restrict__ acc_out) {
  extern __shared__ int16_t tab[];
  griddep_launch_dependents();
  griddep_wait();  // the codes come from the preceding kernel
  const int words = K / 16;  // 32-bit words per packed row
  const int nt = 4 * words;  // tables: one per byte of a word (4 inputs each)
  const int pitch = lut_pitch(nt);

  // Table t = 4 w + b covers inputs 16 w + 4 j + b, j = 0..3 (bit pair j of byte b).
  for (int t = threadIdx.x; t < nt; t += blockDim.x) {
    const int w = t >> 2, b = t & 3;
    int q[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) q[j] = xq[16 * w + 4 * j + b];
#pragma unroll
    for (int mask = 0; mask < 16; ++mask) {
      int v = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) v += (mask >> j & 1) ? q[j] : 0;
      tab[mask * pitch + t] = static_cast<int16_t>(v);
    }
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float gamma = __ldg(gamma_p);
  const float gs = __fdiv_rn(gamma, __ldcg(scale));
  const int rs = __ldcg(rowsum);
  for (int n = blockIdx.x * kLutWarps + warp; n < N; n += gridDim.x * kLutWarps) {
    const uint32_t* row = packed + static_cast<size_t>(n) * words;
    int acc = 0;
    for (int w0 = 0; w0 < words; w0 += 32 * 4) {
      uint32_t wv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int w = w0 + 32 * i + lane;
        wv[i] = w < words ? __ldg(row + w) : 0x55555555u;  // code 1 (t = 0) past the end: adds q_j, never read
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int w = w0 + 32 * i + lane;
        if (w < words) {
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const uint32_t byte = (wv[i] >> (8 * b)) & 0xFFu;
            const int t = 4 * w + b;
            acc += tab[even_bits4(byte) * pitch + t] + 2 * tab[even_bits4(byte >> 1) * pitch + t];
          }
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const int a = acc - rs;
      const float v = __fmul_rn(static_cast<float>(a), gs);
      if constexpr (sizeof(TY) == 4) y[n] = v; else y[n] = __float2bfloat16_rn(v);
      if (acc_out) acc_out[n] = a;
    }
  }
}

int lut_gemv_smem_bytes(int K) {
  const int nt = K / 4;
  return 16 * ((nt + 63) / 64 * 64) * static_cast<int>(sizeof(int16_t));
}

cudaError_t launch_lut_gemv(const uint8_t* packed, const float* gamma, int N, int K, const int8_t* xq,
                            const float* scale, const int32_t* rowsum, void* y, int y_type, int32_t* acc_out,
                            cudaStream_t stream, bool pdl) {
  if (K % 64 != 0 || K > kLutMaxK || N <= 0) return cudaErrorInvalidValue;
  const int smem = lut_gemv_smem_bytes(K);
  static std::atomic<uint64_t> attr_done[2];  // per output type and device
  const int ti = y_type == kOutBF16 ? 1 : 0;
  auto kb = lut_gemv_kernel<__nv_bfloat16>;
  auto kf = lut_gemv_kernel<float>;
  const cudaError_t e = once_per_device(attr_done[ti], [&] {
    return ti ? cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, 48 * 1024 * 4)
              : cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, 48 * 1024 * 4);
  });
  if (e != cudaSuccess) return e;
  // Blocks: a few per SM (as many as fit beside their tables), rows split among their warps.
  int per_sm = (224 * 1024) / (smem + 1024);
  if (per_sm < 1) per_sm = 1;
  if (per_sm > 8) per_sm = 8;
  int grid = per_sm * num_sms();
  const int need = (N + kLutWarps - 1) / kLutWarps;
  if (grid > need) grid = need;
  const uint32_t* pw = reinterpret_cast<const uint32_t*>(packed);
  if (ti) return launch(kb, dim3(grid), dim3(kLutThreads), static_cast<size_t>(smem), stream, pdl, pw, gamma, N, K,
                        xq, scale, rowsum, static_cast<__nv_bfloat16*>(y), acc_out);
  return launch(kf, dim3(grid), dim3(kLutThreads), static_cast<size_t>(smem), stream, pdl, pw, gamma, N, K, xq,
                scale, rowsum, static_cast<float*>(y), acc_out);
}

}  // namespace bl
