// The straight-through backward of a BitLinear, for training with latent
// ("shadow") weights.
//
// "BitNet b1.58 and the 1-Bit AI Architecture Revolution", section "Training
// Dynamics: The Straight-Through Estimator": the backward pass treats the
// quantisation as the identity, so gradients pass through the quantised
// weights to the high-precision shadow weights, which are quantised again
// (bitlinear_pack_weights) before the next forward.  With the forward
// y = xhat . What^T, xhat = q / s per token and What = gamma * t:
//   dx = dy . What = gamma * (dy . t)      [M][K]
//   dW = dy^T . xhat                       [N][K]
// xhat is taken as the backward stores it, bf16(q / s).
//
// Both products run on one bf16 tcgen05 GEMM, D = alpha * A . B^T with A and
// B K-major (row-major along the summed index), fed by three layout kernels:
// t^T as bf16 (-1, 0, 1 exactly) from the packed weights, dy^T, and xhat^T.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace bl {

// ---------------------------------------------------------------------------
// Layout kernels: 64 x 64 tiles through shared memory.
// ---------------------------------------------------------------------------
constexpr int kTile = 64;

// tt[k][n] = t[n][k] as bf16, from packed [N][K/4] (element 16g+4j+b in byte b, bits 2j..2j+1 of word g).
__global__ void __launch_bounds__(256) unpack_transpose_kernel(const uint32_t* __restrict__ packed, int N, int K,
                                                               __nv_bfloat16* __restrict__ tt) {
  __shared__ __nv_bfloat16 tile[kTile][kTile + 2];  // [k][n], padded
  const int n0 = blockIdx.y * kTile, k0 = blockIdx.x * kTile;
  const int words = K / 16;
  // 64 rows x 4 words (64 inputs) of the packed tile: one word per thread.
  const int r = threadIdx.x >> 2, wi = threadIdx.x & 3;
  const int n = n0 + r;
  uint32_t w = 0x55555555u;  // code 1 (t = 0) outside the matrix
  if (n < N) w = __ldg(packed + static_cast<size_t>(n) * words + k0 / 16 + wi);
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int code = static_cast<int>((w >> (8 * b + 2 * j)) & 3u);
      tile[16 * wi + 4 * j + b][r] = __float2bfloat16_rn(static_cast<float>(code - 1));
    }
  __syncthreads();
  // Out: 64 rows k of 64 n (128 bytes), two bf16 per thread per step.
  for (int i = threadIdx.x; i < kTile * kTile / 2; i += blockDim.x) {
    const int kr = i / (kTile / 2), c = 2 * (i % (kTile / 2));
    const int nn = n0 + c;
    if (k0 + kr < K && nn < N) {
      __nv_bfloat162 v;
      v.x = tile[kr][c];
      v.y = tile[kr][c + 1];
      *reinterpret_cast<__nv_bfloat162*>(tt + static_cast<size_t>(k0 + kr) * N + nn) = v;
    }
  }
}

// out[c][r] = f(in[r][c]) for a [R][C] bf16 matrix, or (xhat) bf16(q[r][c] / s[r]) from int8 codes.
template <bool kFromCodes>
__global__ void __launch_bounds__(256) transpose_kernel(const void* __restrict__ in, const float* __restrict__ s,
                                                        int R, int C, __nv_bfloat16* __restrict__ out) {
  __shared__ __nv_bfloat16 tile[kTile][kTile + 2];  // [r][c], padded
  const int r0 = blockIdx.y * kTile, c0 = blockIdx.x * kTile;
  for (int i = threadIdx.x; i < kTile * kTile; i += blockDim.x) {
    const int rr = i / kTile, cc = i % kTile;
    const int r = r0 + rr, c = c0 + cc;
    __nv_bfloat16 v = __float2bfloat16_rn(0.0f);
    if (r < R && c < C) {
      if constexpr (kFromCodes) {
        const int8_t q = static_cast<const int8_t*>(in)[static_cast<size_t>(r) * C + c];
        v = __float2bfloat16_rn(__fdiv_rn(static_cast<float>(q), __ldg(s + r)));
      } else {
        v = static_cast<const __nv_bfloat16*>(in)[static_cast<size_t>(r) * C + c];
      }
    }
    tile[rr][cc] = v;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kTile * kTile; i += blockDim.x) {
    const int cc = i / kTile, rr = i % kTile;
    const int r = r0 + rr, c = c0 + cc;
    if (r < R && c < C) out[static_cast<size_t>(c) * R + r] = tile[rr][cc];
  }
}

// ---------------------------------------------------------------------------
// bf16 GEMM: D[P][Q] = alpha * sum_r A[P][r] * B[Q][r], fp32 accumulation.
// Tiles 128 x 256 x 64 (128 bytes of r per row, 128-byte swizzle); warp 0
// TMA producer, warp 1 tensor-memory owner and MMA issuer (4 x K = 16 per
// k-block), warps 4-7 epilogue; two 256-column accumulators.
// ---------------------------------------------------------------------------
constexpr int kFBM = 128, kFBN = 256, kFBK = 64;
constexpr int kFStages = 4;
constexpr int kFABytes = kFBM * kFBK * 2, kFBBytes = kFBN * kFBK * 2;
constexpr int kFOffA = 0, kFOffB = kFStages * kFABytes, kFOffBar = kFOffB + kFStages * kFBBytes;
constexpr int kFNumBars = 2 * kFStages + 5;
constexpr int kFOffMisc = kFOffBar + kFNumBars * 8;
constexpr int kFSmem = kFOffMisc + 64 + 1024;
constexpr int kFThreads = 256;
// D f32, A bf16, B bf16, both K-major, N = 256, M = 128.
constexpr uint32_t kFIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((kFBN >> 3) << 17) | ((kFBM >> 4) << 24);

template <typename TO>
__global__ void __launch_bounds__(kFThreads, 1) gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmap_a,
                                                                 const __grid_constant__ CUtensorMap tmap_b, int P,
                                                                 int Q, int R, float alpha,
                                                                 const float* __restrict__ alpha_ptr,
                                                                 TO* __restrict__ out, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto full_bar = [&](int i) { return sb + kFOffBar + 8 * i; };
  auto empty_bar = [&](int i) { return sb + kFOffBar + 8 * (kFStages + i); };
  auto tfull_bar = [&](int i) { return sb + kFOffBar + 8 * (2 * kFStages + i); };
  auto tempty_bar = [&](int i) { return sb + kFOffBar + 8 * (2 * kFStages + 2 + i); };
  const uint32_t done_bar = sb + kFOffBar + 8 * (2 * kFStages + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kFOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kFOffMisc + 16);
  volatile int* never = reinterpret_cast<volatile int*>(smem + kFOffMisc + 32);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kFStages; ++i) {
      mbar_init(full_bar(i), 1);
      mbar_init(empty_bar(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), 128);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    *never = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_launch_dependents();
  griddep_wait();  // the operands come from the preceding kernels

  const WaitCtl ctl{status, abort_flag, kWaitLimitNs};
  const int p_tiles = (P + kFBM - 1) / kFBM, q_tiles = (Q + kFBN - 1) / kFBN;
  const int tiles = p_tiles * q_tiles, kblocks = (R + kFBK - 1) / kFBK;

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < tiles; tile += gridDim.x) {
        const int pt = tile % p_tiles, qt = tile / p_tiles;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kFStages;
          if (!mbar_wait(empty_bar(s), ((it / kFStages) & 1) ^ 1, ctl)) { ok = false; break; }
          mbar_arrive_expect_tx(full_bar(s), kFABytes + kFBBytes);
          tma_load_2d(sb + kFOffA + s * kFABytes, &tmap_a, kb * kFBK, pt * kFBM, full_bar(s));
          tma_load_2d(sb + kFOffB + s * kFBBytes, &tmap_b, kb * kFBK, qt * kFBN, full_bar(s));
        }
      }
      if (!ok) {
        const WaitCtl drain{nullptr, never, 100000000ull};
        for (int i = (it > kFStages ? it - kFStages : 0); i < it; ++i)
          mbar_wait(full_bar(i % kFStages), (i / kFStages) & 1, drain);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int it = 0, tc = 0;
      bool ok = true, issued = false;
      for (int tile = blockIdx.x; ok && tile < tiles; tile += gridDim.x, ++tc) {
        const int a = tc & 1;
        if (!mbar_wait(tempty_bar(a), ((tc >> 1) & 1) ^ 1, ctl)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + a * kFBN;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kFStages;
          if (!mbar_wait(full_bar(s), (it / kFStages) & 1, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = sw128_kmajor_desc(sb + kFOffA + s * kFABytes);
          const uint64_t bdesc = sw128_kmajor_desc(sb + kFOffB + s * kFBBytes);
#pragma unroll
          for (int k = 0; k < kFBK / 16; ++k) tc_mma_f16(d_tmem, adesc + 2 * k, bdesc + 2 * k, kFIdesc, (kb | k) != 0);
          issued = true;
          tc_commit(empty_bar(s));
        }
        if (ok) tc_commit(tfull_bar(a));
      }
      if (issued) {
        tc_commit(done_bar);
        const WaitCtl drain{nullptr, never, 100000000ull};
        mbar_wait(done_bar, 0, drain);
      }
    }
  } else if (warp >= 4) {
    const int q = warp & 3;
    const float al = alpha_ptr ? __fmul_rn(alpha, __ldg(alpha_ptr)) : alpha;
    int tc = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tc) {
      const int pt = tile % p_tiles, qt = tile / p_tiles;
      const int a = tc & 1;
      const bool got = mbar_wait(tfull_bar(a), (tc >> 1) & 1, ctl);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int p = pt * kFBM + q * 32 + lane;
#pragma unroll 1
      for (int c = 0; c < kFBN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * kFBN + c * 32, r);
        tmem_ld_wait();
        const int q0 = qt * kFBN + c * 32;
        if (p < P && q0 < Q) {
          TO* row = out + static_cast<size_t>(p) * Q;
          if (q0 + 32 <= Q && (Q % 8) == 0) {
            if constexpr (sizeof(TO) == 4) {
              float4* d = reinterpret_cast<float4*>(row + q0);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                d[i] = make_float4(__fmul_rn(__uint_as_float(r[4 * i]), al), __fmul_rn(__uint_as_float(r[4 * i + 1]), al),
                                   __fmul_rn(__uint_as_float(r[4 * i + 2]), al),
                                   __fmul_rn(__uint_as_float(r[4 * i + 3]), al));
            } else {
              uint32_t h[16];
#pragma unroll
              for (int i = 0; i < 16; ++i)
                h[i] = static_cast<uint32_t>(
                           __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(__uint_as_float(r[2 * i]), al)))) |
                       (static_cast<uint32_t>(__bfloat16_as_ushort(
                            __float2bfloat16_rn(__fmul_rn(__uint_as_float(r[2 * i + 1]), al))))
                        << 16);
              uint4* d = reinterpret_cast<uint4*>(row + q0);
#pragma unroll
              for (int i = 0; i < 4; ++i) d[i] = make_uint4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
            }
          } else {
            for (int i = 0; i < 32; ++i)
              if (q0 + i < Q) row[q0 + i] = static_cast<TO>(__fmul_rn(__uint_as_float(r[i]), al));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty_bar(a));
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

static bool map_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  EncodeTiledFn fn = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kFBK), box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// D[P][Q] = alpha (* *alpha_ptr) * A[P][R] . B[Q][R]^T; A, B bf16 row-major; out fp32 or bf16.
static cudaError_t launch_gemm_bf16(const __nv_bfloat16* A, const __nv_bfloat16* B, int P, int Q, int R, float alpha,
                                   const float* alpha_ptr, void* out, bool out_bf16, uint32_t* status,
                                   cudaStream_t stream) {
  CUtensorMap ta, tb;
  if (!map_bf16_2d(&ta, A, R, P, kFBM) || !map_bf16_2d(&tb, B, R, Q, kFBN)) return cudaErrorInvalidValue;
  static std::atomic<uint64_t> attr_done[2];  // per output type and device
  const cudaError_t e = once_per_device(attr_done[out_bf16 ? 1 : 0], [&] {
    return out_bf16 ? cudaFuncSetAttribute(gemm_bf16_kernel<__nv_bfloat16>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, kFSmem)
                    : cudaFuncSetAttribute(gemm_bf16_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kFSmem);
  });
  if (e != cudaSuccess) return e;
  const int tiles = ((P + kFBM - 1) / kFBM) * ((Q + kFBN - 1) / kFBN);
  const int grid = tiles < num_sms() ? tiles : num_sms();
  if (out_bf16)
    return launch(gemm_bf16_kernel<__nv_bfloat16>, dim3(grid), dim3(kFThreads), kFSmem, stream, true, ta, tb, P, Q,
                  R, alpha, alpha_ptr, static_cast<__nv_bfloat16*>(out), status);
  return launch(gemm_bf16_kernel<float>, dim3(grid), dim3(kFThreads), kFSmem, stream, true, ta, tb, P, Q, R, alpha,
                alpha_ptr, static_cast<float*>(out), status);
}

size_t ste_scratch_bytes(int M, int N, int K) {
  auto r256 = [](size_t v) { return (v + 255) / 256 * 256; };
  return r256(static_cast<size_t>(K) * N * 2) + r256(static_cast<size_t>(N) * M * 2) +
         r256(static_cast<size_t>(K) * M * 2);
}

cudaError_t launch_ste_backward(const uint8_t* packed, const float* gamma, int N, int K, const void* dy, const int8_t* xq,
                                const float* scale, int M, void* dx, bool dx_bf16, float* dw, uint8_t* scratch,
                                uint32_t* status, cudaStream_t stream) {
  auto r256 = [](size_t v) { return (v + 255) / 256 * 256; };
  __nv_bfloat16* tt = reinterpret_cast<__nv_bfloat16*>(scratch);
  __nv_bfloat16* dyt = reinterpret_cast<__nv_bfloat16*>(scratch + r256(static_cast<size_t>(K) * N * 2));
  __nv_bfloat16* xht = reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<uint8_t*>(dyt) +
                                                       r256(static_cast<size_t>(N) * M * 2));
  cudaError_t e = cudaSuccess;
  if (dx) {
    // dx[M][K] = gamma * dy[M][N] . (t^T)[K][N]^T
    e = launch(unpack_transpose_kernel, dim3((K + kTile - 1) / kTile, (N + kTile - 1) / kTile), dim3(256), 0, stream,
               true, reinterpret_cast<const uint32_t*>(packed), N, K, tt);
    if (e != cudaSuccess) return e;
    e = launch_gemm_bf16(static_cast<const __nv_bfloat16*>(dy), tt, M, K, N, 1.0f, gamma, dx, dx_bf16, status, stream);
    if (e != cudaSuccess) return e;
  }
  if (dw) {
    // dW[N][K] = (dy^T)[N][M] . (xhat^T)[K][M]^T
    e = launch(transpose_kernel<false>, dim3((N + kTile - 1) / kTile, (M + kTile - 1) / kTile), dim3(256), 0, stream,
               true, dy, static_cast<const float*>(nullptr), M, N, dyt);
    if (e != cudaSuccess) return e;
    e = launch(transpose_kernel<true>, dim3((K + kTile - 1) / kTile, (M + kTile - 1) / kTile), dim3(256), 0, stream,
               true, static_cast<const void*>(xq), scale, M, K, xht);
    if (e != cudaSuccess) return e;
    e = launch_gemm_bf16(dyt, xht, N, K, M, 1.0f, nullptr, dw, false, status, stream);
  }
  return e;
}

}  // namespace bl
