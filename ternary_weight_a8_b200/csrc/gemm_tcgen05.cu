// Prefill product (many tokens): int8 activations x unpacked ternary codes on
// the 5th-generation tensor cores (tcgen05.mma kind::i8, int32 accumulators
// in tensor memory), with the dequantisation fused into the epilogue.
//
// "BitNet's Real Bet: Designing the Whole Inference Stack", section "A
// low-bit model is a whole-stack design": packed weights move from HBM to
// shared memory, are unpacked there and meet the 8-bit activations.
// "A Two-Billion Ternary Bet": the pack-store-load-unpack-compute sequence.
//
// Tile: 128 tokens x 256 output rows x 128 inputs per k-block.  Warp roles
// in a persistent block of 16 warps (one block per SM):
//   warp 0      TMA producer of the activation tiles (128-byte swizzle);
//   warp 2      TMA producer of the packed weight tiles (256 rows x 32 bytes),
//               on a ring of its own that the unpack warps release as soon
//               as they hold the words in registers, so weight tiles are
//               requested well ahead of the tensor cores;
//   warp 1      tensor-memory owner and the single thread that issues the
//               4 tcgen05.mma (K = 32 each) per k-block;
//   warps 4-11  unpack: packed words -> one 16-byte chunk of codes
//               ((w >> 2j) & 0x03030303, j = 0..3) written at its 128-byte
//               swizzle position, then a proxy fence and an mbarrier arrive;
//   warps 12-15 epilogue: tcgen05.ld of the int32 accumulators, then
//               y = (acc - rowsum[m]) * (gamma / s[m]) stored as fp32 / bf16.
// Two accumulators (2 x 256 tensor-memory columns) let the epilogue of one
// tile overlap the main loop of the next.  Every mbarrier wait is bounded in
// time; a wait that runs out records the timeout in the workspace status
// word and the block winds down without touching global memory further.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace bl {

constexpr int kBM = 128, kBN = 256, kBK = 128;
constexpr int kAStages = 5, kPStages = 6, kUStages = 3;
constexpr int kABytes = kBM * kBK;       // 16 KB activation tile
constexpr int kBPBytes = kBN * kBK / 4;  // 8 KB packed weight tile
constexpr int kBUBytes = kBN * kBK;      // 32 KB unpacked code tile
constexpr int kGemmThreads = 512;
constexpr int kUnpackThreads = 256;  // warps 4-11
constexpr int kOffA = 0;
constexpr int kOffBU = kOffA + kAStages * kABytes;
constexpr int kOffBP = kOffBU + kUStages * kBUBytes;
constexpr int kOffBar = kOffBP + kPStages * kBPBytes;
constexpr int kNumBars = 2 * (kAStages + kPStages + kUStages) + 5;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory per block");
constexpr uint32_t kTmemCols = 512;

// Instruction descriptor: D s32, A s8, B s8, both K-major, N = 256, M = 128.
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((kBN >> 3) << 17) |
                            ((kBM >> 4) << 24);

template <typename TY>
__device__ __forceinline__ void store_row32(TY* __restrict__ y, int32_t* __restrict__ acc_out,
                                            size_t row_off, int n0, int N, const uint32_t (&r)[32],
                                            int rs, float gs) {
  int acc[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) acc[i] = static_cast<int>(r[i]) - rs;
  const bool full = (n0 + 32 <= N);
  if constexpr (sizeof(TY) == 2) {
    if (full && (N % 8) == 0) {
      uint32_t p[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const __nv_bfloat16 lo = __float2bfloat16_rn(__fmul_rn(static_cast<float>(acc[2 * i]), gs));
        const __nv_bfloat16 hi =
            __float2bfloat16_rn(__fmul_rn(static_cast<float>(acc[2 * i + 1]), gs));
        p[i] = static_cast<uint32_t>(__bfloat16_as_ushort(lo)) |
               (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
      }
      uint4* dst = reinterpret_cast<uint4*>(y + row_off + n0);
#pragma unroll
      for (int i = 0; i < 4; ++i) dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
    } else {
      for (int i = 0; i < 32; ++i)
        if (n0 + i < N) y[row_off + n0 + i] = __float2bfloat16_rn(__fmul_rn(static_cast<float>(acc[i]), gs));
    }
  } else {
    if (full && (N % 4) == 0) {
      float4* dst = reinterpret_cast<float4*>(y + row_off + n0);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        dst[i] = make_float4(__fmul_rn(static_cast<float>(acc[4 * i]), gs),
                             __fmul_rn(static_cast<float>(acc[4 * i + 1]), gs),
                             __fmul_rn(static_cast<float>(acc[4 * i + 2]), gs),
                             __fmul_rn(static_cast<float>(acc[4 * i + 3]), gs));
    } else {
      for (int i = 0; i < 32; ++i)
        if (n0 + i < N) y[row_off + n0 + i] = __fmul_rn(static_cast<float>(acc[i]), gs);
    }
  }
  if (acc_out) {
    if (full && (N % 4) == 0) {
      int4* dst = reinterpret_cast<int4*>(acc_out + row_off + n0);
#pragma unroll
      for (int i = 0; i < 8; ++i) dst[i] = make_int4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
    } else {
      for (int i = 0; i < 32; ++i)
        if (n0 + i < N) acc_out[row_off + n0 + i] = acc[i];
    }
  }
}

template <typename TY>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(
    const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
    const float* __restrict__ gamma_ptr, int N, int K, int M, const float* __restrict__ scale,
    const int32_t* __restrict__ rowsum, TY* __restrict__ y, int32_t* __restrict__ acc_out,
    uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  constexpr int kBarP = 2 * kAStages, kBarU = kBarP + 2 * kPStages, kBarT = kBarU + 2 * kUStages;
  auto afull_bar = [&](int i) { return sb + kOffBar + 8 * i; };
  auto aempty_bar = [&](int i) { return sb + kOffBar + 8 * (kAStages + i); };
  auto pfull_bar = [&](int i) { return sb + kOffBar + 8 * (kBarP + i); };
  auto pempty_bar = [&](int i) { return sb + kOffBar + 8 * (kBarP + kPStages + i); };
  auto ufull_bar = [&](int i) { return sb + kOffBar + 8 * (kBarU + i); };
  auto uempty_bar = [&](int i) { return sb + kOffBar + 8 * (kBarU + kUStages + i); };
  auto tfull_bar = [&](int i) { return sb + kOffBar + 8 * (kBarT + i); };
  auto tempty_bar = [&](int i) { return sb + kOffBar + 8 * (kBarT + 2 + i); };
  const uint32_t done_bar = sb + kOffBar + 8 * (kNumBars - 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 16);
  volatile int* never = reinterpret_cast<volatile int*>(smem + kOffMisc + 32);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kAStages; ++i) {
      mbar_init(afull_bar(i), 1);
      mbar_init(aempty_bar(i), 1);
    }
    for (int i = 0; i < kPStages; ++i) {
      mbar_init(pfull_bar(i), 1);
      mbar_init(pempty_bar(i), kUnpackThreads);
    }
    for (int i = 0; i < kUStages; ++i) {
      mbar_init(ufull_bar(i), kUnpackThreads);
      mbar_init(uempty_bar(i), 1);
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
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmap_a);
  if (warp == 2 && lane == 0) tma_prefetch_desc(&tmap_b);
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  griddep_launch_dependents();
  griddep_wait();  // activations, scales and row sums come from the preceding kernel

  const WaitCtl ctl{status, abort_flag, kWaitLimitNs};
  const int m_tiles = (M + kBM - 1) / kBM;
  const int n_tiles = (N + kBN - 1) / kBN;
  const int tiles = m_tiles * n_tiles;
  const int kblocks = (K + kBK - 1) / kBK;

  if (warp == 0 || warp == 2) {
    if (lane == 0) {
      // warp 0: activation tiles; warp 2: packed weight tiles.
      const bool is_a = (warp == 0);
      const int nst = is_a ? kAStages : kPStages;
      int it = 0, s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < tiles; tile += gridDim.x) {
        const int mt = tile % m_tiles, nt = tile / m_tiles;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const uint32_t full = is_a ? afull_bar(s) : pfull_bar(s);
          if (!mbar_wait(is_a ? aempty_bar(s) : pempty_bar(s), ph ^ 1, ctl)) { ok = false; break; }
          if (is_a) {
            mbar_arrive_expect_tx(full, kABytes);
            tma_load_2d(sb + kOffA + s * kABytes, &tmap_a, kb * kBK, mt * kBM, full);
          } else {
            mbar_arrive_expect_tx(full, kBPBytes);
            tma_load_2d(sb + kOffBP + s * kBPBytes, &tmap_b, kb * (kBK / 4), nt * kBN, full);
          }
          if (++s == nst) { s = 0; ph ^= 1; }
        }
      }
      if (!ok) {
        // Let copies already in flight land before the block's shared memory goes away.
        const WaitCtl drain{nullptr, never, 100000000ull};
        for (int i = (it > nst ? it - nst : 0); i < it; ++i)
          mbar_wait(is_a ? afull_bar(i % nst) : pfull_bar(i % nst), (i / nst) & 1, drain);
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
        const uint32_t d_tmem = tmem_base + a * kBN;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kAStages, u = it % kUStages;
          if (!mbar_wait(afull_bar(s), (it / kAStages) & 1, ctl)) { ok = false; break; }
          if (!mbar_wait(ufull_bar(u), (it / kUStages) & 1, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = sw128_kmajor_desc(sb + kOffA + s * kABytes);
          const uint64_t bdesc = sw128_kmajor_desc(sb + kOffBU + u * kBUBytes);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k) {
            tc_mma_i8(d_tmem, adesc + 2 * k, bdesc + 2 * k, kIdesc, (kb | k) != 0);
          }
          issued = true;
          tc_commit(aempty_bar(s));
          tc_commit(uempty_bar(u));
        }
        if (ok) tc_commit(tfull_bar(a));
      }
      if (issued) {
        // Every MMA must be finished before tensor memory is released.
        tc_commit(done_bar);
        const WaitCtl drain{nullptr, never, 100000000ull};
        mbar_wait(done_bar, 0, drain);
      }
    }
  } else if (warp >= 4 && warp < 12) {
    const int ut = threadIdx.x - 128;
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < tiles; tile += gridDim.x) {
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int s = it % kPStages, u = it % kUStages;
        if (!mbar_wait(pfull_bar(s), (it / kPStages) & 1, ctl)) { ok = false; break; }
        constexpr int kPer = kBPBytes / 16 / kUnpackThreads;  // packed uint4 per thread
        const uint4* bp = reinterpret_cast<const uint4*>(smem + kOffBP + s * kBPBytes);
        uint4 codes[kPer][4];
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
          const uint4 v = bp[ut + j * kUnpackThreads];
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t w = w4[i];
            codes[j][i] = make_uint4(w & 0x03030303u, (w >> 2) & 0x03030303u, (w >> 4) & 0x03030303u,
                                     (w >> 6) & 0x03030303u);
          }
        }
        if (!mbar_wait(uempty_bar(u), ((it / kUStages) & 1) ^ 1, ctl)) { ok = false; break; }
        uint8_t* bu = smem + kOffBU + u * kBUBytes;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
          const int q = ut + j * kUnpackThreads;
          const int r = q >> 1;              // weight row in the tile (32 packed bytes per row)
          const int c0 = (q & 1) * 4;        // first 16-byte chunk (= packed word) of this uint4
          uint8_t* rowp = bu + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            *reinterpret_cast<uint4*>(rowp + (((c0 + i) ^ (r & 7)) << 4)) = codes[j][i];
        }
        // The stores above consumed every packed word, so no read of the packed
        // slot can still be in flight: hand it back to its producer.
        mbar_arrive(pempty_bar(s));
        fence_proxy_async_smem();
        mbar_arrive(ufull_bar(u));
      }
    }
  } else if (warp >= 12) {
    const int q = warp & 3;  // tensor-memory lane quarter this warp may read
    const float gamma = __ldg(gamma_ptr);
    int tc = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tc) {
      const int mt = tile % m_tiles, nt = tile / m_tiles;
      const int a = tc & 1;
      // tcgen05.ld below is warp-collective: take the wait's outcome warp-wide.
      const bool got = mbar_wait(tfull_bar(a), (tc >> 1) & 1, ctl);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int m = mt * kBM + q * 32 + lane;
      const bool mvalid = m < M;
      float gs = 0.0f;
      int rs = 0;
      if (mvalid) {
        gs = __fdiv_rn(gamma, __ldg(scale + m));
        rs = __ldg(rowsum + m);
      }
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * kBN + c * 32, r);
        tmem_ld_wait();
        const int n0 = nt * kBN + c * 32;
        if (mvalid && n0 < N) store_row32<TY>(y, acc_out, static_cast<size_t>(m) * N, n0, N, r, rs, gs);
      }
      tc_fence_before();
      mbar_arrive(tempty_bar(a));
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launch
// ---------------------------------------------------------------------------
void* tensor_map_encoder() {
  static void* fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = p;
    }
  }
  return fn;
}

static bool make_map_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                        uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz, uint64_t pitch = 0) {
  EncodeTiledFn fn = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch ? pitch : inner};  // bytes (uint8 elements)
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename TY>
static cudaError_t launch_gemm_t(const ProductArgs& a, cudaStream_t stream, bool pdl) {
  CUtensorMap ta, tb;
  if (!make_map_2d(&ta, a.xq, static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.M), kBK, kBM,
                   CU_TENSOR_MAP_SWIZZLE_128B, static_cast<uint64_t>(a.ldx)) ||
      !make_map_2d(&tb, a.packed, static_cast<uint64_t>(a.K / 4), static_cast<uint64_t>(a.N),
                   kBK / 4, kBN, CU_TENSOR_MAP_SWIZZLE_NONE)) {
    return cudaErrorInvalidValue;
  }
  static bool attr_set = false;  // per template instance; the attribute is per function
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<TY>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int tiles = ((a.M + kBM - 1) / kBM) * ((a.N + kBN - 1) / kBN);
  const int grid = tiles < num_sms() ? tiles : num_sms();
  return launch(gemm_kernel<TY>, dim3(grid), dim3(kGemmThreads), kSmemBytes, stream, pdl, ta, tb,
                a.gamma, a.N, a.K, a.M, a.scale, a.rowsum, static_cast<TY*>(a.y), a.acc_out,
                a.status);
}

cudaError_t launch_gemm(const ProductArgs& a, cudaStream_t stream, bool pdl) {
  if (a.M <= 0) return cudaSuccess;
  return a.y_type == kOutBF16 ? launch_gemm_t<__nv_bfloat16>(a, stream, pdl)
                              : launch_gemm_t<float>(a, stream, pdl);
}

}  // namespace bl
