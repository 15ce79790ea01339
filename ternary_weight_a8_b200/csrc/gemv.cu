// Decode product (M <= 16 tokens): packed ternary weights x int8 activations,
// int32 accumulation, fused dequantisation.
//
// "BitNet's Real Bet: Designing the Whole Inference Stack", section "A
// low-bit model is a whole-stack design": the GPU path moves packed weights
// from HBM to shared memory, unpacks them and computes with the 8-bit
// activations.  "BitNet b1.58 and the 1-Bit AI Architecture Revolution",
// section "The Energy Revolution": the product is integer additions; here
// they run on the tensor cores' int8 path (mma.sync m16n8k32, u8 x s8 -> s32).
//
// Decode streams the weights once, so the kernel is built around the stream:
//  * A block owns 128 output rows (8 consumer warps x 16 rows) and a range of
//    K.  One producer thread streams the block's packed weights with TMA in
//    stages of 128 rows x 128 bytes (512 inputs), written in the 128-byte
//    swizzle so that each lane's 16-byte reads are free of bank conflicts,
//    through a ring of mbarrier-tracked buffers.  Weight loads need nothing
//    from the preceding kernel, so they start before the grid dependency
//    wait (programmatic dependent launch) and overlap the activation
//    quantisation.
//  * The block's int8 activations are copied once into shared memory, with
//    the 16-byte chunks of every 128-byte block rotated by twice the block
//    index, which makes the activation fragment reads conflict-free too.
//  * Each lane takes 16-byte chunks 2t and 2t+1 of rows g and g+8 of its
//    warp's 16 rows into registers and releases the stage at once.
//    Unpacking is one AND per four weights: mask 0x03030303 << 2j keeps the
//    codes of elements 4j..4j+3 of a word in place (scaled by 4^j); four
//    accumulator sets, one per j, are shifted back and added at the end,
//    which is exact because each set is a multiple of 4^j.  The k order
//    inside an mma is free as long as both operands agree, so lane (g, t)
//    feeds its own words to the A fragment and the matching activation bytes
//    to the B fragment.
//  * Stored codes are c = t + 1, so y = (sum c*q - rowsum(q)) * gamma / s.
//    When K is split over blocks, each block stores its partial sums in its
//    own workspace slot; the last block of a row block (an atomic counter
//    tells) adds the slots in split order, applies the epilogue and resets
//    the counter for the next call.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace bl {

constexpr int kGvWarps = 8;
constexpr int kGvRows = 16 * kGvWarps;            // 128 rows per block
constexpr int kGvStageK = 512;                    // inputs per stage
constexpr int kGvStageBytes = kGvRows * 128;      // 16 KB of packed weights
constexpr int kGvThreads = 32 * (kGvWarps + 1);   // + one producer warp
constexpr int kGvConsumers = 32 * kGvWarps;
constexpr int kGvXBudget = 64 * 1024;             // activation bytes staged per block

__device__ __forceinline__ void mma_u8s8_16x8x32(int (&d)[4], uint32_t a0, uint32_t a1,
                                                 uint32_t a2, uint32_t a3, uint32_t b0,
                                                 uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t u4_get(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kGvConsumers) : "memory");
}

// Byte offset of activation chunk (16 bytes) `c` of a staged token row.
__device__ __forceinline__ int x_chunk_off(int c) {
  const int blk = c >> 3, ci = c & 7;
  return blk * 128 + (((ci + 2 * (blk & 3)) & 7) << 4);
}

template <int TG, typename TY>
__global__ void __launch_bounds__(kGvThreads) gemv_kernel(
    const __grid_constant__ CUtensorMap tmap_w, const float* __restrict__ gamma_ptr, int N, int K,
    int M, const int8_t* __restrict__ xq, const float* __restrict__ scale,
    const int32_t* __restrict__ rowsum, TY* __restrict__ y, int32_t* __restrict__ acc_out,
    int32_t* __restrict__ acc_ws, uint32_t* __restrict__ counters, int splits, int st_per_split,
    int nring, int x_pitch, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t ring = sb;
  const uint32_t xs = sb + nring * kGvStageBytes;
  const int x_bytes = ((M * x_pitch + 127) / 128) * 128;
  uint8_t* misc = smem + nring * kGvStageBytes + x_bytes;
  const uint32_t bar0 = smem_u32(misc);  // full[nring], empty[nring]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 16 * nring);
  volatile int* never = abort_flag + 1;
  volatile int* last_flag = abort_flag + 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rb = blockIdx.x / splits, ks = blockIdx.x % splits;
  const int n_st = (K + kGvStageK - 1) / kGvStageK;
  const int st0 = ks * st_per_split;
  const int st1 = min(n_st, st0 + st_per_split);
  const int nst = st1 - st0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < nring; ++i) {
      mbar_init(bar0 + 8 * i, 1);
      mbar_init(bar0 + 8 * (nring + i), kGvWarps);
    }
    *abort_flag = 0;
    *never = 0;
    fence_barrier_init();
  }
  __syncthreads();
  griddep_launch_dependents();
  const WaitCtl ctl{status, abort_flag, kWaitLimitNs};

  if (warp == kGvWarps) {
    // Producer: weights only, so no grid-dependency wait is needed.
    if (lane == 0) {
      tma_prefetch_desc(&tmap_w);
      int i = 0;
      for (; i < nst; ++i) {
        const int slot = i % nring;
        if (!mbar_wait(bar0 + 8 * (nring + slot), ((i / nring) & 1) ^ 1, ctl)) break;
        mbar_arrive_expect_tx(bar0 + 8 * slot, kGvStageBytes);
        tma_load_2d(ring + slot * kGvStageBytes, &tmap_w, (st0 + i) * 128, rb * kGvRows, bar0 + 8 * slot);
      }
      if (i < nst) {  // gave up: let copies in flight land before shared memory is released
        const WaitCtl drain{nullptr, never, 100000000ull};
        for (int j = (i > nring ? i - nring : 0); j < i; ++j)
          mbar_wait(bar0 + 8 * (j % nring), (j / nring) & 1, drain);
      }
    }
    return;
  }

  // ---- consumers ----
  griddep_wait();  // activations, scales and row sums come from the preceding kernel
  const int k0 = st0 * kGvStageK;
  const int kr = min(K, st1 * kGvStageK) - k0;  // multiple of 64
  {
    const int chunks = kr >> 4;
    for (int idx = threadIdx.x; idx < M * chunks; idx += kGvConsumers) {
      const int m = idx / chunks, c = idx - m * chunks;
      const uint4 v = __ldcg(reinterpret_cast<const uint4*>(xq + static_cast<size_t>(m) * K + k0) + c);
      asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(xs + m * x_pitch + x_chunk_off(c)),
                   "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                   : "memory");
    }
  }
  consumer_sync();

  const int g = lane >> 2, t = lane & 3;
  const int r_lo = warp * 16 + g;  // rows of this lane within the block (and + 8)
  int d[TG][4][4];
#pragma unroll
  for (int tg = 0; tg < TG; ++tg)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) d[tg][j][c] = 0;

  bool ok = true;
  for (int i = 0; i < nst; ++i) {
    const int slot = i % nring;
    const bool got = mbar_wait(bar0 + 8 * slot, (i / nring) & 1, ctl);
    if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
    const uint32_t wt = ring + slot * kGvStageBytes;
    // 128-byte swizzle: chunk c of row r sits at chunk position c ^ (r & 7); r & 7 == g here.
    const uint4 wl0 = lds128(wt + r_lo * 128 + (((2 * t) ^ g) << 4));
    const uint4 wl1 = lds128(wt + r_lo * 128 + (((2 * t + 1) ^ g) << 4));
    const uint4 wh0 = lds128(wt + (r_lo + 8) * 128 + (((2 * t) ^ g) << 4));
    const uint4 wh1 = lds128(wt + (r_lo + 8) * 128 + (((2 * t + 1) ^ g) << 4));
    __syncwarp();
    if (lane == 0) mbar_arrive(bar0 + 8 * (nring + slot));  // weights are in registers

    const int qblk = i * 4 + t;  // this lane's 128-input block of the staged activations
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 wl = h ? wl1 : wl0, wh = h ? wh1 : wh0;
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        const int c0 = 4 * h + 2 * p;  // activation chunks c0, c0+1 of block qblk
        uint4 xa[TG], xb[TG];
#pragma unroll
        for (int tg = 0; tg < TG; ++tg) {
          const int m = tg * 8 + g;
          if (m < M) {
            const uint32_t row = xs + m * x_pitch + qblk * 128;
            xa[tg] = lds128(row + (((c0 + 2 * t) & 7) << 4));
            xb[tg] = lds128(row + (((c0 + 1 + 2 * t) & 7) << 4));
          } else {
            xa[tg] = make_uint4(0, 0, 0, 0);
            xb[tg] = make_uint4(0, 0, 0, 0);
          }
        }
        const uint32_t lo0 = u4_get(wl, 2 * p), lo1 = u4_get(wl, 2 * p + 1);
        const uint32_t hi0 = u4_get(wh, 2 * p), hi1 = u4_get(wh, 2 * p + 1);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t mask = 0x03030303u << (2 * j);
          const uint32_t a0 = lo0 & mask, a1 = hi0 & mask, a2 = lo1 & mask, a3 = hi1 & mask;
#pragma unroll
          for (int tg = 0; tg < TG; ++tg)
            mma_u8s8_16x8x32(d[tg][j], a0, a1, a2, a3, u4_get(xa[tg], j), u4_get(xb[tg], j));
        }
      }
    }
  }
  // Every consumer warp gets here (bounded waits); leave together if any wait ran out.
  consumer_sync();
  if (*abort_flag || !ok) return;  // the status word records it; no output is written

  // ---- epilogue ----
  int acc[TG][4];
#pragma unroll
  for (int tg = 0; tg < TG; ++tg)
#pragma unroll
    for (int c = 0; c < 4; ++c)
      acc[tg][c] = d[tg][0][c] + (d[tg][1][c] >> 2) + (d[tg][2][c] >> 4) + (d[tg][3][c] >> 6);

  const float gamma = __ldg(gamma_ptr);
  const int n_base = rb * kGvRows;
  if (splits == 1) {
#pragma unroll
    for (int tg = 0; tg < TG; ++tg)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int n = n_base + r_lo + ((c & 2) ? 8 : 0);
        const int m = tg * 8 + 2 * t + (c & 1);
        if (n < N && m < M) {
          const int a = acc[tg][c] - __ldg(rowsum + m);
          const float v = __fmul_rn(static_cast<float>(a), __fdiv_rn(gamma, __ldg(scale + m)));
          const size_t o = static_cast<size_t>(m) * N + n;
          if constexpr (sizeof(TY) == 4) y[o] = v; else y[o] = __float2bfloat16_rn(v);
          if (acc_out) acc_out[o] = a;
        }
      }
    return;
  }

  // Split K: each block stores its partial sums in its own slot; the block that
  // completes the row block adds the slots in split order (deterministic) and
  // finishes the row block.  Only the per-row-block counter is shared, and the
  // finishing block resets it.
  int32_t* my_slot = acc_ws + (static_cast<size_t>(rb) * splits + ks) * M * kGvRows;
#pragma unroll
  for (int tg = 0; tg < TG; ++tg)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int r = r_lo + ((c & 2) ? 8 : 0);
      const int m = tg * 8 + 2 * t + (c & 1);
      if (m < M) __stcg(my_slot + m * kGvRows + r, acc[tg][c]);
    }
  __threadfence();
  consumer_sync();
  if (threadIdx.x == 0) {
    const uint32_t prev = atomicAdd(counters + rb, 1u);
    *last_flag = (prev + 1 == static_cast<uint32_t>(splits)) ? 1 : 0;
  }
  consumer_sync();
  if (!*last_flag) return;
  __threadfence();
  const int rows = min(kGvRows, N - n_base);
  const int32_t* slots = acc_ws + static_cast<size_t>(rb) * splits * M * kGvRows;
  for (int idx = threadIdx.x; idx < rows * M; idx += kGvConsumers) {
    const int m = idx / rows, r = idx - m * rows;
    int sum = 0;
    for (int s = 0; s < splits; ++s) sum += __ldcg(slots + (static_cast<size_t>(s) * M + m) * kGvRows + r);
    const int a = sum - __ldg(rowsum + m);
    const size_t o = static_cast<size_t>(m) * N + n_base + r;
    const float v = __fmul_rn(static_cast<float>(a), __fdiv_rn(gamma, __ldg(scale + m)));
    if constexpr (sizeof(TY) == 4) y[o] = v; else y[o] = __float2bfloat16_rn(v);
    if (acc_out) acc_out[o] = a;
  }
  if (threadIdx.x == 0) counters[rb] = 0;
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

static GemvPlan plan_gemv_budget(int M, int N, int K, int x_budget) {
  const int sms = num_sms();
  GemvPlan best{};
  double best_cost = 1e30;
  const int n_rb = (N + kGvRows - 1) / kGvRows;
  const int n_st = (K + kGvStageK - 1) / kGvStageK;
  for (int s = 1; s <= n_st && s <= kGemvMaxSplits; ++s) {
    const int spc = (n_st + s - 1) / s;
    const int s_eff = (n_st + spc - 1) / spc;
    if (s_eff != s) continue;
    const int x_pitch = ((spc * kGvStageK + 127) / 128) * 128 + 16;
    if (M * x_pitch > x_budget) continue;
    for (int ring : {2, 3, 4, 6}) {
      if (ring > spc && ring != 2) continue;
      const int r_eff = ring < spc ? ring : spc;
      const int smem = r_eff * kGvStageBytes + ((M * x_pitch + 127) / 128) * 128 + 16 * r_eff + 64 + 1024;
      if (smem > 227 * 1024) continue;
      int occ = (227 * 1024) / smem;
      if (occ > 2048 / kGvThreads) occ = 2048 / kGvThreads;
      const long long ctas = static_cast<long long>(n_rb) * s;
      const long long slots = static_cast<long long>(sms) * occ;
      const long long per_sm = (ctas + sms - 1) / sms;
      const long long waves = (ctas + slots - 1) / slots;
      const int in_flight = static_cast<int>(per_sm < occ ? per_sm : occ) * r_eff;
      // Stages the busiest SM streams, a little extra per split for the partial sums,
      // a penalty for a short tail wave and for too few stages in flight per SM.
      double cost = static_cast<double>(per_sm * spc) * (1.0 + 0.04 * (s - 1));
      if (waves > 1 && waves < 4) cost *= 1.1;
      if (in_flight < 3 && spc >= 3) cost *= 1.25;
      if (cost < best_cost - 1e-9) {
        best_cost = cost;
        best = GemvPlan{n_rb, n_st, s, spc, r_eff, x_pitch, smem};
      }
    }
  }
  return best;
}

GemvPlan plan_gemv(int M, int N, int K) {
  GemvPlan p = plan_gemv_budget(M, N, K, kGvXBudget);
  if (p.splits == 0) p = plan_gemv_budget(M, N, K, 160 * 1024);
  return p;  // splits == 0: the activations do not fit; the caller uses the GEMM
}

template <int TG, typename TY>
static cudaError_t launch_gemv_t(const ProductArgs& a, const GemvPlan& p, cudaStream_t stream, bool pdl) {
  EncodeTiledFn enc = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tw;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K / 4), static_cast<cuuint64_t>(a.N)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K / 4)};
  const cuuint32_t box[2] = {128, kGvRows};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.packed), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
    return cudaErrorInvalidValue;
  }
  static int max_smem_set = 0;
  if (p.smem > 48 * 1024 && p.smem > max_smem_set) {
    cudaError_t e = cudaFuncSetAttribute(gemv_kernel<TG, TY>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         227 * 1024);
    if (e != cudaSuccess) return e;
    max_smem_set = 227 * 1024;
  }
  return launch(gemv_kernel<TG, TY>, dim3(p.n_rb * p.splits), dim3(kGvThreads), static_cast<size_t>(p.smem),
                stream, pdl, tw, a.gamma, a.N, a.K, a.M, a.xq, a.scale, a.rowsum, static_cast<TY*>(a.y),
                a.acc_out, a.acc_ws, a.counters, p.splits, p.st_per_split, p.nring, p.x_pitch, a.status);
}

cudaError_t launch_gemv(const ProductArgs& a, cudaStream_t stream, bool pdl) {
  const GemvPlan p = plan_gemv(a.M, a.N, a.K);
  if (p.splits == 0) return cudaErrorInvalidConfiguration;
  if (p.splits > 1 && (a.acc_ws == nullptr || a.counters == nullptr)) return cudaErrorInvalidValue;
  if (a.M <= 8) {
    return a.y_type == kOutBF16 ? launch_gemv_t<1, __nv_bfloat16>(a, p, stream, pdl)
                                : launch_gemv_t<1, float>(a, p, stream, pdl);
  }
  return a.y_type == kOutBF16 ? launch_gemv_t<2, __nv_bfloat16>(a, p, stream, pdl)
                              : launch_gemv_t<2, float>(a, p, stream, pdl);
}

}  // namespace bl
