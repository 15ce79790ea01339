// Decode product (M <= 16 tokens): packed ternary weights x int8 activations,
// int32 accumulation, fused dequantisation.
//
// "BitNet's Real Bet: Designing the Whole Inference Stack", section "A
// low-bit model is a whole-stack design": the GPU path moves packed weights
// from HBM to shared memory, unpacks them and computes with the per-token
// 8-bit activations.  "BitNet b1.58 and the 1-Bit AI Architecture
// Revolution", section "The Energy Revolution": the product is integer
// additions; here they run on the tensor cores' int8 path (mma.sync
// m16n8k32, u8 x s8 -> s32).
//
// Decode streams the weights once, so the kernel is built around the stream:
//  * A block owns 128 output rows (8 consumer warps x 16 rows) and a range of
//    K.  One producer thread streams the block's packed weights with TMA in
//    stages of 128 rows x 128 bytes (512 inputs), in the 128-byte swizzle so
//    that the lanes' 16-byte reads are free of bank conflicts, through a
//    ring of mbarrier-tracked buffers.  The weights need nothing from the
//    preceding kernel, so their loads start before the grid-dependency wait
//    (programmatic dependent launch).
//  * The block's activations are staged once in shared memory as int8, the
//    16-byte chunks of every 128-byte block rotated by twice the block index
//    so that fragment reads are conflict-free.  When the activations are
//    small the block quantises them itself (per-token absmax over all of K,
//    then its own K range), which saves a launch and a round trip through
//    HBM; otherwise it copies codes written by the quantisation kernel.
//  * Each lane takes 16-byte chunks 2t and 2t+1 of rows g and g+8 of its
//    warp's 16 rows into registers and releases the stage at once.
//    Unpacking is one AND per four weights: mask 0x03030303 << 2j keeps the
//    codes of elements 4j..4j+3 of a word in place (scaled by 4^j); four
//    accumulator sets, one per j, are shifted back and added at the end,
//    exact because each set is a multiple of 4^j.  The k order inside an mma
//    is free as long as both operands agree, so lane (g, t) feeds its own
//    words to the A fragment and the matching activation bytes to B.
//  * Stored codes are c = t + 1, so each block subtracts the sum of its own
//    activation codes: sum_range (c - 1) q = sum_range t q.
//  * Two ways to cover the matrix, chosen by a host planner from a model of
//    the bytes each SM keeps in flight: when there are enough row blocks,
//    persistent blocks each take every gridDim-th row block over all of K,
//    staging the activations once and streaming weights across row blocks
//    without draining the ring; otherwise K is split, the blocks of one row
//    block form a thread block cluster, add their partial sums through
//    distributed shared memory and each finish a slice of the rows.
//    Either way y = acc * (gamma / s).
//  * The kernel is specialised on the number of token slots (1, 2, 4, 8 or
//    16), so a one-token decode does no work for absent tokens.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdlib.h>

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
constexpr int kGvFuseLimit = 16 * 1024;           // M*K up to which blocks quantise themselves

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

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__device__ __forceinline__ uint32_t u4_get(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kGvConsumers) : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

__device__ __forceinline__ int ld_cluster_s32(uint32_t local_addr, uint32_t rank) {
  uint32_t remote;
  int v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(remote) : "memory");
  return v;
}

// Byte offset of activation chunk (16 bytes) `c` of a staged token row.
__device__ __forceinline__ int x_chunk_off(int c) {
  const int blk = c >> 3, ci = c & 7;
  return blk * 128 + (((ci + 2 * (blk & 3)) & 7) << 4);
}

// Sum of the 16 signed bytes of a chunk.
__device__ __forceinline__ int byte_sum16(const uint4& v) {
  int s = __dp4a(static_cast<int>(v.x), 0x01010101, 0);
  s = __dp4a(static_cast<int>(v.y), 0x01010101, s);
  s = __dp4a(static_cast<int>(v.z), 0x01010101, s);
  return __dp4a(static_cast<int>(v.w), 0x01010101, s);
}

// 8 activations as fp32 (bf16 -> fp32 is exact).
__device__ __forceinline__ void load8f(const float* p, float (&f)[8]) {
  const float4 a = __ldcg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldcg(reinterpret_cast<const float4*>(p) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void load8f(const __nv_bfloat16* p, float (&f)[8]) {
  const uint4 u = __ldcg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

template <int TT>
__device__ __forceinline__ void warp_sum_tokens(int (&v)[TT]) {
#pragma unroll
  for (int m = 0; m < TT; ++m)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v[m] += __shfl_xor_sync(0xffffffffu, v[m], o);
}

template <int TT, typename TY, typename TX>
__global__ void __launch_bounds__(kGvThreads, 1) gemv_kernel(
    const __grid_constant__ CUtensorMap tmap_w, const float* __restrict__ gamma_ptr, int N, int K,
    int M, const TX* __restrict__ x, const float* __restrict__ scale, TY* __restrict__ y,
    int32_t* __restrict__ acc_out, int splits, int st_per_split, int nring, int x_pitch,
    uint32_t* status) {
  constexpr int TG = (TT + 7) / 8;          // mma token groups of 8
  constexpr bool kFused = sizeof(TX) != 1;  // activations arrive unquantised
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t ring = sb;
  const int x_bytes = ((M * x_pitch + 127) / 128) * 128;
  const uint32_t xs = sb + nring * kGvStageBytes;
  uint8_t* misc = smem + nring * kGvStageBytes + x_bytes;
  int* red_buf = reinterpret_cast<int*>(misc);                       // [128 rows][TT] partial sums
  float* s_tok = reinterpret_cast<float*>(misc + kGvRows * TT * 4);  // [TT] token scales
  int* rs_tok = reinterpret_cast<int*>(s_tok + TT);                  // [TT] range code sums
  int* wred = rs_tok + TT;                                           // [kGvWarps][TT] reductions
  const uint32_t bar0 = smem_u32(wred + kGvWarps * TT);              // full[nring], empty[nring]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(wred + kGvWarps * TT + 4 * nring);
  volatile int* never = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_rb = (N + kGvRows - 1) / kGvRows;
  const bool clustered = splits > 1;
  // Row blocks of this block: one per cluster when K is split, else every gridDim-th.
  const int rb0 = clustered ? static_cast<int>(blockIdx.x) / splits : static_cast<int>(blockIdx.x);
  const int rb_step = clustered ? n_rb : static_cast<int>(gridDim.x);
  const int n_my_rb = rb0 < n_rb ? (n_rb - 1 - rb0) / rb_step + 1 : 0;
  const int ks = clustered ? static_cast<int>(cluster_rank()) : 0;
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

  int acc[TG][4];
  const int g = lane >> 2, t = lane & 3;
  const int r_lo = warp * 16 + g;  // rows of this lane within the block (and + 8)
  bool ok = true;

  if (warp == kGvWarps) {
    // Producer: weights only, so no grid-dependency wait is needed.
    if (lane == 0) {
      tma_prefetch_desc(&tmap_w);
      const int total = n_my_rb * nst;  // (row block, stage) items, streamed without a break
      int i = 0;
      for (; i < total; ++i) {
        const int slot = i % nring;
        const int rb = rb0 + (i / nst) * rb_step, st = st0 + i % nst;
        if (!mbar_wait(bar0 + 8 * (nring + slot), ((i / nring) & 1) ^ 1, ctl)) break;
        mbar_arrive_expect_tx(bar0 + 8 * slot, kGvStageBytes);
        tma_load_2d(ring + slot * kGvStageBytes, &tmap_w, st * 128, rb * kGvRows, bar0 + 8 * slot);
      }
      if (i < total) {  // gave up: let copies in flight land before shared memory is released
        const WaitCtl drain{nullptr, never, 100000000ull};
        for (int j = (i > nring ? i - nring : 0); j < i; ++j)
          mbar_wait(bar0 + 8 * (j % nring), (j / nring) & 1, drain);
      }
    }
    __syncwarp();
    if (!clustered) return;
  } else {
    // ---- consumers: stage this block's activations ----
    griddep_wait();  // the activations may be the preceding kernel's output
    const int tid = threadIdx.x;
    const int k0 = st0 * kGvStageK;
    const int kr = min(K, st1 * kGvStageK) - k0;  // multiple of 64
    const int chunks = kr >> 4;                   // 16-input chunks of this block's range
    int rs[TT];
#pragma unroll
    for (int m = 0; m < TT; ++m) rs[m] = 0;
    if constexpr (kFused) {
      // Per-token absmax over all of K, then s = 127 / max(amax, 1e-5).
      float am[TT];
#pragma unroll
      for (int m = 0; m < TT; ++m) {
        am[m] = 0.0f;
        if (m < M) {
          for (int v = tid; v < K / 8; v += kGvConsumers) {
            float f[8];
            load8f(x + static_cast<size_t>(m) * K + v * 8, f);
#pragma unroll
            for (int e = 0; e < 8; ++e) am[m] = fmaxf(am[m], fabsf(f[e]));
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) am[m] = fmaxf(am[m], __shfl_xor_sync(0xffffffffu, am[m], o));
      }
      if (lane == 0) {
#pragma unroll
        for (int m = 0; m < TT; ++m) reinterpret_cast<float*>(wred)[warp * TT + m] = am[m];
      }
      consumer_sync();
      if (tid < TT) {
        float a = 0.0f;
        for (int w = 0; w < kGvWarps; ++w) a = fmaxf(a, reinterpret_cast<float*>(wred)[w * TT + tid]);
        s_tok[tid] = __fdiv_rn(127.0f, fmaxf(a, 1e-5f));
      }
      consumer_sync();
      // Quantise this block's range into shared memory: q = clamp(rint(x * s), -128, 127).
#pragma unroll
      for (int m = 0; m < TT; ++m) {
        if (m < M) {
          const float s = s_tok[m];
          for (int c = tid; c < chunks; c += kGvConsumers) {
            const TX* src = x + static_cast<size_t>(m) * K + k0 + c * 16;
            uint32_t w[4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              float f[8];
              load8f(src + 8 * h, f);
#pragma unroll
              for (int e = 0; e < 8; e += 4) {
                uint32_t word = 0;
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                  int q = __float2int_rn(__fmul_rn(f[e + b], s));
                  q = min(max(q, -128), 127);
                  rs[m] += q;
                  word |= (static_cast<uint32_t>(q) & 0xffu) << (8 * b);
                }
                w[2 * h + e / 4] = word;
              }
            }
            sts128(xs + m * x_pitch + x_chunk_off(c), make_uint4(w[0], w[1], w[2], w[3]));
          }
        }
      }
    } else {
      // Codes written by the quantisation kernel.
#pragma unroll
      for (int m = 0; m < TT; ++m) {
        if (m < M) {
          const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const int8_t*>(x) +
                                                            static_cast<size_t>(m) * K + k0);
          for (int c = tid; c < chunks; c += kGvConsumers) {
            const uint4 v = __ldcg(src + c);
            rs[m] += byte_sum16(v);
            sts128(xs + m * x_pitch + x_chunk_off(c), v);
          }
        }
      }
      if (tid < TT && tid < M) s_tok[tid] = __ldcg(scale + tid);
    }
    warp_sum_tokens<TT>(rs);
    if (lane == 0) {
#pragma unroll
      for (int m = 0; m < TT; ++m) wred[warp * TT + m] = rs[m];
    }
    consumer_sync();
    if (tid < TT) {
      int a = 0;
      for (int w = 0; w < kGvWarps; ++w) a += wred[w * TT + tid];
      rs_tok[tid] = a;
    }
    consumer_sync();

    // ---- main loop: this block's row blocks, each over this block's stages ----
    const float gamma = __ldg(gamma_ptr);
    for (int r = 0; r < n_my_rb && ok; ++r) {
      int d[TG][4][4];
#pragma unroll
      for (int tg = 0; tg < TG; ++tg)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int c = 0; c < 4; ++c) d[tg][j][c] = 0;

      for (int i = 0; i < nst; ++i) {
        const int it = r * nst + i;
        const int slot = it % nring;
        const bool got = mbar_wait(bar0 + 8 * slot, (it / nring) & 1, ctl);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        const uint32_t wt = ring + slot * kGvStageBytes;
        // 128-byte swizzle: chunk c of row r sits at chunk position c ^ (r & 7); r & 7 == g here.
        const uint4 wl0 = lds128(wt + r_lo * 128 + (((2 * t) ^ g) << 4));
        const uint4 wl1 = lds128(wt + r_lo * 128 + (((2 * t + 1) ^ g) << 4));
        const uint4 wh0 = lds128(wt + (r_lo + 8) * 128 + (((2 * t) ^ g) << 4));
        const uint4 wh1 = lds128(wt + (r_lo + 8) * 128 + (((2 * t + 1) ^ g) << 4));
        __syncwarp();
        if (lane == 0) mbar_arrive(bar0 + 8 * (nring + slot));  // the weights are in registers

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
#pragma unroll
      for (int tg = 0; tg < TG; ++tg)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int m = tg * 8 + 2 * t + (c & 1);
          acc[tg][c] = d[tg][0][c] + (d[tg][1][c] >> 2) + (d[tg][2][c] >> 4) + (d[tg][3][c] >> 6) -
                       (m < M ? rs_tok[m] : 0);
        }
      if (!clustered && ok) {
        // All of K is in registers: finish the row block.
        const int n_base = (rb0 + r * rb_step) * kGvRows;
#pragma unroll
        for (int tg = 0; tg < TG; ++tg)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int n = n_base + r_lo + ((c & 2) ? 8 : 0);
            const int m = tg * 8 + 2 * t + (c & 1);
            if (n < N && m < M) {
              const float v = __fmul_rn(static_cast<float>(acc[tg][c]), __fdiv_rn(gamma, s_tok[m]));
              const size_t o = static_cast<size_t>(m) * N + n;
              if constexpr (sizeof(TY) == 4) y[o] = v; else y[o] = __float2bfloat16_rn(v);
              if (acc_out) acc_out[o] = acc[tg][c];
            }
          }
      }
    }
  }

  if (!clustered) return;  // (a wait that ran out is in the status word; outputs are then unspecified)
  const float gamma = __ldg(gamma_ptr);
  const int n_base = rb0 * kGvRows;

  // ---- split K: the cluster's blocks add their partial sums through distributed shared memory ----
  if (warp < kGvWarps) {
#pragma unroll
    for (int tg = 0; tg < TG; ++tg)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int r = r_lo + ((c & 2) ? 8 : 0);
        const int m = tg * 8 + 2 * t + (c & 1);
        if (m < TT) red_buf[r * TT + m] = acc[tg][c];
      }
  }
  cluster_sync_all();  // every thread of every block of the cluster arrives here
  bool failed = false;  // did any block of the cluster give up a wait?
  for (int p = 0; p < splits; ++p)
    failed |= ld_cluster_s32(smem_u32(const_cast<int*>(abort_flag)), p) != 0;
  if (warp < kGvWarps && !failed) {
    // This block finishes rows [r0, r1) of the row block.
    const int per = (kGvRows + splits - 1) / splits;
    const int r0 = ks * per, r1 = min(kGvRows, r0 + per);
    const int rows = min(r1, N - n_base) - r0;
    const uint32_t red_addr = smem_u32(red_buf);
    for (int idx = threadIdx.x; idx < rows * M; idx += kGvConsumers) {
      const int m = idx / rows, r = r0 + (idx - m * rows);
      int a = 0;
      for (int p = 0; p < splits; ++p) a += ld_cluster_s32(red_addr + (r * TT + m) * 4, p);
      const size_t o = static_cast<size_t>(m) * N + n_base + r;
      const float v = __fmul_rn(static_cast<float>(a), __fdiv_rn(gamma, s_tok[m]));
      if constexpr (sizeof(TY) == 4) y[o] = v; else y[o] = __float2bfloat16_rn(v);
      if (acc_out) acc_out[o] = a;
    }
  }
  cluster_sync_all();  // no block leaves while another still reads its shared memory
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static int token_slots(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16; }

static int gemv_smem_bytes(int M, int tt, int ring, int x_pitch) {
  return ring * kGvStageBytes + ((M * x_pitch + 127) / 128) * 128 + kGvRows * tt * 4 + 2 * tt * 4 +
         kGvWarps * tt * 4 + 16 * ring + 64 + 1024;
}

// Modelled time (us) of a plan: the busiest SM streams its bytes at the rate its
// stages in flight allow (Little's law, ~1.5 us latency) or at its share of HBM,
// plus a per-block start-up cost per wave and the cluster reduction.
static double gemv_plan_cost(long long busiest_bytes, long long total_bytes, int in_flight_stages, int sms,
                             long long waves, int splits) {
  const double hbm = 6.5e6;     // bytes per us
  const double latency = 1.5;   // us
  const double per_sm_rate = in_flight_stages * static_cast<double>(kGvStageBytes) / latency;
  double t = static_cast<double>(busiest_bytes) / per_sm_rate;
  const double floor_t = static_cast<double>(total_bytes) / hbm;
  if (t < floor_t) t = floor_t;
  t += 2.0 * static_cast<double>(waves);
  if (splits > 1) t += 1.0;
  (void)sms;
  return t;
}

static int env_int(const char* name) {
  const char* v = getenv(name);
  return v ? atoi(v) : 0;
}

static GemvPlan plan_gemv_budget(int M, int N, int K, int x_budget) {
  const int sms = num_sms();
  // Tuning knobs: pin the K split and / or the ring depth the model would choose.
  const int force_s = env_int("BITLINEAR_GEMV_SPLITS");
  const int force_ring = env_int("BITLINEAR_GEMV_RING");
  const int tt = token_slots(M);
  GemvPlan best{};
  double best_cost = 1e30;
  const int n_rb = (N + kGvRows - 1) / kGvRows;
  const int n_st = (K + kGvStageK - 1) / kGvStageK;
  const long long total = static_cast<long long>(n_rb) * n_st * kGvStageBytes;
  for (int s = 1; s <= n_st && s <= kGemvMaxSplits; ++s) {
    const int spc = (n_st + s - 1) / s;
    const int s_eff = (n_st + spc - 1) / spc;
    if (s_eff != s) continue;
    if (force_s > 0 && s != force_s) continue;
    const int x_pitch = ((spc * kGvStageK + 127) / 128) * 128 + 16;
    if (M * x_pitch > x_budget) continue;
    for (int ring : {2, 3, 4, 6, 8}) {
      if (ring > spc && ring != 2) continue;
      if (force_ring > 0 && ring != force_ring && !(ring == 2 && force_ring > spc)) continue;
      const int r_eff = ring < spc ? ring : spc;
      const int smem = gemv_smem_bytes(M, tt, r_eff, x_pitch);
      if (smem > 227 * 1024) continue;
      int occ = (227 * 1024) / smem;
      if (occ > 2048 / kGvThreads) occ = 2048 / kGvThreads;
      const long long slots = static_cast<long long>(sms) * occ;
      long long ctas, busiest;
      int in_flight;
      long long waves;
      if (s == 1) {
        // Persistent blocks over all of K: as many as fit at once, up to one per row block.
        ctas = n_rb < slots ? n_rb : slots;
        const long long per_sm = (ctas + sms - 1) / sms;
        const long long rb_per_cta = (n_rb + ctas - 1) / ctas;
        busiest = per_sm * rb_per_cta * n_st * kGvStageBytes;
        in_flight = static_cast<int>(per_sm) * r_eff;
        waves = 1;
      } else {
        ctas = static_cast<long long>(n_rb) * s;
        const long long per_sm = (ctas + sms - 1) / sms;
        busiest = per_sm * spc * kGvStageBytes;
        waves = (ctas + slots - 1) / slots;
        in_flight = static_cast<int>(per_sm < occ ? per_sm : occ) * r_eff;
      }
      const double cost = gemv_plan_cost(busiest, total, in_flight, sms, waves, s);
      if (cost < best_cost - 1e-9) {
        best_cost = cost;
        best = GemvPlan{n_rb, n_st, s, spc, r_eff, x_pitch, smem, static_cast<int>(ctas)};
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

bool gemv_fuses_quant(int M, int K) { return static_cast<long long>(M) * K <= kGvFuseLimit; }

template <int TT, typename TY, typename TX>
static cudaError_t launch_gemv_t(const GemvArgs& a, const GemvPlan& p, cudaStream_t stream, bool pdl) {
  EncodeTiledFn enc = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tw;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K / 4), static_cast<cuuint64_t>(a.N)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K / 4)};
  const cuuint32_t box[2] = {128, kGvRows};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.packed), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
    return cudaErrorInvalidValue;
  }
  auto kernel = gemv_kernel<TT, TY, TX>;
  static bool attr_set = false;  // per template instance
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid);
  cfg.blockDim = dim3(kGvThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(p.smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (p.splits > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = p.splits;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, tw, a.gamma, a.N, a.K, a.M, static_cast<const TX*>(a.x), a.scale,
                            static_cast<TY*>(a.y), a.acc_out, p.splits, p.st_per_split, p.nring, p.x_pitch,
                            a.status);
}

template <int TT, typename TY>
static cudaError_t launch_gemv_x(const GemvArgs& a, const GemvPlan& p, cudaStream_t stream, bool pdl) {
  switch (a.x_type) {
    case kInBF16: return launch_gemv_t<TT, TY, __nv_bfloat16>(a, p, stream, pdl);
    case kInF32: return launch_gemv_t<TT, TY, float>(a, p, stream, pdl);
    default: return launch_gemv_t<TT, TY, int8_t>(a, p, stream, pdl);
  }
}

template <typename TY>
static cudaError_t launch_gemv_y(const GemvArgs& a, const GemvPlan& p, cudaStream_t stream, bool pdl) {
  switch (token_slots(a.M)) {
    case 1: return launch_gemv_x<1, TY>(a, p, stream, pdl);
    case 2: return launch_gemv_x<2, TY>(a, p, stream, pdl);
    case 4: return launch_gemv_x<4, TY>(a, p, stream, pdl);
    case 8: return launch_gemv_x<8, TY>(a, p, stream, pdl);
    default: return launch_gemv_x<16, TY>(a, p, stream, pdl);
  }
}

cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t stream, bool pdl) {
  const GemvPlan p = plan_gemv(a.M, a.N, a.K);
  if (p.splits == 0) return cudaErrorInvalidConfiguration;
  return a.y_type == kOutBF16 ? launch_gemv_y<__nv_bfloat16>(a, p, stream, pdl)
                              : launch_gemv_y<float>(a, p, stream, pdl);
}

}  // namespace bl
