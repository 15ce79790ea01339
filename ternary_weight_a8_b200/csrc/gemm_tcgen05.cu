// Prefill product (many tokens): int8 activations x unpacked ternary codes on
// the 5th-generation tensor cores (tcgen05.mma kind::i8, int32 accumulators
// in tensor memory), with the dequantisation fused into the epilogue.
//
// "BitNet's Real Bet: Designing the Whole Inference Stack", section "A
// low-bit model is a whole-stack design": packed weights move from HBM to
// shared memory, are unpacked there and meet the 8-bit activations.
// "A Two-Billion Ternary Bet": the pack-store-load-unpack-compute sequence.
//
// Tiles: 128 tokens per CTA x 256 output rows x 128 inputs per k-block.
// Two forms of one kernel:
//   CG = 1  one CTA per tile (used for up to 128 tokens);
//   CG = 2  a cluster of two CTAs on two SMs shares a 256-token x 256-row
//           tile through tcgen05.mma.cta_group::2: each CTA loads its own 128
//           tokens and unpacks only its half (128 rows) of the weight tile, so
//           per SM the unpack stores and the tensor cores' shared-memory reads
//           of codes are halved.  The MMA thread of the even CTA issues for
//           both; commits are multicast to both CTAs.
// Warp roles in a persistent block (one per SM) of 16 warps (12 in the pair form):
//   warp 0      TMA producer of the activation tiles (128-byte swizzle);
//   warp 2      TMA producer of the packed weight tiles, on a ring of its own
//               that the unpack warps release once their stores have consumed
//               the words, so weight tiles are requested well ahead;
//   warp 1      tensor-memory owner; in the even CTA, the single thread that
//               issues the 4 tcgen05.mma (K = 32 each) per k-block;
//   warps 4-11  unpack (4-7 in the pair form): packed words -> 16-byte chunks of codes
//               ((w >> 2j) & 0x03030303, j = 0..3) written at its 128-byte
//               swizzle position, a proxy fence, then one arrive per warp;
//   next 4      epilogue: tcgen05.ld of the int32 accumulators, then
//               y = (acc - rowsum[m]) * (gamma / s[m]) stored as fp32 / bf16.
// Two accumulators (2 x 256 tensor-memory columns) let the epilogue of one
// tile overlap the main loop of the next.  Every mbarrier wait is bounded in
// time; a wait that runs out records the timeout in the workspace status
// word, raises the abort flag of both CTAs of the pair, and the block winds
// down without touching global memory further.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace bl {

constexpr int kBM = 128, kBN = 256, kBK = 128;
constexpr int kABytes = kBM * kBK;  // 16 KB activation tile per CTA
constexpr int kEpiWarps = 4;        // the last four warps of the block
constexpr uint32_t kTmemCols = 512;

template <int CG>
struct GemmCfg {
  // Warps 4 .. 4 + kUnpackWarps - 1 unpack, the next four run the epilogue.
  // The pair form unpacks half a weight tile per CTA and needs half the
  // unpack warps (measured: as fast, and the smaller block is slightly faster).
  static constexpr int kUnpackWarps = CG == 1 ? 8 : 4;
  static constexpr int kUnpackThreads = 32 * kUnpackWarps;
  static constexpr int kEpiWarp0 = 4 + kUnpackWarps;
  static constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
  static constexpr int kRowsB = kBN / CG;            // weight rows unpacked by one CTA
  static constexpr int kBPBytes = kRowsB * kBK / 4;  // packed weight tile per CTA
  static constexpr int kBUBytes = kRowsB * kBK;      // unpacked code tile per CTA
  static constexpr int kAStages = CG == 1 ? 5 : 6;
  static constexpr int kPStages = CG == 1 ? 6 : 6;
  static constexpr int kUStages = CG == 1 ? 3 : 4;
  // Output staging of the pair form: per epilogue warp two 32 x 32 boxes of
  // up to 4-byte elements, written out by TMA bulk-tensor stores.
  static constexpr int kOutWarpBytes = CG == 2 ? 2 * 4096 : 0;
  static constexpr int kOffA = 0;
  static constexpr int kOffBU = kOffA + kAStages * kABytes;
  static constexpr int kOffBP = kOffBU + kUStages * kBUBytes;
  static constexpr int kOffOut = kOffBP + kPStages * kBPBytes;
  static constexpr int kOffBar = kOffOut + kEpiWarps * kOutWarpBytes;
  static constexpr int kNumBars = 2 * (kAStages + kPStages + kUStages) + 5;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack
  // Instruction descriptor: D s32, A s8, B s8, both K-major, N = 256, M = 128 * CG.
  static constexpr uint32_t kIdesc =
      (2u << 4) | (1u << 7) | (1u << 10) | ((kBN >> 3) << 17) | (((kBM * CG) >> 4) << 24);
  static_assert(kSmemBytes <= 232448, "shared memory per block");
  static_assert(kBPBytes / 16 % kUnpackThreads == 0, "packed words per unpack thread");
  static_assert(kEpiWarp0 % 4 == 0, "epilogue warp w reads tensor-memory lanes 32 * (w % 4) ..");
  static_assert(kOffOut % 1024 == 0, "swizzled staging alignment");
};

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

// One 32-token x 32-output box of the epilogue through shared memory: lane i
// holds token row i.  The box is written in the swizzle of its tensor map
// (64-byte rows for bf16, 128-byte rows for 4-byte elements) so that the
// lanes' 16-byte stores are free of bank conflicts, then one lane issues the
// TMA store, which skips elements outside the output.
__device__ __forceinline__ void stage_box_b16(uint8_t* buf, int lane, const uint32_t (&p)[16]) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    *reinterpret_cast<uint4*>(buf + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
        make_uint4(p[4 * j], p[4 * j + 1], p[4 * j + 2], p[4 * j + 3]);
}
__device__ __forceinline__ void stage_box_b32(uint8_t* buf, int lane, const uint32_t (&w)[32]) {
#pragma unroll
  for (int j = 0; j < 8; ++j)
    *reinterpret_cast<uint4*>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
        make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
}

template <typename TY>
__device__ __forceinline__ void stage_y(uint8_t* buf, int lane, const uint32_t (&r)[32], int rs, float gs) {
  if constexpr (sizeof(TY) == 2) {
    uint32_t p[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const __nv_bfloat16 lo =
          __float2bfloat16_rn(__fmul_rn(static_cast<float>(static_cast<int>(r[2 * i]) - rs), gs));
      const __nv_bfloat16 hi =
          __float2bfloat16_rn(__fmul_rn(static_cast<float>(static_cast<int>(r[2 * i + 1]) - rs), gs));
      p[i] = static_cast<uint32_t>(__bfloat16_as_ushort(lo)) |
             (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
    }
    stage_box_b16(buf, lane, p);
  } else {
    uint32_t w[32];
#pragma unroll
    for (int i = 0; i < 32; ++i)
      w[i] = __float_as_uint(__fmul_rn(static_cast<float>(static_cast<int>(r[i]) - rs), gs));
    stage_box_b32(buf, lane, w);
  }
}

// Output values already computed in fp32 (held as bits): a staged box, or direct stores.
template <typename TY>
__device__ __forceinline__ void stage_vals(uint8_t* buf, int lane, const uint32_t (&v)[32]) {
  if constexpr (sizeof(TY) == 2) {
    uint32_t p[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      p[i] = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[2 * i])))) |
             (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[2 * i + 1])))) << 16);
    stage_box_b16(buf, lane, p);
  } else {
    stage_box_b32(buf, lane, v);
  }
}

template <typename TY>
__device__ __forceinline__ void store_vals32(TY* __restrict__ y, size_t row_off, int n0, int N, const uint32_t (&v)[32]) {
  for (int i = 0; i < 32; ++i)
    if (n0 + i < N) {
      if constexpr (sizeof(TY) == 2) {
        y[row_off + n0 + i] = __float2bfloat16_rn(__uint_as_float(v[i]));
      } else {
        y[row_off + n0 + i] = __uint_as_float(v[i]);
      }
    }
}

// Bounded wait for the GEMM: as mbar_wait, and in the pair form a wait that
// gives up raises the abort flag of the peer CTA too.
template <int CG>
__device__ __forceinline__ bool gemm_wait(uint32_t bar, uint32_t parity, const WaitCtl& ctl,
                                          uint32_t peer_abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, 200000u)) return true;
    if (*ctl.abort) return false;
    if (global_ns() - t0 > ctl.limit_ns) {
      *ctl.abort = 1;
      if (CG == 2) st_shared_cluster_u32(peer_abort, 1u);
      if (ctl.status) atomicOr(ctl.status, kStatusTimeout);
      return false;
    }
  }
}

// Arrive on a barrier of the even CTA of the pair (this CTA's own when CG = 1).
template <int CG>
__device__ __forceinline__ void arrive_leader(uint32_t bar) {
  if constexpr (CG == 1) {
    mbar_arrive(bar);
  } else {
    mbar_arrive_cluster(mapa_shared(bar, 0));
  }
}

template <int CG>
__device__ __forceinline__ void commit_to(uint32_t bar) {
  if constexpr (CG == 1) {
    tc_commit(bar);
  } else {
    tc_commit_pair_mc(bar, static_cast<uint16_t>(0x3));
  }
}

// The FFN's gate and up products in one GEMM (glu_act >= 0): a tile holds
// 128 rows of the gate weights (tmap_b) in accumulator columns 0..127 and the
// same 128 rows of the up weights (tmap_b2) in columns 128..255 (in the pair
// form the even CTA loads the gate half, the odd one the up half), and the
// epilogue stores h = act(gate) * up (each output rounded to TY first, as
// stored BitLinear outputs are, then h rounded to TY) instead of y.
struct GemmGlu {
  int act;              // -1: plain GEMM; else the GluAct of h
  const float* gamma2;  // the up BitLinear's gamma
};

template <typename TY, int CG>
__global__ void __maxnreg__(128) gemm_kernel(
    const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
    const __grid_constant__ CUtensorMap tmap_b2, const __grid_constant__ CUtensorMap tmap_y,
    const __grid_constant__ CUtensorMap tmap_acc, int tma_out, const GemmGlu glu,
    const float* __restrict__ gamma_ptr, int N, int K, int M, const float* __restrict__ scale,
    const int32_t* __restrict__ rowsum, TY* __restrict__ y, int32_t* __restrict__ acc_out,
    uint32_t* status) {
  using C = GemmCfg<CG>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  constexpr int kBarP = 2 * C::kAStages, kBarU = kBarP + 2 * C::kPStages, kBarT = kBarU + 2 * C::kUStages;
  auto afull_bar = [&](int i) { return sb + C::kOffBar + 8 * i; };
  auto aempty_bar = [&](int i) { return sb + C::kOffBar + 8 * (C::kAStages + i); };
  auto pfull_bar = [&](int i) { return sb + C::kOffBar + 8 * (kBarP + i); };
  auto pempty_bar = [&](int i) { return sb + C::kOffBar + 8 * (kBarP + C::kPStages + i); };
  auto ufull_bar = [&](int i) { return sb + C::kOffBar + 8 * (kBarU + i); };
  auto uempty_bar = [&](int i) { return sb + C::kOffBar + 8 * (kBarU + C::kUStages + i); };
  auto tfull_bar = [&](int i) { return sb + C::kOffBar + 8 * (kBarT + i); };
  auto tempty_bar = [&](int i) { return sb + C::kOffBar + 8 * (kBarT + 2 + i); };
  const uint32_t done_bar = sb + C::kOffBar + 8 * (C::kNumBars - 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 16);
  volatile int* never = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 32);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
  const uint32_t peer_abort = CG == 2 ? mapa_shared(sb + C::kOffMisc + 16, rank ^ 1u) : 0u;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kAStages; ++i) {
      mbar_init(afull_bar(i), 1);   // the even CTA's expect-tx arrive (bytes of both CTAs)
      mbar_init(aempty_bar(i), 1);  // MMA commit
    }
    for (int i = 0; i < C::kPStages; ++i) {
      mbar_init(pfull_bar(i), 1);
      mbar_init(pempty_bar(i), C::kUnpackWarps);
    }
    for (int i = 0; i < C::kUStages; ++i) {
      mbar_init(ufull_bar(i), C::kUnpackWarps * CG);  // unpack warps of both CTAs
      mbar_init(uempty_bar(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), kEpiWarps * CG);  // epilogue warps of both CTAs
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    *never = 0;
    fence_barrier_init();
  }
  const bool is_glu = glu.act >= 0;
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmap_a);
  if (warp == 2 && lane == 0) {
    tma_prefetch_desc(&tmap_b);
    if (is_glu) tma_prefetch_desc(&tmap_b2);
  }
  if (warp == 1) {
    if constexpr (CG == 1) {
      tmem_alloc(smem_u32(tmem_slot), kTmemCols);
      tmem_relinquish();
    } else {
      tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
      tmem_relinquish_pair();
    }
  }
  tc_fence_before();
  if constexpr (CG == 1) {
    __syncthreads();
  } else {
    cluster_sync_all();  // barriers of both CTAs initialised before any remote arrive
  }
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // Only the roles that touch the activations, scales, row sums or outputs
  // wait for the preceding kernel; the weight tiles (never written by a
  // kernel that lets its dependents start early) are fetched and unpacked
  // meanwhile.
  griddep_launch_dependents();

  const WaitCtl ctl{status, abort_flag, kWaitLimitNs};
  const int m_tiles = (M + kBM * CG - 1) / (kBM * CG);
  const int tile_n = is_glu ? kBN / 2 : kBN;  // output columns per tile
  const int n_tiles = (N + tile_n - 1) / tile_n;
  const int tiles = m_tiles * n_tiles;
  const int kblocks = (K + kBK - 1) / kBK;
  const int cluster_id = blockIdx.x / CG, n_clusters = gridDim.x / CG;

  if (warp == 0 || warp == 2) {
    if (lane == 0) {
      // warp 0: activation tiles; warp 2: packed weight tiles.
      const bool is_a = (warp == 0);
      if (is_a) griddep_wait();  // the activation codes come from the preceding kernel
      const int nst = is_a ? C::kAStages : C::kPStages;
      int it = 0, s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = cluster_id; ok && tile < tiles; tile += n_clusters) {
        const int mt = tile % m_tiles, nt = tile / m_tiles;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          if (!gemm_wait<CG>(is_a ? aempty_bar(s) : pempty_bar(s), ph ^ 1, ctl, peer_abort)) {
            ok = false;
            break;
          }
          if (is_a) {
            const uint32_t dst = sb + C::kOffA + s * kABytes;
            const int row = mt * kBM * CG + static_cast<int>(rank) * kBM;
            if constexpr (CG == 1) {
              mbar_arrive_expect_tx(afull_bar(s), kABytes);
              tma_load_2d(dst, &tmap_a, kb * kBK, row, afull_bar(s));
            } else {
              if (rank == 0) mbar_arrive_expect_tx(afull_bar(s), CG * kABytes);
              tma_load_2d_pair(dst, &tmap_a, kb * kBK, row, mapa_shared(afull_bar(s), 0));
            }
          } else {
            mbar_arrive_expect_tx(pfull_bar(s), C::kBPBytes);
            const uint32_t dst = sb + C::kOffBP + s * C::kBPBytes;
            if (!is_glu) {
              tma_load_2d(dst, &tmap_b, kb * (kBK / 4), nt * kBN + static_cast<int>(rank) * C::kRowsB, pfull_bar(s));
            } else if constexpr (CG == 1) {
              // 128 gate rows, then the same 128 rows of up.
              tma_load_2d(dst, &tmap_b, kb * (kBK / 4), nt * (kBN / 2), pfull_bar(s));
              tma_load_2d(dst + (kBN / 2) * (kBK / 4), &tmap_b2, kb * (kBK / 4), nt * (kBN / 2), pfull_bar(s));
            } else {
              tma_load_2d(dst, rank == 0 ? &tmap_b : &tmap_b2, kb * (kBK / 4), nt * (kBN / 2), pfull_bar(s));
            }
          }
          if (++s == nst) { s = 0; ph ^= 1; }
        }
      }
      if (!ok) {
        // Let copies already in flight land before the block's shared memory goes away.
        const WaitCtl drain{nullptr, never, 100000000ull};
        if (!is_a || CG == 1) {
          for (int i = (it > nst ? it - nst : 0); i < it; ++i)
            gemm_wait<1>(is_a ? afull_bar(i % nst) : pfull_bar(i % nst), (i / nst) & 1, drain, 0u);
        } else {
          // Completion of the pair's activation copies is counted in the even
          // CTA; give copies in flight a fixed millisecond instead.
          const uint64_t t0 = global_ns();
          while (global_ns() - t0 < 1000000ull) __nanosleep(10000);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      int it = 0, tc = 0;
      bool ok = true, issued = false;
      for (int tile = cluster_id; ok && tile < tiles; tile += n_clusters, ++tc) {
        const int a = tc & 1;
        if (!gemm_wait<CG>(tempty_bar(a), ((tc >> 1) & 1) ^ 1, ctl, peer_abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + a * kBN;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % C::kAStages, u = it % C::kUStages;
          if (!gemm_wait<CG>(afull_bar(s), (it / C::kAStages) & 1, ctl, peer_abort)) { ok = false; break; }
          if (!gemm_wait<CG>(ufull_bar(u), (it / C::kUStages) & 1, ctl, peer_abort)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = sw128_kmajor_desc(sb + C::kOffA + s * kABytes);
          const uint64_t bdesc = sw128_kmajor_desc(sb + C::kOffBU + u * C::kBUBytes);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k) {
            if constexpr (CG == 1) {
              tc_mma_i8(d_tmem, adesc + 2 * k, bdesc + 2 * k, C::kIdesc, (kb | k) != 0);
            } else {
              tc_mma_i8_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, C::kIdesc, (kb | k) != 0);
            }
          }
          issued = true;
          commit_to<CG>(aempty_bar(s));
          commit_to<CG>(uempty_bar(u));
        }
        if (ok) commit_to<CG>(tfull_bar(a));
      }
      if (issued) {
        // Every MMA must be finished before tensor memory is released (the odd
        // CTA learns of it through the closing cluster barrier).
        if constexpr (CG == 1) {
          tc_commit(done_bar);
        } else {
          tc_commit_pair(done_bar);
        }
        const WaitCtl drain{nullptr, never, 100000000ull};
        gemm_wait<1>(done_bar, 0, drain, 0u);
      }
    }
  } else if (warp >= 4 && warp < C::kEpiWarp0) {
    const int ut = threadIdx.x - 128;
    int it = 0;
    bool ok = true;
    for (int tile = cluster_id; ok && tile < tiles; tile += n_clusters) {
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int s = it % C::kPStages, u = it % C::kUStages;
        // Wait outcomes are made warp-uniform: the warp then syncs and arrives as one.
        ok = __all_sync(0xffffffffu, gemm_wait<1>(pfull_bar(s), (it / C::kPStages) & 1, ctl, peer_abort));
        if (!ok) break;
        constexpr int kPer = C::kBPBytes / 16 / C::kUnpackThreads;  // packed uint4 per thread
        const uint4* bp = reinterpret_cast<const uint4*>(smem + C::kOffBP + s * C::kBPBytes);
        uint4 codes[kPer][4];
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
          const uint4 v = bp[ut + j * C::kUnpackThreads];
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t w = w4[i];
            codes[j][i] = make_uint4(w & 0x03030303u, (w >> 2) & 0x03030303u, (w >> 4) & 0x03030303u,
                                     (w >> 6) & 0x03030303u);
          }
        }
        ok = __all_sync(0xffffffffu,
                        gemm_wait<CG>(uempty_bar(u), ((it / C::kUStages) & 1) ^ 1, ctl, peer_abort));
        if (!ok) break;
        uint8_t* bu = smem + C::kOffBU + u * C::kBUBytes;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
          const int q = ut + j * C::kUnpackThreads;
          const int r = q >> 1;        // weight row in the CTA's tile (32 packed bytes per row)
          const int c0 = (q & 1) * 4;  // first 16-byte chunk (= packed word) of this uint4
          uint8_t* rowp = bu + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            *reinterpret_cast<uint4*>(rowp + (((c0 + i) ^ (r & 7)) << 4)) = codes[j][i];
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          // The warp's stores consumed its packed words: release the packed
          // slot, and report the codes to the MMA issuer.
          mbar_arrive(pempty_bar(s));
          arrive_leader<CG>(ufull_bar(u));
        }
      }
    }
  } else if (warp >= C::kEpiWarp0) {
    const int q = warp & 3;  // tensor-memory lane quarter this warp may read
    griddep_wait();          // scales and row sums come from the preceding kernel; y may be read by it
    const float gamma = __ldg(gamma_ptr);
    const float gamma2 = is_glu ? __ldg(glu.gamma2) : 0.0f;
    const bool staged = C::kOutWarpBytes > 0 && tma_out;
    uint8_t* obuf = smem + C::kOffOut + (warp - C::kEpiWarp0) * C::kOutWarpBytes;
    int ob = 0;  // staging buffer of the next box
    if (staged && lane == 0) {
      tma_prefetch_desc(&tmap_y);
      if (acc_out) tma_prefetch_desc(&tmap_acc);
    }
    int tc = 0;
    for (int tile = cluster_id; tile < tiles; tile += n_clusters, ++tc) {
      const int mt = tile % m_tiles, nt = tile / m_tiles;
      const int a = tc & 1;
      // tcgen05.ld below is warp-collective: take the wait's outcome warp-wide.
      const bool got = gemm_wait<CG>(tfull_bar(a), (tc >> 1) & 1, ctl, peer_abort);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int m0 = mt * kBM * CG + static_cast<int>(rank) * kBM + q * 32;  // first row of this warp
      const int m = m0 + lane;
      const bool mvalid = m < M;
      float gs = 0.0f, gs2 = 0.0f;
      int rs = 0;
      if (mvalid) {
        gs = __fdiv_rn(gamma, __ldg(scale + m));
        if (is_glu) gs2 = __fdiv_rn(gamma2, __ldg(scale + m));
        rs = __ldg(rowsum + m);
      }
      if (is_glu) {
        // 32 output columns at a time: the gate accumulators at column c, the
        // up accumulators at column c + 128.
#pragma unroll 1
        for (int c = 0; c < kBN / 64; ++c) {
          uint32_t r[32], r2[32];
          const uint32_t t0 = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * kBN + c * 32;
          tmem_ld_32x32b_x32(t0, r);
          tmem_ld_32x32b_x32(t0 + kBN / 2, r2);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float g = round_to<TY>(__fmul_rn(static_cast<float>(static_cast<int>(r[i]) - rs), gs));
            const float u = round_to<TY>(__fmul_rn(static_cast<float>(static_cast<int>(r2[i]) - rs), gs2));
            r[i] = __float_as_uint(glu_value<TY>(g, u, glu.act));
          }
          const int n0 = nt * (kBN / 2) + c * 32;
          if (staged) {
            if (n0 < N && m0 < M) {  // warp-uniform
              if (lane == 0) bulk_wait_group_read<1>();
              __syncwarp();
              uint8_t* b = obuf + ob * 4096;
              stage_vals<TY>(b, lane, r);
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&tmap_y, smem_u32(b), n0, m0);
                bulk_commit_group();
              }
              ob ^= 1;
            }
          } else if (mvalid && n0 < N) {
            store_vals32<TY>(y, static_cast<size_t>(m) * N, n0, N, r);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_leader<CG>(tempty_bar(a));
        continue;
      }
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * kBN + c * 32, r);
        tmem_ld_wait();
        const int n0 = nt * kBN + c * 32;
        if (staged) {
          if (n0 < N && m0 < M) {  // warp-uniform
            if (acc_out) {
              // y and the accumulators: one box each, both buffers, every step.
              if (lane == 0) bulk_wait_group_read<0>();
              __syncwarp();
              stage_y<TY>(obuf, lane, r, rs, gs);
              uint32_t w[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) w[i] = static_cast<uint32_t>(static_cast<int>(r[i]) - rs);
              stage_box_b32(obuf + 4096, lane, w);
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&tmap_y, smem_u32(obuf), n0, m0);
                tma_store_2d(&tmap_acc, smem_u32(obuf + 4096), n0, m0);
                bulk_commit_group();
              }
            } else {
              // The buffer's previous box (two groups ago) must have been read.
              if (lane == 0) bulk_wait_group_read<1>();
              __syncwarp();
              uint8_t* b = obuf + ob * 4096;
              stage_y<TY>(b, lane, r, rs, gs);
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&tmap_y, smem_u32(b), n0, m0);
                bulk_commit_group();
              }
              ob ^= 1;
            }
          }
        } else if (mvalid && n0 < N) {
          store_row32<TY>(y, acc_out, static_cast<size_t>(m) * N, n0, N, r, rs, gs);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_leader<CG>(tempty_bar(a));
    }
    if (staged && lane == 0) bulk_wait_group_all();  // stores done before the block's shared memory goes away
  }

  tc_fence_before();
  if constexpr (CG == 1) {
    __syncthreads();
  } else {
    cluster_sync_all();  // no CTA leaves while its peer may still signal it
  }
  if (warp == 1) {
    tc_fence_after();
    if constexpr (CG == 1) {
      tmem_dealloc(tmem_base, kTmemCols);
    } else {
      tmem_dealloc_pair(tmem_base, kTmemCols);
    }
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

// 2-D map over a row-major matrix of `outer` rows of `inner` elements, rows
// `pitch` bytes apart (default: dense).
static bool make_map_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                        uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz, uint64_t pitch = 0,
                        CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_UINT8, uint32_t esize = 1) {
  EncodeTiledFn fn = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch ? pitch : inner * esize};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename TY, int CG>
static cudaError_t launch_gemm_t(const ProductArgs& a, cudaStream_t stream, bool pdl) {
  using C = GemmCfg<CG>;
  const bool glu = a.glu_act >= 0;
  if (glu && (!a.packed2 || !a.gamma2 || a.acc_out)) return cudaErrorInvalidValue;
  // A GLU tile takes 128 rows of each weight tensor (one load each, or one per CTA of the pair).
  const uint32_t rows_b = glu ? kBN / 2 : C::kRowsB;
  CUtensorMap ta, tb, tb2 = {};
  if (!make_map_2d(&ta, a.xq, static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.M), kBK, kBM,
                   CU_TENSOR_MAP_SWIZZLE_128B, static_cast<uint64_t>(a.ldx)) ||
      !make_map_2d(&tb, a.packed, static_cast<uint64_t>(a.K / 4), static_cast<uint64_t>(a.N), kBK / 4, rows_b,
                   CU_TENSOR_MAP_SWIZZLE_NONE) ||
      (glu && !make_map_2d(&tb2, a.packed2, static_cast<uint64_t>(a.K / 4), static_cast<uint64_t>(a.N), kBK / 4,
                           rows_b, CU_TENSOR_MAP_SWIZZLE_NONE))) {
    return cudaErrorInvalidValue;
  }
  // The pair form writes its outputs by TMA when the rows are 16-byte
  // multiples and the buffers 16-byte aligned; otherwise by plain stores.
  CUtensorMap ty = {}, tacc = {};
  const uint64_t esz = sizeof(TY);
  int tma_out = CG == 2 && (static_cast<uint64_t>(a.N) * esz) % 16 == 0 &&
                (static_cast<uint64_t>(a.N) * 4) % 16 == 0 && reinterpret_cast<uintptr_t>(a.y) % 16 == 0 &&
                reinterpret_cast<uintptr_t>(a.acc_out) % 16 == 0;
  if (tma_out) {
    const bool ok_y = make_map_2d(&ty, a.y, static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.M), 32, 32,
                                  esz == 2 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B, 0,
                                  esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                                  static_cast<uint32_t>(esz));
    const bool ok_acc = !a.acc_out || make_map_2d(&tacc, a.acc_out, static_cast<uint64_t>(a.N),
                                                  static_cast<uint64_t>(a.M), 32, 32, CU_TENSOR_MAP_SWIZZLE_128B,
                                                  0, CU_TENSOR_MAP_DATA_TYPE_INT32, 4);
    if (!ok_y || !ok_acc) return cudaErrorInvalidValue;
  }
  // Per template instance and device (function attributes belong to the
  // device's context): the shared-memory attribute and the resident clusters.
  static std::atomic<int> max_clusters_of[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) dev = -1;
  int max_clusters = dev >= 0 ? max_clusters_of[dev].load(std::memory_order_acquire) : 0;
  if (max_clusters == 0) {
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<TY, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (e != cudaSuccess) return e;
    int n = num_sms() / CG;
    if (CG > 1) {
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3(CG * n);
      q.blockDim = dim3(C::kThreads);
      q.dynamicSmemBytes = C::kSmemBytes;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = CG;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      q.attrs = at;
      q.numAttrs = 1;
      int c = 0;
      e = cudaOccupancyMaxActiveClusters(&c, gemm_kernel<TY, CG>, &q);
      if (e != cudaSuccess) return e;
      if (c > 0 && c < n) n = c;
    }
    max_clusters = n > 0 ? n : 1;
    if (dev >= 0) max_clusters_of[dev].store(max_clusters, std::memory_order_release);
  }
  const int tile_n = glu ? kBN / 2 : kBN;
  const int tiles = ((a.M + kBM * CG - 1) / (kBM * CG)) * ((a.N + tile_n - 1) / tile_n);
  const int clusters = tiles < max_clusters ? tiles : max_clusters;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CG * clusters);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (CG > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = CG;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  const GemmGlu gg{a.glu_act, a.gamma2};
  return cudaLaunchKernelEx(&cfg, gemm_kernel<TY, CG>, ta, tb, tb2, ty, tacc, tma_out, gg, a.gamma, a.N, a.K, a.M,
                            a.scale, a.rowsum, static_cast<TY*>(a.y), a.acc_out, a.status);
}

// Up to 128 tokens one CTA per tile; beyond, CTA pairs on 256-token tiles.
cudaError_t launch_gemm(const ProductArgs& a, cudaStream_t stream, bool pdl) {
  if (a.M <= 0) return cudaSuccess;
  const bool pair = a.M > kBM;
  if (a.y_type == kOutBF16)
    return pair ? launch_gemm_t<__nv_bfloat16, 2>(a, stream, pdl) : launch_gemm_t<__nv_bfloat16, 1>(a, stream, pdl);
  return pair ? launch_gemm_t<float, 2>(a, stream, pdl) : launch_gemm_t<float, 1>(a, stream, pdl);
}

}  // namespace bl
