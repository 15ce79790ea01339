// Decode product on the 5th-generation tensor cores for 2 to 16 tokens:
// the ternary codes of 128 weight rows are the A operand of
// tcgen05.mma.kind::i8, taken from tensor memory, the tokens' int8 codes the
// B operand (N = 16) in shared memory, the int32 sums in tensor memory.
//
// "BitNet's Real Bet: Designing the Whole Inference Stack", section "A
// low-bit model is a whole-stack design": packed weights move from HBM to
// shared memory, are unpacked there and meet the 8-bit activations.  On
// B200 the unpacked codes never go back to shared memory: the unpack warps
// expand each packed word in registers (c = (w >> 2j) & 0x03030303 gives
// four codes of consecutive inputs) and write them to tensor memory with
// tcgen05.st, where the MMA reads them.  A decode step moves far more weight
// bytes than it does arithmetic, so shared memory stays free for a deep
// ring of packed-weight stages.
//
// Measured on B200 (70B-class chain, 214 MB of packed weights): ~97-102 us
// per step at 2 to 16 tokens, against 41-61 us for the CUDA-core form, with
// one or four accumulator chains and one or two stages unpacked at a time
// alike.  Each 128 x 16 x 32 MMA holds the tensor core about 125 cycles,
// as long as a 128 x 256 x 32 one: the pace is set by the tensor core
// taking in the A operand, 4 KB of unpacked codes per MMA, about 32 bytes
// per clock per SM, while streaming the packed weights at the HBM rate
// would need four times that (the codes are four times the packed bytes).
// So this form is selected only on request (bitlinear_set_decode_form).
//
// Work unit: 128 output rows x all of K of one layer; several independent
// layers share a launch, longest K first, units handed out by the ticket
// counter of the decode kernel (block b starts with unit b).  A stage is 512
// inputs: 16 KB of packed weights (128-byte swizzle) and the 16 tokens'
// codes of those inputs (4 blocks of 16 rows x 128 bytes, the 128-byte
// swizzled K-major layout the MMA reads), 9 stages in flight per block, one
// block per SM.
//
// Warp roles (448 threads):
//   warp 0        TMA producer (packed weights, then, after the grid
//                 dependency, the activation codes of each stage);
//   warp 1        tensor-memory owner; its lane 0 issues the MMAs
//                 (16 per stage, K = 32 each) and the commits;
//   warps 2-9     unpack, two groups of four taking alternate stages (two
//                 stages in flight): warp w writes tensor-memory lanes
//                 32 (w % 4) .. +31, one weight row per thread;
//   warps 10-13   epilogue: tcgen05.ld of the 16 token sums of a row, then
//                 y = (acc - rowsum[m]) * (gamma / s[m]) for m < M.
// Tensor memory (512 columns): three A buffers of 128 columns (a stage's
// 512 codes per row, four per column) and two accumulators of 4 x 16
// columns, so the unpack of the next stages and the epilogue of the last
// unit overlap the MMAs.  Each of a stage's four 128-input blocks adds into
// its own 16 columns: four independent chains of MMAs instead of one, which
// the epilogue sums (exact int32).  Every wait is bounded; a role that gives up raises the block's
// abort flag and the block winds down without touching global memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

namespace bl {

namespace {

constexpr int kTcRows = 128;                  // MMA M: output rows per unit
constexpr int kTcTok = 16;                    // MMA N: token slots
constexpr int kTcStageK = 512;                // inputs per stage
constexpr int kTcWBytes = kTcRows * kTcStageK / 4;  // 16 KB of packed weights per stage
constexpr int kTcXBytes = 4 * kTcTok * 128;   // 8 KB of codes per stage (4 blocks of 128 inputs)
constexpr int kTcSlot = kTcWBytes + kTcXBytes;
constexpr int kTcRing = 9;
constexpr int kTcABufs = 3;                   // A buffers in tensor memory
constexpr int kTcACols = kTcStageK / 4;       // 128 columns per A buffer
constexpr int kTcDCol0 = kTcABufs * kTcACols; // first accumulator column
constexpr int kTcDCols = 4 * kTcTok;          // one accumulator: 4 partial sums of 16 tokens
constexpr uint32_t kTcTmemCols = 512;
constexpr int kTcUnpackWarps = 8;
constexpr int kTcUnpackGroups = 2;            // groups of 4 unpack warps taking alternate stages
constexpr int kTcGroupWarps = kTcUnpackWarps / kTcUnpackGroups;
constexpr int kTcEpiWarp0 = 10;
constexpr int kTcThreads = 32 * (kTcEpiWarp0 + 4);
constexpr int kTcMaxLayers = kGvMaxLayers;
constexpr int kTcTagEnd = -1;
// Instruction descriptor: D s32, A s8, B s8, both K-major, N = 16, M = 128.
constexpr uint32_t kTcIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((kTcTok >> 3) << 17) | ((kTcRows >> 4) << 24);
static_assert(kTcDCol0 + 2 * kTcDCols <= static_cast<int>(kTcTmemCols), "tensor memory columns");
static_assert(kTcSlot % 1024 == 0 && kTcWBytes % 1024 == 0, "swizzle atoms");

struct TcLayer {
  CUtensorMap wmap;  // packed weights [N][K/4]: box 128 bytes x 128 rows, 128-byte swizzle
  CUtensorMap xmap;  // codes viewed as [K/128 blocks][M tokens][128]: box 128 x 16 x 4, 128-byte swizzle
  const float* scale;
  const int32_t* rowsum;
  const float* gamma;
  void* y;
  int32_t* acc_out;
  int N, K, unit0;
};

struct TcParams {
  TcLayer layer[kTcMaxLayers];
  int n_layers, M, total_units, one_unit;
  uint32_t* status;
  uint32_t* tickets;
};

// Shared-memory layout after the ring (1024-byte aligned base).
constexpr int kTcOffBar = kTcRing * kTcSlot;
// barriers: full[R], empty[R], afull[3], aempty[3], dfull[2], dempty[2], done
constexpr int kTcNumBars = 2 * kTcRing + 2 * kTcABufs + 4 + 1;
constexpr int kTcOffMisc = kTcOffBar + kTcNumBars * 8;
// misc: tmem base (4), abort (4), never (4), tags[R], stage[R], nstage[R], dtag[2]
constexpr int kTcMiscBytes = 16 + 3 * 4 * kTcRing + 8;
constexpr int kTcSmemBytes = kTcOffMisc + kTcMiscBytes + 1024;  // + alignment slack
static_assert(kTcSmemBytes <= 232448, "shared memory per block");

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// D[tmem] (+)= A[tmem] x B[smem desc]^T, int8 inputs, int32 accumulators.
__device__ __forceinline__ void tc_mma_i8_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}

template <typename TY>
__global__ void __launch_bounds__(kTcThreads, 1) gemv_tc_kernel(const __grid_constant__ TcParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto full_bar = [&](int i) { return sb + kTcOffBar + 8 * i; };
  auto empty_bar = [&](int i) { return sb + kTcOffBar + 8 * (kTcRing + i); };
  auto afull_bar = [&](int i) { return sb + kTcOffBar + 8 * (2 * kTcRing + i); };
  auto aempty_bar = [&](int i) { return sb + kTcOffBar + 8 * (2 * kTcRing + kTcABufs + i); };
  auto dfull_bar = [&](int i) { return sb + kTcOffBar + 8 * (2 * kTcRing + 2 * kTcABufs + i); };
  auto dempty_bar = [&](int i) { return sb + kTcOffBar + 8 * (2 * kTcRing + 2 * kTcABufs + 2 + i); };
  const uint32_t done_bar = sb + kTcOffBar + 8 * (kTcNumBars - 1);
  uint8_t* misc = smem + kTcOffMisc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  volatile int* never = reinterpret_cast<volatile int*>(misc + 8);
  volatile int* tags = reinterpret_cast<volatile int*>(misc + 16);  // unit of each slot
  volatile int* stg = tags + kTcRing;                               // stage of the unit
  volatile int* nstg = stg + kTcRing;                               // stages of the unit
  volatile int* dtag = nstg + kTcRing;                              // unit of each accumulator

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kTcRing; ++i) {
      mbar_init(full_bar(i), 1);
      mbar_init(empty_bar(i), kTcGroupWarps + 1);  // one group's unpack warps (weights) + MMA commit (codes)
    }
    for (int i = 0; i < kTcABufs; ++i) {
      mbar_init(afull_bar(i), kTcGroupWarps);
      mbar_init(aempty_bar(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(dfull_bar(i), 2);  // MMA commit + the MMA thread's arrive after writing dtag
      mbar_init(dempty_bar(i), 4);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    *never = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTcTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_launch_dependents();
  const WaitCtl ctl{P.status, abort_flag, kWaitLimitNs};
  const int M = P.M;

  auto layer_of = [&](int u) {
    int l = 0;
    while (l + 1 < P.n_layers && u >= P.layer[l + 1].unit0) ++l;
    return l;
  };

  if (warp == 0) {
    // ---- producer ----
    if (lane == 0) {
      int it = 0;
      bool ok = true, waited = false;
      int unit = static_cast<int>(blockIdx.x);
      auto next_unit = [&]() {
        if (P.one_unit) return P.total_units;
        if (!waited) {
          griddep_wait();  // the ticket counter is reset by the preceding launch
          waited = true;
        }
        return static_cast<int>(gridDim.x) + static_cast<int>(atomicAdd(P.tickets, 1u));
      };
      // The first unit's first ring of weight stages goes out before the grid
      // dependency (weights are never written by a kernel that lets its
      // dependents start early), their codes once the preceding kernel is done.
      int pre = 0;
      if (unit < P.total_units) {
        const TcLayer& L = P.layer[layer_of(unit)];
        const int nst = (L.K + kTcStageK - 1) / kTcStageK;
        pre = nst < kTcRing ? nst : kTcRing;
        for (int j = 0; j < pre; ++j) {
          tags[j] = unit;
          stg[j] = j;
          nstg[j] = nst;
          mbar_arrive_expect_tx(full_bar(j), kTcSlot);
          tma_load_2d(sb + j * kTcSlot, &L.wmap, j * (kTcStageK / 4), (unit - L.unit0) * kTcRows, full_bar(j));
        }
        griddep_wait();
        waited = true;
        for (int j = 0; j < pre; ++j)
          tma_load_3d(sb + j * kTcSlot + kTcWBytes, &L.xmap, 0, 0, 4 * j, full_bar(j));
        it = pre;
      }
      int st0 = pre;
      while (ok && unit < P.total_units) {
        const TcLayer& L = P.layer[layer_of(unit)];
        const int nst = (L.K + kTcStageK - 1) / kTcStageK;
        for (int st = st0; st < nst; ++st, ++it) {
          const int s = it % kTcRing;
          if (!mbar_wait(empty_bar(s), ((it / kTcRing) & 1) ^ 1, ctl)) { ok = false; break; }
          tags[s] = unit;
          stg[s] = st;
          nstg[s] = nst;
          mbar_arrive_expect_tx(full_bar(s), kTcSlot);
          tma_load_2d(sb + s * kTcSlot, &L.wmap, st * (kTcStageK / 4), (unit - L.unit0) * kTcRows, full_bar(s));
          if (!waited) {
            griddep_wait();
            waited = true;
          }
          tma_load_3d(sb + s * kTcSlot + kTcWBytes, &L.xmap, 0, 0, 4 * st, full_bar(s));
        }
        st0 = 0;
        if (!ok) break;
        unit = next_unit();
      }
      if (ok) {
        // End markers in the next slot of every unpack group.
        for (int e = 0; e < kTcUnpackGroups; ++e, ++it) {
          const int s = it % kTcRing;
          if (!mbar_wait(empty_bar(s), ((it / kTcRing) & 1) ^ 1, ctl)) break;
          tags[s] = kTcTagEnd;
          mbar_arrive(full_bar(s));
        }
      } else {
        // Gave up: let copies in flight land before shared memory is released.
        const WaitCtl drain{nullptr, never, 100000000ull};
        for (int j = (it > kTcRing ? it - kTcRing : 0); j < it; ++j)
          mbar_wait(full_bar(j % kTcRing), (j / kTcRing) & 1, drain);
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----
    if (lane == 0) {
      int it = 0, uc = 0;
      bool ok = true, issued = false;
      while (true) {
        const int s = it % kTcRing, b = it % kTcABufs;
        if (!mbar_wait(full_bar(s), (it / kTcRing) & 1, ctl)) { ok = false; break; }
        const int unit = tags[s];
        const int d = uc & 1;
        if (unit == kTcTagEnd) {
          // Tell the epilogue (both arrivals of its barrier; no MMA pending on it).
          if (mbar_wait(dempty_bar(d), ((uc >> 1) & 1) ^ 1, ctl)) {
            dtag[d] = kTcTagEnd;
            mbar_arrive(dfull_bar(d));
            mbar_arrive(dfull_bar(d));
          }
          break;
        }
        const int st = stg[s], nst = nstg[s];
        if (st == 0) {
          if (!mbar_wait(dempty_bar(d), ((uc >> 1) & 1) ^ 1, ctl)) { ok = false; break; }
        }
        if (!mbar_wait(afull_bar(b), (it / kTcABufs) & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + kTcDCol0 + kTcDCols * d;
        const uint32_t a_tmem = tmem_base + kTcACols * b;
        const uint32_t x0 = sb + s * kTcSlot + kTcWBytes;
        // k outer, blocks inner: consecutive MMAs go to the four partial sums in turn.
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
          for (int blk = 0; blk < 4; ++blk)
            tc_mma_i8_tmem_a(d_tmem + kTcTok * blk, a_tmem + (blk * 4 + k) * 8,
                             sw128_kmajor_desc(x0 + blk * (kTcTok * 128)) + 2 * k, kTcIdesc, (st | k) != 0);
        issued = true;
        tc_commit(empty_bar(s));   // the stage's codes are read
        tc_commit(aempty_bar(b));  // the A buffer is read
        if (st == nst - 1) {
          dtag[d] = unit;
          tc_commit(dfull_bar(d));
          mbar_arrive(dfull_bar(d));
          ++uc;
        }
        ++it;
      }
      (void)ok;
      if (issued) {
        // Every MMA is finished before tensor memory is released.
        tc_commit(done_bar);
        const WaitCtl drain{nullptr, never, 100000000ull};
        mbar_wait(done_bar, 0, drain);
      }
    }
  } else if (warp < kTcEpiWarp0) {
    // ---- unpack: one weight row per thread; group g takes stages g, g + 2, ... ----
    const int q = warp & 3, group = (warp - 2) / kTcGroupWarps;
    const int r = 32 * q + lane;  // weight row of the unit = tensor-memory lane
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    int it = group;
    while (true) {
      const int s = it % kTcRing, b = it % kTcABufs;
      const bool got = mbar_wait(full_bar(s), (it / kTcRing) & 1, ctl);
      if (!__all_sync(0xffffffffu, got)) break;
      if (tags[s] == kTcTagEnd) break;
      const bool free_a = mbar_wait(aempty_bar(b), ((it / kTcABufs) & 1) ^ 1, ctl);
      if (!__all_sync(0xffffffffu, free_a)) break;
      tc_fence_after();
      // The row's 8 chunks (128-byte swizzle: chunk c at c ^ (r & 7)).
      const uint32_t row = sb + s * kTcSlot + r * 128;
      uint4 pk[8];
#pragma unroll
      for (int c = 0; c < 8; ++c)
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(pk[c].x), "=r"(pk[c].y), "=r"(pk[c].z), "=r"(pk[c].w)
                     : "r"(row + ((c ^ (r & 7)) << 4)));
#pragma unroll
      for (int part = 0; part < 4; ++part) {
        // Packed words 8 part .. +7: word g holds inputs 16g .. 16g + 15 of the
        // stage; (w >> 2j) & 0x03030303 are inputs 16g + 4j .. +3 = column 4g + j.
        uint32_t out[32];
#pragma unroll
        for (int wi = 0; wi < 8; ++wi) {
          const uint4 v = pk[2 * part + (wi >> 2)];
          const uint32_t w = (wi & 3) == 0 ? v.x : (wi & 3) == 1 ? v.y : (wi & 3) == 2 ? v.z : v.w;
#pragma unroll
          for (int j = 0; j < 4; ++j) out[4 * wi + j] = (w >> (2 * j)) & 0x03030303u;
        }
        tmem_st_32x32b_x32(tmem_base + lane_base + kTcACols * b + 32 * part, out);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(afull_bar(b));
        mbar_arrive(empty_bar(s));  // the stage's packed words are consumed
      }
      it += kTcUnpackGroups;
    }
  } else {
    // ---- epilogue ----
    griddep_wait();  // scales and row sums come from the preceding kernel
    const int q = warp & 3;
    const int r = 32 * q + lane;
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    int uc = 0;
    while (true) {
      const int d = uc & 1;
      const bool got = mbar_wait(dfull_bar(d), (uc >> 1) & 1, ctl);
      if (!__all_sync(0xffffffffu, got)) break;
      const int unit = dtag[d];
      if (unit == kTcTagEnd) break;
      tc_fence_after();
      uint32_t v[16], p[16];
      tmem_ld_32x32b_x16(tmem_base + lane_base + kTcDCol0 + kTcDCols * d, v);
#pragma unroll
      for (int blk = 1; blk < 4; ++blk) {
        tmem_ld_32x32b_x16(tmem_base + lane_base + kTcDCol0 + kTcDCols * d + kTcTok * blk, p);
        tmem_ld_wait();
#pragma unroll
        for (int m = 0; m < kTcTok; ++m) v[m] += p[m];
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dempty_bar(d));
      const TcLayer& L = P.layer[layer_of(unit)];
      const int n = (unit - L.unit0) * kTcRows + r;
      if (n < L.N) {
        const float gamma = __ldg(L.gamma);
        TY* y = static_cast<TY*>(L.y);
#pragma unroll
        for (int m = 0; m < kTcTok; ++m) {
          if (m < M) {
            const int a = static_cast<int>(v[m]) - __ldcg(L.rowsum + m);
            const float val = __fmul_rn(static_cast<float>(a), __fdiv_rn(gamma, __ldcg(L.scale + m)));
            const size_t o = static_cast<size_t>(m) * L.N + n;
            if constexpr (sizeof(TY) == 4) y[o] = val; else y[o] = __float2bfloat16_rn(val);
            if (L.acc_out) L.acc_out[o] = a;
          }
        }
      }
      ++uc;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTcTmemCols);
  }
  // The block that finishes last resets the ticket counter for the next launch.
  if (P.one_unit) return;
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(P.tickets + 1, 1u) == gridDim.x - 1) {
      atomicExch(P.tickets, 0u);
      atomicExch(P.tickets + 1, 0u);
    }
  }
}

}  // namespace

bool gemv_tc_eligible(const GemvLayerArgs* layers, int n_layers, int M) {
  if (M < 2 || M > kTcTok || n_layers < 1 || n_layers > kTcMaxLayers) return false;
  for (int i = 0; i < n_layers; ++i)
    if (layers[i].ldx % 128 != 0 || layers[i].ldx < layers[i].K) return false;
  return true;
}

cudaError_t launch_gemv_tc(const GemvLayerArgs* layers, int n_layers, int M, int y_type, uint32_t* status,
                           uint32_t* tickets, cudaStream_t stream, bool pdl) {
  if (!gemv_tc_eligible(layers, n_layers, M)) return cudaErrorInvalidValue;
  EncodeTiledFn enc = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
  if (!enc) return cudaErrorNotSupported;
  // Largest K first: the longest units are handed out first.
  int order[kTcMaxLayers];
  for (int i = 0; i < n_layers; ++i) order[i] = i;
  for (int i = 1; i < n_layers; ++i)
    for (int j = i; j > 0 && layers[order[j]].K > layers[order[j - 1]].K; --j) {
      const int t = order[j];
      order[j] = order[j - 1];
      order[j - 1] = t;
    }
  TcParams P;
  memset(&P, 0, sizeof(P));
  int units = 0;
  for (int i = 0; i < n_layers; ++i) {
    const GemvLayerArgs& a = layers[order[i]];
    TcLayer& L = P.layer[i];
    {
      const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K / 4), static_cast<cuuint64_t>(a.N)};
      const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K / 4)};
      const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(kTcRows)};
      const cuuint32_t estr[2] = {1, 1};
      if (enc(&L.wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.packed), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
    {
      // Codes [M][ldx] as [ldx/128 blocks][M tokens][128 bytes]: a box is 4
      // blocks of 16 token rows (rows past M and blocks past ldx read as zero).
      const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(M), static_cast<cuuint64_t>(a.ldx / 128)};
      const cuuint64_t strides[2] = {static_cast<cuuint64_t>(a.ldx), 128};
      const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(kTcTok), 4};
      const cuuint32_t estr[3] = {1, 1, 1};
      if (enc(&L.xmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(a.x), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
    L.scale = a.scale;
    L.rowsum = a.rowsum;
    L.gamma = a.gamma;
    L.y = a.y;
    L.acc_out = a.acc_out;
    L.N = a.N;
    L.K = a.K;
    L.unit0 = units;
    units += (a.N + kTcRows - 1) / kTcRows;
  }
  P.n_layers = n_layers;
  P.M = M;
  P.total_units = units;
  P.status = status;
  P.tickets = tickets;
  const int sms = num_sms();
  const int grid = units < sms ? units : sms;
  P.one_unit = units <= grid ? 1 : 0;
  static std::atomic<uint64_t> attr_done[2];  // per output type and device
  const int yi = y_type == kOutBF16 ? 1 : 0;
  auto kernel = yi ? gemv_tc_kernel<__nv_bfloat16> : gemv_tc_kernel<float>;
  cudaError_t e = once_per_device(attr_done[yi], [&] {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemBytes);
  });
  if (e != cudaSuccess) return e;
  return launch(kernel, dim3(grid), dim3(kTcThreads), static_cast<size_t>(kTcSmemBytes), stream, pdl, P);
}

}  // namespace bl
