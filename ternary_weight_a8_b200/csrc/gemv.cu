// Decode product (M <= 16 tokens) for one BitLinear or a group of independent
// BitLinears: packed ternary weights x int8 activations, int32 accumulation,
// fused dequantisation, in one persistent launch.
//
// "BitNet's Real Bet: Designing the Whole Inference Stack", section "A
// low-bit model is a whole-stack design": the GPU path moves packed weights
// from HBM to shared memory, unpacks them and computes with the per-token
// 8-bit activations.  "BitNet b1.58 and the 1-Bit AI Architecture
// Revolution", section "The Energy Revolution": the product is integer
// additions; here they run on the tensor cores' int8 path (mma.sync
// m16n8k32, u8 x s8 -> s32) for two or more tokens, and as byte dot products
// (dp4a) for one token.
//
// Decode streams every weight byte once, so the kernel is built around one
// uninterrupted weight stream per SM:
//  * Work unit: 64 output rows of one layer over all of its K (32 rows for one
//    token; three blocks per SM).  Units are
//    ordered largest-K layer first; each block takes its first unit by index
//    and the rest from a ticket counter in the workspace, so the blocks end
//    within a fraction of a unit of one another.  The block that finishes
//    last resets the counter for the next launch.  With no more units than
//    blocks, each block takes its own unit and the counter is not touched.
//  * One producer thread streams the block's units with TMA in stages of 64
//    rows x 256 bytes (1024 inputs, two 128-byte halves), in the 128-byte
//    swizzle so that the lanes' 16-byte reads are conflict-free, through a deep ring of
//    mbarrier-tracked buffers that runs on from one unit to the next.  A whole
//    ring of the first unit's weight loads is issued before the
//    grid-dependency wait (programmatic dependent launch): weights never
//    depend on the preceding kernel, so they stream while it still runs.
//  * Activations quantised by the quantisation kernel stream with the
//    weights: each stage also brings the stage's 1024 inputs of every token,
//    loaded through a 3-D tensor map (token, 128-input block, byte) in the
//    128-byte swizzle, so shared-memory row 4m + q holds block q of token m
//    and the fragment reads of the eight lanes of a phase hit eight
//    different 16-byte bank groups.  Tiny activations (a one-token step of a
//    small model) are instead quantised by the block itself in one read
//    (per-token absmax over all of K, s = 127 / max(amax, 1e-5),
//    q = rint(x * s)) and staged whole, the 16-byte chunks of every 128-byte
//    block rotated by twice the block index; that saves a launch.
//  * Two or more tokens: each lane takes 16-byte chunks 2t and 2t+1 of rows g and g+8 of its
//    warp's 16 rows into registers; a warp releases a stage once it has
//    read everything it needs from it (at once when the activations are
//    staged whole, after the stage's products when they stream with it).
//    Unpacking is one AND per four weights: mask 0x03030303 << 2j keeps the
//    codes of elements 4j..4j+3 of a word in place (scaled by 4^j); four
//    accumulator sets, one per j, are shifted back and added at the end,
//    exact because each set is a multiple of 4^j.  The k order inside an mma
//    is free as long as both operands agree, so lane (g, t) feeds its own
//    words to the A fragment and the matching activation bytes to B.
//  * One token: the mma's eight token columns would be seven-eighths idle, and
//    one warp per SM sub-partition issues mma.sync too slowly for a short,
//    latency-bound step.  Lane (rs, ch) instead takes 16-byte chunk ch of rows
//    rs, rs+4, rs+8, rs+12 of its warp's 16 and the matching 64 codes: the
//    same AND per four weights, then one dp4a (unsigned codes x signed codes)
//    per four weights into the four accumulator sets; the eight lanes of a
//    row group finish with a three-step butterfly.  Without a split the unit
//    is 32 rows over stages of 2048 inputs (narrow units: each half-stage
//    holds the 32 rows over two 512-input ranges 1024 apart, so a lane's four
//    rows are two rows over two ranges): twice the units, each half as long,
//    so the blocks end closer together (with in-kernel quantisation only when
//    the 64-row units would leave SMs idle).
//  * Short, wide layers (few 64-row units for the SMs) are split along K: a
//    cluster of ks CTAs shares each unit, rank r taking the contiguous stage
//    range [r*nst/ks, (r+1)*nst/ks).  Every CTA folds its accumulator sets per
//    lane; ranks 1..ks-1 leave them in their own shared memory and arrive on
//    rank 0's mbarrier (release, cluster scope); rank 0 reads them through
//    distributed shared memory, adds them and finishes the unit.  A cluster
//    barrier at the end keeps every CTA alive while a peer may still read its
//    shared memory or arrive on its barrier.  The split is a template
//    parameter, so launches that do not split run none of its code.
//  * Stored codes are c = t + 1: acc = sum c*q - sum q, and
//    y = acc * (gamma / s) is stored straight from registers.
//  * The kernel is specialised on the number of token slots (1, 2, 4, 8 or
//    16), so a one-token decode does no work for absent tokens.
//  * The FFN's gate and up BitLinears can run as one launch that also forms
//    h = act(gate) * up and quantises it for the down BitLinear (GvGlu below).
#include <cuda.h>
#include <cuda_bf16.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

namespace bl {

constexpr int kGvWarps = 4;
constexpr int kGvRows = 16 * kGvWarps;           // 64 rows per unit
constexpr int kGvStageK = 1024;                  // inputs per stage
constexpr int kGvStageBytes = kGvRows * 256;     // 16 KB of packed weights (two 128-byte halves)
constexpr int kGvThreads = 32 * (kGvWarps + 1);  // + one producer warp
constexpr int kGvConsumers = 32 * kGvWarps;
constexpr int kGvBlocksPerSM = 3;
constexpr int kGvSmemPerBlock = 75 * 1024;
constexpr int kGvMaxRing = 16;
constexpr int kGvMaxSplit = 8;        // CTAs of a cluster sharing one unit (the portable cluster limit)
constexpr int kGvTagEnd = -1;
constexpr int kGvFuseChunks = 2;      // 16-input chunks a consumer thread quantises itself
constexpr int kGvFuseChunks1 = 5;     // the same for one bf16 token of a single layer
constexpr int kGvFuseElems = 4096;    // M*K up to which the blocks quantise activations themselves

struct GvLayer {
  CUtensorMap tmap;  // packed weights [N][K/4]: box 128 bytes x 64 rows, 128-byte swizzle
  CUtensorMap xmap;  // int8 codes as [M][K/128][128]: box 128 x 4 x token slots, 128-byte swizzle
  const void* x;     // raw activations (quantised in the kernel) or int8 codes
  const float* scale;
  const int32_t* rowsum;
  const float* gamma;
  void* y;
  int32_t* acc_out;
  int N, K, unit0;  // unit0: index of the layer's first unit
};

// Shared-memory bytes of half a stage's activation tile: token slots x 4 blocks x 128,
// rounded to the 1024-byte period of the 128-byte swizzle.
__host__ __device__ constexpr int x_half_bytes(int tt) { return ((tt * 4 * 128 + 1023) / 1024) * 1024; }

// The FFN's gate and up BitLinears in one launch, with the gated activation
// and the quantisation of its result (the down BitLinear's input) done by the
// same launch.  With two or more tokens a unit is 32 output rows: each
// half-stage of its weights holds those 32 gate rows, then the same 32 up
// rows, so that a lane's mma fragment (rows g and g + 8 of its warp's 16)
// holds the gate and up sums of one output row.  With one token a unit is 16
// output rows over stages of 2048 inputs: each half-stage holds the 16 gate
// rows over two 512-input ranges 1024 apart, then the same up rows over the
// same ranges, so that a dp4a lane holds both sums of one row.  The lane
// rounds both outputs to the activation type, as stored outputs are, forms
// h = act(gate) * up, stores h and keeps the warp's running maximum of |h|
// per token in registers.  When the units run out, the block folds its
// warps' maxima in shared memory, publishes them (one atomic max per token,
// each token's word on a 128-byte line of its own) and counts itself done,
// with one fence.  Then the quantisation is spread over the grid: global warp
// w takes the 512-element slices w, w + W, ... of h (W warps in the grid);
// its block waits until every block is done, quantises with the final
// per-token scale and adds its code sums, then counts itself finished; the
// last block to finish writes the scales and code sums.
struct GvGlu {
  int on;
  int act;                // kGluRelu2 or kGluSilu
  int gate, up;           // their layer slots
  int q_warps;            // warps with quantisation slices: min(slices, warps in the grid)
  int q_blocks;           // blocks holding those warps
  void* h;                // [M][N] h, activation type
  int8_t* xq;             // [M][N] codes of h
  float* scale;           // [M]
  int32_t* rowsum;        // [M]
  uint32_t* amax;         // per token m, word 32 m: max |h| as float bits; zero at launch
  int32_t* rsum;          // per token m, word 32 m: sum of h's codes; zero at launch
  uint32_t* done;         // [2] zero at launch: blocks done with units, quantisation blocks finished
};

struct GvParams {
  GvLayer layer[kGvMaxLayers];
  int n_layers, M, total_units, nring, x_pitch;
  uint32_t* status;
  uint32_t* tickets;  // [0] next ticket, [1] blocks done
  int one_unit;       // as many blocks as units: each block takes its own unit, no tickets
  int ksplit;         // CTAs of a cluster that share one unit, each over its own range of stages
  int narrow;         // 32-row units of 2048-input stages (one token, streamed codes, ksplit 1)
  GvGlu glu;          // the fused gate/up launch (ksplit is 1 then)
};

// Stages [sb, se) of a unit with nst stages taken by cluster rank `rank` of `ks`.
__host__ __device__ inline void stage_range(int nst, int ks, int rank, int& sb, int& se) {
  sb = rank * nst / ks;
  se = (rank + 1) * nst / ks;
}

// Shared-memory bytes of one CTA's partial sums in a K-split launch: one
// 16-byte vector per consumer thread and mma token group.
__host__ __device__ constexpr int gv_part_bytes(int tt) { return ((tt + 7) / 8) * kGvConsumers * 16; }

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

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// Sum of the four products of unsigned bytes of a with signed bytes of b, plus c.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
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

// The same barrier, returning the OR of every consumer thread's `v` (one
// decision for the whole block).
__device__ __forceinline__ bool consumer_sync_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(v ? 1u : 0u), "n"(kGvConsumers)
      : "memory");
  return r != 0;
}

// Byte offset of activation chunk (16 bytes) `c` of a staged token row.
__device__ __forceinline__ int x_chunk_off(int c) {
  const int blk = c >> 3, ci = c & 7;
  return blk * 128 + (((ci + 2 * (blk & 3)) & 7) << 4);
}

// Low bytes of four ints, packed little-endian into one word.
__device__ __forceinline__ uint32_t pack4_s8(int a, int b, int c, int d) {
  const uint32_t lo = __byte_perm(static_cast<uint32_t>(a), static_cast<uint32_t>(b), 0x5140);
  const uint32_t hi = __byte_perm(static_cast<uint32_t>(c), static_cast<uint32_t>(d), 0x5140);
  return __byte_perm(lo, hi, 0x5410);
}

// Sum of the 16 signed bytes of a chunk.
__device__ __forceinline__ int byte_sum16(const uint4& v) {
  int s = __dp4a(static_cast<int>(v.x), 0x01010101, 0);
  s = __dp4a(static_cast<int>(v.y), 0x01010101, s);
  s = __dp4a(static_cast<int>(v.z), 0x01010101, s);
  return __dp4a(static_cast<int>(v.w), 0x01010101, s);
}

// One chunk of 16 raw activations, held as loaded.
struct RawChunk {
  uint4 v[4];  // bf16: v[0..1]; fp32: v[0..3]
};

template <typename TX>
__device__ __forceinline__ void load_chunk(const TX* p, RawChunk& r) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
  r.v[0] = __ldcg(q);
  r.v[1] = __ldcg(q + 1);
  if constexpr (sizeof(TX) == 4) {
    r.v[2] = __ldcg(q + 2);
    r.v[3] = __ldcg(q + 3);
  }
}

template <typename TX>
__device__ __forceinline__ float chunk_elem(const RawChunk& r, int e) {
  if constexpr (sizeof(TX) == 4) {
    return __uint_as_float(u4_get(r.v[e >> 2], e & 3));
  } else {
    const uint32_t w = u4_get(r.v[e >> 3], (e >> 1) & 3);  // bf16 -> fp32 is exact
    return __uint_as_float((e & 1) ? (w & 0xffff0000u) : (w << 16));
  }
}

// Reduction of one value per thread over the threads of each token group
// (group = kGvConsumers / TT consecutive consumer threads).  Returns the
// group's result in every thread of the group.
template <int TT, bool kMax>
__device__ __forceinline__ float group_reduce(float v, float* scratch) {
  constexpr int G = kGvConsumers / TT;
  constexpr int lanes = G < 32 ? G : 32;
#pragma unroll
  for (int o = lanes / 2; o > 0; o >>= 1) {
    const float u = __shfl_xor_sync(0xffffffffu, v, o);
    v = kMax ? fmaxf(v, u) : v + u;
  }
  if constexpr (G <= 32) {
    return v;
  } else {
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) scratch[warp] = v;
    consumer_sync();
    const int w0 = (warp / (G / 32)) * (G / 32);
    float r = scratch[w0];
    for (int w = 1; w < G / 32; ++w) r = kMax ? fmaxf(r, scratch[w0 + w]) : r + scratch[w0 + w];
    consumer_sync();
    return r;
  }
}

template <int TT>
__device__ __forceinline__ int group_reduce_int(int v, int* scratch) {
  constexpr int G = kGvConsumers / TT;
  constexpr int lanes = G < 32 ? G : 32;
#pragma unroll
  for (int o = lanes / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if constexpr (G <= 32) {
    return v;
  } else {
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) scratch[warp] = v;
    consumer_sync();
    const int w0 = (warp / (G / 32)) * (G / 32);
    int r = scratch[w0];
    for (int w = 1; w < G / 32; ++w) r += scratch[w0 + w];
    consumer_sync();
    return r;
  }
}

// Stages layer L's activations for all tokens: int8 codes in the rotated
// layout at xs, the token scales and the code sums in shared memory.
template <int TT, typename TX>
__device__ __forceinline__ void stage_activations(const GvLayer& L, int M, uint32_t xs, int x_pitch,
                                                  float* s_tok, int* rs_tok, float* scratch) {
  constexpr int G = kGvConsumers / TT;  // threads per token slot
  const int tid = threadIdx.x;
  const int m = tid / G, j = tid % G;
  const int K = L.K;
  const int chunks = K >> 4;
  {
    // At most kChunks chunks per thread (the host keeps M*K within that).
    constexpr int kChunks = sizeof(TX) == 4 ? kGvFuseChunks / 2 : TT == 1 ? kGvFuseChunks1 : kGvFuseChunks;
    RawChunk raw[kChunks];
    const TX* src = static_cast<const TX*>(L.x) + static_cast<size_t>(m) * K;
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
      const int c = j + i * G;
      if (m < M && c < chunks) load_chunk<TX>(src + c * 16, raw[i]);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
      const int c = j + i * G;
      if (m < M && c < chunks) {
#pragma unroll
        for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(chunk_elem<TX>(raw[i], e)));
      }
    }
    amax = group_reduce<TT, true>(amax, scratch);
    const float s = __fdiv_rn(127.0f, fmaxf(amax, 1e-5f));
    int rs = 0;
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
      const int c = j + i * G;
      if (m < M && c < chunks) {
        uint32_t w[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          int q[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            q[e] = __float2int_rn(__fmul_rn(chunk_elem<TX>(raw[i], 4 * b + e), s));
            q[e] = min(max(q[e], -128), 127);
          }
          w[b] = pack4_s8(q[0], q[1], q[2], q[3]);
          rs = __dp4a(static_cast<int>(w[b]), 0x01010101, rs);
        }
        sts128(xs + m * x_pitch + x_chunk_off(c), make_uint4(w[0], w[1], w[2], w[3]));
      }
    }
    rs = group_reduce_int<TT>(rs, reinterpret_cast<int*>(scratch));
    if (j == 0 && m < TT) {
      rs_tok[m] = rs;
      s_tok[m] = s;
    }
  }
  consumer_sync();
}

// ---------------------------------------------------------------------------
// The gated activation and its quantisation inside the gate/up launch
// ---------------------------------------------------------------------------
template <typename TY>
__device__ __forceinline__ float ld_act(const void* p, size_t i) {
  if constexpr (sizeof(TY) == 4) {
    return __ldcg(static_cast<const float*>(p) + i);
  } else {
    const unsigned short b = __ldcg(static_cast<const unsigned short*>(p) + i);
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
  }
}

static_assert(kGluRelu2 == 0 && kGluSilu == 1, "glu_value's activation codes");

// Polls a counter in global memory (lane 0) until it reaches `target`;
// bounded like every wait.  Warp-uniform result.
__device__ __forceinline__ bool wait_count(const uint32_t* p, uint32_t target, const WaitCtl& ctl) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) {
    const uint64_t t0 = global_ns();
    while (true) {
      uint32_t v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
      if (v >= target) break;
      if (*ctl.abort) { ok = false; break; }
      if (global_ns() - t0 > ctl.limit_ns) {
        *ctl.abort = 1;
        if (ctl.status) atomicOr(ctl.status, kStatusTimeout);
        ok = false;
        break;
      }
      __nanosleep(256);
    }
  }
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  __syncwarp();
  return ok;
}

// Token m's word of a per-token array of the fused gate/up launch: one
// 128-byte line each, so that atomics on different tokens meet in different
// L2 slices.
constexpr int kGluTokStride = 32;

// The consumer warps of a block of the fused gate/up launch are done with
// their units (every consumer warp calls this once, also after giving up, so
// that the barriers match): their per-token maxima of |h| are folded through
// `red` (64 floats of this block's shared memory, free once every consumer
// warp is past its last stage) and published with one atomic max per token;
// then the block's h stores and those maxima are made visible (the barrier
// orders the other warps' stores before warp 0's fence) and the block is
// counted.  A block that gave up publishes nothing (the others' waits run out).
template <int TG, bool kAlu>
__device__ __forceinline__ void glu_block_done(const GvParams& P, const float (&hmax)[TG][2], float* red,
                                               const WaitCtl& ctl) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Every consumer warp is past the ring before it is reused; one decision on giving up.
  if (consumer_sync_or(*ctl.abort != 0)) return;
  if constexpr (kAlu) {
    if (lane == 0) red[warp * 16] = hmax[0][0];
  } else {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int tg = 0; tg < TG; ++tg)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int m = tg * 8 + 2 * t + e;
        if (g == 0 && m < P.M) red[warp * 16 + m] = hmax[tg][e];
      }
  }
  consumer_sync();
  if (warp == 0) {
    if (lane < P.M) {
      float v = red[lane];
#pragma unroll
      for (int w = 1; w < kGvWarps; ++w) v = fmaxf(v, red[w * 16 + lane]);
      if (v > 0.0f) atomicMax(P.glu.amax + kGluTokStride * lane, __float_as_uint(v));
    }
    __syncwarp();
    if (lane == 0) {
      __threadfence();
      atomicAdd(P.glu.done, 1u);
    }
  }
}

// The quantisation of h ([M][N], N % 16 == 0, so no 16-element chunk crosses
// a token) by this warp: slices of 512 elements, one 16-element chunk per
// lane, once every consumer warp of the grid is done with its units.  Codes
// as the quantisation kernel makes them: s = 127 / max(amax, 1e-5),
// q = clamp(rint(h * s), -128, 127).
constexpr int kGluSlice = 512;

template <typename TY>
__device__ __noinline__ void glu_quant_slices(const GvParams& P, int N, const WaitCtl& ctl) {
  const GvGlu& G = P.glu;
  if (static_cast<int>(blockIdx.x) >= G.q_blocks) return;  // block-uniform
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, M = P.M;
  const int W = static_cast<int>(gridDim.x) * kGvWarps;
  const int gw = static_cast<int>(blockIdx.x) * kGvWarps + warp;
  // Warp 0 waits for every block; the barrier passes the outcome on (and
  // orders warp 0's acquire before the other warps' loads of h).
  bool bad = false;
  if (warp == 0) bad = !wait_count(G.done, gridDim.x, ctl);
  if (consumer_sync_or(bad || *ctl.abort != 0)) return;  // (every warp returns: no barrier follows)
  const long long total = static_cast<long long>(M) * N;
  for (long long e = static_cast<long long>(gw) * kGluSlice + 16 * lane; gw < G.q_warps && e < total;
       e += static_cast<long long>(W) * kGluSlice) {
    const int m = static_cast<int>(e / N);
    const float s = __fdiv_rn(127.0f, fmaxf(__uint_as_float(__ldcg(G.amax + kGluTokStride * m)), 1e-5f));
    float hv[16];
    if constexpr (sizeof(TY) == 4) {
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(G.h) + e);
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const float4 v = __ldcg(src + b);
        hv[4 * b] = v.x;
        hv[4 * b + 1] = v.y;
        hv[4 * b + 2] = v.z;
        hv[4 * b + 3] = v.w;
      }
    } else {
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const unsigned short*>(G.h) + e);
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const uint4 v = __ldcg(src + b);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          hv[8 * b + 2 * k] = __uint_as_float(w4[k] << 16);
          hv[8 * b + 2 * k + 1] = __uint_as_float(w4[k] & 0xffff0000u);
        }
      }
    }
    uint32_t w[4];
    int sum = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      int c[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        c[k] = __float2int_rn(__fmul_rn(hv[4 * b + k], s));
        c[k] = min(max(c[k], -128), 127);
      }
      w[b] = pack4_s8(c[0], c[1], c[2], c[3]);
      sum = __dp4a(static_cast<int>(w[b]), 0x01010101, sum);
    }
    *reinterpret_cast<uint4*>(G.xq + e) = make_uint4(w[0], w[1], w[2], w[3]);
    // One atomic per warp when the warp's chunks are of one token.
    const unsigned active = __activemask();
    const int lead = __ffs(active) - 1;
    const int m0 = __shfl_sync(active, m, lead);
    if (__all_sync(active, m == m0)) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(active, sum, o);
      if (lane == lead) atomicAdd(G.rsum + kGluTokStride * m, sum);
    } else {
      atomicAdd(G.rsum + kGluTokStride * m, sum);
    }
  }
  // The block that finishes the last quantisation work writes the scales and code sums.
  consumer_sync();
  if (warp == 0) {
    uint32_t old = 0;
    if (lane == 0) {
      __threadfence();
      old = atomicAdd(G.done + 1, 1u);
    }
    old = __shfl_sync(0xffffffffu, old, 0);
    if (static_cast<int>(old) == G.q_blocks - 1) {
      __threadfence();
      if (lane < M) {
        G.scale[lane] = __fdiv_rn(127.0f, fmaxf(__uint_as_float(__ldcg(G.amax + kGluTokStride * lane)), 1e-5f));
        G.rowsum[lane] = __ldcg(G.rsum + kGluTokStride * lane);
      }
    }
  }
}

// kMode: 0 plain, 1 K-split over clusters, 2 the fused gate/up launch,
// 3 narrow units (one token).
template <int TT, typename TY, typename TX, int kMode>
__global__ void __launch_bounds__(kGvThreads, kGvBlocksPerSM) gemv_group_kernel(const __grid_constant__ GvParams P) {
  constexpr bool kSplit = kMode == 1;
  constexpr bool kGlu = kMode == 2;
  constexpr bool kNarrow = kMode == 3;
  constexpr int TG = (TT + 7) / 8;           // mma token groups of 8
  constexpr bool kStream = sizeof(TX) == 1;  // int8 codes stream with the weights
  constexpr bool kAlu = TT == 1;             // one token: dp4a dot products instead of the mma path
  static_assert(!kNarrow || kAlu, "narrow units are a one-token form");
  // The fused gate/up launch at one token: units of 16 gate and the same 16
  // up rows over stages of 2048 inputs (each half-stage: the gate rows over two
  // 512-input ranges 1024 apart, then the up rows over the same ranges).
  constexpr bool kGluNarrow = kGlu && kAlu;
  constexpr bool kWide = kNarrow || kGluNarrow;  // stages of 2048 inputs
  // Inputs per stage: a narrow unit's stage is 32 rows of twice the inputs.
  constexpr int kStageIn = kWide ? 2 * kGvStageK : kGvStageK;
  constexpr int kXHalf = x_half_bytes(TT);   // one half-stage activation tile
  constexpr int kSlot = kGvStageBytes + (kStream ? 2 * kXHalf : 0);
  static_assert(!kWide || !kStream || 2 * kXHalf >= 16 * 128, "a 2048-input stage's codes: 16 blocks of 128");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nring = P.nring, M = P.M;
  const uint32_t sb = smem_u32(smem);
  const uint32_t ring = sb;
  const uint32_t xs = sb + nring * kSlot;  // whole-K activations (in-kernel quantisation only)
  const int ks = kSplit ? P.ksplit : 1;    // CTAs sharing one unit (a cluster of ks)
  const int x_bytes = kStream ? 0 : ((M * P.x_pitch + 127) / 128) * 128;
  const uint32_t part = xs + x_bytes;      // this CTA's partial sums (K-split only)
  uint8_t* misc = smem + nring * kSlot + x_bytes + (ks > 1 ? gv_part_bytes(TT) : 0);
  float* s_tok = reinterpret_cast<float*>(misc);          // [16]
  int* rs_tok = reinterpret_cast<int*>(misc + 64);         // [16]
  float* scratch = reinterpret_cast<float*>(misc + 128);   // [kGvWarps]
  int* tags = reinterpret_cast<int*>(misc + 160);          // [kGvMaxRing]: unit of each stage
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 224);
  volatile int* never = abort_flag + 1;
  const uint32_t bar0 = smem_u32(misc + 256);              // full[nring], empty[nring], then red
  const uint32_t red_bar = bar0 + 16 * nring;              // K-split: the peers' partial sums are in place
  const int rank = ks > 1 ? static_cast<int>(blockIdx.x) % ks : 0;
  const int unit_first = static_cast<int>(blockIdx.x) / ks;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < nring; ++i) {
      mbar_init(bar0 + 8 * i, 1);
      mbar_init(bar0 + 8 * (nring + i), kGvWarps);
    }
    if (ks > 1) mbar_init(red_bar, (ks - 1) * kGvWarps);
    *abort_flag = 0;
    *never = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (ks > 1) cluster_sync_all();  // the peers' barriers are initialised before any remote arrive
  griddep_launch_dependents();
  const WaitCtl ctl{P.status, abort_flag, kWaitLimitNs};

  if (warp == kGvWarps) {
    // ---- producer: one thread streams the block's units ----
    if (lane == 0) {
      int slot = 0, phase = 0, issued = 0;
      bool waited = false;  // grid dependency
      bool ok = true;
      int unit = unit_first;
      // The layer, row block and stage range of a unit.  A unit of the fused
      // gate/up launch is 32 output rows (16 at one token, over 2048-input
      // stages; see GvGlu).  A narrow unit is 32 rows too: each half-stage
      // holds them over one 512-input range, then over the range 1024 inputs
      // further on.
      auto locate = [&](int u, const GvLayer*& Lp, int& rb, int& s0, int& s1) {
        if constexpr (kGlu) {
          Lp = &P.layer[P.glu.gate];
          rb = u;
          s0 = 0;
          s1 = (Lp->K + kStageIn - 1) / kStageIn;
        } else {
          int l = 0;
          while (l + 1 < P.n_layers && u >= P.layer[l + 1].unit0) ++l;
          Lp = &P.layer[l];
          rb = u - Lp->unit0;
          stage_range((Lp->K + kStageIn - 1) / kStageIn, ks, rank, s0, s1);
        }
      };
      auto load_weights = [&](const GvLayer& L, int rb, int st, uint32_t full, uint32_t dst) {
        if constexpr (kGluNarrow) {
          const GvLayer& LU = P.layer[P.glu.up];
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int b = 0; b < 4; ++b)  // gate range 0, gate range 1, up range 0, up range 1
              tma_load_2d(dst + hf * (kGvStageBytes / 2) + b * (kGvRows / 4) * 128, b < 2 ? &L.tmap : &LU.tmap,
                          (2 * st + (b & 1)) * 256 + hf * 128, rb * (kGvRows / 4), full);
        } else if constexpr (kGlu) {
          const GvLayer& LU = P.layer[P.glu.up];
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const uint32_t d = dst + hf * (kGvStageBytes / 2);
            tma_load_2d(d, &L.tmap, st * 256 + hf * 128, rb * (kGvRows / 2), full);
            tma_load_2d(d + (kGvRows / 2) * 128, &LU.tmap, st * 256 + hf * 128, rb * (kGvRows / 2), full);
          }
        } else if constexpr (kNarrow) {
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int sb = 0; sb < 2; ++sb)
              tma_load_2d(dst + hf * (kGvStageBytes / 2) + sb * (kGvRows / 2) * 128, &L.tmap,
                          (2 * st + sb) * 256 + hf * 128, rb * (kGvRows / 2), full);
        } else {
          tma_load_2d(dst, &L.tmap, st * 256, rb * kGvRows, full);
          tma_load_2d(dst + kGvStageBytes / 2, &L.tmap, st * 256 + 128, rb * kGvRows, full);
        }
      };
      // The stage's activation tiles (streamed codes), in the same slot after
      // the weights; a narrow stage's 2048 codes are one 16-block tile.
      auto load_act = [&](const GvLayer& L, int st, uint32_t full, uint32_t dst) {
        if constexpr (kWide) {
          tma_load_3d(dst + kGvStageBytes, &L.xmap, 0, 16 * st, 0, full);
        } else {
          tma_load_3d(dst + kGvStageBytes, &L.xmap, 0, 8 * st, 0, full);
          tma_load_3d(dst + kGvStageBytes + kXHalf, &L.xmap, 0, 8 * st + 4, 0, full);
        }
      };
      constexpr uint32_t kStageTx = kGvStageBytes + (!kStream ? 0 : kWide ? 16 * 128 : 2 * TT * 4 * 128);
      // The next ticket (none when each block takes only its own unit).
      auto next_unit = [&]() {
        if (P.one_unit) return P.total_units;
        if (!waited) {
          griddep_wait();  // the ticket counter is reset by the preceding launch
          waited = true;
        }
        return static_cast<int>(gridDim.x) + static_cast<int>(atomicAdd(P.tickets, 1u));
      };
      int st0 = -1;  // first stage of the current unit still to issue (-1: all)
      if constexpr (kStream) {
        // Before the grid dependency: the weights of the first unit's first
        // stages (a whole ring of them); their activation tiles, written by
        // the preceding kernel, follow once it has finished.
        if (unit < P.total_units) {
          const GvLayer* Lp;
          int rb, s0, s1;
          locate(unit, Lp, rb, s0, s1);
          const int pre = s1 - s0 < nring ? s1 - s0 : nring;
          for (int j = 0; j < pre; ++j) {  // fresh slots 0 .. pre-1
            tags[j] = unit;
            mbar_arrive_expect_tx(bar0 + 8 * j, kStageTx);
            load_weights(*Lp, rb, s0 + j, bar0 + 8 * j, ring + j * kSlot);
          }
          griddep_wait();  // the codes come from the preceding kernel
          waited = true;
          for (int j = 0; j < pre; ++j) load_act(*Lp, s0 + j, bar0 + 8 * j, ring + j * kSlot);
          issued = pre;
          slot = pre % nring;
          phase = pre == nring ? 1 : 0;
          st0 = s0 + pre;
        }
      }
      while (ok && unit < P.total_units) {
        const GvLayer* Lp;
        int rb, s0, s1;
        locate(unit, Lp, rb, s0, s1);
        for (int st = st0 >= 0 ? st0 : s0; st < s1; ++st) {
          if (!mbar_wait(bar0 + 8 * (nring + slot), phase ^ 1, ctl)) { ok = false; break; }
          tags[slot] = unit;
          const uint32_t full = bar0 + 8 * slot, dst = ring + slot * kSlot;
          mbar_arrive_expect_tx(full, kStageTx);
          load_weights(*Lp, rb, st, full, dst);
          if constexpr (kStream) {
            if (!waited) {
              griddep_wait();  // the codes come from the preceding kernel
              waited = true;
            }
            load_act(*Lp, st, full, dst);
          }
          ++issued;
          if (++slot == nring) { slot = 0; phase ^= 1; }
        }
        st0 = -1;
        if (!ok) break;
        unit = next_unit();
      }
      if (ok) {
        // End marker: one more phase on the next slot, with no data.
        if (mbar_wait(bar0 + 8 * (nring + slot), phase ^ 1, ctl)) {
          tags[slot] = kGvTagEnd;
          mbar_arrive(bar0 + 8 * slot);
        }
      } else {
        // Gave up: let copies in flight land before shared memory is released.
        const WaitCtl drain{nullptr, never, 100000000ull};
        for (int j = (issued > nring ? issued - nring : 0); j < issued; ++j)
          mbar_wait(bar0 + 8 * (j % nring), (j / nring) & 1, drain);
      }
    }
  } else {
    // ---- consumers ----
    griddep_wait();  // activations may be the preceding kernel's output
    const int g = lane >> 2, t = lane & 3;
    // The lane's two rows of the stage in the mma path: g and g + 8 of the
    // warp's 16; in the fused gate/up launch, gate row 8 * warp + g and the
    // same up row, 32 rows further on.
    const int row_lo = kGlu ? warp * 8 + g : warp * 16 + g;
    const int row_hi = kGlu ? 32 + warp * 8 + g : row_lo + 8;
    // Byte offsets of this lane's weight chunks 2t, 2t+1 of those rows within a
    // 128-byte-swizzled half-stage: chunk c of row r sits at chunk position c ^ (r & 7).
    const uint32_t w_lo0 = row_lo * 128 + (((2 * t) ^ g) << 4), w_lo1 = row_lo * 128 + (((2 * t + 1) ^ g) << 4);
    const uint32_t w_hi0 = row_hi * 128 + (((2 * t) ^ g) << 4), w_hi1 = row_hi * 128 + (((2 * t + 1) ^ g) << 4);
    // Streamed activations: row 4m + t of a half tile holds block t of token m.
    uint32_t x_row[TG];
    int x_sw[TG];
#pragma unroll
    for (int tg = 0; tg < TG; ++tg) {
      const int m = tg * 8 + g;
      x_row[tg] = (4 * m + t) * 128;
      x_sw[tg] = (4 * m + t) & 7;
    }
    const void* staged = nullptr;  // input whose activations are in shared memory (layers may share one)
    int staged_k = 0;
    int slot = 0, phase = 0;
    if constexpr (!kStream) {
      // The first unit is the block's index, so its activations can be
      // quantised while its first weight stage is still on the way.
      if (unit_first < P.total_units) {
        int l = kGlu ? P.glu.gate : 0;
        if constexpr (!kGlu) {
          while (l + 1 < P.n_layers && unit_first >= P.layer[l + 1].unit0) ++l;
        }
        stage_activations<TT, TX>(P.layer[l], M, xs, P.x_pitch, s_tok, rs_tok, scratch);
        staged = P.layer[l].x;
        staged_k = P.layer[l].K;
      }
    }
    float hmax[TG][2];      // the fused gate/up launch: this lane's running max of |h| per token
#pragma unroll
    for (int tg = 0; tg < TG; ++tg) hmax[tg][0] = hmax[tg][1] = 0.0f;
    while (true) {
      const bool got0 = mbar_wait(bar0 + 8 * slot, phase, ctl);
      if (!__all_sync(0xffffffffu, got0)) break;
      const int unit = tags[slot];
      if (unit == kGvTagEnd) {
        break;
      }
      int l = kGlu ? P.glu.gate : 0;
      if constexpr (!kGlu) {
        while (l + 1 < P.n_layers && unit >= P.layer[l + 1].unit0) ++l;
      }
      const GvLayer& L = P.layer[l];
      int s0, s1;  // this CTA's stages of the unit
      stage_range((L.K + kStageIn - 1) / kStageIn, ks, rank, s0, s1);
      if constexpr (!kStream) {
        if (L.x != staged || L.K != staged_k) {
          consumer_sync();  // every warp is done with the previous input's activations
          stage_activations<TT, TX>(L, M, xs, P.x_pitch, s_tok, rs_tok, scratch);
          staged = L.x;
          staged_k = L.K;
        }
      }

      // The epilogue's scalars, loaded now so their latency hides behind the products.
      const float gamma = __ldg(L.gamma);
      const float gamma_up = kGlu ? __ldg(P.layer[P.glu.up].gamma) : 0.0f;
      int rsum_m[TG][2];
      float s_m[TG][2];
#pragma unroll
      for (int tg = 0; tg < TG; ++tg)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int m = tg * 8 + 2 * t + e;
          rsum_m[tg][e] = 0;
          s_m[tg][e] = 1.0f;
          if constexpr (kStream && !kAlu) {
            if (m < M) {
              rsum_m[tg][e] = __ldcg(L.rowsum + m);
              s_m[tg][e] = __ldcg(L.scale + m);
            }
          }
        }

      int rsum1 = 0;  // the one-token path's epilogue scalars (every lane)
      float s1tok = 1.0f;
      if constexpr (kAlu && kStream) {
        rsum1 = __ldcg(L.rowsum);
        s1tok = __ldcg(L.scale);
      }

      int d[TG][4][4];      // mma path: accumulator fragments
      int dr[kAlu ? 4 : 1][4];   // one-token path: the lane's four rows, one set per code position j
#pragma unroll
      for (int tg = 0; tg < TG; ++tg)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int c = 0; c < 4; ++c) d[tg][j][c] = 0;
#pragma unroll
      for (int r = 0; r < (kAlu ? 4 : 1); ++r)
#pragma unroll
        for (int j = 0; j < 4; ++j) dr[r][j] = 0;
      bool ok = true;
      for (int i = s0; i < s1 && ok; ++i) {
        if (i > s0) {
          const bool got = mbar_wait(bar0 + 8 * slot, phase, ctl);
          if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        }
        const uint32_t wt = ring + slot * kSlot;
        if constexpr (kAlu) {
          // Lane (rs, ch) = (lane >> 3, lane & 7) takes 16-byte chunk ch of four
          // rows of its warp in each half (inputs 64ch .. 64ch+63 of the half)
          // and the matching 64 codes: one AND and one dp4a per four weights,
          // no idle mma columns.  Each 8-lane phase reads one 128-byte swizzled
          // row.  Rows: warp*16 + rs + 4*it; in a narrow unit the first two are
          // rows warp*8 + rs + 4*it, the last two the same rows over the inputs
          // 1024 further on; in the fused gate/up launch row warp*4 + rs of each
          // of the four boxes (gate, gate 1024 further on, up, up further on).
          const int ch = lane & 7, rs = lane >> 3;
          uint4 wv[2][4];
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int it = 0; it < 4; ++it) {
              // (one-token gate/up units: row rs of the warp's 4 in box it)
              const int row = kGluNarrow ? it * 16 + warp * 4 + rs
                              : kNarrow ? (it < 2 ? warp * 8 + rs + 4 * it : 32 + warp * 8 + rs + 4 * (it - 2))
                                        : warp * 16 + rs + 4 * it;
              wv[hf][it] = lds128(wt + hf * (kGvStageBytes / 2) + row * 128 + ((ch ^ (row & 7)) << 4));
            }
          if constexpr (!kStream) {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar0 + 8 * (nring + slot));  // the slot held only weights, now in registers
          }
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            if constexpr (kWide) {
              // Rows it < 2 over inputs (2i)*1024 + hf*512 + 64ch .. +63, rows
              // it >= 2 over the same 1024 further on (one-token gate/up
              // units: boxes it = 0, 2 over the first range, 1, 3 over the
              // second): streamed codes are block b = sb*8 + hf*4 + ch/2 of
              // the stage's 16-block tile.
#pragma unroll
              for (int sb = 0; sb < 2; ++sb) {
                const int k0 = (2 * i + sb) * kGvStageK + hf * (kGvStageK / 2) + 64 * ch;
                if (k0 < L.K) {
                  const int b = sb * 8 + hf * 4 + (ch >> 1);
                  uint4 xc[4];
#pragma unroll
                  for (int u = 0; u < 4; ++u) {
                    if constexpr (kStream) {
                      xc[u] = lds128(wt + kGvStageBytes + b * 128 + (((4 * (ch & 1) + u) ^ (b & 7)) << 4));
                    } else {
                      xc[u] = lds128(xs + x_chunk_off((k0 >> 4) + u));
                    }
                  }
#pragma unroll
                  for (int q = 0; q < 2; ++q) {
                    const int it = kGluNarrow ? sb + 2 * q : 2 * sb + q;
#pragma unroll
                    for (int v = 0; v < 4; ++v)
#pragma unroll
                      for (int j = 0; j < 4; ++j)
                        dr[it][j] = dp4a_us(u4_get(wv[hf][it], v) & (0x03030303u << (2 * j)), u4_get(xc[v], j), dr[it][j]);
                  }
                }
              }
              continue;
            }
            const int k0 = i * kGvStageK + hf * (kGvStageK / 2) + 64 * ch;
            if (k0 < L.K) {  // inputs past K have zero weights (K is a multiple of 64)
              uint4 xc[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                if constexpr (kStream) {
                  const int q = ch >> 1, ci = 4 * (ch & 1) + u;  // 128-input block; token 0 owns rows 0..3
                  xc[u] = lds128(wt + kGvStageBytes + hf * kXHalf + q * 128 + ((ci ^ q) << 4));
                } else {
                  xc[u] = lds128(xs + x_chunk_off((k0 >> 4) + u));
                }
              }
#pragma unroll
              for (int it = 0; it < 4; ++it)
#pragma unroll
                for (int v = 0; v < 4; ++v)
#pragma unroll
                  for (int j = 0; j < 4; ++j)
                    dr[it][j] = dp4a_us(u4_get(wv[hf][it], v) & (0x03030303u << (2 * j)), u4_get(xc[v], j), dr[it][j]);
            }
          }
          if constexpr (kStream) {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar0 + 8 * (nring + slot));  // done with the slot's activations too
          }
        } else {
          uint4 w[2][4];  // [half][lo0, lo1, hi0, hi1]
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const uint32_t base = wt + hf * (kGvStageBytes / 2);
            w[hf][0] = lds128(base + w_lo0);
            w[hf][1] = lds128(base + w_lo1);
            w[hf][2] = lds128(base + w_hi0);
            w[hf][3] = lds128(base + w_hi1);
          }
          if constexpr (!kStream) {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar0 + 8 * (nring + slot));  // the slot held only weights, now in registers
          }

#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const uint32_t xt = wt + kGvStageBytes + hf * kXHalf;  // streamed: this half's tile
            const int qblk = i * 8 + hf * 4 + t;                   // this lane's 128-input block (whole-K staging)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint4 wl = w[hf][h], wh = w[hf][2 + h];
#pragma unroll
              for (int p = 0; p < 2; ++p) {
                const int c0 = 4 * h + 2 * p;  // activation chunks c0, c0+1 of the lane's block
                uint4 xa[TG], xb[TG];
#pragma unroll
                for (int tg = 0; tg < TG; ++tg) {
                  const int m = tg * 8 + g;
                  if (m < M) {
                    if constexpr (kStream) {
                      const uint32_t row = xt + x_row[tg];
                      xa[tg] = lds128(row + ((c0 ^ x_sw[tg]) << 4));
                      xb[tg] = lds128(row + (((c0 + 1) ^ x_sw[tg]) << 4));
                    } else {
                      const uint32_t row = xs + m * P.x_pitch + qblk * 128;
                      xa[tg] = lds128(row + (((c0 + 2 * t) & 7) << 4));
                      xb[tg] = lds128(row + (((c0 + 1 + 2 * t) & 7) << 4));
                    }
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
          if constexpr (kStream) {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar0 + 8 * (nring + slot));  // done with the slot's activations too
          }
        }
        if (++slot == nring) { slot = 0; phase ^= 1; }
      }
      if (!ok) break;

      // This CTA's sums per lane: the four code-position sets shifted back (exact,
      // each set being a multiple of 4^j).
      int pc[TG][4];
      if constexpr (kAlu) {
#pragma unroll
        for (int r = 0; r < 4; ++r) pc[0][r] = dr[r][0] + (dr[r][1] >> 2) + (dr[r][2] >> 4) + (dr[r][3] >> 6);
        if constexpr (kNarrow) {  // rows rs and rs + 4: the two input ranges summed
          pc[0][0] += pc[0][2];
          pc[0][1] += pc[0][3];
        } else if constexpr (kGluNarrow) {  // the gate row's and the up row's sums over both ranges
          pc[0][0] += pc[0][1];
          pc[0][1] = pc[0][2] + pc[0][3];
        }
      } else if constexpr (kSplit) {  // (the mma epilogue below combines them itself otherwise)
#pragma unroll
        for (int tg = 0; tg < TG; ++tg)
#pragma unroll
          for (int c = 0; c < 4; ++c)
            pc[tg][c] = d[tg][0][c] + (d[tg][1][c] >> 2) + (d[tg][2][c] >> 4) + (d[tg][3][c] >> 6);
      }
      if (ks > 1) {
        // K-split: each CTA of the cluster holds the same lanes' sums over its own
        // stages; rank 0 adds the others' (read from their shared memory) and
        // finishes the unit.
        const uint32_t mine = part + (warp * 32 + lane) * 16;
        if (rank != 0) {
#pragma unroll
          for (int tg = 0; tg < TG; ++tg)
            sts128(mine + tg * kGvConsumers * 16, make_uint4(pc[tg][0], pc[tg][1], pc[tg][2], pc[tg][3]));
          __syncwarp();
          if (lane == 0) mbar_arrive_release_cluster(mapa_shared(red_bar, 0));
          continue;
        }
        const bool got = mbar_wait(red_bar, 0, ctl);
        if (!__all_sync(0xffffffffu, got)) break;
        fence_acq_rel_cluster();
        for (int r = 1; r < ks; ++r)
#pragma unroll
          for (int tg = 0; tg < TG; ++tg) {
            const uint4 v = ld_shared_cluster_v4(mapa_shared(mine + tg * kGvConsumers * 16, r));
            pc[tg][0] += static_cast<int>(v.x);
            pc[tg][1] += static_cast<int>(v.y);
            pc[tg][2] += static_cast<int>(v.z);
            pc[tg][3] += static_cast<int>(v.w);
          }
      }

      // Finish the unit: y = (sum c*q - sum q) * (gamma / s).  The fused
      // gate/up launch instead forms h = act(gate) * up from the lane's gate
      // and up sums of the same output row (each output rounded to the
      // activation type first, as a stored output is), stores h and folds
      // |h| into the per-token maxima.
      const int n_base =
          (kGlu ? unit : unit - L.unit0) * (kGluNarrow ? kGvRows / 4 : (kGlu || kNarrow) ? kGvRows / 2 : kGvRows);
      TY* y = static_cast<TY*>(L.y);
      if constexpr (kGluNarrow) {
        // Gate and up sums of row rs of the warp's 4, over the 8 lanes of the row group.
        int gs = pc[0][0], us = pc[0][1];
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) {
          gs += __shfl_xor_sync(0xffffffffu, gs, o);
          us += __shfl_xor_sync(0xffffffffu, us, o);
        }
        const int n = n_base + warp * 4 + (lane >> 3);
        const int rsum = kStream ? rsum1 : rs_tok[0];
        const float sm = kStream ? s1tok : s_tok[0];
        float habs = 0.0f;
        if ((lane & 7) == 0 && n < L.N) {
          const float g_v = round_to<TY>(__fmul_rn(static_cast<float>(gs - rsum), __fdiv_rn(gamma, sm)));
          const float u_v = round_to<TY>(__fmul_rn(static_cast<float>(us - rsum), __fdiv_rn(gamma_up, sm)));
          const float h = glu_value<TY>(g_v, u_v, P.glu.act);
          TY* hp = static_cast<TY*>(P.glu.h);
          if constexpr (sizeof(TY) == 4) hp[n] = h; else hp[n] = __float2bfloat16_rn(h);
          habs = fabsf(h);
        }
        habs = fmaxf(habs, __shfl_xor_sync(0xffffffffu, habs, 8));
        habs = fmaxf(habs, __shfl_xor_sync(0xffffffffu, habs, 16));
        hmax[0][0] = fmaxf(hmax[0][0], habs);
        continue;
      }
      if constexpr (kNarrow) {
        // Rows rs (lanes with ch < 4 after the first step) and rs + 4 of the
        // warp's 8, summed over the 8 lanes of the row group.
        const bool upper = (lane & 4) != 0;
        int v = (upper ? pc[0][1] : pc[0][0]) + __shfl_xor_sync(0xffffffffu, upper ? pc[0][0] : pc[0][1], 4);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        const int n = n_base + warp * 8 + (lane >> 3) + 4 * ((lane >> 2) & 1);
        if ((lane & 3) == 0 && n < L.N) {
          const int a = v - (kStream ? rsum1 : rs_tok[0]);
          const float val = __fmul_rn(static_cast<float>(a), __fdiv_rn(gamma, kStream ? s1tok : s_tok[0]));
          if constexpr (sizeof(TY) == 4) y[n] = val; else y[n] = __float2bfloat16_rn(val);
          if (L.acc_out) L.acc_out[n] = a;
        }
        continue;
      } else if constexpr (kAlu) {
        // A butterfly over the 8 lanes of a row group leaves the lane's row
        // number (lane >> 3) + 4*((lane >> 1) & 3) of the warp's 16 summed in
        // lanes 2r and 2r + 1.
        int v[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) v[r] = pc[0][r];
#pragma unroll
        for (int st = 0; st < 2; ++st) {
          const int off = 4 >> st, half = 2 >> st;
          const bool upper = (lane & off) != 0;
#pragma unroll
          for (int r = 0; r < half; ++r) {
            const int send = upper ? v[r] : v[r + half];
            const int keep_v = upper ? v[r + half] : v[r];
            v[r] = keep_v + __shfl_xor_sync(0xffffffffu, send, off);
          }
        }
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
        const int rsum = kStream ? rsum1 : rs_tok[0];
        const float sm = kStream ? s1tok : s_tok[0];
        const int n = n_base + warp * 16 + (lane >> 3) + 4 * ((lane >> 1) & 3);
        if ((lane & 1) == 0 && n < L.N) {
          const int a = v[0] - rsum;
          const float val = __fmul_rn(static_cast<float>(a), __fdiv_rn(gamma, sm));
          if constexpr (sizeof(TY) == 4) y[n] = val; else y[n] = __float2bfloat16_rn(val);
          if (L.acc_out) L.acc_out[n] = a;
        }
        continue;
      }
      if constexpr (kGlu) {
        // Fragment c holds row g (c < 2: a gate row) or g + 8 (the same up row)
        // for token 2t + (c & 1).
#pragma unroll
        for (int tg = 0; tg < TG; ++tg)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int n = n_base + warp * 8 + g;
            const int m = tg * 8 + 2 * t + e;
            float habs = 0.0f;
            if (n < L.N && m < M) {
              const int rsum = kStream ? rsum_m[tg][e] : rs_tok[m];
              const float sm = kStream ? s_m[tg][e] : s_tok[m];
              const int ag = d[tg][0][e] + (d[tg][1][e] >> 2) + (d[tg][2][e] >> 4) + (d[tg][3][e] >> 6) - rsum;
              const int au = d[tg][0][e + 2] + (d[tg][1][e + 2] >> 2) + (d[tg][2][e + 2] >> 4) +
                             (d[tg][3][e + 2] >> 6) - rsum;
              const float g_v = round_to<TY>(__fmul_rn(static_cast<float>(ag), __fdiv_rn(gamma, sm)));
              const float u_v = round_to<TY>(__fmul_rn(static_cast<float>(au), __fdiv_rn(gamma_up, sm)));
              const float h = glu_value<TY>(g_v, u_v, P.glu.act);
              TY* hp = static_cast<TY*>(P.glu.h);
              const size_t o = static_cast<size_t>(m) * L.N + n;
              if constexpr (sizeof(TY) == 4) hp[o] = h; else hp[o] = __float2bfloat16_rn(h);
              habs = fabsf(h);
            }
            // Per token: the 8 lanes (g) holding it.
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) habs = fmaxf(habs, __shfl_xor_sync(0xffffffffu, habs, o));
            hmax[tg][e] = fmaxf(hmax[tg][e], habs);
          }
        continue;
      }
#pragma unroll
      for (int tg = 0; tg < TG; ++tg)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int n = n_base + row_lo + ((c & 2) ? 8 : 0);
          const int m = tg * 8 + 2 * t + (c & 1);
          if (n < L.N && m < M) {
            const int rsum = kStream ? rsum_m[tg][c & 1] : rs_tok[m];
            const float sm = kStream ? s_m[tg][c & 1] : s_tok[m];
            const int a = (kSplit ? pc[tg][c] : d[tg][0][c] + (d[tg][1][c] >> 2) + (d[tg][2][c] >> 4) + (d[tg][3][c] >> 6)) - rsum;
            const float v = __fmul_rn(static_cast<float>(a), __fdiv_rn(gamma, sm));
            const size_t o = static_cast<size_t>(m) * L.N + n;
            if constexpr (sizeof(TY) == 4) y[o] = v; else y[o] = __float2bfloat16_rn(v);
            if (L.acc_out) L.acc_out[o] = a;
          }
        }
    }
    if constexpr (kGlu) {
      // Every consumer warp, after its last unit or after giving up.
      glu_block_done<TG, kAlu>(P, hmax, reinterpret_cast<float*>(smem), ctl);
      glu_quant_slices<TY>(P, P.layer[P.glu.gate].N, ctl);
    }
  }

  // No CTA of a K-split cluster leaves while a peer may still read its shared
  // memory or arrive on its barrier.
  if (ks > 1) cluster_sync_all();
  // The block that finishes last resets the ticket counter for the next launch.
  if (P.one_unit) return;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(P.tickets + 1, 1u) == gridDim.x - 1) {
      atomicExch(P.tickets, 0u);
      atomicExch(P.tickets + 1, 0u);
    }
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static int token_slots(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16; }

int gemv_x_pitch(int K) { return ((K + 127) / 128) * 128 + 16; }

// Shared memory of one block: the ring, then (in-kernel quantisation only) the
// whole-K activations, then (K-split only) the partial sums, then the small
// arrays and barriers.
int gemv_smem_bytes(int M, int K_max, int nring, bool stream, int ksplit = 1) {
  const int slot = kGvStageBytes + (stream ? 2 * x_half_bytes(token_slots(M)) : 0);
  const int staged = stream ? 0 : ((M * gemv_x_pitch(K_max) + 127) / 128) * 128;
  const int part = ksplit > 1 ? gv_part_bytes(token_slots(M)) : 0;
  return nring * slot + staged + part + 256 + 16 * nring + 16 + 1024;
}

bool gemv_fuses_quant(int M, int K, int x_bf16, bool single) {
  // Every block quantises the activations it uses, so only tiny ones are worth it;
  // each consumer thread then holds at most kGvFuseChunks chunks of 16 inputs.
  // One bf16 token of a single layer: up to kGvFuseChunks1 chunks, as long as
  // the whole input fits beside a ring of four stages (K up to 9856): every
  // block reads the input (L2-resident after the first) instead of waiting
  // for a quantisation launch.
  const int G = kGvConsumers / token_slots(M);
  const int chunks_per_thread = (K / 16 + G - 1) / G;
  if (single && M == 1 && x_bf16)
    return chunks_per_thread <= kGvFuseChunks1 && gemv_smem_bytes(1, K, 4, false) <= kGvSmemPerBlock;
  const int max_chunks = x_bf16 ? kGvFuseChunks : (kGvFuseChunks + 1) / 2;
  return M >= 1 && M <= 16 && static_cast<long long>(M) * K <= kGvFuseElems && chunks_per_thread <= max_chunks &&
         gemv_smem_bytes(M, K, 4, false) <= kGvSmemPerBlock;
}

template <int TT, typename TY, typename TX>
static cudaError_t launch_group_t(const GvParams& P, int grid, int smem, cudaStream_t stream, bool pdl) {
  // Separate instances for the plain launch, the K-split and the fused
  // gate/up launch, so that each runs none of the others' code.
  static std::atomic<uint64_t> attr_done[4];  // per template instance and device
  constexpr bool kHasNarrow = TT == 1;
  const int mode = P.glu.on ? 2 : P.ksplit > 1 ? 1 : P.narrow ? 3 : 0;
  if (mode == 3 && !kHasNarrow) return cudaErrorInvalidValue;
  auto kernel = mode == 2   ? gemv_group_kernel<TT, TY, TX, 2>
                : mode == 1 ? gemv_group_kernel<TT, TY, TX, 1>
                : mode == 3 ? gemv_group_kernel<TT, TY, TX, kHasNarrow ? 3 : 0>
                            : gemv_group_kernel<TT, TY, TX, 0>;
  cudaError_t e = once_per_device(attr_done[mode], [&] {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGvSmemPerBlock);
  });
  if (e != cudaSuccess) return e;
  const int sp = mode == 1 ? 1 : 0;
  if (!sp) return launch(kernel, dim3(grid), dim3(kGvThreads), static_cast<size_t>(smem), stream, pdl, P);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGvThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = P.ksplit;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, P);
}

template <int TT, typename TY>
static cudaError_t launch_group_x(int x_type, const GvParams& P, int grid, int smem, cudaStream_t stream, bool pdl) {
  switch (x_type) {
    case kInBF16: return launch_group_t<TT, TY, __nv_bfloat16>(P, grid, smem, stream, pdl);
    case kInF32: return launch_group_t<TT, TY, float>(P, grid, smem, stream, pdl);
    default: return launch_group_t<TT, TY, int8_t>(P, grid, smem, stream, pdl);
  }
}

template <typename TY>
static cudaError_t launch_group_y(int x_type, const GvParams& P, int grid, int smem, cudaStream_t stream, bool pdl) {
  switch (token_slots(P.M)) {
    case 1: return launch_group_x<1, TY>(x_type, P, grid, smem, stream, pdl);
    case 2: return launch_group_x<2, TY>(x_type, P, grid, smem, stream, pdl);
    case 4: return launch_group_x<4, TY>(x_type, P, grid, smem, stream, pdl);
    case 8: return launch_group_x<8, TY>(x_type, P, grid, smem, stream, pdl);
    default: return launch_group_x<16, TY>(x_type, P, grid, smem, stream, pdl);
  }
}

thread_local int g_force_ksplit = 0;  // 0: automatic

void gemv_force_ksplit(int ks) { g_force_ksplit = ks > 0 ? ks : 0; }

thread_local int g_force_form = 0;  // 0: by size

void gemv_force_form(int form) { g_force_form = form; }

// Zeroed scratch of a fused gate/up launch: amax and rsum (one 128-byte line
// per token, 16 tokens each), then done[2].
size_t gemv_glu_scratch_bytes(int N) {
  (void)N;
  return 2 * 16 * kGluTokStride * 4 + 256;
}

cudaError_t launch_gemv_group(const GemvLayerArgs* layers, int n_layers, int M, int x_type, int y_type,
                              uint32_t* status, uint32_t* tickets, cudaStream_t stream, bool pdl,
                              const GemvGluArgs* glu) {
  if (n_layers < 1 || n_layers > kGvMaxLayers || M < 1 || M > 16) return cudaErrorInvalidValue;
  if (glu && (n_layers != 2 || layers[0].N != layers[1].N || layers[0].K != layers[1].K || layers[0].N % 16 != 0 ||
              !glu->zeroed || !glu->h || !glu->xq || !glu->scale || !glu->rowsum))
    return cudaErrorInvalidValue;
  // The tensor-core form only when forced: it measures slower at every token
  // count (its MMAs cost as much per 128 x 32 block of codes as full-width ones).
  if (!glu && x_type == kInInt8 && g_force_form == 2 && gemv_tc_eligible(layers, n_layers, M))
    return launch_gemv_tc(layers, n_layers, M, y_type, status, tickets, stream, pdl);
  EncodeTiledFn enc = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
  if (!enc) return cudaErrorNotSupported;
  const bool stream_x = x_type == kInInt8;
  const int tt = token_slots(M);
  // Largest K first: the longest units are handed out first.
  int order[kGvMaxLayers];
  for (int i = 0; i < n_layers; ++i) order[i] = i;
  for (int i = 1; i < n_layers; ++i)
    for (int j = i; j > 0 && layers[order[j]].K > layers[order[j - 1]].K; --j) {
      const int tmp = order[j];
      order[j] = order[j - 1];
      order[j - 1] = tmp;
    }
  GvParams P;
  memset(&P, 0, sizeof(P));
  int units = 0, k_max = 64, nst_min = 1 << 30;
  for (int i = 0; i < n_layers; ++i) {
    const GemvLayerArgs& a = layers[order[i]];
    if (stream_x && (a.ldx % 128 != 0 || a.ldx < a.K)) return cudaErrorInvalidValue;
    units += (a.N + kGvRows - 1) / kGvRows;
    if (a.K > k_max) k_max = a.K;
    const int nst = (a.K + kGvStageK - 1) / kGvStageK;
    if (nst < nst_min) nst_min = nst;
  }
  P.n_layers = n_layers;
  P.M = M;
  P.x_pitch = gemv_x_pitch(k_max);
  P.status = status;
  P.tickets = tickets;
  // Few units for the SMs (a short, wide layer): a cluster of ks CTAs shares
  // each unit, every CTA over its own contiguous range of the unit's stages.
  // One token: about one CTA per SM to decide whether to split, about 1.35 once
  // split.  More tokens, where one warp per SM sub-partition issuing mma.sync
  // is the limit: about two.  ks is that target
  // over the unit count, rounded; at most 8, at most the fewest stages of any
  // layer, and no more CTAs than are resident at once.
  const int sms = num_sms();
  const int target = tt == 1 ? sms : 2 * sms;
  int ks = units < target ? (target + units / 2) / units : 1;
  // One token split at all: about 1.35 CTAs per SM measured better than one
  // (the 3B 8640->3200 layer 7.8 -> 7.3 us, 11008->4096 10.0 -> 8.7 us, none
  // slower); groups that would not split are left whole, since splitting them
  // gives up the narrow units (4096->8192: 5.1 -> 6.0 us).
  if (tt == 1 && ks >= 2) ks = (sms * 27 / 20 + units / 2) / units;
  if (g_force_ksplit > 0) ks = g_force_ksplit;
  while (ks > 1 && units * ks > kGvBlocksPerSM * sms) --ks;
  if (ks > kGvMaxSplit) ks = kGvMaxSplit;
  if (ks > nst_min) ks = nst_min;
  if (ks < 1 || glu) ks = 1;  // the fused gate/up launch hands its quantisation units out by ticket
  P.ksplit = ks;
  // One token without a split: units of 32 rows, so that the last units
  // handed out are half as long.  With the activations quantised by every
  // block itself, only when the 64-row units would leave SMs without one
  // (the 3B 3200->8640 layer: 5.9 -> 4.9 us; the 2B step, 148 units for 148
  // SMs, went from 3.8 to 4.6 us as 296 blocks each quantising the token).
  const bool narrow = tt == 1 && ks == 1 && !glu && (stream_x || units < sms);
  P.narrow = narrow ? 1 : 0;
  // Rows per unit: 16 (+ 16 up rows) in the fused gate/up launch at one token,
  // 32 (+ 32) with more tokens, 32 for narrow units, 64 otherwise.
  const bool glu_narrow = glu && tt == 1;
  const int unit_rows = glu_narrow ? kGvRows / 4 : (narrow || glu) ? kGvRows / 2 : kGvRows;
  units = 0;
  for (int i = 0; i < n_layers; ++i) {
    const GemvLayerArgs& a = layers[order[i]];
    GvLayer& L = P.layer[i];
    {
      // Boxes of one unit's rows (16 or 32 for the fused gate/up launch, 32 for narrow units).
      const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K / 4), static_cast<cuuint64_t>(a.N)};
      const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K / 4)};
      const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(unit_rows)};
      const cuuint32_t estr[2] = {1, 1};
      if (enc(&L.tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.packed), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
        return cudaErrorInvalidValue;
      }
    }
    if (stream_x) {
      // Codes [M][ldx] viewed as [M][ldx/128][128]; blocks past K are zero in
      // the buffer, blocks past ldx are filled with zeros by the copy.  A
      // narrow stage takes its 16 blocks in one box.
      const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(a.ldx / 128), static_cast<cuuint64_t>(M)};
      const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(a.ldx)};
      const cuuint32_t box[3] = {128, (narrow || glu_narrow) ? 16u : 4u, static_cast<cuuint32_t>(tt)};
      const cuuint32_t estr[3] = {1, 1, 1};
      if (enc(&L.xmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(a.x), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
        return cudaErrorInvalidValue;
      }
    }
    L.x = a.x;
    L.scale = a.scale;
    L.rowsum = a.rowsum;
    L.gamma = a.gamma;
    L.y = a.y;
    L.acc_out = a.acc_out;
    L.N = a.N;
    L.K = a.K;
    L.unit0 = units;
    units += (a.N + unit_rows - 1) / unit_rows;
  }
  // A unit of the fused gate/up launch covers the same rows of both layers.
  if (glu) units = (layers[0].N + unit_rows - 1) / unit_rows;
  P.total_units = units;
  if (glu) {
    // Units of 32 rows of both layers; the quantisation slices go to the grid's
    // warps once the grid size is known (below).
    GvGlu& G = P.glu;
    G.on = 1;
    G.act = glu->act;
    for (int i = 0; i < n_layers; ++i) {
      if (order[i] == 0) G.gate = i;
      if (order[i] == 1) G.up = i;
    }
    G.h = glu->h;
    G.xq = glu->xq;
    G.scale = glu->scale;
    G.rowsum = glu->rowsum;
    uint32_t* z = glu->zeroed;
    G.amax = z;
    G.rsum = reinterpret_cast<int32_t*>(z + 16 * kGluTokStride);
    G.done = z + 2 * 16 * kGluTokStride;
  }
  // kGvBlocksPerSM blocks per SM, each with the deepest weight ring that fits beside its other data.
  const int slot = kGvStageBytes + (stream_x ? 2 * x_half_bytes(tt) : 0);
  const int fixed = gemv_smem_bytes(M, k_max, 0, stream_x, ks);
  int nring = (kGvSmemPerBlock - fixed) / (slot + 16);
  if (nring > kGvMaxRing) nring = kGvMaxRing;
  if (nring < 2) return cudaErrorInvalidConfiguration;
  P.nring = nring;
  const int smem = gemv_smem_bytes(M, k_max, nring, stream_x, ks);
  const int slots = kGvBlocksPerSM * sms;
  int grid = ks > 1 ? units * ks : (units < slots ? units : slots);
  // One token with more units than resident blocks: as few blocks as take
  // them in equal numbers, so that no few blocks are left each with one more
  // unit at the end (the gate/up pair at the 70B width: 896 units, 299 blocks
  // of three, 33.9 -> 32.9 us).  With more tokens the mma path needs every
  // block: there it measured slower (35.3 -> 36.6 us at 8 tokens).
  if (ks == 1 && tt == 1 && units > slots) {
    const int per = (units + slots - 1) / slots;
    grid = (units + per - 1) / per;
  }
  P.one_unit = ks > 1 || units <= slots ? 1 : 0;
  if (glu) {
    const long long slices = (static_cast<long long>(M) * layers[0].N + kGluSlice - 1) / kGluSlice;
    const long long warps = static_cast<long long>(grid) * kGvWarps;
    P.glu.q_warps = static_cast<int>(slices < warps ? slices : warps);
    P.glu.q_blocks = (P.glu.q_warps + kGvWarps - 1) / kGvWarps;
  }
  return y_type == kOutBF16 ? launch_group_y<__nv_bfloat16>(x_type, P, grid, smem, stream, pdl)
                            : launch_group_y<float>(x_type, P, grid, smem, stream, pdl);
}

}  // namespace bl
