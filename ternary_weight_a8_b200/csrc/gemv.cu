// Decode product (M <= 16 tokens): packed ternary weights x int8 activations,
// int32 accumulation, fused dequantisation.
//
// "BitNet's Real Bet: Designing the Whole Inference Stack", section "A
// low-bit model is a whole-stack design": the GPU path moves packed weights
// from HBM on chip, unpacks them and computes with the 8-bit activations.
// "BitNet b1.58 and the 1-Bit AI Architecture Revolution", section "The
// Energy Revolution": the product is integer additions; here the additions
// run on the tensor cores' int8 path (mma.sync m16n8k32, u8 x s8 -> s32).
//
// Decode is bound by the weight stream, so the kernel keeps every weight byte
// in registers from a single 16-byte streaming load and never stages it in
// shared memory.  Unpacking costs one AND per four weights: for j = 0..3 the
// mask 0x03030303 << 2j keeps the codes of elements 4j..4j+3 of each 32-bit
// word in place, i.e. scaled by 4^j; four accumulator sets (one per j) are
// shifted back by 2j and added, which is exact because each is a multiple of
// 4^j.  The k order inside one mma is free as long as weights and
// activations agree, so the fragment of lane (g, t) is read directly from
// the packed word layout.
//
// Work split: a row group is 16 output rows, a segment 256 inputs (64 packed
// bytes per row).  A block owns `rg_per_cta` row groups over all of K; its 8
// warps share the (row group, segment) items and add their partial sums into
// shared memory, then the block applies  y = (acc - rowsum) * (gamma / s).
// The first weight loads are issued before waiting on the preceding kernel
// (programmatic dependent launch), so the weight stream overlaps the
// activation quantisation.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace bl {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;

__device__ __forceinline__ void mma_u8s8_16x8x32(int (&d)[4], uint32_t a0, uint32_t a1,
                                                 uint32_t a2, uint32_t a3, uint32_t b0,
                                                 uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t u4_get(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

template <int TG>
struct XFrag {
  uint4 v[TG][4];  // token (tg*8 + g): 64 activation bytes at k = seg*256 + 64t .. +63
};

template <int TG>
__device__ __forceinline__ void load_x(XFrag<TG>& xf, const int8_t* __restrict__ xq, int M, int K,
                                       int seg, int g, int t) {
  const int k0 = seg * 256 + 64 * t;
#pragma unroll
  for (int tg = 0; tg < TG; ++tg) {
    const int m = tg * 8 + g;
    if (m < M && k0 < K) {
      const uint4* p = reinterpret_cast<const uint4*>(xq + static_cast<size_t>(m) * K + k0);
#pragma unroll
      for (int i = 0; i < 4; ++i) xf.v[tg][i] = __ldg(p + i);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) xf.v[tg][i] = make_uint4(0, 0, 0, 0);
    }
  }
}

struct WFrag {
  uint4 lo, hi;  // rows (16 rg + g) and (16 rg + g + 8): packed bytes of k = seg*256 + 64t .. +63
};

__device__ __forceinline__ WFrag load_w(const uint8_t* __restrict__ packed, int N, int K, int rg,
                                        int seg, int g, int t) {
  WFrag w;
  const int kbytes = K / 4;
  const int koff = seg * 64 + 16 * t;  // byte offset of this lane's chunk within a row
  const int r0 = rg * 16 + g;
  const bool kin = koff < kbytes;
  w.lo = (kin && r0 < N) ? ldg_stream_u4(packed + static_cast<size_t>(r0) * kbytes + koff)
                         : make_uint4(0, 0, 0, 0);
  w.hi = (kin && r0 + 8 < N) ? ldg_stream_u4(packed + static_cast<size_t>(r0 + 8) * kbytes + koff)
                             : make_uint4(0, 0, 0, 0);
  return w;
}

// 8 (or 16) mma per token group for one item; adds the exact sums into shared memory.
template <int TG>
__device__ __forceinline__ void compute_item(const WFrag& w, const XFrag<TG>& xf, int* acc_s,
                                             int rl, int g, int t) {
  int d[TG][4][4];
#pragma unroll
  for (int tg = 0; tg < TG; ++tg)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) d[tg][j][c] = 0;

#pragma unroll
  for (int p = 0; p < 2; ++p) {
    const int i0 = 2 * p, i1 = 2 * p + 1;
    const uint32_t lo0 = u4_get(w.lo, i0), lo1 = u4_get(w.lo, i1);
    const uint32_t hi0 = u4_get(w.hi, i0), hi1 = u4_get(w.hi, i1);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t mask = 0x03030303u << (2 * j);
      const uint32_t a0 = lo0 & mask, a1 = hi0 & mask, a2 = lo1 & mask, a3 = hi1 & mask;
#pragma unroll
      for (int tg = 0; tg < TG; ++tg) {
        mma_u8s8_16x8x32(d[tg][j], a0, a1, a2, a3, u4_get(xf.v[tg][i0], j), u4_get(xf.v[tg][i1], j));
      }
    }
  }
  constexpr int TT = TG * 8;
#pragma unroll
  for (int tg = 0; tg < TG; ++tg) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int v = d[tg][0][c] + (d[tg][1][c] >> 2) + (d[tg][2][c] >> 4) + (d[tg][3][c] >> 6);
      const int row = rl * 16 + g + ((c & 2) ? 8 : 0);
      const int tok = tg * 8 + 2 * t + (c & 1);
      red_shared_add(acc_s + row * TT + tok, v);
    }
  }
}

template <int TG, typename TY>
__global__ void __launch_bounds__(kGemvThreads, 2) gemv_kernel(
    const uint8_t* __restrict__ packed, const float* __restrict__ gamma_ptr, int N, int K,
    const int8_t* __restrict__ xq, const float* __restrict__ scale,
    const int32_t* __restrict__ rowsum, int M, TY* __restrict__ y, int32_t* __restrict__ acc_out,
    int rg_per_cta) {
  extern __shared__ int acc_s[];  // [rg_per_cta * 16][TG * 8]
  constexpr int TT = TG * 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int n_rg = (N + 15) / 16;
  const int rg0 = blockIdx.x * rg_per_cta;
  const int rg_cnt = min(rg_per_cta, n_rg - rg0);
  const int nseg = (K + 255) / 256;
  const int items = rg_cnt * nseg;

  for (int i = threadIdx.x; i < rg_cnt * 16 * TT; i += kGemvThreads) acc_s[i] = 0;

  // This warp's items: a contiguous range in (segment-major, row-group-minor)
  // order, so that consecutive items mostly share one activation segment.
  const int per = (items + kGemvWarps - 1) / kGemvWarps;
  const int ib = min(items, warp * per), ie = min(items, ib + per);

  // Prefetch the first two items' weights before the dependency wait.
  WFrag w0 = {}, w1 = {};
  if (ib < ie) w0 = load_w(packed, N, K, rg0 + ib % rg_cnt, ib / rg_cnt, g, t);
  if (ib + 1 < ie) w1 = load_w(packed, N, K, rg0 + (ib + 1) % rg_cnt, (ib + 1) / rg_cnt, g, t);

  griddep_launch_dependents();
  griddep_wait();
  __syncthreads();  // acc_s zeroed

  XFrag<TG> xf;
  int cur_seg = -1;
  for (int it = ib; it < ie; it += 2) {
    // Issue the next pair's loads before computing this pair.
    WFrag n0 = {}, n1 = {};
    if (it + 2 < ie) n0 = load_w(packed, N, K, rg0 + (it + 2) % rg_cnt, (it + 2) / rg_cnt, g, t);
    if (it + 3 < ie) n1 = load_w(packed, N, K, rg0 + (it + 3) % rg_cnt, (it + 3) / rg_cnt, g, t);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int item = it + u;
      if (item < ie) {
        const int seg = item / rg_cnt, rl = item % rg_cnt;
        if (seg != cur_seg) {
          load_x<TG>(xf, xq, M, K, seg, g, t);
          cur_seg = seg;
        }
        compute_item<TG>(u == 0 ? w0 : w1, xf, acc_s, rl, g, t);
      }
    }
    w0 = n0;
    w1 = n1;
  }
  __syncthreads();

  // Epilogue: y[m][n] = (acc - rowsum[m]) * (gamma / s[m]).
  const float gamma = __ldg(gamma_ptr);
  const int rows = rg_cnt * 16;
  const int nb = rg0 * 16;
  for (int idx = threadIdx.x; idx < rows * M; idx += kGemvThreads) {
    const int m = idx / rows, r = idx % rows;
    const int n = nb + r;
    if (n >= N) continue;
    const int acc = acc_s[r * TT + m] - __ldg(rowsum + m);
    const float v = __fmul_rn(static_cast<float>(acc), __fdiv_rn(gamma, __ldg(scale + m)));
    const size_t o = static_cast<size_t>(m) * N + n;
    if constexpr (sizeof(TY) == 4) {
      y[o] = v;
    } else {
      y[o] = __float2bfloat16_rn(v);
    }
    if (acc_out) acc_out[o] = acc;
  }
}

template <int TG, typename TY>
static cudaError_t launch_gemv_t(const ProductArgs& a, cudaStream_t stream, bool pdl) {
  const int n_rg = (a.N + 15) / 16;
  const int target = 2 * num_sms();
  const int rg_per_cta = (n_rg + target - 1) / target;
  const int grid = (n_rg + rg_per_cta - 1) / rg_per_cta;
  const size_t smem = static_cast<size_t>(rg_per_cta) * 16 * TG * 8 * sizeof(int);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(gemv_kernel<TG, TY>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  return launch(gemv_kernel<TG, TY>, dim3(grid), dim3(kGemvThreads), smem, stream, pdl, a.packed,
                a.gamma, a.N, a.K, a.xq, a.scale, a.rowsum, a.M, static_cast<TY*>(a.y), a.acc_out,
                rg_per_cta);
}

cudaError_t launch_gemv(const ProductArgs& a, cudaStream_t stream, bool pdl) {
  if (a.M <= 8) {
    return a.y_type == kOutBF16 ? launch_gemv_t<1, __nv_bfloat16>(a, stream, pdl)
                                : launch_gemv_t<1, float>(a, stream, pdl);
  }
  return a.y_type == kOutBF16 ? launch_gemv_t<2, __nv_bfloat16>(a, stream, pdl)
                              : launch_gemv_t<2, float>(a, stream, pdl);
}

}  // namespace bl
