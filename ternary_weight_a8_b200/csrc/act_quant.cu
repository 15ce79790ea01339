// Per-token 8-bit activation quantisation, for one input or several at once.
//
// "BitNet's Real Bet: Designing the Whole Inference Stack", section "A
// low-bit model is a whole-stack design": activations take a separate
// per-token 8-bit path.  "A Two-Billion Ternary Bet": activations are
// quantised dynamically.  Reading (the pages print no formula): symmetric
// absmax, s = 127 / max(amax, 1e-5), q = clamp(rint(x * s), -128, 127), in
// fp32 with round-half-to-even.  The kernel also writes sum_k q[m][k], which
// the tensor-core GEMM uses to turn sums over the stored codes c = t + 1 into
// sums over t.
//
// One block per (input, token).  A token of up to 32768 inputs is read once
// into registers (16-input chunks, up to four per thread): block absmax,
// then quantise from registers, pack four codes per word with byte permutes
// and add the codes with dp4a.  Longer tokens are read a second time.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace bl {

constexpr int kQuantMaxThreads = 512;
constexpr int kQuantRegChunks = 4;

struct QuantItem {
  const void* x;
  int8_t* xq;  // rows of ldq bytes; [K, ldq) is written as zeros
  float* scale;
  int32_t* rowsum;
  int K, ldq;
};

struct QuantParams {
  QuantItem item[kQuantMaxItems];
  int n_items;
};

struct Chunk16 {
  uint4 v[4];  // bf16: v[0..1]; fp32: v[0..3]
};

template <typename TX>
__device__ __forceinline__ void load16(const TX* p, Chunk16& r) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
  r.v[0] = __ldcg(q);
  r.v[1] = __ldcg(q + 1);
  if constexpr (sizeof(TX) == 4) {
    r.v[2] = __ldcg(q + 2);
    r.v[3] = __ldcg(q + 3);
  }
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

template <typename TX>
__device__ __forceinline__ float elem(const Chunk16& r, int e) {
  if constexpr (sizeof(TX) == 4) {
    return __uint_as_float(word_of(r.v[e >> 2], e & 3));
  } else {
    const uint32_t w = word_of(r.v[e >> 3], (e >> 1) & 3);  // bf16 -> fp32 is exact
    return __uint_as_float((e & 1) ? (w & 0xffff0000u) : (w << 16));
  }
}

template <typename TX>
__device__ __forceinline__ float chunk_absmax(const Chunk16& r) {
  float a = 0.0f;
#pragma unroll
  for (int e = 0; e < 16; ++e) a = fmaxf(a, fabsf(elem<TX>(r, e)));
  return a;
}

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  const uint32_t lo = __byte_perm(static_cast<uint32_t>(a), static_cast<uint32_t>(b), 0x5140);
  const uint32_t hi = __byte_perm(static_cast<uint32_t>(c), static_cast<uint32_t>(d), 0x5140);
  return __byte_perm(lo, hi, 0x5410);
}

// q for the 16 inputs of a chunk, written as one 16-byte store; returns sum q.
template <typename TX>
__device__ __forceinline__ int quant_chunk(const Chunk16& r, float s, int8_t* dst) {
  uint32_t w[4];
  int sum = 0;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    int q[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      q[e] = __float2int_rn(__fmul_rn(elem<TX>(r, 4 * b + e), s));
      q[e] = min(max(q[e], -128), 127);
    }
    w[b] = pack4(q[0], q[1], q[2], q[3]);
    sum = __dp4a(static_cast<int>(w[b]), 0x01010101, sum);
  }
  *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  return sum;
}

template <typename T, typename Op>
__device__ __forceinline__ T block_reduce(T v, Op op, T* smem) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  if (lane == 0) smem[warp] = v;
  __syncthreads();
  T r = smem[0];
  for (int i = 1; i < nw; ++i) r = op(r, smem[i]);
  __syncthreads();
  return r;
}

template <typename TX>
__global__ void __launch_bounds__(kQuantMaxThreads) act_quant_kernel(const __grid_constant__ QuantParams P) {
  __shared__ float red_f[kQuantMaxThreads / 32];
  __shared__ int red_i[kQuantMaxThreads / 32];
  griddep_launch_dependents();
  griddep_wait();  // x may be the preceding kernel's output; q may still be read by it

  const QuantItem& it = P.item[blockIdx.y];
  const int m = blockIdx.x, K = it.K, chunks = K >> 4, T = blockDim.x;
  const TX* xr = static_cast<const TX*>(it.x) + static_cast<size_t>(m) * K;
  int8_t* qr = it.xq + static_cast<size_t>(m) * it.ldq;
  for (int c = K + 16 * threadIdx.x; c < it.ldq; c += 16 * T)  // row padding (K % 16 == 0)
    *reinterpret_cast<uint4*>(qr + c) = make_uint4(0, 0, 0, 0);
  const bool in_regs = chunks <= T * kQuantRegChunks;

  Chunk16 reg[kQuantRegChunks];
  float amax = 0.0f;
  if (in_regs) {
#pragma unroll
    for (int i = 0; i < kQuantRegChunks; ++i) {
      const int c = threadIdx.x + i * T;
      if (c < chunks) load16<TX>(xr + c * 16, reg[i]);
    }
#pragma unroll
    for (int i = 0; i < kQuantRegChunks; ++i) {
      const int c = threadIdx.x + i * T;
      if (c < chunks) amax = fmaxf(amax, chunk_absmax<TX>(reg[i]));
    }
  } else {
    for (int c = threadIdx.x; c < chunks; c += T) {
      Chunk16 r;
      load16<TX>(xr + c * 16, r);
      amax = fmaxf(amax, chunk_absmax<TX>(r));
    }
  }
  amax = block_reduce(amax, [](float a, float b) { return fmaxf(a, b); }, red_f);
  const float s = __fdiv_rn(127.0f, fmaxf(amax, 1e-5f));

  int sum = 0;
  if (in_regs) {
#pragma unroll
    for (int i = 0; i < kQuantRegChunks; ++i) {
      const int c = threadIdx.x + i * T;
      if (c < chunks) sum += quant_chunk<TX>(reg[i], s, qr + c * 16);
    }
  } else {
    for (int c = threadIdx.x; c < chunks; c += T) {
      Chunk16 r;
      load16<TX>(xr + c * 16, r);
      sum += quant_chunk<TX>(r, s, qr + c * 16);
    }
  }
  sum = block_reduce(sum, [](int a, int b) { return a + b; }, red_i);
  if (threadIdx.x == 0) {
    it.scale[m] = s;
    if (it.rowsum) it.rowsum[m] = sum;
  }
}

// ---------------------------------------------------------------------------
// RMSNorm fused with the quantisation: the normalisation that precedes a
// BitLinear ("BitNet's Real Bet: Designing the Whole Inference Stack",
// native-training section: RMSNorm, sub-layer normalisation).  Reading (no
// formula on the pages): v = x * r * g, r = 1 / sqrt(mean(x^2) + eps); the
// squares are summed in double (exact squares, one rounding per add, so the
// order changes r only in double's last bits), r is rounded once to fp32,
// x * r then * g are fp32 multiplies, and v is rounded to the activation
// type exactly as an unfused norm would store it; then the same per-token
// quantisation as above.  One block per token, the token held in registers.
// ---------------------------------------------------------------------------
struct NormParams {
  const void* x;
  const float* gain;  // [K] or null
  float eps;
  void* x_norm;       // [M][K] in the activation type, or null
  int8_t* xq;         // [M][K]
  float* scale;
  int32_t* rowsum;    // or null
  int K;
};

// v = round_to_TX(x * r [* g]) for the 16 inputs of chunk c.
template <typename TX>
__device__ __forceinline__ void norm_chunk(const Chunk16& raw, float r, const float* gain, int c, float (&v)[16]) {
  float gv[16];
  if (gain) {
    const float4* gp = reinterpret_cast<const float4*>(gain + 16 * c);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 t = __ldg(gp + i);
      gv[4 * i] = t.x;
      gv[4 * i + 1] = t.y;
      gv[4 * i + 2] = t.z;
      gv[4 * i + 3] = t.w;
    }
  }
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    float t = __fmul_rn(elem<TX>(raw, e), r);
    if (gain) t = __fmul_rn(t, gv[e]);
    if constexpr (sizeof(TX) == 2) t = __bfloat162float(__float2bfloat16_rn(t));
    v[e] = t;
  }
}

// Codes of 16 values (one 16-byte store), and the values themselves in the
// activation type when `vout` is set; returns the sum of the codes.
template <typename TX>
__device__ __forceinline__ int quant_store16(const float (&v)[16], float s, int8_t* dst, TX* vout) {
  uint32_t w[4];
  int sum = 0;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    int q[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) q[e] = min(max(__float2int_rn(__fmul_rn(v[4 * b + e], s)), -128), 127);
    w[b] = pack4(q[0], q[1], q[2], q[3]);
    sum = __dp4a(static_cast<int>(w[b]), 0x01010101, sum);
  }
  *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  if (vout) {
    if constexpr (sizeof(TX) == 2) {
      uint32_t h[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        h[e] = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v[2 * e]))) |
               (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v[2 * e + 1]))) << 16);
      uint4* d = reinterpret_cast<uint4*>(vout);
      d[0] = make_uint4(h[0], h[1], h[2], h[3]);
      d[1] = make_uint4(h[4], h[5], h[6], h[7]);
    } else {
      float4* d = reinterpret_cast<float4*>(vout);
#pragma unroll
      for (int e = 0; e < 4; ++e) d[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
    }
  }
  return sum;
}

template <typename TX>
__global__ void __launch_bounds__(kQuantMaxThreads) rmsnorm_quant_kernel(const __grid_constant__ NormParams P) {
  __shared__ double red_d[kQuantMaxThreads / 32];
  __shared__ float red_f[kQuantMaxThreads / 32];
  __shared__ int red_i[kQuantMaxThreads / 32];
  griddep_launch_dependents();
  griddep_wait();  // x may be the preceding kernel's output; q may still be read by it

  const int m = blockIdx.x, K = P.K, chunks = K >> 4, T = blockDim.x;
  const TX* xr = static_cast<const TX*>(P.x) + static_cast<size_t>(m) * K;
  int8_t* qr = P.xq + static_cast<size_t>(m) * K;
  TX* nr = P.x_norm ? static_cast<TX*>(P.x_norm) + static_cast<size_t>(m) * K : nullptr;
  const bool in_regs = chunks <= T * kQuantRegChunks;
  Chunk16 reg[kQuantRegChunks];
  if (in_regs) {
#pragma unroll
    for (int i = 0; i < kQuantRegChunks; ++i) {
      const int c = threadIdx.x + i * T;
      if (c < chunks) load16<TX>(xr + c * 16, reg[i]);
    }
  }
  // fn(chunk, c) over this thread's chunks: from registers, or read again.
  auto for_each_chunk = [&](auto&& fn) {
    if (in_regs) {
#pragma unroll
      for (int i = 0; i < kQuantRegChunks; ++i) {
        const int c = threadIdx.x + i * T;
        if (c < chunks) fn(reg[i], c);
      }
    } else {
      for (int c = threadIdx.x; c < chunks; c += T) {
        Chunk16 raw;
        load16<TX>(xr + c * 16, raw);
        fn(raw, c);
      }
    }
  };

  // Mean of squares, in double (each square exact, one rounding per add).
  double ss = 0.0;
  for_each_chunk([&](const Chunk16& ch, int) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const double v = static_cast<double>(elem<TX>(ch, e));
      ss = __fma_rn(v, v, ss);
    }
  });
  ss = block_reduce(ss, [](double a, double b) { return __dadd_rn(a, b); }, red_d);
  const double ms = __ddiv_rn(ss, static_cast<double>(K));
  const float r = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(ms, static_cast<double>(P.eps)))));

  // Absmax of the normalised token.  When the token is in registers the
  // normalised values of the thread's first kNormKeep chunks stay there too.
  constexpr int kNormKeep = 2;
  float vkeep[kNormKeep][16];
  float amax = 0.0f;
  for_each_chunk([&](const Chunk16& ch, int c) {
    float v[16];
    norm_chunk<TX>(ch, r, P.gain, c, v);
    const int i = (c - static_cast<int>(threadIdx.x)) / T;
#pragma unroll
    for (int k = 0; k < kNormKeep; ++k)
      if (in_regs && i == k) {
#pragma unroll
        for (int e = 0; e < 16; ++e) vkeep[k][e] = v[e];
      }
#pragma unroll
    for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(v[e]));
  });
  amax = block_reduce(amax, [](float a, float b) { return fmaxf(a, b); }, red_f);
  const float s = __fdiv_rn(127.0f, fmaxf(amax, 1e-5f));

  // Codes (and the normalised activations when asked for).
  int sum = 0;
  for_each_chunk([&](const Chunk16& ch, int c) {
    float v[16];
    const int i = (c - static_cast<int>(threadIdx.x)) / T;
    if (in_regs && i < kNormKeep) {
#pragma unroll
      for (int k = 0; k < kNormKeep; ++k)
        if (i == k) {
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = vkeep[k][e];
        }
    } else {
      norm_chunk<TX>(ch, r, P.gain, c, v);
    }
    sum += quant_store16<TX>(v, s, qr + c * 16, nr ? nr + c * 16 : nullptr);
  });
  sum = block_reduce(sum, [](int a, int b) { return a + b; }, red_i);
  if (threadIdx.x == 0) {
    P.scale[m] = s;
    if (P.rowsum) P.rowsum[m] = sum;
  }
}

cudaError_t launch_rmsnorm_quant(const void* x, int x_bf16, int M, int K, const float* gain, float eps, void* x_norm,
                                 int8_t* xq, float* scale, int32_t* rowsum, cudaStream_t stream, bool pdl) {
  if (M <= 0) return cudaSuccess;
  const NormParams P{x, gain, eps, x_norm, xq, scale, rowsum, K};
  int threads = ((K / 16 + 1) / 2 + 31) / 32 * 32;  // about two chunks per thread, 64 .. 512
  if (threads < 64) threads = 64;
  if (threads > kQuantMaxThreads) threads = kQuantMaxThreads;
  if (x_bf16) return launch(rmsnorm_quant_kernel<__nv_bfloat16>, dim3(M), dim3(threads), 0, stream, pdl, P);
  return launch(rmsnorm_quant_kernel<float>, dim3(M), dim3(threads), 0, stream, pdl, P);
}

// ---------------------------------------------------------------------------
// The FFN's gated activation fused with the quantisation of the down
// BitLinear's input ("BitNet's Real Bet: Designing the Whole Inference
// Stack", native-training section: SwiGLU, squared ReLU; "A Two-Billion
// Ternary Bet": squared-ReLU-style activations).  Reading (no formula on the
// pages): h = act(gate) * up on the stored gate/up values, in fp32, rounded
// to the activation type; act = max(z, 0)^2 as (g * g) * u, or SiLU as
// z / (1 + expf(-z)) * u; then the per-token quantisation.  One block per
// token, h kept in registers between its absmax and its codes.
// ---------------------------------------------------------------------------
struct GluParams {
  const void* gate;
  const void* up;
  int act;         // kGluRelu2 or kGluSilu
  void* h;         // [M][N] in the activation type, or null
  int8_t* xq;      // [M][N]
  float* scale;
  int32_t* rowsum; // or null
  int N;
};

template <typename TX>
__device__ __forceinline__ void glu_chunk(const Chunk16& g, const Chunk16& u, int act, float (&h)[16]) {
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float z = elem<TX>(g, e), w = elem<TX>(u, e);
    float t;
    if (act == kGluRelu2) {
      const float p = z > 0.0f ? z : 0.0f;
      t = __fmul_rn(__fmul_rn(p, p), w);
    } else {
      t = __fmul_rn(__fdiv_rn(z, __fadd_rn(1.0f, expf(-z))), w);
    }
    if constexpr (sizeof(TX) == 2) t = __bfloat162float(__float2bfloat16_rn(t));
    h[e] = t;
  }
}

template <typename TX>
__global__ void __launch_bounds__(kQuantMaxThreads) glu_quant_kernel(const __grid_constant__ GluParams P) {
  __shared__ float red_f[kQuantMaxThreads / 32];
  __shared__ int red_i[kQuantMaxThreads / 32];
  griddep_launch_dependents();
  griddep_wait();  // gate and up are the preceding kernel's outputs

  const int m = blockIdx.x, N = P.N, chunks = N >> 4, T = blockDim.x;
  const TX* gr = static_cast<const TX*>(P.gate) + static_cast<size_t>(m) * N;
  const TX* ur = static_cast<const TX*>(P.up) + static_cast<size_t>(m) * N;
  int8_t* qr = P.xq + static_cast<size_t>(m) * N;
  TX* hr = P.h ? static_cast<TX*>(P.h) + static_cast<size_t>(m) * N : nullptr;
  constexpr int kKeep = 2;  // chunks per thread whose h stays in registers
  const bool keep = chunks <= T * kKeep;
  float hk[kKeep][16];

  float amax = 0.0f;
  for (int i = 0, c = threadIdx.x; c < chunks; ++i, c += T) {
    Chunk16 g, u;
    load16<TX>(gr + c * 16, g);
    load16<TX>(ur + c * 16, u);
    float h[16];
    glu_chunk<TX>(g, u, P.act, h);
#pragma unroll
    for (int k = 0; k < kKeep; ++k)
      if (keep && i == k) {
#pragma unroll
        for (int e = 0; e < 16; ++e) hk[k][e] = h[e];
      }
#pragma unroll
    for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(h[e]));
  }
  amax = block_reduce(amax, [](float a, float b) { return fmaxf(a, b); }, red_f);
  const float s = __fdiv_rn(127.0f, fmaxf(amax, 1e-5f));

  int sum = 0;
  for (int i = 0, c = threadIdx.x; c < chunks; ++i, c += T) {
    float h[16];
    if (keep) {
#pragma unroll
      for (int k = 0; k < kKeep; ++k)
        if (i == k) {
#pragma unroll
          for (int e = 0; e < 16; ++e) h[e] = hk[k][e];
        }
    } else {
      Chunk16 g, u;
      load16<TX>(gr + c * 16, g);
      load16<TX>(ur + c * 16, u);
      glu_chunk<TX>(g, u, P.act, h);
    }
    sum += quant_store16<TX>(h, s, qr + c * 16, hr ? hr + c * 16 : nullptr);
  }
  sum = block_reduce(sum, [](int a, int b) { return a + b; }, red_i);
  if (threadIdx.x == 0) {
    P.scale[m] = s;
    if (P.rowsum) P.rowsum[m] = sum;
  }
}

cudaError_t launch_glu_quant(const void* gate, const void* up, int x_bf16, int M, int N, int act, void* h,
                             int8_t* xq, float* scale, int32_t* rowsum, cudaStream_t stream, bool pdl) {
  if (M <= 0) return cudaSuccess;
  if (act != kGluRelu2 && act != kGluSilu) return cudaErrorInvalidValue;
  const GluParams P{gate, up, act, h, xq, scale, rowsum, N};
  int threads = ((N / 16 + 1) / 2 + 31) / 32 * 32;  // about two chunks per thread, 64 .. 512
  if (threads < 64) threads = 64;
  if (threads > kQuantMaxThreads) threads = kQuantMaxThreads;
  if (x_bf16) return launch(glu_quant_kernel<__nv_bfloat16>, dim3(M), dim3(threads), 0, stream, pdl, P);
  return launch(glu_quant_kernel<float>, dim3(M), dim3(threads), 0, stream, pdl, P);
}

cudaError_t launch_act_quant_group(const QuantArgs* items, int n_items, int M, int x_bf16, cudaStream_t stream,
                                   bool pdl) {
  if (M <= 0 || n_items <= 0) return cudaSuccess;
  if (n_items > kQuantMaxItems) return cudaErrorInvalidValue;
  QuantParams P = {};
  int k_max = 0;
  for (int i = 0; i < n_items; ++i) {
    P.item[i] = QuantItem{items[i].x, items[i].xq, items[i].scale, items[i].rowsum, items[i].K, items[i].ldq};
    if (items[i].K > k_max) k_max = items[i].K;
  }
  P.n_items = n_items;
  // About two chunks per thread, in whole warps, 64 .. 512 threads.
  int threads = ((k_max / 16 + 1) / 2 + 31) / 32 * 32;
  if (threads < 64) threads = 64;
  if (threads > kQuantMaxThreads) threads = kQuantMaxThreads;
  const dim3 grid(M, n_items);
  if (x_bf16) return launch(act_quant_kernel<__nv_bfloat16>, grid, dim3(threads), 0, stream, pdl, P);
  return launch(act_quant_kernel<float>, grid, dim3(threads), 0, stream, pdl, P);
}

cudaError_t launch_act_quant(const void* x, int x_bf16, int M, int K, int ldq, int8_t* xq, float* scale,
                             int32_t* rowsum, cudaStream_t stream, bool pdl) {
  const QuantArgs a{x, xq, scale, rowsum, K, ldq};
  return launch_act_quant_group(&a, 1, M, x_bf16, stream, pdl);
}

}  // namespace bl
