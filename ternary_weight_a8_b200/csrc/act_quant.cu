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
  uint4* zero;  // a region to clear (16-byte vectors), or null
  long long zero_vecs;
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

  if (P.zero) {
    // This block's slice of the region to clear (the following decode launch's split scratch).
    const long long nb = static_cast<long long>(gridDim.x) * gridDim.y;
    const long long b = static_cast<long long>(blockIdx.y) * gridDim.x + blockIdx.x;
    const long long v0 = P.zero_vecs * b / nb, v1 = P.zero_vecs * (b + 1) / nb;
    for (long long v = v0 + threadIdx.x; v < v1; v += blockDim.x) P.zero[v] = make_uint4(0, 0, 0, 0);
  }
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

// The gains of chunk c (16 floats).
__device__ __forceinline__ void load_gain16(const float* gain, int c, float4 (&g)[4]) {
  const float4* gp = reinterpret_cast<const float4*>(gain + 16 * c);
#pragma unroll
  for (int i = 0; i < 4; ++i) g[i] = __ldg(gp + i);
}

// v = round_to_TX(x * r [* g]) for the 16 inputs of a chunk, g its gains.
template <typename TX>
__device__ __forceinline__ void norm_vals(const Chunk16& raw, float r, bool has_gain, const float4 (&g)[4],
                                          float (&v)[16]) {
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    float t = __fmul_rn(elem<TX>(raw, e), r);
    if (has_gain) {
      const float4 q = g[e >> 2];
      t = __fmul_rn(t, (e & 3) == 0 ? q.x : (e & 3) == 1 ? q.y : (e & 3) == 2 ? q.z : q.w);
    }
    if constexpr (sizeof(TX) == 2) t = __bfloat162float(__float2bfloat16_rn(t));
    v[e] = t;
  }
}

// The same, loading the gains of chunk c.
template <typename TX>
__device__ __forceinline__ void norm_chunk(const Chunk16& raw, float r, const float* gain, int c, float (&v)[16]) {
  float4 g[4];
  if (gain) load_gain16(gain, c, g);
  norm_vals<TX>(raw, r, gain != nullptr, g, v);
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
  // When the token is in registers, the gains of the thread's first kNormKeep
  // chunks are fetched with it (off the path between the two reductions), and
  // the normalised values of those chunks are kept for the codes.
  constexpr int kNormKeep = 2;
  float4 gpre[kNormKeep][4];
  if (in_regs) {
#pragma unroll
    for (int i = 0; i < kQuantRegChunks; ++i) {
      const int c = threadIdx.x + i * T;
      if (c < chunks) load16<TX>(xr + c * 16, reg[i]);
    }
    if (P.gain) {
#pragma unroll
      for (int k = 0; k < kNormKeep; ++k) {
        const int c = threadIdx.x + k * T;
        if (c < chunks) load_gain16(P.gain, c, gpre[k]);
      }
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

  // Absmax of the normalised token.
  float vkeep[kNormKeep][16];
  float amax = 0.0f;
  for_each_chunk([&](const Chunk16& ch, int c) {
    float v[16];
    const int i = (c - static_cast<int>(threadIdx.x)) / T;
    if (in_regs && P.gain && i < kNormKeep) {
      float4 g[4];
#pragma unroll
      for (int k = 0; k < kNormKeep; ++k)
        if (i == k) {
#pragma unroll
          for (int q = 0; q < 4; ++q) g[q] = gpre[k][q];
        }
      norm_vals<TX>(ch, r, true, g, v);
    } else {
      norm_chunk<TX>(ch, r, P.gain, c, v);
    }
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

static cudaError_t launch_rmsnorm_quant_cluster(const NormParams& P, int M, int x_bf16, cudaStream_t stream, bool pdl,
                                                bool* done);

cudaError_t launch_rmsnorm_quant(const void* x, int x_bf16, int M, int K, const float* gain, float eps, void* x_norm,
                                 int8_t* xq, float* scale, int32_t* rowsum, cudaStream_t stream, bool pdl) {
  if (M <= 0) return cudaSuccess;
  const NormParams P{x, gain, eps, x_norm, xq, scale, rowsum, K};
  bool done = false;
  cudaError_t ce = launch_rmsnorm_quant_cluster(P, M, x_bf16, stream, pdl, &done);
  if (done || ce != cudaSuccess) return ce;
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

static cudaError_t launch_glu_quant_cluster(const GluParams& P, int M, int x_bf16, cudaStream_t stream, bool pdl,
                                            bool* done);

cudaError_t launch_glu_quant(const void* gate, const void* up, int x_bf16, int M, int N, int act, void* h,
                             int8_t* xq, float* scale, int32_t* rowsum, cudaStream_t stream, bool pdl) {
  if (M <= 0) return cudaSuccess;
  if (act != kGluRelu2 && act != kGluSilu) return cudaErrorInvalidValue;
  const GluParams P{gate, up, act, h, xq, scale, rowsum, N};
  bool done = false;
  cudaError_t ce = launch_glu_quant_cluster(P, M, x_bf16, stream, pdl, &done);
  if (done || ce != cudaSuccess) return ce;
  int threads = ((N / 16 + 1) / 2 + 31) / 32 * 32;  // about two chunks per thread, 64 .. 512
  if (threads < 64) threads = 64;
  if (threads > kQuantMaxThreads) threads = kQuantMaxThreads;
  if (x_bf16) return launch(glu_quant_kernel<__nv_bfloat16>, dim3(M), dim3(threads), 0, stream, pdl, P);
  return launch(glu_quant_kernel<float>, dim3(M), dim3(threads), 0, stream, pdl, P);
}

// ---------------------------------------------------------------------------
// Decode sizes: a token split over a thread-block cluster
// ---------------------------------------------------------------------------
// With few tokens one block per token leaves most SMs idle and serialises a
// long token through one block's loads and reductions.  Here a cluster of
// C <= 8 CTAs (128 threads each) shares a token: CTA c takes the contiguous
// chunk range [c * chunks / C, (c + 1) * chunks / C), its chunks held in
// registers; each reduction is a block reduction, then the C partial results
// are read from the CTAs' shared memory (distributed shared memory) after a
// cluster barrier, every CTA adding them in rank order.  One more barrier at
// the end keeps every CTA's shared memory alive until its peers have read it.
constexpr int kClusterThreads = 128;
constexpr int kClusterMax = 8;
constexpr int kClusterChunks = 4;  // 16-input chunks per thread, in registers

__device__ __forceinline__ float ld_cluster_f32(const float* p, int rank) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(mapa_shared(smem_u32(p), rank)) : "memory");
  return v;
}
__device__ __forceinline__ int ld_cluster_s32(const int* p, int rank) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(mapa_shared(smem_u32(p), rank)) : "memory");
  return v;
}
__device__ __forceinline__ double ld_cluster_f64(const double* p, int rank) {
  double v;
  asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(mapa_shared(smem_u32(p), rank)) : "memory");
  return v;
}

// Cluster-wide reductions; `slot` is a shared variable used by this reduction only.
__device__ __forceinline__ float cluster_max(float v, float* red, float* slot, int csize) {
  v = block_reduce(v, [](float a, float b) { return fmaxf(a, b); }, red);
  if (threadIdx.x == 0) *slot = v;
  cluster_sync_all();
  float r = 0.0f;
  for (int c = 0; c < csize; ++c) r = fmaxf(r, ld_cluster_f32(slot, c));
  return r;
}
__device__ __forceinline__ int cluster_sum(int v, int* red, int* slot, int csize) {
  v = block_reduce(v, [](int a, int b) { return a + b; }, red);
  if (threadIdx.x == 0) *slot = v;
  cluster_sync_all();
  int r = 0;
  for (int c = 0; c < csize; ++c) r += ld_cluster_s32(slot, c);
  return r;
}
__device__ __forceinline__ double cluster_sum(double v, double* red, double* slot, int csize) {
  v = block_reduce(v, [](double a, double b) { return __dadd_rn(a, b); }, red);
  if (threadIdx.x == 0) *slot = v;
  cluster_sync_all();
  double r = 0.0;
  for (int c = 0; c < csize; ++c) r = __dadd_rn(r, ld_cluster_f64(slot, c));
  return r;
}

// The chunk range of cluster rank `rank` (of csize) over `chunks` chunks, and
// this thread's chunks in it: c0 + threadIdx.x + i * kClusterThreads.
struct ClusterSlice {
  int c0, c1;
};
__device__ __forceinline__ ClusterSlice cluster_slice(int chunks, int rank, int csize) {
  return ClusterSlice{static_cast<int>(static_cast<long long>(chunks) * rank / csize),
                      static_cast<int>(static_cast<long long>(chunks) * (rank + 1) / csize)};
}

// act_quant over a cluster per (item, token): blockIdx.x = token * C + rank, blockIdx.y = item.
template <typename TX>
__global__ void __launch_bounds__(kClusterThreads) act_quant_cluster_kernel(const __grid_constant__ QuantParams P) {
  __shared__ float red_f[kClusterThreads / 32];
  __shared__ int red_i[kClusterThreads / 32];
  __shared__ float slot_max;
  __shared__ int slot_sum;
  griddep_launch_dependents();
  griddep_wait();  // x may be the preceding kernel's output; q may still be read by it
  const int csize = static_cast<int>(cluster_nctarank());
  const int rank = static_cast<int>(cluster_ctarank());
  if (P.zero) {
    const long long nb = static_cast<long long>(gridDim.x) * gridDim.y;
    const long long b = static_cast<long long>(blockIdx.y) * gridDim.x + blockIdx.x;
    const long long v0 = P.zero_vecs * b / nb, v1 = P.zero_vecs * (b + 1) / nb;
    for (long long v = v0 + threadIdx.x; v < v1; v += blockDim.x) P.zero[v] = make_uint4(0, 0, 0, 0);
  }
  const QuantItem& it = P.item[blockIdx.y];
  const int m = blockIdx.x / csize, K = it.K, chunks = K >> 4;
  const TX* xr = static_cast<const TX*>(it.x) + static_cast<size_t>(m) * K;
  int8_t* qr = it.xq + static_cast<size_t>(m) * it.ldq;
  if (rank == csize - 1)
    for (int c = K + 16 * threadIdx.x; c < it.ldq; c += 16 * kClusterThreads)  // row padding
      *reinterpret_cast<uint4*>(qr + c) = make_uint4(0, 0, 0, 0);
  const ClusterSlice sl = cluster_slice(chunks, rank, csize);
  Chunk16 reg[kClusterChunks];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < kClusterChunks; ++i) {
    const int c = sl.c0 + threadIdx.x + i * kClusterThreads;
    if (c < sl.c1) load16<TX>(xr + c * 16, reg[i]);
  }
#pragma unroll
  for (int i = 0; i < kClusterChunks; ++i) {
    const int c = sl.c0 + threadIdx.x + i * kClusterThreads;
    if (c < sl.c1) amax = fmaxf(amax, chunk_absmax<TX>(reg[i]));
  }
  amax = cluster_max(amax, red_f, &slot_max, csize);
  const float s = __fdiv_rn(127.0f, fmaxf(amax, 1e-5f));
  int sum = 0;
#pragma unroll
  for (int i = 0; i < kClusterChunks; ++i) {
    const int c = sl.c0 + threadIdx.x + i * kClusterThreads;
    if (c < sl.c1) sum += quant_chunk<TX>(reg[i], s, qr + c * 16);
  }
  sum = cluster_sum(sum, red_i, &slot_sum, csize);
  if (rank == 0 && threadIdx.x == 0) {
    it.scale[m] = s;
    if (it.rowsum) it.rowsum[m] = sum;
  }
  cluster_sync_all();  // peers may still read this CTA's slots
}

// RMSNorm + quantisation over a cluster per token (blockIdx.x = token * C + rank).
template <typename TX>
__global__ void __launch_bounds__(kClusterThreads) rmsnorm_quant_cluster_kernel(const __grid_constant__ NormParams P) {
  __shared__ double red_d[kClusterThreads / 32];
  __shared__ float red_f[kClusterThreads / 32];
  __shared__ int red_i[kClusterThreads / 32];
  __shared__ double slot_ss;
  __shared__ float slot_max;
  __shared__ int slot_sum;
  griddep_launch_dependents();
  griddep_wait();  // x may be the preceding kernel's output; q may still be read by it
  const int csize = static_cast<int>(cluster_nctarank());
  const int rank = static_cast<int>(cluster_ctarank());
  const int m = blockIdx.x / csize, K = P.K, chunks = K >> 4;
  const TX* xr = static_cast<const TX*>(P.x) + static_cast<size_t>(m) * K;
  int8_t* qr = P.xq + static_cast<size_t>(m) * K;
  TX* nr = P.x_norm ? static_cast<TX*>(P.x_norm) + static_cast<size_t>(m) * K : nullptr;
  const ClusterSlice sl = cluster_slice(chunks, rank, csize);
  Chunk16 reg[kClusterChunks];
#pragma unroll
  for (int i = 0; i < kClusterChunks; ++i) {
    const int c = sl.c0 + threadIdx.x + i * kClusterThreads;
    if (c < sl.c1) load16<TX>(xr + c * 16, reg[i]);
  }
  double ss = 0.0;
#pragma unroll
  for (int i = 0; i < kClusterChunks; ++i) {
    const int c = sl.c0 + threadIdx.x + i * kClusterThreads;
    if (c < sl.c1) {
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const double v = static_cast<double>(elem<TX>(reg[i], e));
        ss = __fma_rn(v, v, ss);
      }
    }
  }
  ss = cluster_sum(ss, red_d, &slot_ss, csize);
  const double ms = __ddiv_rn(ss, static_cast<double>(K));
  const float r = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(ms, static_cast<double>(P.eps)))));
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < kClusterChunks; ++i) {
    const int c = sl.c0 + threadIdx.x + i * kClusterThreads;
    if (c < sl.c1) {
      float v[16];
      norm_chunk<TX>(reg[i], r, P.gain, c, v);
#pragma unroll
      for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(v[e]));
    }
  }
  amax = cluster_max(amax, red_f, &slot_max, csize);
  const float s = __fdiv_rn(127.0f, fmaxf(amax, 1e-5f));
  int sum = 0;
#pragma unroll
  for (int i = 0; i < kClusterChunks; ++i) {
    const int c = sl.c0 + threadIdx.x + i * kClusterThreads;
    if (c < sl.c1) {
      float v[16];
      norm_chunk<TX>(reg[i], r, P.gain, c, v);
      sum += quant_store16<TX>(v, s, qr + c * 16, nr ? nr + c * 16 : nullptr);
    }
  }
  sum = cluster_sum(sum, red_i, &slot_sum, csize);
  if (rank == 0 && threadIdx.x == 0) {
    P.scale[m] = s;
    if (P.rowsum) P.rowsum[m] = sum;
  }
  cluster_sync_all();  // peers may still read this CTA's slots
}

// The gated activation + quantisation over a cluster per token.
template <typename TX>
__global__ void __launch_bounds__(kClusterThreads) glu_quant_cluster_kernel(const __grid_constant__ GluParams P) {
  __shared__ float red_f[kClusterThreads / 32];
  __shared__ int red_i[kClusterThreads / 32];
  __shared__ float slot_max;
  __shared__ int slot_sum;
  griddep_launch_dependents();
  griddep_wait();  // gate and up are the preceding kernel's outputs
  const int csize = static_cast<int>(cluster_nctarank());
  const int rank = static_cast<int>(cluster_ctarank());
  const int m = blockIdx.x / csize, N = P.N, chunks = N >> 4;
  const TX* gr = static_cast<const TX*>(P.gate) + static_cast<size_t>(m) * N;
  const TX* ur = static_cast<const TX*>(P.up) + static_cast<size_t>(m) * N;
  int8_t* qr = P.xq + static_cast<size_t>(m) * N;
  TX* hr = P.h ? static_cast<TX*>(P.h) + static_cast<size_t>(m) * N : nullptr;
  const ClusterSlice sl = cluster_slice(chunks, rank, csize);
  constexpr int kKeep = 2;  // chunks per thread whose h stays in registers
  float hk[kKeep][16];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < kClusterChunks; ++i) {
    const int c = sl.c0 + threadIdx.x + i * kClusterThreads;
    if (c < sl.c1) {
      Chunk16 g, u;
      load16<TX>(gr + c * 16, g);
      load16<TX>(ur + c * 16, u);
      float h[16];
      glu_chunk<TX>(g, u, P.act, h);
#pragma unroll
      for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(h[e]));
      if (i < kKeep) {
#pragma unroll
        for (int e = 0; e < 16; ++e) hk[i < kKeep ? i : 0][e] = h[e];
      }
    }
  }
  amax = cluster_max(amax, red_f, &slot_max, csize);
  const float s = __fdiv_rn(127.0f, fmaxf(amax, 1e-5f));
  int sum = 0;
#pragma unroll
  for (int i = 0; i < kClusterChunks; ++i) {
    const int c = sl.c0 + threadIdx.x + i * kClusterThreads;
    if (c < sl.c1) {
      float h[16];
      if (i < kKeep) {
#pragma unroll
        for (int e = 0; e < 16; ++e) h[e] = hk[i < kKeep ? i : 0][e];
      } else {
        Chunk16 g, u;
        load16<TX>(gr + c * 16, g);
        load16<TX>(ur + c * 16, u);
        glu_chunk<TX>(g, u, P.act, h);
      }
      sum += quant_store16<TX>(h, s, qr + c * 16, hr ? hr + c * 16 : nullptr);
    }
  }
  sum = cluster_sum(sum, red_i, &slot_sum, csize);
  if (rank == 0 && threadIdx.x == 0) {
    P.scale[m] = s;
    if (P.rowsum) P.rowsum[m] = sum;
  }
  cluster_sync_all();  // peers may still read this CTA's slots
}

// CTAs per token for the cluster form (0: use one block per token).  Only
// tokens longer than one block holds at two chunks per thread (512 threads)
// gain: below that the cluster's launch and barriers cost more than they save
// (measured: a one-token RMSNorm at K = 8192 went from 4.3 to 6.7 us as two
// CTAs, the gated activation at N = 28672 from 7.6 to 5.1 us as seven).  The
// plain quantisation reads one input per element instead of two: one block
// holds up to four chunks per thread in registers, and the cluster pays only
// past that (a one-token quantisation at K = 28672: 4.1 us as one block,
// 4.7 us as a cluster; the 70B chain step 39.1 against 39.8 us).
static int cluster_size_for(int M, int k_max, int min_chunks = 2 * kQuantMaxThreads) {
  const int chunks = k_max / 16;
  if (M > 16 || chunks <= min_chunks) return 0;
  int c = (chunks + 2 * kClusterThreads - 1) / (2 * kClusterThreads);  // about two chunks per thread
  if (c > kClusterMax) c = kClusterMax;
  if (chunks > c * kClusterThreads * kClusterChunks) return 0;  // does not fit the registers
  return c;
}

template <typename Kern, typename Params>
static cudaError_t launch_cluster(Kern kernel, dim3 grid, int csize, cudaStream_t stream, bool pdl, const Params& P) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kClusterThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(csize);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, P);
}

static cudaError_t launch_rmsnorm_quant_cluster(const NormParams& P, int M, int x_bf16, cudaStream_t stream, bool pdl,
                                                bool* done) {
  const int csize = cluster_size_for(M, P.K);
  *done = csize > 0;
  if (csize == 0) return cudaSuccess;
  if (x_bf16) return launch_cluster(rmsnorm_quant_cluster_kernel<__nv_bfloat16>, dim3(M * csize), csize, stream, pdl, P);
  return launch_cluster(rmsnorm_quant_cluster_kernel<float>, dim3(M * csize), csize, stream, pdl, P);
}

static cudaError_t launch_glu_quant_cluster(const GluParams& P, int M, int x_bf16, cudaStream_t stream, bool pdl,
                                            bool* done) {
  const int csize = cluster_size_for(M, P.N);
  *done = csize > 0;
  if (csize == 0) return cudaSuccess;
  if (x_bf16) return launch_cluster(glu_quant_cluster_kernel<__nv_bfloat16>, dim3(M * csize), csize, stream, pdl, P);
  return launch_cluster(glu_quant_cluster_kernel<float>, dim3(M * csize), csize, stream, pdl, P);
}

cudaError_t launch_act_quant_group(const QuantArgs* items, int n_items, int M, int x_bf16, cudaStream_t stream,
                                   bool pdl, void* zero, size_t zero_bytes) {
  if (M <= 0 || n_items <= 0) return cudaSuccess;
  if (n_items > kQuantMaxItems) return cudaErrorInvalidValue;
  if ((reinterpret_cast<uintptr_t>(zero) | zero_bytes) % 16 != 0) return cudaErrorInvalidValue;
  QuantParams P = {};
  P.zero = zero_bytes ? static_cast<uint4*>(zero) : nullptr;
  P.zero_vecs = static_cast<long long>(zero_bytes / 16);
  int k_max = 0;
  for (int i = 0; i < n_items; ++i) {
    P.item[i] = QuantItem{items[i].x, items[i].xq, items[i].scale, items[i].rowsum, items[i].K, items[i].ldq};
    if (items[i].K > k_max) k_max = items[i].K;
  }
  P.n_items = n_items;
  const int csize = cluster_size_for(M, k_max, kQuantRegChunks * kQuantMaxThreads);
  if (csize > 0) {
    const dim3 grid(M * csize, n_items);
    if (x_bf16) return launch_cluster(act_quant_cluster_kernel<__nv_bfloat16>, grid, csize, stream, pdl, P);
    return launch_cluster(act_quant_cluster_kernel<float>, grid, csize, stream, pdl, P);
  }
  // About two chunks per thread, in whole warps, 64 .. 512 threads.
  int threads = ((k_max / 16 + 1) / 2 + 31) / 32 * 32;
  if (threads < 64) threads = 64;
  if (threads > kQuantMaxThreads) threads = kQuantMaxThreads;
  const dim3 grid(M, n_items);
  if (x_bf16) return launch(act_quant_kernel<__nv_bfloat16>, grid, dim3(threads), 0, stream, pdl, P);
  return launch(act_quant_kernel<float>, grid, dim3(threads), 0, stream, pdl, P);
}

cudaError_t launch_act_quant(const void* x, int x_bf16, int M, int K, int ldq, int8_t* xq, float* scale,
                             int32_t* rowsum, cudaStream_t stream, bool pdl, void* zero, size_t zero_bytes) {
  const QuantArgs a{x, xq, scale, rowsum, K, ldq};
  return launch_act_quant_group(&a, 1, M, x_bf16, stream, pdl, zero, zero_bytes);
}

}  // namespace bl
