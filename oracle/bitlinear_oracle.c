/*
 * CPU oracle for the BitLinear W1.58A8 forward.
 *
 * TEST INFRASTRUCTURE ONLY.  The parity tests, the package's smoke check and
 * the bench's CPU-baseline leg are the only callers.  The CUDA library never
 * links, loads or calls this file, and this file includes nothing of it.
 *
 * Plain, slow, scalar C: one loop per step, in the order the pages give the
 * steps, so that each function can be checked against its passage by eye.
 * Built with -O2 -ffp-contract=off and no fast-math, so on x86-64 every fp32
 * operation below is one IEEE-754 single-precision operation (SSE) and every
 * double operation one IEEE-754 double operation.
 *
 * Sources (web pages on BitNet b1.58):
 *  [AbsMean] "BitNet b1.58 and the 1-Bit AI Architecture Revolution",
 *            section "The BitLinear Layer and AbsMean Quantization": gamma is
 *            the mean absolute value of the whole weight matrix; each weight
 *            is divided by (gamma + eps), eps = 1e-5, rounded to the nearest
 *            integer and clamped to [-1, 1]; gamma is returned beside the
 *            ternary matrix.
 *  [Stack]   "BitNet's Real Bet: Designing the Whole Inference Stack",
 *            section "A low-bit model is a whole-stack design": weights in
 *            {-1, 0, +1}, activations on a separate per-token 8-bit path
 *            (W1.58A8); the GPU path stores four ternary values in one int8.
 *  [Energy]  same blog as [AbsMean], section "The Energy Revolution": the
 *            product reduces to integer additions of 8-bit activations.
 *  [GLU]     "BitNet's Real Bet: Designing the Whole Inference Stack" (native
 *            training section: the 2024 model uses SwiGLU, the 2B4T model
 *            squared ReLU) and "A Two-Billion Ternary Bet" (squared-ReLU-style
 *            activations tame gradient scale): the gated activation between
 *            the gate/up BitLinears and the down BitLinear of the FFN.
 *  [STE]     "BitNet b1.58 and the 1-Bit AI Architecture Revolution", section
 *            "Training Dynamics: The Straight-Through Estimator": the backward
 *            pass treats the quantisation as the identity, so gradients pass
 *            through the quantised weights to the high-precision shadow
 *            weights, which are quantised again before the next forward.
 *  [Norm]    "BitNet's Real Bet: Designing the Whole Inference Stack" (native
 *            training section: the 2024 model uses RMSNorm, the 2B4T model
 *            sub-layer normalisation) and "A Two-Billion Ternary Bet"
 *            (sub-layer normalisation stabilises training): the normalisation
 *            that precedes a BitLinear's activation quantisation.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *  - gamma is summed in double precision in a fixed order: each row's |w|
 *    over k ascending, then the row sums over n ascending; the mean is that
 *    sum divided by N*K in double, rounded once to fp32.
 *  - The divide, round and clamp of the ternarisation run in fp32 (the
 *    section's weights are fp32 tensors); rounding is to nearest, ties to
 *    even.  The divisor is gamma + 1e-5: the section fixes eps = 1e-5 as the
 *    guard added to gamma (an all-zero matrix then ternarises to zeros).
 *  - Per-token 8-bit quantisation is symmetric absmax: s = 127 / max(amax,
 *    1e-5) in fp32, q = clamp(rint(x * s), -128, 127) (ties to even).
 *  - Dequantisation is y = acc * gamma / s, evaluated in double (gamma, not
 *    gamma + eps: the section keeps gamma itself beside the ternary matrix).
 *  - Storage: code c = t + 1 in {0, 1, 2}, two bits each, four to a byte;
 *    32-bit little-endian word g of a row holds elements 16g .. 16g+15, and
 *    element 16g + 4j + b sits in byte b at bits [2j, 2j+1].
 *  - RMSNorm (the pages name it without a formula): v = x * r * g with
 *    r = 1 / sqrt(mean(x^2) + eps), g an optional per-channel gain; the
 *    squares are summed in double over k ascending, r is formed in double
 *    and rounded once to fp32, the products x * r then * g are fp32, and v
 *    is rounded to the activation type (bf16 round-to-nearest-even for bf16
 *    inputs), as an unfused norm that writes its output would store it.
 *  - Gated activation (named, no formula): h = act(gate) * up with
 *    act = ReLU(z)^2 (2B4T) or SiLU(z) = z / (1 + e^-z) (SwiGLU); gate and up
 *    are the BitLinear outputs as stored (activation type); h is rounded to
 *    the activation type.  Squared ReLU is two fp32 multiplies, (g * g) * u
 *    with g = max(gate, 0); SiLU is evaluated exactly (double) and rounded
 *    once, the GPU's fp32 evaluation being held to a stated bar.
 *  - Straight-through backward: the forward is y = xhat . What^T with
 *    xhat = q / s (per token) and What = gamma * t; the quantisers pass
 *    gradients unchanged, so dx = dy . What = gamma * (dy . t) and
 *    dW = dy^T . xhat.  xhat enters as the backward stores it: q / s in fp32
 *    rounded to bf16.  Both products are evaluated in double.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_EPS 1e-5f

/* [AbsMean]: gamma is the average absolute value of the entire weight matrix. */
float oracle_absmean_gamma(const float* W, int64_t N, int64_t K, double* sum_out) {
  double total = 0.0;
  for (int64_t n = 0; n < N; ++n) {
    double row = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      row += fabs((double)W[n * K + k]);
    }
    total += row;
  }
  if (sum_out) *sum_out = total;
  if (N * K == 0) return 0.0f;
  return (float)(total / (double)(N * K));
}

/* [AbsMean]: every weight divided by the gamma scale (plus eps), rounded to the
 * nearest integer, clamped so that no value leaves [-1, 1]. */
void oracle_ternarize(const float* W, int64_t count, float gamma, int8_t* T) {
  float d = gamma + ORACLE_EPS;
  for (int64_t i = 0; i < count; ++i) {
    float r = W[i] / d;
    float t = rintf(r);
    if (t > 1.0f) t = 1.0f;
    if (t < -1.0f) t = -1.0f;
    T[i] = (int8_t)t;
  }
}

/* [Stack]: four ternary values per byte, in this library's 2-bit layout. */
int oracle_pack(const int8_t* T, int64_t N, int64_t K, uint8_t* P) {
  if (K % 16 != 0) return -1;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < K / 16; ++g) {
      uint32_t word = 0;
      for (int j = 0; j < 4; ++j) {
        for (int b = 0; b < 4; ++b) {
          int8_t t = T[n * K + 16 * g + 4 * j + b];
          if (t < -1 || t > 1) return -2;
          uint32_t code = (uint32_t)(t + 1);
          word |= code << (8 * b + 2 * j);
        }
      }
      uint8_t* dst = P + n * (K / 4) + 4 * g;
      dst[0] = (uint8_t)(word & 0xff);
      dst[1] = (uint8_t)((word >> 8) & 0xff);
      dst[2] = (uint8_t)((word >> 16) & 0xff);
      dst[3] = (uint8_t)((word >> 24) & 0xff);
    }
  }
  return 0;
}

/* Inverse of oracle_pack.  Returns -1 if a code 3 (not a ternary value) appears. */
int oracle_unpack(const uint8_t* P, int64_t N, int64_t K, int8_t* T) {
  if (K % 16 != 0) return -2;
  int bad = 0;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < K / 16; ++g) {
      const uint8_t* src = P + n * (K / 4) + 4 * g;
      uint32_t word = (uint32_t)src[0] | ((uint32_t)src[1] << 8) | ((uint32_t)src[2] << 16) |
                      ((uint32_t)src[3] << 24);
      for (int j = 0; j < 4; ++j) {
        for (int b = 0; b < 4; ++b) {
          uint32_t code = (word >> (8 * b + 2 * j)) & 3u;
          if (code == 3u) bad = 1;
          T[n * K + 16 * g + 4 * j + b] = (int8_t)((int)code - 1);
        }
      }
    }
  }
  return bad ? -1 : 0;
}

/* [Stack]: per-token 8-bit activations (absmax reading, see header). */
void oracle_quant_act(const float* x, int64_t M, int64_t K, int8_t* q, float* s, int32_t* rowsum) {
  for (int64_t m = 0; m < M; ++m) {
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(x[m * K + k]);
      if (a > amax) amax = a;
    }
    float scale = 127.0f / fmaxf(amax, ORACLE_EPS);
    int64_t sum = 0;
    for (int64_t k = 0; k < K; ++k) {
      float v = rintf(x[m * K + k] * scale);
      if (v > 127.0f) v = 127.0f;
      if (v < -128.0f) v = -128.0f;
      q[m * K + k] = (int8_t)v;
      sum += (int8_t)v;
    }
    s[m] = scale;
    if (rowsum) rowsum[m] = (int32_t)sum;
  }
}

/*
 * [Energy]: acc[m][n] = sum_k q[m][k] * t[n][k], exact in 64-bit integers.
 * Returns 0, or -1 if some sum does not fit in int32.
 */
int oracle_accumulate(const int8_t* q, const int8_t* T, int64_t M, int64_t N, int64_t K,
                      int32_t* acc) {
  int overflow = 0;
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t n = 0; n < N; ++n) {
      int64_t sum = 0;
      for (int64_t k = 0; k < K; ++k) {
        sum += (int64_t)q[m * K + k] * (int64_t)T[n * K + k];
      }
      if (sum > INT32_MAX || sum < INT32_MIN) overflow = 1;
      acc[m * N + n] = (int32_t)sum;
    }
  }
  return overflow ? -1 : 0;
}

/* y[m][n] = acc[m][n] * gamma / s[m], in double. */
void oracle_dequant(const int32_t* acc, float gamma, const float* s, int64_t M, int64_t N,
                    double* y) {
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t n = 0; n < N; ++n) {
      y[m * N + n] = (double)acc[m * N + n] * (double)gamma / (double)s[m];
    }
  }
}

/* double -> fp32, round to nearest even. */
void oracle_round_f32(const double* y, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = (float)y[i];
}

/* double -> bf16 bit pattern, rounded once to nearest even (not via fp32). */
static uint16_t oracle_bf16_of(double y) {
  uint16_t sign = signbit(y) ? 0x8000u : 0u;
  if (isnan(y)) return 0x7fc0u;
  double a = fabs(y);
  if (a == 0.0) return sign;
  if (isinf(a)) return (uint16_t)(sign | 0x7f80u);
  int e;
  frexp(a, &e);              /* a = f * 2^e, f in [0.5, 1) */
  int qexp = e - 8;          /* bf16 keeps 8 significant bits */
  if (qexp < -133) qexp = -133; /* subnormal spacing 2^-133 */
  double r = rint(ldexp(a, -qexp));
  double v = ldexp(r, qexp); /* at most 8 significant bits: exact in fp32 */
  float f = (float)v;        /* overflows to inf past the fp32 range */
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f7f0000u) u = 0x7f800000u;
  return (uint16_t)(sign | (uint16_t)((u >> 16) & 0x7fffu));
}

void oracle_round_bf16(const double* y, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_of(y[i]);
}

/* [Norm]: per-token RMSNorm, output rounded to the activation type (values as fp32). */
void oracle_rmsnorm(const float* x, int64_t M, int64_t K, const float* g, float eps, int out_bf16,
                    float* out) {
  for (int64_t m = 0; m < M; ++m) {
    double ss = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      double v = (double)x[m * K + k];
      ss += v * v;
    }
    double ms = ss / (double)K;
    float r = (float)(1.0 / sqrt(ms + (double)eps));
    for (int64_t k = 0; k < K; ++k) {
      float v = x[m * K + k] * r;
      if (g) v = v * g[k];
      if (out_bf16) {
        uint16_t h = oracle_bf16_of((double)v);
        uint32_t u = (uint32_t)h << 16;
        memcpy(&v, &u, 4);
      }
      out[m * K + k] = v;
    }
  }
}

/* [GLU]: h = act(gate) * up, rounded to the activation type (values as fp32).
 * act 0: squared ReLU in fp32; act 1: SiLU, exact then rounded once. */
void oracle_glu(const float* gate, const float* up, int64_t count, int act, int out_bf16, float* out) {
  for (int64_t i = 0; i < count; ++i) {
    float h;
    if (act == 0) {
      float g = gate[i] > 0.0f ? gate[i] : 0.0f;
      h = (g * g) * up[i];
    } else {
      double z = (double)gate[i];
      h = (float)(z / (1.0 + exp(-z)) * (double)up[i]);
    }
    if (out_bf16) {
      uint16_t b = oracle_bf16_of(act == 0 ? (double)h : (double)gate[i] / (1.0 + exp(-(double)gate[i])) *
                                                            (double)up[i]);
      uint32_t u = (uint32_t)b << 16;
      memcpy(&h, &u, 4);
    }
    out[i] = h;
  }
}

/* [STE]: dx[m][k] = gamma * sum_n dy[m][n] * t[n][k], in double. */
void oracle_ste_grad_input(const float* dy, const int8_t* T, float gamma, int64_t M, int64_t N, int64_t K,
                           double* dx) {
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t k = 0; k < K; ++k) {
      double sum = 0.0;
      for (int64_t n = 0; n < N; ++n) sum += (double)dy[m * N + n] * (double)T[n * K + k];
      dx[m * K + k] = (double)gamma * sum;
    }
  }
}

/* [STE]: the stored dequantised activations, xhat = bf16(fp32(q / s)), as fp32 values. */
void oracle_ste_xhat(const int8_t* q, const float* s, int64_t M, int64_t K, float* xhat) {
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t k = 0; k < K; ++k) {
      float v = (float)q[m * K + k] / s[m];
      uint16_t h = oracle_bf16_of((double)v);
      uint32_t u = (uint32_t)h << 16;
      memcpy(&v, &u, 4);
      xhat[m * K + k] = v;
    }
  }
}

/* [STE]: dW[n][k] = sum_m dy[m][n] * xhat[m][k], in double. */
void oracle_ste_grad_weight(const float* dy, const float* xhat, int64_t M, int64_t N, int64_t K, double* dw) {
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      double sum = 0.0;
      for (int64_t m = 0; m < M; ++m) sum += (double)dy[m * N + n] * (double)xhat[m * K + k];
      dw[n * K + k] = sum;
    }
  }
}
