/*
 * bitlinear.h — C ABI of the B200 (sm_100a) BitLinear W1.58A8 forward.
 *
 * The operation, from the BitNet b1.58 pages:
 *  - "BitNet b1.58 and the 1-Bit AI Architecture Revolution", section "The
 *    BitLinear Layer and AbsMean Quantization": gamma is the mean absolute
 *    value of the whole latent weight matrix; every weight is divided by
 *    (gamma + 1e-5), rounded to the nearest integer and clamped to [-1, 1];
 *    gamma is kept beside the ternary matrix.
 *  - "BitNet's Real Bet: Designing the Whole Inference Stack", section "A
 *    low-bit model is a whole-stack design": weights in {-1, 0, +1},
 *    activations on a separate per-token 8-bit path (W1.58A8); the GPU path
 *    stores four ternary values in one int8, moves packed weights from HBM to
 *    on-chip memory, unpacks them and computes with the 8-bit activations.
 *  - same blog, section "The Energy Revolution": the product is integer
 *    additions of 8-bit activations (int32 accumulation here).
 *  - "A Two-Billion Ternary Bet": activations are quantised dynamically.
 *
 * Definitions this library implements (readings where the pages are silent):
 *  gamma   = fp32( (sum_n sum_k |W[n][k]|) / (N*K) ), sums in double, k
 *            ascending within a row, then rows ascending.
 *  t[n][k] = clamp(rint(W[n][k] / (gamma + 1e-5f)), -1, 1), fp32 ops, ties to even.
 *  s[m]    = 127 / max(max_k |x[m][k]|, 1e-5), fp32.
 *  q[m][k] = clamp(rint(x[m][k] * s[m]), -128, 127), fp32 ops, ties to even.
 *  acc     = sum_k q[m][k] * t[n][k]   (int32, exact)
 *  y[m][n] = acc * gamma / s[m]          (fp32 arithmetic, then the output type)
 *
 * Packed weight layout ("four ternary values in one int8"): uint8 [N][K/4],
 * row-major.  Code c = t + 1 in {0, 1, 2}.  The 32-bit little-endian word g of
 * a row holds elements 16g .. 16g+15; element 16g + 4j + b sits in byte b at
 * bits [2j, 2j+1].  So (word >> 2j) & 0x03030303 holds the four consecutive
 * codes 16g+4j .. 16g+4j+3, one per byte.
 *
 * Conventions for every call:
 *  - Pointers named "device" must be CUDA device (or managed, or mapped
 *    pinned host) memory, 16-byte aligned; the workspace must be 256-byte
 *    aligned.  Host-only pointers are rejected with BL_ERR_INVALID_ARG.
 *  - The caller owns and allocates every buffer.  The library allocates no
 *    device memory.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *    only enqueue work; they do not synchronise, except
 *    bitlinear_device_status.
 *  - Shapes: 1 <= N <= 2^24, 64 <= K, K % 64 == 0, 0 <= M.  M == 0 is a no-op.
 *  - Return value: BL_OK or a negative BL_ERR_* code; the message of the most
 *    recent failure on the calling thread is bitlinear_last_error().
 *  - Device-side failures (a bounded wait that ran out) set a bit in the
 *    workspace's status word; bitlinear_device_status reads and clears it.
 *  - A workspace starts with a 256-byte status word, which must be zero
 *    before first use (zero the workspace once after allocating it).  Calls
 *    that overlap on the GPU must not share a workspace.
 *  - The product kernels are launched as programmatic dependents of the
 *    kernel before them on the stream: they start loading the packed
 *    weights while that kernel finishes, and wait for it before reading
 *    anything else (activations, codes, scales, gamma) or writing.  So the
 *    packed weights must not be written by the kernel launched immediately
 *    before the call.  bitlinear_pack_weights ends with a memory operation
 *    (not a kernel) for this reason; weights written by earlier work on the
 *    stream, or copied in by a memory copy, need nothing more.
 */
#ifndef BITLINEAR_H
#define BITLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element types of activations and outputs. */
typedef enum { BL_F32 = 0, BL_BF16 = 1 } bl_dtype;

/* Status codes. */
enum {
  BL_OK = 0,
  BL_ERR_INVALID_ARG = -1,         /* null / host-only pointer, bad dtype, negative size */
  BL_ERR_UNSUPPORTED_SHAPE = -2,   /* K % 64 != 0, K < 64, N < 1, sizes past int32 indexing */
  BL_ERR_MISALIGNED = -3,          /* device pointer not 16-byte (workspace: 256-byte) aligned */
  BL_ERR_WORKSPACE_TOO_SMALL = -4, /* workspace_bytes below the *_workspace_bytes() figure */
  BL_ERR_CUDA = -5,                /* a CUDA runtime call or kernel launch failed */
  BL_ERR_DEVICE_TIMEOUT = -6       /* a device-side bounded wait ran out (device_status only) */
};

/*
 * Workspace bytes bitlinear_pack_weights needs for an N x K matrix
 * (status word + N per-row double sums).
 */
size_t bitlinear_pack_workspace_bytes(int N, int K);

/*
 * Offline weight path: absmean gamma, ternarisation and 2-bit packing
 * ("The BitLinear Layer and AbsMean Quantization"; "A low-bit model is a
 * whole-stack design").
 *   W       device fp32 [N][K], row-major (nn.Linear: out x in) latent weights; read only.
 *   packed  device uint8 [N][K/4] out, layout above.
 *   gamma   device fp32 [1] out.
 *   workspace / workspace_bytes: >= bitlinear_pack_workspace_bytes(N, K).
 * The gamma sum order is fixed (see above), so results are bit-reproducible.
 */
int bitlinear_pack_weights(const float* W, int N, int K, uint8_t* packed, float* gamma,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Per-token 8-bit activation quantisation ("A low-bit model is a whole-stack
 * design"; "A Two-Billion Ternary Bet"), one pass per token.
 *   x       device [M][K] of x_dtype (BL_F32 or BL_BF16); read only.
 *   xq      device int8 [M][K] out: q.
 *   scale   device fp32 [M] out: s.
 *   rowsum  device int32 [M] out, or NULL: sum_k q[m][k].
 */
int bitlinear_quant_act(const void* x, int x_dtype, int M, int K, int8_t* xq, float* scale,
                        int32_t* rowsum, void* stream);

/*
 * The normalisation before a BitLinear fused with its activation
 * quantisation: RMSNorm (the 2024 model) / sub-layer normalisation (the 2B4T
 * model), "BitNet's Real Bet: Designing the Whole Inference Stack", native
 * training section; "BitNet b1.58 and the 1-Bit AI Architecture Revolution",
 * section "Empirical Performance and The New Scaling Law".  The pages give no
 * formula; the reading is v = x * r * g, r = 1 / sqrt(mean_k x^2 + eps),
 * with the squares summed in double, r rounded once to fp32, fp32 products
 * (x * r, then * g), and v rounded to x_dtype as an unfused norm would store
 * it; v is then quantised exactly as bitlinear_quant_act does.  One pass
 * over x per token.
 *   x       device [M][K] of x_dtype (BL_F32 or BL_BF16); read only; 16-byte aligned.
 *   gain    device fp32 [K] (the norm's per-channel weight), or NULL for 1.
 *   eps     the norm's epsilon (>= 0, finite).
 *   x_norm  device [M][K] of x_dtype out, or NULL: v itself (the residual
 *           branch may need it).
 *   xq, scale, rowsum: as bitlinear_quant_act (rowsum may be NULL).
 * Errors: as bitlinear_quant_act; BL_ERR_INVALID_ARG for a negative or
 * non-finite eps.
 */
int bitlinear_rmsnorm_quant(const void* x, int x_dtype, int M, int K, const float* gain, float eps, void* x_norm,
                            int8_t* xq, float* scale, int32_t* rowsum, void* stream);

/* The FFN's gated activation (see bitlinear_glu_quant). */
typedef enum { BL_GLU_RELU2 = 0, BL_GLU_SILU = 1 } bl_glu;

/*
 * The FFN's gated activation between the gate/up BitLinears and the down
 * BitLinear, fused with the quantisation of the down BitLinear's input:
 * squared ReLU (the 2B4T model) or SwiGLU (the 2024 model), "BitNet's Real
 * Bet: Designing the Whole Inference Stack", native training section; "A
 * Two-Billion Ternary Bet" (squared-ReLU-style activations).  The pages give
 * no formula; the reading is h = act(gate) * up on the stored gate and up
 * values, in fp32: BL_GLU_RELU2 (g * g) * up with g = max(gate, 0),
 * BL_GLU_SILU gate / (1 + expf(-gate)) * up; h is rounded to x_dtype and
 * quantised exactly as bitlinear_quant_act does.  One pass per token.
 *   gate, up device [M][N] of x_dtype (BL_F32 or BL_BF16), e.g. the y of the
 *           gate and up BitLinears; read only; 16-byte aligned.
 *   act     BL_GLU_RELU2 or BL_GLU_SILU.
 *   h       device [M][N] of x_dtype out, or NULL: h itself.
 *   xq, scale, rowsum: as bitlinear_quant_act with K = N (rowsum may be NULL);
 *           they feed bitlinear_forward_quantized of the down BitLinear.
 * N >= 64 and N % 64 == 0 (the down BitLinear's K).  Errors: as
 * bitlinear_quant_act; BL_ERR_INVALID_ARG for an unknown act.
 */
int bitlinear_glu_quant(const void* gate, const void* up, int x_dtype, int M, int N, int act, void* h,
                        int8_t* xq, float* scale, int32_t* rowsum, void* stream);

/* Workspace bytes bitlinear_gate_up_glu needs for M tokens, gate/up N x K. */
size_t bitlinear_gate_up_glu_workspace_bytes(int M, int N, int K);

/*
 * The FFN's gate and up BitLinears, the gated activation between them and the
 * down BitLinear, and the quantisation of its result for the down BitLinear,
 * as one call ("BitNet's Real Bet: Designing the Whole Inference Stack",
 * native training section: SwiGLU for the 2024 model, squared ReLU for 2B4T;
 * "A Two-Billion Ternary Bet": squared-ReLU-style activations).  The result
 * equals, bit for bit, bitlinear_layer_chain of the gate and up BitLinears
 * on x (outputs in x_dtype) followed by bitlinear_glu_quant of their outputs.
 *   packed_gate, gamma_gate, packed_up, gamma_up: the two BitLinears (each its
 *           own gamma), N x K each; N % 64 == 0 (N is the down BitLinear's K).
 *   x       device [M][K] of x_dtype, the FFN's (normalised) input.
 *   act     BL_GLU_RELU2 or BL_GLU_SILU, as bitlinear_glu_quant.
 *   h       device [M][N] of x_dtype out, or NULL: h itself.
 *   xq, scale, rowsum: device int8 [M][N], fp32 [M], int32 [M] out: the
 *           codes of h, as bitlinear_quant_act would make them; they feed the
 *           down BitLinear (bitlinear_forward_quantized, or a chain layer's
 *           xq / scale / rowsum).
 *   workspace / workspace_bytes: >= bitlinear_gate_up_glu_workspace_bytes(M, N, K),
 *           its first 256 bytes zero.
 * M <= 8: one quantisation launch (or, for tiny x, none) and one decode
 * launch that computes gate and up, forms h as soon as both halves of a
 * group of rows are in, keeps the per-token maxima of |h| and, once every
 * row is in, quantises h with the final scales (no further launch).  That
 * launch waits grid-wide for its blocks, which it sizes for three per SM of
 * the whole device: on a device partitioned so that fewer can be resident
 * (an MPS limit on SMs, say) the wait runs out after 2 s and the call
 * reports BL_ERR_DEVICE_TIMEOUT through the workspace status word.
 * 9 <= M <= 16: the gate and up products into the workspace, then the
 * gated-activation kernel (there the fused launch's grid-wide step cost more
 * than the launch it saves).  Larger M: the quantisation of x, one
 * tensor-core GEMM whose tiles pair 128 gate rows with the same 128 up rows
 * so that its epilogue writes h, then the quantisation of h.
 */
int bitlinear_gate_up_glu(const uint8_t* packed_gate, const float* gamma_gate, const uint8_t* packed_up,
                          const float* gamma_up, int N, int K, const void* x, int x_dtype, int M, int act, void* h,
                          int8_t* xq, float* scale, int32_t* rowsum, void* workspace, size_t workspace_bytes,
                          void* stream);

/*
 * The product and dequantisation of one token by table lookup instead of
 * multiplication: the T-MAC approach ("BitNet b1.58 and the 1-Bit AI
 * Architecture Revolution", section "The CPU Revival: bitnet.cpp and T-MAC":
 * four ternary weights leave few partial sums, precomputed and looked up,
 * with the sign structure reducing the tables to 16 binary combinations).
 * Here each 16-entry table holds the subset sums of the 4 codes of q that
 * share a packed byte, and a byte's two bit planes index it
 * (sum c*q = T[lo] + 2 T[hi]).  The result equals bitlinear_forward_quantized's
 * bit for bit (acc) and at its bars (y); it exists to compare the two
 * decode algorithms.
 *   packed, gamma, N, K: as bitlinear_forward; K % 64 == 0 and K <= 24576
 *           (the tables take 8 bytes of shared memory per input).
 *   xq, scale, rowsum: one token's codes [K], scale [1], code sum [1] as
 *           bitlinear_quant_act wrote them (rowsum required).
 *   M       must be 1.
 *   y, y_dtype, acc_out: as bitlinear_forward_quantized.
 * No workspace.  Errors: BL_ERR_UNSUPPORTED_SHAPE for M != 1 or K out of
 * range; the rest as bitlinear_forward_quantized.
 */
int bitlinear_forward_lut(const uint8_t* packed, const float* gamma, int N, int K, const int8_t* xq,
                          const float* scale, const int32_t* rowsum, int M, void* y, int y_dtype, int32_t* acc_out,
                          void* stream);

/* Workspace bytes bitlinear_ste_backward needs for M tokens of an N x K BitLinear. */
size_t bitlinear_ste_workspace_bytes(int M, int N, int K);

/*
 * The straight-through backward of a BitLinear, for training on latent
 * ("shadow") weights: "BitNet b1.58 and the 1-Bit AI Architecture
 * Revolution", section "Training Dynamics: The Straight-Through Estimator"
 * (the backward treats the quantisation as the identity; gradients reach the
 * high-precision shadow weights, which are quantised again, with
 * bitlinear_pack_weights, before the next forward).  With the forward
 * y = xhat . What^T, xhat = q / s and What = gamma * t:
 *   dx = gamma * (dy . t)   and   dW = dy^T . xhat,
 * xhat taken as the backward stores it, bf16(q / s).  Both products run on
 * the tensor cores (bf16 operands, fp32 accumulation).
 *   packed, gamma, N, K: the weights of the forward (N % 64 == 0, K % 64 == 0).
 *   dy      device bf16 [M][N]: the output gradient; M % 8 == 0.
 *   xq, scale: the forward's codes [M][K] and scales [M] (bitlinear_quant_act).
 *   dx      device [M][K] of dx_dtype out, or NULL to skip.
 *   dw      device fp32 [N][K] out, or NULL to skip (the gradient of the latent weights).
 *   workspace / workspace_bytes: >= bitlinear_ste_workspace_bytes(M, N, K), first 256 bytes zero.
 */
int bitlinear_ste_backward(const uint8_t* packed, const float* gamma, int N, int K, const void* dy,
                           const int8_t* xq, const float* scale, int M, void* dx, int dx_dtype, float* dw,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes bitlinear_forward needs (status word + q, s, rowsum). */
size_t bitlinear_workspace_bytes(int M, int N, int K);

/*
 * The BitLinear W1.58A8 forward: quantise x per token, ternary x int8
 * product with int32 accumulation, fused dequantisation by gamma and s.
 *   packed  device uint8 [N][K/4] (from bitlinear_pack_weights); gamma device fp32 [1].
 *   x       device [M][K] of x_dtype.
 *   y       device [M][N] of y_dtype out.
 *   acc_out device int32 [M][N] out, or NULL: the exact accumulators
 *           sum_k q*t (for parity checks).
 *   workspace / workspace_bytes: >= bitlinear_workspace_bytes(M, N, K), its
 *           first 256 bytes zero.
 * M <= 16 runs the decode GEMV kernel (which quantises small activations
 * itself: M * K up to 4096, or one bf16 token of up to 9856 inputs; else the
 * quantisation kernel runs first); larger M the quantisation kernel and the
 * tcgen05 tensor-core GEMM.
 */
int bitlinear_forward(const uint8_t* packed, const float* gamma, int N, int K, const void* x,
                      int x_dtype, int M, void* y, int y_dtype, int32_t* acc_out, void* workspace,
                      size_t workspace_bytes, void* stream);

/*
 * The product and dequantisation on activations already quantised by
 * bitlinear_quant_act (xq, scale, rowsum as it wrote them; rowsum required).
 * Only the workspace's status word is used (256 bytes suffice).
 */
int bitlinear_forward_quantized(const uint8_t* packed, const float* gamma, int N, int K,
                                const int8_t* xq, const float* scale, const int32_t* rowsum,
                                int M, void* y, int y_dtype, int32_t* acc_out, void* workspace,
                                size_t workspace_bytes, void* stream);

/*
 * One BitLinear of a chain: weights, gamma, shape, input [M][K], output [M][N].
 *   x       device [M][K] activations of the chain's x_dtype; ignored (may be
 *           NULL) when xq is set.
 *   xq, scale, rowsum: NULL, or the layer's input already quantised, as
 *           bitlinear_quant_act or bitlinear_glu_quant wrote it (codes
 *           [M][K], scales [M], code sums [M]): the chain then quantises
 *           nothing for this layer.
 *   acc_out NULL, or device int32 [M][N] out: the layer's exact accumulators
 *           (for parity checks).
 */
typedef struct {
  const uint8_t* packed;
  const float* gamma;
  int N;
  int K;
  const void* x;
  void* y;
  const int8_t* xq;
  const float* scale;
  const int32_t* rowsum;
  int32_t* acc_out;
} bl_layer;

/* Workspace bytes bitlinear_layer_chain needs for these layers at M tokens. */
size_t bitlinear_chain_workspace_bytes(const bl_layer* layers, int n_layers, int M);

/*
 * Runs n_layers BitLinear forwards back to back on one stream.  Consecutive
 * layers that read the same x pointer with the same K (e.g. FFN gate and up)
 * share one activation quantisation; each keeps its own gamma.  At decode
 * sizes (M <= 16), consecutive layers that are independent of one another
 * (no layer reads what another writes) run in one launch of the decode
 * kernel.  `layers` is a host array, read during the call only; at most 64
 * layers.  The workspace (>= bitlinear_chain_workspace_bytes) starts with a
 * zero status block, as every workspace does.
 */
int bitlinear_layer_chain(const bl_layer* layers, int n_layers, int M, int x_dtype, int y_dtype,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronises `stream`, returns BL_OK or BL_ERR_DEVICE_TIMEOUT from the
 * workspace's status word, and clears the word.
 */
int bitlinear_device_status(void* workspace, void* stream);

/*
 * Exercises the device-side bounded wait: launches one block that waits on a
 * barrier nothing completes, with a limit of `limit_us` microseconds
 * (1 .. 1000000); the wait gives up, sets the status word and returns.  A
 * following bitlinear_device_status reports BL_ERR_DEVICE_TIMEOUT.
 */
int bitlinear_selftest_wait_timeout(void* workspace, size_t workspace_bytes, int limit_us,
                                    void* stream);

/*
 * The forward of bitlinear_forward for callers that cannot allocate device
 * memory.  (The pages have no counterpart: this is a deployment aid.)
 *
 * Who needs it: code where cudaMalloc is off limits because it can
 * synchronise the device (latency-critical decode loops, real-time
 * threads); plug-ins inside an engine that owns all device memory through
 * its own pool and offers them no allocator; callers that hold a device-wide
 * lock they must not block under.  Such callers pass only inputs and
 * outputs (arguments as for bitlinear_forward, without the workspace).
 *
 * The scratch is a fixed 1 MiB array in device memory that the library
 * declares once; every GPU that loads the library holds it until the
 * process exits.  What a call needs of it depends on the kernel that runs:
 * 256 bytes when the decode kernel quantises the activations itself (M * K
 * up to 4096, or one bf16 token of up to 9856 inputs), else 256 bytes plus
 * about M * K bytes for the codes (exactly
 * bitlinear_workspace_bytes(M, N, K)).  Larger calls are refused with
 * BL_ERR_WORKSPACE_TOO_SMALL.  All calls share the array and each call first
 * clears its 256-byte control block, so calls in one stream are safe but
 * calls that overlap on the GPU (other streams, other host threads) race on
 * it.  The first call on a device (and the first after the device's context
 * changes, e.g. after cudaDeviceReset) looks up the array's device address
 * with that device current and caches it per device and context; make that
 * first call before any stream capture.  Device-side wait failures are
 * recorded in the shared control block and wiped by the next call's clear:
 * read them between calls with bitlinear_noalloc_status.
 */
int bitlinear_forward_noalloc(const uint8_t* packed, const float* gamma, int N, int K, const void* x,
                              int x_dtype, int M, void* y, int y_dtype, int32_t* acc_out, void* stream);

/*
 * For bitlinear_forward_noalloc callers: synchronises `stream`, then returns
 * BL_OK or BL_ERR_DEVICE_TIMEOUT from the shared control block's status word
 * (as bitlinear_device_status does for a workspace) and clears the word.
 * Call it after a no-allocation call and before the next one.  Allocates
 * nothing.
 */
int bitlinear_noalloc_status(void* stream);

/* Forces the product kernel: 0 = by M (default), 1 = GEMV (M <= 16 only), 2 = GEMM.  Per thread. */
int bitlinear_set_path(int path);

/*
 * Forces how many CTAs (a thread-block cluster, 1 .. 8) share each unit of
 * 64 weight rows in the decode kernel, each over its own range of K, on the
 * calling thread: 0 (default) lets the kernel choose (it splits short, wide
 * layers, whose units are too few for the SMs).  The split is capped by the
 * layer's 1024-input stages and by the CTAs resident at once.  For tests and
 * tuning; the fused gate/up call never splits.
 */
int bitlinear_set_decode_split(int ctas);

/*
 * Chooses the form of the decode product for 2 to 16 tokens whose input is
 * int8 codes (every decode call quantises first unless the decode kernel
 * quantises tiny inputs itself), on the calling thread: 0 (default) and 1
 * the CUDA-core form (mma.sync); 2 the tensor-core form (tcgen05.mma
 * kind::i8 with the unpacked ternary codes in tensor memory, one block per
 * SM) whenever the call is eligible (2 to 16 tokens on codes, not the fused
 * gate/up call).  Both give bit-identical results; the tensor-core form is
 * slower (each of its 128-row x 16-token MMAs costs about as much as a
 * full-width one, so feeding the unpacked codes through the tensor cores,
 * not HBM, sets its pace), so it is never chosen by default.  For tests and
 * measurement.  Returns BL_ERR_INVALID_ARG for any other value.
 */
int bitlinear_set_decode_form(int form);

/* Message of the most recent failure on the calling thread ("" if none). */
const char* bitlinear_last_error(void);

/* Library version, as MAJOR*10000 + MINOR*100 + PATCH. */
int bitlinear_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H */
