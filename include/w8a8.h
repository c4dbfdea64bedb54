/*
 * w8a8.h - C ABI of libw8a8.so, a B200 (sm_100a) W8A8 quantized Linear.
 *
 * The operation (OneTrainer wiki "Quantization", int W8A8 and float W8A8
 * paragraphs, "Technical:" lines): weights are quantized tensor-wise to int8
 * or float8 e4m3, activations are quantized token-wise during training, and
 * the Linear layer's matrix multiplication runs in int8 / float8.  The GGUF A8
 * int paragraph adds weights re-quantized from GGUF blocks to int8 axis-wise;
 * the SVDQuant paragraph adds a bfloat16 low-rank branch.
 *
 * Notation: X[M,K] bf16 activations, W[N,K] bf16 weight (nn.Linear layout),
 * Y[M,N] = X W^T, all row-major.  Codes are int8 or OCP E4M3FN bytes; scales
 * are fp32.  QMAX = 127 (int8) or 448 (e4m3).
 *
 * Conventions shared by every call
 *  - Ownership: the caller owns every buffer.  All data pointers are DEVICE
 *    pointers unless stated otherwise.  The library never allocates, frees or
 *    synchronizes inside a compute call; workspace is passed in by the caller
 *    (size from w8a8_workspace_bytes).
 *  - Streams: all work is enqueued on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream).  Calls return as soon as the work is enqueued.
 *    Calls on one stream take effect in stream order, whatever produced
 *    their inputs (a previous call, e.g. a weight preparation, or any other
 *    kernel): a call's kernels may be launched while the kernel before them
 *    finishes (programmatic dependent launch) and set themselves up, but
 *    read nothing before it has completed.  The one early read - the weight
 *    tiles of a few-row or split product in w8a8_linear_fwd(_ex),
 *    w8a8_linear_fwd_noalloc, w8a8_linear_dgrad and svdq_linear_fwd(_e4m3) -
 *    comes after that call's own row quantizer, which waits for every
 *    earlier kernel on the stream first.
 *  - Alignment: every device pointer must be 16-byte aligned
 *    (W8A8_ERR_MISALIGNED otherwise) - the alignment to 16 that fixed the
 *    misaligned-address offloading bug in OneTrainer PR #1034, Known issues.
 *  - Shapes: M >= 0 (M == 0 is a no-op that returns W8A8_OK), N >= 1,
 *    K >= 16 and K % 16 == 0 (tensor-copy row strides are 16-byte multiples;
 *    cf. the cuBLASLt m/k shape limits in bitsandbytes #1401, Next steps).
 *    Other shapes return W8A8_ERR_UNSUPPORTED_SHAPE before any launch.
 *  - Inputs are finite (no NaN/Inf); results for non-finite inputs are
 *    unspecified.
 *  - Tracing: every compute call is one NVTX range named after the call
 *    (nested when one call is built on another), so a profiler's timeline
 *    groups each call's launches; without a profiling tool the ranges cost
 *    nothing measurable.
 *  - Errors: argument errors return before any launch.  A failed launch
 *    returns W8A8_ERR_CUDA.  A device that is not compute capability 10.0
 *    returns W8A8_ERR_UNSUPPORTED_DEVICE; there is no CPU fallback.  Kernels
 *    never trap: every wait on the GPU is bounded, and a wait that runs out
 *    records W8A8_ERR_DEVICE_TIMEOUT in a per-device status word that
 *    w8a8_device_status() reads.  w8a8_last_error() gives a message for the
 *    last failing call of the calling thread.
 */
#ifndef W8A8_H
#define W8A8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared without the CUDA headers. */
struct CUstream_st;
typedef struct CUstream_st* w8a8_stream_t;

typedef enum {
  W8A8_OK = 0,
  W8A8_ERR_INVALID_ARG = 1,
  W8A8_ERR_UNSUPPORTED_SHAPE = 2,
  W8A8_ERR_MISALIGNED = 3,
  W8A8_ERR_WORKSPACE = 4,
  W8A8_ERR_CUDA = 5,
  W8A8_ERR_DEVICE_TIMEOUT = 6,
  W8A8_ERR_UNSUPPORTED_DEVICE = 7,
  W8A8_ERR_DEVICE_BOUNDS = 8   /* debug build only: a device-side index check failed */
} w8a8_status;

typedef enum { W8A8_INT8 = 0, W8A8_E4M3 = 1 } w8a8_qtype;
typedef enum { W8A8_TENSOR = 0, W8A8_AXIS = 1 } w8a8_wgran;
typedef enum { W8A8_ACT_NONE = 0, W8A8_ACT_GELU = 1, W8A8_ACT_GELU_TANH = 2 } w8a8_act;
typedef enum {
  W8A8_OP_LINEAR_FWD = 0,      /* w8a8_linear_fwd                          */
  W8A8_OP_LINEAR_DGRAD = 1,    /* w8a8_linear_dgrad                        */
  W8A8_OP_SVDQ_FWD = 2,        /* svdq_linear_fwd                          */
  W8A8_OP_QUANTIZE_WEIGHT = 3, /* w8a8_quantize_weight (TENSOR needs 256 B) */
  W8A8_OP_BF16_FWD = 4,        /* bf16_linear_fwd                          */
  W8A8_OP_WEIGHT_ONLY_FWD = 5, /* float8_linear_fwd, gguf_linear_fwd        */
  W8A8_OP_BF16_DGRAD = 6,      /* bf16_linear_dgrad                        */
  W8A8_OP_WEIGHT_ONLY_DGRAD = 7 /* float8_linear_dgrad, gguf_linear_dgrad  */
} w8a8_op;

/* ------------------------------------------------------------------------
 * Token-wise calibrate + quantize (bitsandbytes #1401, Enhancements: the
 * fused kernel for activation scale calibration and quantization,
 * int8_vectorwise_quant; OneTrainer wiki: activations quantized token-wise).
 * For every row m of X:  a = max_k |x[m,k]|,  s[m] = (a < 1e-10 ? 1e-10 :
 * a / QMAX) (fp32 division),  q[m,k] = code(x[m,k] / s[m]) with int8 codes
 * rounded half-to-even and clamped to +-127, e4m3 codes rounded to nearest
 * even and saturated to +-448.  One pass over X.
 *   x_bf16    [M, ldx] bf16, the first K columns are read; ldx % 8 == 0
 *   q_out     [M, ldq] bytes (int8 or e4m3), ldq >= K, ldq % 16 == 0
 *   row_scale [M] fp32
 * ---------------------------------------------------------------------- */
w8a8_status w8a8_quantize_rows(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                               w8a8_qtype qt, void* q_out, int64_t ldq, float* row_scale,
                               w8a8_stream_t stream);

/* ------------------------------------------------------------------------
 * Weight quantization (OneTrainer wiki, float8 / float W8A8 / int W8A8:
 * "Tensor-wise quantization of weights"; GGUF A8: axis-wise).
 *   TENSOR: one scale s = floor(absmax(W)) / QMAX for all N*K values; needs
 *           ws_bytes >= w8a8_workspace_bytes(W8A8_OP_QUANTIZE_WEIGHT, ...)
 *           (256 bytes, cleared by the call itself); scale is [1].
 *   AXIS:   one scale per output row n, the token-wise rule applied to W's
 *           rows; no workspace; scale is [N].
 *   w_bf16 [N, K] contiguous bf16;  q_out [N, K] bytes.
 * ---------------------------------------------------------------------- */
w8a8_status w8a8_quantize_weight(const void* w_bf16, int64_t N, int64_t K, w8a8_qtype qt,
                                 w8a8_wgran g, void* q_out, float* scale,
                                 void* ws, size_t ws_bytes, w8a8_stream_t stream);

/* ------------------------------------------------------------------------
 * GGUF Q8_0 (entrenar 0.7.8, src/quant/gguf_quant/q8_0.rs: struct Q8_0 and
 * Q8_0::quantize / Q8_0::dequantize).  A block holds 32 values in 34 bytes:
 * the f16 scale (little-endian) followed by 32 int8 codes.  n values take
 * ceil(n/32) blocks; a short last block is padded with zero codes.
 *   quantize: per block max_abs = max|v|, scale = (max_abs < 1e-10 ? 1e-10 :
 *             max_abs / 127) in fp32, code = clamp(round(v / scale), -128,
 *             127) with round = ties away from zero; the stored scale is the
 *             f16 (round-to-nearest-even) of the fp32 scale.
 *   dequantize: y = f16 scale * code (exact in fp32), n values.
 *   x / y: [n] fp32.  blocks: q8_0_bytes(n) bytes, 16-byte aligned base.
 *   n >= 0 (0 is a no-op); no K constraint applies here.
 * ---------------------------------------------------------------------- */
size_t q8_0_bytes(int64_t n);
w8a8_status q8_0_quantize(const float* x, int64_t n, void* blocks, w8a8_stream_t stream);
w8a8_status q8_0_dequantize(const void* blocks, int64_t n, float* y, w8a8_stream_t stream);
/* GGUF dequantized to bf16 (OneTrainer wiki, GGUF: weights dequantized to the
 * train data type): y[i] = bf16_rne(f16(d) * q), the product exact in fp32.
 * n >= 0 values (any n; the last block may be short).  y_bf16 [n]. */
w8a8_status q8_0_dequantize_bf16(const void* blocks, int64_t n, void* y_bf16, w8a8_stream_t stream);

/* Re-quantize a Q8_0 weight to axis-wise int8 (OneTrainer wiki, GGUF A8 int:
 * weights re-quantized from GGUF to int8 axis-wise).  Row n of W[N,K] is the
 * K/32 consecutive blocks starting at block n*K/32.  Each value is
 * dequantized exactly (f16 scale * code), then row n takes the token-wise
 * int8 rule: s[n] = floor(max|deq|)/127, q = clamp(rne(deq/s[n]), +-127).
 * K % 32 == 0 and K <= 131072.   q_out [N, K] int8;  scale [N] fp32. */
w8a8_status q8_0_to_axis_int8(const void* blocks, int64_t N, int64_t K, int8_t* q_out,
                              float* scale, w8a8_stream_t stream);

/* Re-quantize a Q8_0 weight to axis-wise float8 e4m3 (OneTrainer wiki, GGUF
 * A8 float: weights re-quantized from GGUF to float8 axis-wise; the Linear
 * matmuls then run in float8).  The same rows and dequantization as
 * q8_0_to_axis_int8, with the e4m3 rule of the token-wise quantizer:
 * s[n] = floor(max|deq|)/448, q = e4m3_rne_satfinite(deq/s[n]) (OCP E4M3FN;
 * a -0 value keeps its sign, code 0x80).  K % 32 == 0 and K <= 131072.
 * q_out [N, K] e4m3 bytes;  scale [N] fp32.  The result feeds
 * w8a8_linear_fwd with W8A8_E4M3 and W8A8_AXIS. */
w8a8_status q8_0_to_axis_e4m3(const void* blocks, int64_t N, int64_t K, uint8_t* q_out,
                              float* scale, w8a8_stream_t stream);

/* ------------------------------------------------------------------------
 * Weight-only types (OneTrainer wiki, "float8": tensor-wise e4m3 weights, and
 * "GGUF"; both dequantized to the train data type during training).  The
 * weight stays 8-bit in memory; each forward dequantizes it to bf16 in the
 * workspace and runs a bf16 Linear on the tensor cores:
 *     y = bf16( fp32(sum_k x[m,k] W[n,k]) (+ bias[n]) )
 * with fp32 sums (kind::f16 MMAs; split along K, partial sums added in split
 * order, when the output makes few tiles) and one fp32 RN bias add.
 * Shapes and alignment as w8a8_linear_fwd (K >= 16, K % 16 == 0, 16-byte
 * aligned pointers); M == 0 is a no-op.
 * ---------------------------------------------------------------------- */
/* e4m3 codes -> bf16(value * scale[0]), n % 16 == 0.  w_bf16 [n]. */
w8a8_status w8a8_dequantize_e4m3_bf16(const void* q, int64_t n, const float* scale, void* w_bf16,
                                      w8a8_stream_t stream);
/* The bf16 Linear alone: x [M, K], w [N, K], bias [N] or NULL, y [M, N], all
 * bf16.  ws: w8a8_workspace_bytes(W8A8_OP_BF16_FWD, M, N, K, 0) bytes (0 when
 * the product is not split; ws may then be NULL). */
w8a8_status bf16_linear_fwd(const void* x_bf16, int64_t M, int64_t N, int64_t K, const void* w_bf16,
                            const void* bias_bf16, void* y_bf16, void* ws, size_t ws_bytes,
                            w8a8_stream_t stream);
/* float8: wq [N, K] e4m3 codes with tensor-wise w_scale [1] (as
 * w8a8_quantize_weight with W8A8_E4M3, W8A8_TENSOR).  W = bf16(dec(wq) *
 * w_scale[0]).  ws: w8a8_workspace_bytes(W8A8_OP_WEIGHT_ONLY_FWD, M, N, K, 0)
 * bytes; holds W [N, K] bf16, then the split partial sums. */
w8a8_status float8_linear_fwd(const void* x_bf16, int64_t M, int64_t N, int64_t K, const void* wq,
                              const float* w_scale, const void* bias_bf16, void* y_bf16, void* ws,
                              size_t ws_bytes, w8a8_stream_t stream);
/* GGUF: the weight as Q8_0 blocks over its N*K values in row-major order.
 * W = bf16(f16(d) * q).  ws as float8_linear_fwd. */
w8a8_status gguf_linear_fwd(const void* x_bf16, int64_t M, int64_t N, int64_t K, const void* blocks,
                            const void* bias_bf16, void* y_bf16, void* ws, size_t ws_bytes,
                            w8a8_stream_t stream);

/* The input gradients of the weight-only types (the LoRA training through
 * the frozen, dequantized weight):  dX = bf16( fp32(sum_n dY[m,n] W[n,k]) ),
 * the bf16 weight read with its rows as the contraction (no transposed
 * copy).  dy [M, N] bf16 with N % 8 == 0, dx [M, K] bf16, K % 16 == 0.
 * ws: w8a8_workspace_bytes(W8A8_OP_BF16_DGRAD, ...) for the bf16 weight,
 * W8A8_OP_WEIGHT_ONLY_DGRAD for the float8 / GGUF weights (the dequantized
 * weight first, then the split partial sums). */
w8a8_status bf16_linear_dgrad(const void* dy_bf16, int64_t M, int64_t N, int64_t K, const void* w_bf16,
                              void* dx_bf16, void* ws, size_t ws_bytes, w8a8_stream_t stream);
w8a8_status float8_linear_dgrad(const void* dy_bf16, int64_t M, int64_t N, int64_t K, const void* wq,
                                const float* w_scale, void* dx_bf16, void* ws, size_t ws_bytes,
                                w8a8_stream_t stream);
w8a8_status gguf_linear_dgrad(const void* dy_bf16, int64_t M, int64_t N, int64_t K, const void* blocks,
                              void* dx_bf16, void* ws, size_t ws_bytes, w8a8_stream_t stream);

/* ------------------------------------------------------------------------
 * W8A8 Linear forward (OneTrainer wiki, int/float W8A8): quantize X
 * token-wise (as w8a8_quantize_rows), multiply the codes with the weight
 * codes on the 5th-generation tensor cores (int8 x int8 -> int32, or
 * e4m3 x e4m3 -> fp32), then the fused epilogue
 *     y = bf16( ((acc * s_x[m]) * w_scale[n or 0]) + bias[n] )
 * with every product and sum rounded to fp32 on its own.
 *   x_bf16 [M, K] contiguous;  wq [N, K] codes of qt;  w_scale [1] (TENSOR)
 *   or [N] (AXIS);  bias_bf16 [N] or NULL;  y_bf16 [M, N] contiguous.
 *   ws: w8a8_workspace_bytes(W8A8_OP_LINEAR_FWD, M, N, K, 0) bytes; holds
 *   the activation codes and row scales of this call, and the int32 partial
 *   sums when an int8 product with few output tiles is split along K (the
 *   size depends on the shape only, never on the device).
 * A few tokens run as one weight-streaming launch on the CUDA cores that
 * quantizes the rows itself and leaves ws untouched: int8 with M <= 2 and
 * K <= 16384 (dp4a; the same bits as every other path), e4m3 with M == 1
 * and K <= 32768 (codes decoded to fp32, exact products, fp32 sums in
 * another order: within the e4m3 bound).  Up to 128 tokens otherwise run the
 * transposed tensor-core product (the weight as the 128-row operand).
 * ---------------------------------------------------------------------- */
w8a8_status w8a8_linear_fwd(const void* x_bf16, int64_t M, int64_t N, int64_t K,
                            w8a8_qtype qt, const void* wq, const float* w_scale, w8a8_wgran g,
                            const void* bias_bf16, void* y_bf16,
                            void* ws, size_t ws_bytes, w8a8_stream_t stream);

/* w8a8_linear_fwd for a chain of projections (an MLP block): the same
 * product, with
 *   act     W8A8_ACT_GELU (0.5 v (1 + erf(v / sqrt 2))) or W8A8_ACT_GELU_TANH
 *           (0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3)))) applied to the
 *           fp32 epilogue value before the bf16 rounding (fp32 math
 *           functions: within a few fp32 ulp of the exact function);
 *   y_amax  [M] uint32 or NULL: receives max_n |y[m, n]| of the bf16 outputs
 *           as fp32 bits (the GEMM epilogue folds each tile's rows in with
 *           atomicMax; the call clears the buffer first);
 *   x_amax  [M] uint32 or NULL: max_k |x[m, k]| as fp32 bits, e.g. the
 *           y_amax of the call that produced x.  The token-wise quantizer
 *           then skips its reduction; the codes are the same as without it
 *           when x_amax is the true row absmax.
 * x_amax and y_amax must not be the same buffer.  With act, x_amax or y_amax
 * set, the few-token weight-streaming kernel is not used.  Workspace as
 * w8a8_linear_fwd.  (The pages blame the unfused quantization for W8A8's
 * need of a compiler, OneTrainer wiki: A8 is faster only with compiled
 * transformer blocks.) */
w8a8_status w8a8_linear_fwd_ex(const void* x_bf16, int64_t M, int64_t N, int64_t K,
                               w8a8_qtype qt, const void* wq, const float* w_scale, w8a8_wgran g,
                               const void* bias_bf16, w8a8_act act, const uint32_t* x_amax,
                               uint32_t* y_amax, void* y_bf16, void* ws, size_t ws_bytes,
                               w8a8_stream_t stream);

/* ------------------------------------------------------------------------
 * W8A8 Linear input gradient for LoRA training with frozen quantized weights
 * (OneTrainer PR #1034: "train LoRA twice as fast"; wiki: activations are
 * quantized token-wise during training):  dX = Q(dY) Q(W), i.e.
 *     dx[m,k] = bf16( (acc[m,k] * s_dy[m]) * w_scale[0] ),
 *     acc[m,k] = sum_n dyq[m,n] * wq[n,k].
 * The tensor cores read the same wq[N,K] codes as the forward, with N as the
 * contraction dimension (no transposed copy).  Tensor-wise weights only
 * (g must be W8A8_TENSOR).  N % 16 == 0.
 *   dy_bf16 [M, N];  wq [N, K];  dx_bf16 [M, K].
 *   ws: w8a8_workspace_bytes(W8A8_OP_LINEAR_DGRAD, M, N, K, 0) bytes (codes,
 *   row scales and, for an int8 product with few output tiles, the int32
 *   partial sums of the split contraction).
 * ---------------------------------------------------------------------- */
w8a8_status w8a8_linear_dgrad(const void* dy_bf16, int64_t M, int64_t N, int64_t K,
                              w8a8_qtype qt, const void* wq, const float* w_scale, w8a8_wgran g,
                              void* dx_bf16, void* ws, size_t ws_bytes, w8a8_stream_t stream);

/* ------------------------------------------------------------------------
 * SVDQuant int W8A8 forward (OneTrainer PR #1034, "SVDQuant", after arXiv
 * 2411.05007; wiki: SVDQuant data type bfloat16):  W^T ~= L1 L2 + R^T with
 * the residual R quantized int8 tensor-wise, so
 *     T = bf16(X L1)                                   [M, r], fp32 sums
 *     y = bf16( (((acc_R * s_x[m]) * r_scale) + bias[n]) + sum_j T[m,j] L2[j,n] )
 * where acc_R = Q(X) Q(R)^T on the tensor cores, the low-rank sum is an fp32
 * accumulation of bf16 products (on the tensor cores from zero, or in the
 * epilogue) and each outer step is one fp32 RN operation.  r is 8, 16, 24 or
 * 32 (W8A8_ERR_UNSUPPORTED_SHAPE otherwise).
 *   rq [N, K] int8;  r_scale [1];  l1_bf16 [K, r];  l2_bf16 [r, N];
 *   bias_bf16 [N] or NULL;  y_bf16 [M, N].
 *   ws: w8a8_workspace_bytes(W8A8_OP_SVDQ_FWD, M, N, K, r) bytes; also
 *   holds T [M, r] bf16 (after the codes and row scales) and, when the T
 *   product is split along K, its fp32 partial sums.
 * ---------------------------------------------------------------------- */
w8a8_status svdq_linear_fwd(const void* x_bf16, int64_t M, int64_t N, int64_t K,
                            const void* rq, const float* r_scale, int r,
                            const void* l1_bf16, const void* l2_bf16, const void* bias_bf16,
                            void* y_bf16, void* ws, size_t ws_bytes, w8a8_stream_t stream);

/* SVDQuant on float W8A8 (OneTrainer wiki, SVDQuant paragraph: it combines
 * with all quantized data types except GGUF): svdq_linear_fwd with e4m3
 * residual codes and e4m3 token-wise activation codes.  The residual product
 * accumulates in fp32 on the tensor cores (kind::f8f6f4), then the same
 * epilogue and low-rank sum.  rq [N, K] e4m3 bytes (tensor-wise, as
 * w8a8_quantize_weight with W8A8_E4M3); every other argument as in
 * svdq_linear_fwd, including the workspace size. */
w8a8_status svdq_linear_fwd_e4m3(const void* x_bf16, int64_t M, int64_t N, int64_t K,
                                 const void* rq, const float* r_scale, int r,
                                 const void* l1_bf16, const void* l2_bf16, const void* bias_bf16,
                                 void* y_bf16, void* ws, size_t ws_bytes, w8a8_stream_t stream);

/* ------------------------------------------------------------------------
 * The two tensor-core products on codes that are already quantized (the
 * second half of w8a8_linear_fwd / w8a8_linear_dgrad), for callers that
 * quantize once and multiply many times.  Same epilogue and rules as above.
 *   fwd:   xq [M, ldq] codes (ldq >= K, ldq % 16 == 0), x_scale [M], wq [N, K],
 *          y [M, N] = epilogue( xq wq^T ).
 *   dgrad: dyq [M, ldq] (ldq >= N, ldq % 16 == 0), dy_scale [M], wq [N, K],
 *          dx [M, K] = epilogue( dyq wq ), tensor-wise w_scale only.
 * ---------------------------------------------------------------------- */
w8a8_status w8a8_qgemm_fwd(const void* xq, int64_t ldq, const float* x_scale,
                           int64_t M, int64_t N, int64_t K, w8a8_qtype qt,
                           const void* wq, const float* w_scale, w8a8_wgran g,
                           const void* bias_bf16, void* y_bf16, w8a8_stream_t stream);
w8a8_status w8a8_qgemm_dgrad(const void* dyq, int64_t ldq, const float* dy_scale,
                             int64_t M, int64_t N, int64_t K, w8a8_qtype qt,
                             const void* wq, const float* w_scale, void* dx_bf16,
                             w8a8_stream_t stream);

/* ------------------------------------------------------------------------
 * w8a8_linear_fwd without a caller workspace.  (No counterpart on the pages:
 * this is a calling convenience of this library.)
 *
 * Some callers cannot hand the library device memory for scratch: code that
 * runs where allocating is not allowed or not possible (an embedding runtime
 * or plugin host that owns all device memory and exposes no allocator, a
 * latency-critical path that must not call cudaMalloc because it can
 * synchronize the device, a language binding with no CUDA allocator).  This
 * entry point computes exactly what w8a8_linear_fwd computes (the same
 * kernels for the same shapes, so the same bits), but keeps the
 * activation codes and row scales in a fixed scratch array that is part of
 * the library itself (a file-scope __device__ array of
 * W8A8_NOALLOC_SCRATCH_BYTES; every GPU that loads the library holds it
 * until the process exits).  It calls no cudaMalloc / cudaFree and no
 * allocating library routine.  The caller still passes x, wq, w_scale, bias
 * and the output y.
 *
 * Limits: M * K <= W8A8_NOALLOC_MAX_CODES and M <= W8A8_NOALLOC_MAX_ROWS;
 * larger problems return W8A8_ERR_WORKSPACE before any launch (use
 * w8a8_linear_fwd with a workspace instead).
 * Set-up: the first call in each CUDA context (normally one per device: its
 * primary context) looks up the scratch array's device address
 * (cudaGetSymbolAddress) with that device current, and keeps it for that
 * context; make that first call before any stream capture.  A new context
 * (after cudaDeviceReset, or a second context on a device) gets its own
 * lookup on its first call.
 * Sharing: all calls on a device use the same scratch, which keeps the last
 * call's contents (every byte a call reads was written earlier by the same
 * call, so nothing needs clearing).  Calls whose kernels overlap on the GPU
 * (different streams, or graphs replayed concurrently) race on the scratch;
 * order them on one stream.
 * ---------------------------------------------------------------------- */
#define W8A8_NOALLOC_MAX_CODES (64ull << 20)
#define W8A8_NOALLOC_MAX_ROWS 65536ll
#define W8A8_NOALLOC_SCRATCH_BYTES (W8A8_NOALLOC_MAX_CODES + 4ull * W8A8_NOALLOC_MAX_ROWS)
w8a8_status w8a8_linear_fwd_noalloc(const void* x_bf16, int64_t M, int64_t N, int64_t K,
                                    w8a8_qtype qt, const void* wq, const float* w_scale,
                                    w8a8_wgran g, const void* bias_bf16, void* y_bf16,
                                    w8a8_stream_t stream);

/* Workspace size in bytes for `op` at the given sizes (r only for SVDQ). */
size_t w8a8_workspace_bytes(int op, int64_t M, int64_t N, int64_t K, int r);

/* ------------------------------------------------------------------------
 * Device status and diagnostics (not on the pages; the failure-detection
 * side of the library).
 *  w8a8_device_status: synchronizes `stream`, then returns the first
 *    device-side error recorded on the current device since the last reset
 *    (W8A8_OK if none), and clears it when reset != 0.
 *  w8a8_set_wait_limit_ns: bound of every device-side wait on the current
 *    device (default 2e9 ns).  Synchronous; call outside stream capture.
 *  w8a8_selftest_wait: launches one block that waits on a barrier which
 *    nothing completes, bounded by `limit_ns`; the wait runs out, records
 *    W8A8_ERR_DEVICE_TIMEOUT and the kernel returns normally.
 *  w8a8_e4m3_encode: y[i] = E4M3FN code of x[i] (RNE, saturating), the same
 *    device conversion the quantizers use.  x [n] fp32, y [n] bytes.
 *  w8a8_last_error: message of the last failing call on this thread.
 * ---------------------------------------------------------------------- */
w8a8_status w8a8_device_status(w8a8_stream_t stream, int reset);
w8a8_status w8a8_set_wait_limit_ns(uint64_t limit_ns);
w8a8_status w8a8_selftest_wait(uint64_t limit_ns, w8a8_stream_t stream);

/* ------------------------------------------------------------------------
 * Debug build (the same sources compiled with W8A8_DEBUG_CHECKS=1 into
 * libw8a8_debug.so; not on the pages).  Every plain (non-TMA) global-memory
 * access of a kernel first checks the index it derived against the extent
 * the call's shape implies; an index outside that extent records
 * W8A8_ERR_DEVICE_BOUNDS and the check's site in the status word read by
 * w8a8_device_status, and the access is skipped - nothing faults.  TMA copies
 * need no check (the hardware clips stores and zero-fills loads at the
 * tensor map's bounds).  The release build, libw8a8.so, has no checks.
 *  w8a8_selftest_bounds: one kernel evaluates a check one past the end of
 *    an extent (it touches no memory): the debug build then records
 *    W8A8_ERR_DEVICE_BOUNDS (site 0xBFFF); the release build records nothing.
 *  w8a8_debug_checks: 1 in the debug build, 0 in the release build.
 * ---------------------------------------------------------------------- */
w8a8_status w8a8_selftest_bounds(w8a8_stream_t stream);
int w8a8_debug_checks(void);
w8a8_status w8a8_e4m3_encode(const float* x, int64_t n, uint8_t* y, w8a8_stream_t stream);
const char* w8a8_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* W8A8_H */
