/*
 * oracle.h - plain CPU reference for the W8A8 quantized Linear.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this code: only the tests, the smoke check and the bench's CPU-baseline
 * leg use it.  It shares no code, header, table or helper with the CUDA
 * library; every codec below is written from the format's own definition.
 *
 * Sources (web pages; cited by title and section):
 *  [OT-PR]  OneTrainer PR #1034 "New quant types, activation quantization",
 *           section "W8A8 quant types" and "SVDQuant".
 *  [OT-WIKI] OneTrainer wiki "Quantization": the float W8A8, int W8A8,
 *           GGUF A8 int, GGUF A8 float and SVDQuant paragraphs
 *           ("Technical:" lines).
 *  [BNB]    bitsandbytes #1401 "LLM.int8() Refactoring: Part 1", section
 *           "Enhancements / Improved kernels for inference" (the fused
 *           row calibrate-and-quantize op int8_vectorwise_quant).
 *  [Q80]    docs.rs entrenar 0.7.8, src/quant/gguf_quant/q8_0.rs:
 *           struct Q8_0 docs, Q8_0::quantize, Q8_0::dequantize, size helpers.
 *
 * Conventions: X[M,K] bf16 activations, W[N,K] bf16 weight (nn.Linear
 * layout), Y[M,N] = X W^T, all row-major.  bf16/f16 values travel as their
 * uint16 bit patterns, e4m3 codes as uint8, int8 codes as int8.
 */
#ifndef W8A8_ORACLE_H
#define W8A8_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_INT8 = 0, ORC_E4M3 = 1 };
enum { ORC_TENSOR = 0, ORC_AXIS = 1 };

/* ---- scalar codecs (format definitions) ---------------------------------- */
float    orc_bf16_to_f32(uint16_t h);
uint16_t orc_f32_to_bf16(float f);           /* round to nearest, ties to even */
float    orc_f16_to_f32(uint16_t h);
uint16_t orc_f32_to_f16(float f);            /* RNE, subnormals, overflow -> inf */
float    orc_e4m3_to_f32(uint8_t c);         /* OCP E4M3FN decode */
uint8_t  orc_f32_to_e4m3(float f);           /* RNE, saturate to +-448 */
int8_t   orc_f32_to_int8_sym(float v);       /* RNE, clamp to [-127,127] */

/* bulk versions for the tests */
void orc_bf16_to_f32_n(const uint16_t* h, float* f, int64_t n);
void orc_f32_to_bf16_n(const float* f, uint16_t* h, int64_t n);
void orc_f16_to_f32_n(const uint16_t* h, float* f, int64_t n);
void orc_f32_to_f16_n(const float* f, uint16_t* h, int64_t n);
void orc_e4m3_to_f32_n(const uint8_t* c, float* f, int64_t n);
void orc_f32_to_e4m3_n(const float* f, uint8_t* c, int64_t n);

/* ---- quantizers ----------------------------------------------------------- */
/* Token-wise (row) absmax calibration + quantization [OT-WIKI int/float W8A8;
 * BNB int8_vectorwise_quant].  q is [M,K] contiguous, s is [M]. */
void orc_quantize_rows(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                       int qt, uint8_t* q, float* s);

/* Weight quantization: tensor-wise (one scale) or axis-wise (one scale per
 * output row n) [OT-WIKI float8 / int W8A8 / GGUF A8 int]. */
void orc_quantize_weight(const uint16_t* w, int64_t N, int64_t K, int qt,
                         int gran, uint8_t* q, float* s);

/* ---- GGUF Q8_0 [Q80] ------------------------------------------------------ */
int64_t orc_q8_0_bytes(int64_t n);           /* ceil(n/32) * 34 */
/* blocks: ceil(n/32) x {f16 scale, 32 x int8}; scales_f32 (nullable) receives
 * the f32 scale of every block, as kept by the Q8_0 struct. */
void orc_q8_0_quantize(const float* x, int64_t n, uint8_t* blocks, float* scales_f32);
/* GGUF dequantize: f16 scale times code, n values. */
void orc_q8_0_dequantize(const uint8_t* blocks, int64_t n, float* y);
/* Struct dequantize: f32 scale per block times code. */
void orc_q8_0_dequantize_f32(const float* scales_f32, const int8_t* codes,
                             int64_t n, float* y);
/* GGUF -> axis-wise re-quantization [OT-WIKI GGUF A8 int (qt ORC_INT8),
 * GGUF A8 float (qt ORC_E4M3)]: q [N,K] one-byte codes, s [N]. */
void orc_q8_0_to_axis(const uint8_t* blocks, int64_t N, int64_t K, int qt,
                      uint8_t* q, float* s);
void orc_q8_0_to_axis_int8(const uint8_t* blocks, int64_t N, int64_t K,
                           int8_t* q, float* s);

/* ---- activation and row absmax (the MLP chain) --------------------------- */
/* act 1: GELU 0.5 v (1 + erf(v / sqrt 2)); act 2: the tanh form; in double,
 * rounded once to fp32.  act 0 copies. */
void orc_act(const float* v, int64_t n, int act, float* out);
/* amax[m] = max_n |y[m, n]| of bf16 values. */
void orc_row_absmax_bf16(const uint16_t* y, int64_t M, int64_t N, float* amax);

/* ---- weight-only types [OT-WIKI float8, GGUF] ---------------------------- */
/* w = bf16(e4m3_value(q) * s) for n codes (tensor-wise scale s). */
void orc_dequant_e4m3_bf16(const uint8_t* q, int64_t n, float s, uint16_t* w);
/* w = bf16(f16(d) * q) for the first n values of the blocks. */
void orc_q8_0_dequantize_bf16(const uint8_t* blocks, int64_t n, uint16_t* w);
/* bf16 Linear: acc = sum x w (fp64), absacc = sum |x w|, y32 = fp32(acc)
 * (+ bias, fp32 RN), y = bf16(y32).  x [M,K], w [N,K], bias [N] or NULL. */
void orc_linear_bf16(const uint16_t* x, const uint16_t* w, int64_t M, int64_t N, int64_t K,
                     const uint16_t* bias, double* acc, double* absacc, float* y32, uint16_t* y);

/* ---- 8-bit matrix products ------------------------------------------------ */
/* acc[m,n] = sum_k A[m,k] * B[n,k] in int64; returns 0, or 1 if any sum
 * leaves the int32 range (then acc holds the truncated values). */
int orc_gemm_i8_nt(const int8_t* A, const int8_t* B, int64_t M, int64_t N,
                   int64_t K, int32_t* acc);
/* acc[m,k] = sum_n A[m,n] * B[n,k] (B read along its rows: the dgrad form). */
int orc_gemm_i8_nn(const int8_t* A, const int8_t* B, int64_t M, int64_t N,
                   int64_t K, int32_t* acc);
/* e4m3 codes decoded, products and sums in fp64; absacc = sum |a*b|. */
void orc_gemm_e4m3_nt(const uint8_t* A, const uint8_t* B, int64_t M, int64_t N,
                      int64_t K, double* acc, double* absacc);
void orc_gemm_e4m3_nn(const uint8_t* A, const uint8_t* B, int64_t M, int64_t N,
                      int64_t K, double* acc, double* absacc);

/* ---- dequantizing epilogue ------------------------------------------------- */
/* y32 = ((float)acc * s_row[m]) * s_w[n or 0] (+ (float)bias[n]), each an
 * fp32 round-to-nearest operation, no fused multiply-add; y = bf16(y32). */
void orc_epilogue_i32(const int32_t* acc, int64_t M, int64_t N,
                      const float* s_row, const float* s_w, int w_axis,
                      const uint16_t* bias, float* y32, uint16_t* y);
/* fp8 form: the same products in fp64, rounded once to fp32, then bf16. */
void orc_epilogue_f64(const double* acc, int64_t M, int64_t N,
                      const float* s_row, const float* s_w, int w_axis,
                      const uint16_t* bias, float* y32, uint16_t* y);

/* ---- SVDQuant low-rank branch [OT-PR SVDQuant; OT-WIKI SVDQuant] ---------- */
/* t64[m,j] = sum_k x[m,k] * L1[k,j] (fp64), t[m,j] = bf16(fp32(t64)). */
void orc_lowrank_down(const uint16_t* x, const uint16_t* l1, int64_t M,
                      int64_t K, int64_t r, double* t64, uint16_t* t);
/* lr[m,n] = sum_j T[m,j] * L2[j,n] (fp64), lr_abs = sum_j |T*L2|. */
void orc_lowrank_up(const uint16_t* t, const uint16_t* l2, int64_t M,
                    int64_t r, int64_t N, double* lr, double* lr_abs);

#ifdef __cplusplus
}
#endif
#endif
