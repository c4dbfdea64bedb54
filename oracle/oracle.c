/*
 * oracle.c - plain CPU reference for the W8A8 quantized Linear.
 *
 * TEST INFRASTRUCTURE ONLY (see oracle.h).  Slow, obviously correct loops;
 * each function names the page passage it follows.  Compile with
 * -ffp-contract=off so that every fp32 multiply and add rounds on its own.
 *
 * Readings where the pages are silent are stated beside the code:
 *  - rounding of W8A8 codes: round to nearest, ties to even; Q8_0 codes:
 *    ties away from zero (Rust f32::round in Q8_0::quantize);
 *  - W8A8 clamp +-127 (symmetric); Q8_0 clamp [-128,127] as in Q8_0::quantize;
 *  - every absmax scale gets the 1e-10 floor that Q8_0::quantize uses;
 *  - x / s is an IEEE fp32 division, as Q8_0::quantize writes val / scale;
 *  - e4m3 is OCP E4M3FN (max 448), RNE then saturate to +-448.
 */
#include "oracle.h"

#include <math.h>
#ifndef M_PI
#define M_PI 3.14159265358979323846
#endif
#include <stdlib.h>
#include <string.h>

static uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float bits_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* ========================================================================== */
/* Codecs                                                                      */
/* ========================================================================== */

/* bfloat16 is the upper half of an IEEE binary32 pattern. */
float orc_bf16_to_f32(uint16_t h) { return bits_f32((uint32_t)h << 16); }

/* Keep the upper 16 bits; the discarded 16 bits decide the rounding: above
 * one half rounds up, exactly one half rounds to the even upper half. */
uint16_t orc_f32_to_bf16(float f) {
  uint32_t u = f32_bits(f);
  if (isnan(f)) return (uint16_t)((u >> 16) | 0x0040u);  /* quiet NaN */
  uint32_t hi = u >> 16, lo = u & 0xFFFFu;
  if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi += 1u;
  return (uint16_t)hi;
}

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
float orc_f16_to_f32(uint16_t h) {
  int s = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 31) v = m ? NAN : INFINITY;
  else if (e == 0) v = ldexp((double)m, -24);               /* subnormal */
  else v = ldexp((double)(1024 + m), e - 15 - 10);
  return (float)(s ? -v : v);
}

/* fp32 -> binary16, round to nearest even.  All scalings below are by powers
 * of two and therefore exact in double; nearbyint() rounds ties to even. */
uint16_t orc_f32_to_f16(float f) {
  uint16_t sign = signbit(f) ? 0x8000u : 0u;
  if (isnan(f)) return (uint16_t)(sign | 0x7E00u);
  double a = fabs((double)f);
  if (isinf(f)) return (uint16_t)(sign | 0x7C00u);
  if (a < ldexp(1.0, -14)) {                   /* subnormal range, step 2^-24 */
    double k = nearbyint(a * ldexp(1.0, 24));  /* k == 1024 is the min normal */
    return (uint16_t)(sign | (uint16_t)k);
  }
  int e2;
  frexp(a, &e2);
  int E = e2 - 1;                              /* a = 1.f * 2^E */
  double m = nearbyint((ldexp(a, -E) - 1.0) * 1024.0);
  if (m == 1024.0) { m = 0.0; E += 1; }
  if (E > 15) return (uint16_t)(sign | 0x7C00u);  /* overflow -> inf */
  return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)m);
}

/* OCP E4M3FN: 1 sign, 4 exponent (bias 7), 3 mantissa bits, no infinities,
 * S.1111.111 is NaN, largest finite 1.75 * 2^8 = 448, subnormal step 2^-9. */
float orc_e4m3_to_f32(uint8_t c) {
  int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
  if (e == 15 && m == 7) return NAN;
  double v = (e == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 7 - 3);
  return (float)(s ? -v : v);
}

/* fp32 -> E4M3FN, round to nearest even, then saturate to +-448 (the
 * "RNE saturating" encoding of the float W8A8 configuration).  Direct from
 * fp32, no intermediate rounding.  Zero keeps its sign. */
uint8_t orc_f32_to_e4m3(float f) {
  uint8_t sign = signbit(f) ? 0x80u : 0u;
  if (isnan(f)) return (uint8_t)(sign | 0x7Fu);
  double a = fabs((double)f);
  if (a >= 448.0) return (uint8_t)(sign | 0x7Eu);   /* saturate (incl. inf) */
  if (a < ldexp(1.0, -6)) {                          /* subnormal, step 2^-9 */
    double k = nearbyint(a * 512.0);                 /* k == 8 is min normal */
    return (uint8_t)(sign | (uint8_t)k);
  }
  int e2;
  frexp(a, &e2);
  int E = e2 - 1;                                    /* E in [-6, 8] */
  double m = nearbyint((ldexp(a, -E) - 1.0) * 8.0);
  if (m == 8.0) { m = 0.0; E += 1; }
  return (uint8_t)(sign | (uint8_t)((E + 7) << 3) | (uint8_t)m);
}

/* W8A8 int code: nearest integer, ties to even, clamped to +-127. */
int8_t orc_f32_to_int8_sym(float v) {
  float r = nearbyintf(v);
  if (r > 127.0f) r = 127.0f;
  if (r < -127.0f) r = -127.0f;
  return (int8_t)r;
}

void orc_bf16_to_f32_n(const uint16_t* h, float* f, int64_t n) {
  for (int64_t i = 0; i < n; ++i) f[i] = orc_bf16_to_f32(h[i]);
}
void orc_f32_to_bf16_n(const float* f, uint16_t* h, int64_t n) {
  for (int64_t i = 0; i < n; ++i) h[i] = orc_f32_to_bf16(f[i]);
}
void orc_f16_to_f32_n(const uint16_t* h, float* f, int64_t n) {
  for (int64_t i = 0; i < n; ++i) f[i] = orc_f16_to_f32(h[i]);
}
void orc_f32_to_f16_n(const float* f, uint16_t* h, int64_t n) {
  for (int64_t i = 0; i < n; ++i) h[i] = orc_f32_to_f16(f[i]);
}
void orc_e4m3_to_f32_n(const uint8_t* c, float* f, int64_t n) {
  for (int64_t i = 0; i < n; ++i) f[i] = orc_e4m3_to_f32(c[i]);
}
void orc_f32_to_e4m3_n(const float* f, uint8_t* c, int64_t n) {
  for (int64_t i = 0; i < n; ++i) c[i] = orc_f32_to_e4m3(f[i]);
}

/* ========================================================================== */
/* W8A8 quantizers                                                             */
/* ========================================================================== */

static float qmax_of(int qt) { return qt == ORC_E4M3 ? 448.0f : 127.0f; }

/* absmax scale with the 1e-10 floor of Q8_0::quantize, fp32 division. */
static float absmax_scale(float a, int qt) {
  return (a < 1e-10f) ? 1e-10f : a / qmax_of(qt);
}

static uint8_t encode_code(float v, int qt) {
  if (qt == ORC_E4M3) return orc_f32_to_e4m3(v);
  return (uint8_t)orc_f32_to_int8_sym(v);
}

/* Token-wise quantization [OT-WIKI float/int W8A8 "Activations are quantized
 * token-wise"; BNB int8_vectorwise_quant]: for each row m,
 *   a = max_k |x[m,k]|,  s_m = floor(a)/QMAX,  q[m,k] = code(x[m,k] / s_m). */
void orc_quantize_rows(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                       int qt, uint8_t* q, float* s) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    const uint16_t* row = x + m * ldx;
    float a = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float v = fabsf(orc_bf16_to_f32(row[k]));
      if (v > a) a = v;
    }
    float sm = absmax_scale(a, qt);
    s[m] = sm;
    for (int64_t k = 0; k < K; ++k)
      q[m * K + k] = encode_code(orc_bf16_to_f32(row[k]) / sm, qt);
  }
}

/* Weight quantization [OT-WIKI float8 / float W8A8 / int W8A8: "Tensor-wise
 * quantization of weights"; GGUF A8 int: "re-quantized ... axis-wise"]. */
void orc_quantize_weight(const uint16_t* w, int64_t N, int64_t K, int qt,
                         int gran, uint8_t* q, float* s) {
  if (gran == ORC_AXIS) {
    orc_quantize_rows(w, N, K, K, qt, q, s);
    return;
  }
  float a = 0.0f;
  for (int64_t i = 0; i < N * K; ++i) {
    float v = fabsf(orc_bf16_to_f32(w[i]));
    if (v > a) a = v;
  }
  float sw = absmax_scale(a, qt);
  s[0] = sw;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < N * K; ++i)
    q[i] = encode_code(orc_bf16_to_f32(w[i]) / sw, qt);
}

/* ========================================================================== */
/* GGUF Q8_0 [Q80]                                                             */
/* ========================================================================== */

#define Q80_BLOCK 32          /* GGUF_BLOCK_SIZE: "Each block: 32 values"     */
#define Q80_BYTES 34          /* "-> 34 bytes (2 scale + 32 data)"            */

int64_t orc_q8_0_bytes(int64_t n) { return ((n + Q80_BLOCK - 1) / Q80_BLOCK) * Q80_BYTES; }

/* Q8_0::quantize: per block of 32 (the last one may be short),
 *   max_abs = max |v|;  scale = max_abs < 1e-10 ? 1e-10 : max_abs / 127;
 *   q = clamp(round(v / scale), -128, 127), round = ties away from zero;
 *   short blocks are padded with zero codes.
 * The f32 scale is stored as f16 (round to nearest even) in the 34-byte block
 * ("stored as f32, converted to f16 on export"). */
void orc_q8_0_quantize(const float* x, int64_t n, uint8_t* blocks, float* scales_f32) {
  int64_t nb = (n + Q80_BLOCK - 1) / Q80_BLOCK;
#pragma omp parallel for schedule(static)
  for (int64_t b = 0; b < nb; ++b) {
    int64_t start = b * Q80_BLOCK;
    int64_t end = start + Q80_BLOCK < n ? start + Q80_BLOCK : n;
    float max_abs = 0.0f;
    for (int64_t i = start; i < end; ++i) {
      float v = fabsf(x[i]);
      if (v > max_abs) max_abs = v;
    }
    float scale = (max_abs < 1e-10f) ? 1e-10f : max_abs / 127.0f;
    if (scales_f32) scales_f32[b] = scale;
    uint8_t* blk = blocks + b * Q80_BYTES;
    uint16_t d = orc_f32_to_f16(scale);
    blk[0] = (uint8_t)(d & 0xFF);          /* little-endian f16 */
    blk[1] = (uint8_t)(d >> 8);
    for (int64_t j = 0; j < Q80_BLOCK; ++j) {
      int8_t code = 0;                      /* padding of a short block */
      if (start + j < end) {
        float r = roundf(x[start + j] / scale);
        if (r < -128.0f) r = -128.0f;
        if (r > 127.0f) r = 127.0f;
        code = (int8_t)r;
      }
      blk[2 + j] = (uint8_t)code;
    }
  }
}

static float block_scale_f16(const uint8_t* blk) {
  uint16_t d = (uint16_t)(blk[0] | (blk[1] << 8));
  return orc_f16_to_f32(d);
}

/* GGUF dequantization: value = f16 scale * code (the product of an 11-bit and
 * an 8-bit significand is exact in fp32). */
void orc_q8_0_dequantize(const uint8_t* blocks, int64_t n, float* y) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    const uint8_t* blk = blocks + (i / Q80_BLOCK) * Q80_BYTES;
    y[i] = block_scale_f16(blk) * (float)(int8_t)blk[2 + i % Q80_BLOCK];
  }
}

/* Q8_0::dequantize on the struct: f32::from(q) * scales[i / 32]. */
void orc_q8_0_dequantize_f32(const float* scales_f32, const int8_t* codes,
                             int64_t n, float* y) {
  for (int64_t i = 0; i < n; ++i) y[i] = (float)codes[i] * scales_f32[i / Q80_BLOCK];
}

/* GGUF A8 int / GGUF A8 float [OT-WIKI]: weights "re-quantized from GGUF to
 * int8 axis-wise" / "to float8 (e4m3) axis-wise".  Each weight row n holds
 * K/32 consecutive blocks; dequantize (exact), then the token-wise rule on
 * that row: s_n = floor(absmax)/QMAX, q = code(deq / s_n), with QMAX and the
 * code of the target type (int8: 127, RNE, clamp; e4m3: 448, RNE-satfinite).
 * q holds N*K one-byte codes. */
void orc_q8_0_to_axis(const uint8_t* blocks, int64_t N, int64_t K, int qt,
                      uint8_t* q, float* s) {
  int64_t bpr = K / Q80_BLOCK;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    float* deq = (float*)malloc((size_t)K * sizeof(float));
    orc_q8_0_dequantize(blocks + n * bpr * Q80_BYTES, K, deq);
    float a = 0.0f;
    for (int64_t k = 0; k < K; ++k)
      if (fabsf(deq[k]) > a) a = fabsf(deq[k]);
    float sn = absmax_scale(a, qt);
    s[n] = sn;
    for (int64_t k = 0; k < K; ++k) q[n * K + k] = encode_code(deq[k] / sn, qt);
    free(deq);
  }
}

void orc_q8_0_to_axis_int8(const uint8_t* blocks, int64_t N, int64_t K,
                           int8_t* q, float* s) {
  orc_q8_0_to_axis(blocks, N, K, ORC_INT8, (uint8_t*)q, s);
}

/* ========================================================================== */
/* The activation between two projections and the row absmax of an output     */
/* (not on the pages: the optional GELU of a DiT MLP block, read plainly; the */
/* row absmax is a property of the output, max_n |y[m,n]|).                   */
/* ========================================================================== */

/* GELU, exact form: 0.5 v (1 + erf(v / sqrt 2)); tanh form: 0.5 v (1 +
 * tanh(sqrt(2/pi) (v + 0.044715 v^3))).  In double, rounded once to fp32. */
void orc_act(const float* v, int64_t n, int act, float* out) {
  for (int64_t i = 0; i < n; ++i) {
    double x = (double)v[i], r = x;
    if (act == 1) r = 0.5 * x * (1.0 + erf(x / sqrt(2.0)));
    if (act == 2) r = 0.5 * x * (1.0 + tanh(sqrt(2.0 / M_PI) * (x + 0.044715 * x * x * x)));
    out[i] = (float)r;
  }
}

/* amax[m] = max_n |bf16 y[m, n]| as fp32. */
void orc_row_absmax_bf16(const uint16_t* y, int64_t M, int64_t N, float* amax) {
  for (int64_t m = 0; m < M; ++m) {
    float a = 0.0f;
    for (int64_t n = 0; n < N; ++n) {
      float v = fabsf(orc_bf16_to_f32(y[m * N + n]));
      if (v > a) a = v;
    }
    amax[m] = a;
  }
}

/* ========================================================================== */
/* Weight-only types [OT-WIKI float8: "Tensor-wise quantization of weights in */
/* float8 e4m3. Dequantized to your Train Data Type"; GGUF: "dequantized to   */
/* Train Data Type"]: the weight becomes bf16, then a bf16 Linear.            */
/* ========================================================================== */

/* w = bf16(dec(q) * s): the e4m3 value times the tensor-wise scale, one fp32
 * RN product, then bf16 RNE. */
void orc_dequant_e4m3_bf16(const uint8_t* q, int64_t n, float s, uint16_t* w) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) w[i] = orc_f32_to_bf16(orc_e4m3_to_f32(q[i]) * s);
}

/* w = bf16(f16(d) * q): the exact GGUF value, then bf16 RNE. */
void orc_q8_0_dequantize_bf16(const uint8_t* blocks, int64_t n, uint16_t* w) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    const uint8_t* blk = blocks + (i / Q80_BLOCK) * Q80_BYTES;
    w[i] = orc_f32_to_bf16(block_scale_f16(blk) * (float)(int8_t)blk[2 + i % Q80_BLOCK]);
  }
}

/* The bf16 Linear: acc[m,n] = sum_k x[m,k] w[n,k] in fp64 (bf16 products are
 * exact), absacc = sum |x w|; y32 = fp32(acc) (+ bias as one fp32 RN add),
 * y = bf16(y32). */
void orc_linear_bf16(const uint16_t* x, const uint16_t* w, int64_t M, int64_t N, int64_t K,
                     const uint16_t* bias, double* acc, double* absacc, float* y32, uint16_t* y) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      double sum = 0.0, asum = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        double p = (double)orc_bf16_to_f32(x[m * K + k]) * (double)orc_bf16_to_f32(w[n * K + k]);
        sum += p;
        asum += fabs(p);
      }
      acc[m * N + n] = sum;
      absacc[m * N + n] = asum;
      float v = (float)sum;
      if (bias) v = v + orc_bf16_to_f32(bias[n]);
      y32[m * N + n] = v;
      y[m * N + n] = orc_f32_to_bf16(v);
    }
}

/* ========================================================================== */
/* 8-bit matrix products [OT-PR "8bit matrix multiplications"; OT-WIKI        */
/* "matrix multiplications are performed in int8 / float8"]                   */
/* ========================================================================== */

int orc_gemm_i8_nt(const int8_t* A, const int8_t* B, int64_t M, int64_t N,
                   int64_t K, int32_t* acc) {
  int overflow = 0;
#pragma omp parallel for schedule(static) reduction(| : overflow)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      int64_t sum = 0;
      for (int64_t k = 0; k < K; ++k) sum += (int64_t)A[m * K + k] * (int64_t)B[n * K + k];
      if (sum > INT32_MAX || sum < INT32_MIN) overflow = 1;
      acc[m * N + n] = (int32_t)sum;
    }
  return overflow;
}

int orc_gemm_i8_nn(const int8_t* A, const int8_t* B, int64_t M, int64_t N,
                   int64_t K, int32_t* acc) {
  int overflow = 0;
#pragma omp parallel for schedule(static) reduction(| : overflow)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k) {
      int64_t sum = 0;
      for (int64_t n = 0; n < N; ++n) sum += (int64_t)A[m * N + n] * (int64_t)B[n * K + k];
      if (sum > INT32_MAX || sum < INT32_MIN) overflow = 1;
      acc[m * K + k] = (int32_t)sum;
    }
  return overflow;
}

void orc_gemm_e4m3_nt(const uint8_t* A, const uint8_t* B, int64_t M, int64_t N,
                      int64_t K, double* acc, double* absacc) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      double sum = 0.0, asum = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        double p = (double)orc_e4m3_to_f32(A[m * K + k]) * (double)orc_e4m3_to_f32(B[n * K + k]);
        sum += p;
        asum += fabs(p);
      }
      acc[m * N + n] = sum;
      if (absacc) absacc[m * N + n] = asum;
    }
}

void orc_gemm_e4m3_nn(const uint8_t* A, const uint8_t* B, int64_t M, int64_t N,
                      int64_t K, double* acc, double* absacc) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k) {
      double sum = 0.0, asum = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        double p = (double)orc_e4m3_to_f32(A[m * N + n]) * (double)orc_e4m3_to_f32(B[n * K + k]);
        sum += p;
        asum += fabs(p);
      }
      acc[m * K + k] = sum;
      if (absacc) absacc[m * K + k] = asum;
    }
}

/* ========================================================================== */
/* Dequantizing epilogue: acc x row scale x weight scale (+ bias) -> bf16      */
/* ========================================================================== */

void orc_epilogue_i32(const int32_t* acc, int64_t M, int64_t N,
                      const float* s_row, const float* s_w, int w_axis,
                      const uint16_t* bias, float* y32, uint16_t* y) {
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      float t = (float)acc[m * N + n] * s_row[m];
      float u = t * s_w[w_axis ? n : 0];
      if (bias) u = u + orc_bf16_to_f32(bias[n]);
      if (y32) y32[m * N + n] = u;
      if (y) y[m * N + n] = orc_f32_to_bf16(u);
    }
}

void orc_epilogue_f64(const double* acc, int64_t M, int64_t N,
                      const float* s_row, const float* s_w, int w_axis,
                      const uint16_t* bias, float* y32, uint16_t* y) {
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      double u = acc[m * N + n] * (double)s_row[m] * (double)s_w[w_axis ? n : 0];
      if (bias) u += (double)orc_bf16_to_f32(bias[n]);
      float u32 = (float)u;
      if (y32) y32[m * N + n] = u32;
      if (y) y[m * N + n] = orc_f32_to_bf16(u32);
    }
}

/* ========================================================================== */
/* SVDQuant low-rank branch: Y += (X L1) L2 with bf16 factors                  */
/* ========================================================================== */

void orc_lowrank_down(const uint16_t* x, const uint16_t* l1, int64_t M,
                      int64_t K, int64_t r, double* t64, uint16_t* t) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t j = 0; j < r; ++j) {
      double sum = 0.0;
      for (int64_t k = 0; k < K; ++k)
        sum += (double)orc_bf16_to_f32(x[m * K + k]) * (double)orc_bf16_to_f32(l1[k * r + j]);
      if (t64) t64[m * r + j] = sum;
      if (t) t[m * r + j] = orc_f32_to_bf16((float)sum);
    }
}

void orc_lowrank_up(const uint16_t* t, const uint16_t* l2, int64_t M,
                    int64_t r, int64_t N, double* lr, double* lr_abs) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      double sum = 0.0, asum = 0.0;
      for (int64_t j = 0; j < r; ++j) {
        double p = (double)orc_bf16_to_f32(t[m * r + j]) * (double)orc_bf16_to_f32(l2[j * N + n]);
        sum += p;
        asum += fabs(p);
      }
      lr[m * N + n] = sum;
      if (lr_abs) lr_abs[m * N + n] = asum;
    }
}
