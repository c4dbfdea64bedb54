// gemv.cuh - the int8 W8A8 forward for a few tokens (M <= kGemvMaxRows), in
// one launch on the CUDA cores: a weight-streaming product, bound by HBM,
// where a tensor-core tile would be almost all padding.
//
// Every block quantizes the M activation rows itself (the row quantizer's
// arithmetic: absmax, scale with the 1e-10 floor, codes from the refined
// quotient) into shared memory, then its warps stream weight rows with
// 16-byte loads and accumulate dp4a products in int32 (exact), and write
//     y[m, n] = bf16( ((acc * s_x[m]) * s_w[n or 0]) + bias[n] )
// with the same fp32 RN steps as the GEMM epilogue.  The result is the
// quantize + GEMM path's bit for bit.
#pragma once
#include "quantize.cuh"
#include "weight_only.cuh"

namespace w8a8 {

constexpr int kGemvMaxRows = 8;    // rows the kernel supports
constexpr int kGemvUseRows = 2;    // rows for which it beats quantize + GEMM (the library's choice)
constexpr int kGemvThreads = 256;
constexpr int kGemvMaxK = 16384;   // M * K codes in shared memory: at most 128 KB

// M rows of x [M, K] bf16 -> codes in shared memory (row stride K) and the
// row scales (s_out, shared).  All threads of the block take part.
template <int M>
__device__ __forceinline__ void gemv_quantize_rows(const __nv_bfloat16* __restrict__ x, int64_t ldx, int K,
                                                   uint8_t* codes, float* s_out, float* red) {
  const int nv = K >> 3;
  for (int m = 0; m < M; ++m) {
    const uint4* row = reinterpret_cast<const uint4*>(x + m * ldx);
    uint32_t mb = 0;
    for (int v = threadIdx.x; v < nv; v += kGemvThreads)
      if (in_bounds(v, nv, 0xB303)) mb = absmax8(__ldg(row + v), mb);
    const float a = block_max(bf2_absmax_final(mb), red);
    const float s = absmax_scale<0>(a);
    const float y = __frcp_rn(s);
    if (threadIdx.x == 0) s_out[m] = s;
    uint2* out = reinterpret_cast<uint2*>(codes + m * K);
    for (int v = threadIdx.x; v < nv; v += kGemvThreads)
      if (in_bounds(v, nv, 0xB303)) out[v] = encode8<0>(__ldg(row + v), s, y);
  }
  __syncthreads();
}

// One warp per weight row n (grid-stride over rows): lane l takes the
// 16-byte units l, l + 32, ... of the row.
template <int M>
__global__ void __launch_bounds__(kGemvThreads, 4) gemv_int8_kernel(const __nv_bfloat16* __restrict__ x, int64_t ldx,
                                                                int N, int K, const int8_t* __restrict__ wq,
                                                                const float* __restrict__ s_col, int axis,
                                                                const __nv_bfloat16* __restrict__ bias,
                                                                __nv_bfloat16* __restrict__ y) {
  extern __shared__ __align__(16) uint8_t gemv_smem[];
  __shared__ float red[32];
  __shared__ float sx[kGemvMaxRows];
  griddep_launch();
  griddep_wait();   // x may be the previous kernel's output
  gemv_quantize_rows<M>(x, ldx, K, gemv_smem, sx, red);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = K >> 4;   // 16-byte units per row
  const float sw0 = axis ? 0.0f : s_col[0];
  for (int n = blockIdx.x * (kGemvThreads / 32) + warp; n < N; n += gridDim.x * (kGemvThreads / 32)) {
    if (!in_bounds(n, N, 0xB301)) break;   // warp-uniform
    const uint4* wrow = reinterpret_cast<const uint4*>(wq + static_cast<int64_t>(n) * K);
    int acc[M];
#pragma unroll
    for (int m = 0; m < M; ++m) acc[m] = 0;
    // up to eight 16-byte weight units in flight per lane (4096 codes of a
    // row at once), then the dot products
    for (int base = lane; base < nv; base += 256) {
      uint4 w8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (base + 32 * u < nv && in_bounds(base + 32 * u, nv, 0xB301)) w8[u] = __ldg(wrow + base + 32 * u);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (base + 32 * u < nv) {
#pragma unroll
          for (int m = 0; m < M; ++m) {
            const uint4 c = *reinterpret_cast<const uint4*>(gemv_smem + m * K + 16 * (base + 32 * u));
            acc[m] = __dp4a(static_cast<int>(w8[u].x), static_cast<int>(c.x), acc[m]);
            acc[m] = __dp4a(static_cast<int>(w8[u].y), static_cast<int>(c.y), acc[m]);
            acc[m] = __dp4a(static_cast<int>(w8[u].z), static_cast<int>(c.z), acc[m]);
            acc[m] = __dp4a(static_cast<int>(w8[u].w), static_cast<int>(c.w), acc[m]);
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < M; ++m) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[m] += __shfl_xor_sync(0xFFFFFFFFu, acc[m], o);
    }
    if (lane < M) {
      int a = acc[0];
#pragma unroll
      for (int m = 1; m < M; ++m)
        if (lane == m) a = acc[m];
      float f = __int2float_rn(a);
      f = __fmul_rn(__fmul_rn(f, sx[lane]), axis ? __ldg(s_col + n) : sw0);
      if (bias != nullptr) f = __fadd_rn(f, __bfloat162float(bias[n]));
      if (in_bounds(static_cast<int64_t>(lane) * N + n, static_cast<int64_t>(M) * N, 0xB302))
        y[static_cast<int64_t>(lane) * N + n] = __float2bfloat16_rn(f);
    }
  }
}

// ---------------------------------------------------------------------------
// The e4m3 forward for a few tokens (M <= kGemvE4m3MaxRows), e.g. GGUF A8
// float at decode: e4m3 has no exact CUDA-core dot product like dp4a, so the
// codes are multiplied as 16-bit floats.  Every block quantizes the M rows to
// e4m3 (the row quantizer's arithmetic) and keeps their values as f16 in
// shared memory (every e4m3 value is an f16 value); a warp per weight row
// converts each pair of weight codes to an f16 pair (cvt.rn.f16x2.e4m3x2,
// exact) and accumulates with the mixed-precision fma.rn.f32.f16: the product
// of two f16 operands is exact in fp32 (4-bit by 4-bit significands here), so
// each step is one fp32 RN add, in k order.  acc then takes the GEMM
// epilogue's fp32 RN steps.  The sum is in another order than the tensor
// cores', within the fp8 bound.
//
// Shared layout: the activations of row m, in 16-value units U (16 U .. 16 U
// + 15) of two 16-byte halves (8 f16 each), half h of unit U at byte
// (((U / 32) * 2 + h) * 32 + U % 32) * 16, so that the 32 lanes of a warp
// (lane l takes units l, l + 32, ...) read 32 consecutive 16-byte words: no
// bank conflict.
constexpr int kGemvE4m3MaxRows = 4;
constexpr int kGemvE4m3SmemBytes = 128 * 1024;   // the K limit: M * (K rounded up to 512) * 4 <= this
                                                 // (the f16 activations take half)

__device__ __forceinline__ int gemv_e4m3_half_off(int u, int h) {   // byte offset of half h of unit u
  return ((((u >> 5) * 2 + h) << 5) + (u & 31)) << 4;
}
// Two e4m3 codes (bits 15..0 of v; the code in bits 7..0 comes first) -> their
// values as an f16 pair, the first in the low half.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t v) {
  uint32_t h2;
  asm("{\n\t.reg .b16 lo;\n\tcvt.u16.u32 lo, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, lo;\n\t}" : "=r"(h2) : "r"(v));
  return h2;
}
// acc + w.lo a.lo, then + w.hi a.hi: fp32 fma of f16 operands (exact products
// of e4m3 values), one RN rounding each.
__device__ __forceinline__ float fma_f16x2_f32(uint32_t w2, uint32_t a2, float acc) {
  float r;
  asm("{\n\t.reg .b16 w0, w1, a0, a1;\n\tmov.b32 {w0, w1}, %1;\n\tmov.b32 {a0, a1}, %2;\n\t"
      "fma.rn.f32.f16 %0, w0, a0, %3;\n\tfma.rn.f32.f16 %0, w1, a1, %0;\n\t}"
      : "=f"(r)
      : "r"(w2), "r"(a2), "f"(acc));
  return r;
}

// blocks per SM: as many as the registers allow (the weight stream needs
// many loads in flight; one row per warp at a time)
template <int M>
constexpr int gemv_e4m3_min_blocks() { return M == 1 ? 4 : (M == 2 ? 3 : 2); }

template <int M>
__global__ void __launch_bounds__(kGemvThreads, gemv_e4m3_min_blocks<M>()) gemv_e4m3_kernel(const __nv_bfloat16* __restrict__ x, int64_t ldx,
                                                                 int N, int K, const uint8_t* __restrict__ wq,
                                                                 const float* __restrict__ s_col, int axis,
                                                                 const __nv_bfloat16* __restrict__ bias,
                                                                 __nv_bfloat16* __restrict__ y) {
  extern __shared__ __align__(16) uint8_t gemv_smem[];
  __shared__ float red[32];
  __shared__ float sx[kGemvE4m3MaxRows];
  griddep_launch();
  griddep_wait();   // x may be the previous kernel's output
  const int nv = K >> 3;             // 8-value vectors per row
  const int row_b = (((K + 511) >> 9) << 9) * 2;   // bytes per row in shared memory
  for (int m = 0; m < M; ++m) {
    const uint4* row = reinterpret_cast<const uint4*>(x + m * ldx);
    uint32_t mb = 0;
    for (int v = threadIdx.x; v < nv; v += kGemvThreads)
      if (in_bounds(v, nv, 0xB303)) mb = absmax8(__ldg(row + v), mb);
    const float a = block_max(bf2_absmax_final(mb), red);
    const float s = absmax_scale<1>(a);
    const float yr = __frcp_rn(s);
    if (threadIdx.x == 0) sx[m] = s;
    for (int v = threadIdx.x; v < nv; v += kGemvThreads) {
      // values 8 v .. 8 v + 7: half (v & 1) of unit v / 2
      const uint2 c = encode8<1>(__ldg(row + v), s, yr);
      const uint4 h = make_uint4(e4m3x2_to_f16x2(c.x), e4m3x2_to_f16x2(c.x >> 16), e4m3x2_to_f16x2(c.y),
                                 e4m3x2_to_f16x2(c.y >> 16));
      *reinterpret_cast<uint4*>(gemv_smem + m * row_b + gemv_e4m3_half_off(v >> 1, v & 1)) = h;
    }
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nu = K >> 4;   // 16-code units per weight row
  const float sw0 = axis ? 0.0f : s_col[0];
  for (int n = blockIdx.x * (kGemvThreads / 32) + warp; n < N; n += gridDim.x * (kGemvThreads / 32)) {
    if (!in_bounds(n, N, 0xB301)) break;   // warp-uniform
    const uint4* wrow = reinterpret_cast<const uint4*>(wq + static_cast<int64_t>(n) * K);
    float acc[M];
#pragma unroll
    for (int m = 0; m < M; ++m) acc[m] = 0.0f;
    for (int base = lane; base < nu; base += 256) {
      uint4 w8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (base + 32 * u < nu && in_bounds(base + 32 * u, nu, 0xB301)) w8[u] = __ldg(wrow + base + 32 * u);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int U = base + 32 * u;
        if (U < nu) {
          const uint32_t cw[4] = {w8[u].x, w8[u].y, w8[u].z, w8[u].w};
          uint32_t wh[8];   // f16 pairs of codes 2 i, 2 i + 1 of the unit
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            wh[2 * j] = e4m3x2_to_f16x2(cw[j]);
            wh[2 * j + 1] = e4m3x2_to_f16x2(cw[j] >> 16);
          }
#pragma unroll
          for (int m = 0; m < M; ++m) {
            const uint8_t* ar = gemv_smem + m * row_b;
            const uint4 a0 = *reinterpret_cast<const uint4*>(ar + gemv_e4m3_half_off(U, 0));
            const uint4 a1 = *reinterpret_cast<const uint4*>(ar + gemv_e4m3_half_off(U, 1));
            acc[m] = fma_f16x2_f32(wh[0], a0.x, acc[m]);
            acc[m] = fma_f16x2_f32(wh[1], a0.y, acc[m]);
            acc[m] = fma_f16x2_f32(wh[2], a0.z, acc[m]);
            acc[m] = fma_f16x2_f32(wh[3], a0.w, acc[m]);
            acc[m] = fma_f16x2_f32(wh[4], a1.x, acc[m]);
            acc[m] = fma_f16x2_f32(wh[5], a1.y, acc[m]);
            acc[m] = fma_f16x2_f32(wh[6], a1.z, acc[m]);
            acc[m] = fma_f16x2_f32(wh[7], a1.w, acc[m]);
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < M; ++m) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[m] += __shfl_xor_sync(0xFFFFFFFFu, acc[m], o);
    }
    if (lane < M) {
      float a = acc[0];
#pragma unroll
      for (int m = 1; m < M; ++m)
        if (lane == m) a = acc[m];
      float f = __fmul_rn(__fmul_rn(a, sx[lane]), axis ? __ldg(s_col + n) : sw0);
      if (bias != nullptr) f = __fadd_rn(f, __bfloat162float(bias[n]));
      if (in_bounds(static_cast<int64_t>(lane) * N + n, static_cast<int64_t>(M) * N, 0xB302))
        y[static_cast<int64_t>(lane) * N + n] = __float2bfloat16_rn(f);
    }
  }
}

}  // namespace w8a8
