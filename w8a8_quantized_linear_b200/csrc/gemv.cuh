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
// codes are decoded to fp32 and multiplied there.  Every block quantizes the
// M rows to e4m3 (the row quantizer's arithmetic) and keeps their values,
// times 2^112, in shared memory; a warp per weight row decodes each weight
// code with integer operations to its value times 2^-120 (e4m3_top_byte_scaled)
// and accumulates fl(w a 2^-8) products - exact: 4-bit by 4-bit significands,
// no subnormal - in fp32.  acc * 2^8 (exact) then takes the GEMM epilogue's
// fp32 RN steps.  The sum is in another order than the tensor cores', within
// the fp8 bound.
//
// Shared layout: the activations of row m, in 16-value units U (16 U .. 16 U
// + 15), with the 4 float4 quads of unit U stored at ((U / 32) * 4 + quad) *
// 128 + (U % 32) * 4, so that the 32 lanes of a warp (lane l takes units l,
// l + 32, ...) read 32 consecutive float4: no bank conflict.
constexpr int kGemvE4m3MaxRows = 4;
constexpr int kGemvE4m3SmemBytes = 128 * 1024;   // M * (K rounded up to 512) * 4

__device__ __forceinline__ int gemv_e4m3_slot(int k) {   // float index of value k within its row
  const int u = k >> 4, quad = (k >> 2) & 3;
  return (((u >> 5) * 4 + quad) << 7) + ((u & 31) << 2) + (k & 3);
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
  float* const act = reinterpret_cast<float*>(gemv_smem);
  __shared__ float red[32];
  __shared__ float sx[kGemvE4m3MaxRows];
  griddep_launch();
  griddep_wait();   // x may be the previous kernel's output
  const int nv = K >> 3;             // 8-value vectors per row
  const int row_f = ((K + 511) >> 9) << 9;   // floats per row in shared memory
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
      const uint2 c = encode8<1>(__ldg(row + v), s, yr);
      const uint32_t cw[2] = {c.x, c.y};
      float f[8];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        // code value * 2^-120, then * 2^116 * 2^116 = value * 2^112 (exact)
        f[4 * j] = e4m3_top_byte_scaled(cw[j] << 24);
        f[4 * j + 1] = e4m3_top_byte_scaled(cw[j] << 16);
        f[4 * j + 2] = e4m3_top_byte_scaled(cw[j] << 8);
        f[4 * j + 3] = e4m3_top_byte_scaled(cw[j]);
      }
      float* dst = act + m * row_f;
#pragma unroll
      for (int i = 0; i < 8; i += 4) {
        float4 q4;
        q4.x = __fmul_rn(__fmul_rn(f[i], 0x1p116f), 0x1p116f);
        q4.y = __fmul_rn(__fmul_rn(f[i + 1], 0x1p116f), 0x1p116f);
        q4.z = __fmul_rn(__fmul_rn(f[i + 2], 0x1p116f), 0x1p116f);
        q4.w = __fmul_rn(__fmul_rn(f[i + 3], 0x1p116f), 0x1p116f);
        *reinterpret_cast<float4*>(dst + gemv_e4m3_slot(8 * v + i)) = q4;
      }
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
          float wv[16];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            wv[4 * j] = e4m3_top_byte_scaled(cw[j] << 24);
            wv[4 * j + 1] = e4m3_top_byte_scaled(cw[j] << 16);
            wv[4 * j + 2] = e4m3_top_byte_scaled(cw[j] << 8);
            wv[4 * j + 3] = e4m3_top_byte_scaled(cw[j]);
          }
          const int slot = (((U >> 5) * 4) << 7) + ((U & 31) << 2);
#pragma unroll
          for (int m = 0; m < M; ++m) {
            const float* ar = act + m * row_f + slot;
#pragma unroll
            for (int quad = 0; quad < 4; ++quad) {
              const float4 a4 = *reinterpret_cast<const float4*>(ar + quad * 128);
              acc[m] = __fmaf_rn(wv[4 * quad], a4.x, acc[m]);
              acc[m] = __fmaf_rn(wv[4 * quad + 1], a4.y, acc[m]);
              acc[m] = __fmaf_rn(wv[4 * quad + 2], a4.z, acc[m]);
              acc[m] = __fmaf_rn(wv[4 * quad + 3], a4.w, acc[m]);
            }
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
      float f = __fmul_rn(a, 256.0f);   // the products carried 2^-8
      f = __fmul_rn(__fmul_rn(f, sx[lane]), axis ? __ldg(s_col + n) : sw0);
      if (bias != nullptr) f = __fadd_rn(f, __bfloat162float(bias[n]));
      if (in_bounds(static_cast<int64_t>(lane) * N + n, static_cast<int64_t>(M) * N, 0xB302))
        y[static_cast<int64_t>(lane) * N + n] = __float2bfloat16_rn(f);
    }
  }
}

}  // namespace w8a8
