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

namespace w8a8 {

constexpr int kGemvMaxRows = 8;
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
    for (int v = threadIdx.x; v < nv; v += kGemvThreads) mb = absmax8(__ldg(row + v), mb);
    const float a = block_max(bf2_absmax_final(mb), red);
    const float s = absmax_scale<0>(a);
    const float y = __frcp_rn(s);
    if (threadIdx.x == 0) s_out[m] = s;
    uint2* out = reinterpret_cast<uint2*>(codes + m * K);
    for (int v = threadIdx.x; v < nv; v += kGemvThreads) out[v] = encode8<0>(__ldg(row + v), s, y);
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
        if (base + 32 * u < nv) w8[u] = __ldg(wrow + base + 32 * u);
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
      y[static_cast<int64_t>(lane) * N + n] = __float2bfloat16_rn(f);
    }
  }
}

}  // namespace w8a8
