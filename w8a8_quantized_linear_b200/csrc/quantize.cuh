// quantize.cuh - token-wise absmax calibration + quantization in one pass
// (the fused row calibrate-and-quantize of bitsandbytes #1401), and the
// tensor-wise weight quantizer.  Bandwidth-bound: 16-byte coalesced loads and
// stores, warp-shuffle reductions, no tensor cores.
#pragma once
#include "device.cuh"

namespace w8a8 {

constexpr int kRowVecs = 4;   // 16-byte vectors per thread kept in registers

// Code of v for the two activation formats.
template <int QT>
__device__ __forceinline__ float qmax_of() { return QT == 1 ? 448.0f : 127.0f; }

// absmax scale with the 1e-10 floor, IEEE fp32 division.
template <int QT>
__device__ __forceinline__ float absmax_scale(float a) {
  return (a < 1e-10f) ? 1e-10f : __fdiv_rn(a, qmax_of<QT>());
}

// 8 bf16 (one uint4) -> 8 codes (one uint2), each x / s divided in fp32.
template <int QT>
__device__ __forceinline__ uint2 encode8(uint4 v, float s) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float a0 = __fdiv_rn(bf16_lo(w[2 * h]), s), a1 = __fdiv_rn(bf16_hi(w[2 * h]), s);
    const float a2 = __fdiv_rn(bf16_lo(w[2 * h + 1]), s), a3 = __fdiv_rn(bf16_hi(w[2 * h + 1]), s);
    if constexpr (QT == 1) {
      out[h] = static_cast<uint32_t>(cvt_e4m3x2(a0, a1)) | (static_cast<uint32_t>(cvt_e4m3x2(a2, a3)) << 16);
    } else {
      out[h] = int8_code(a0) | (int8_code(a1) << 8) | (int8_code(a2) << 16) | (int8_code(a3) << 24);
    }
  }
  return make_uint2(out[0], out[1]);
}

__device__ __forceinline__ float absmax8(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) a = fmaxf(a, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
  return a;
}

// Block-wide max; every thread gets the result.  red: >= 32 floats of smem.
__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = (blockDim.x + 31) >> 5;
  __syncthreads();                 // red may still be read from the previous row
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = (lane < nw) ? red[lane] : 0.0f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) r = fmaxf(r, __shfl_xor_sync(0xFFFFFFFFu, r, o));
  return r;
}

// One block per row (grid-stride over rows).  The row's 16-byte vectors
// v = tid + j*blockDim are held in registers for j < kRowVecs; longer rows
// re-read the remainder (an L2 hit) in the second pass.
template <int QT>
__global__ void __launch_bounds__(1024) quantize_rows_kernel(const __nv_bfloat16* __restrict__ x, int64_t ldx,
                                                             int64_t M, int64_t K, uint8_t* __restrict__ q,
                                                             int64_t ldq, float* __restrict__ scale) {
  __shared__ float red[32];
  const int64_t nv = K >> 3;
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    const uint4* row = reinterpret_cast<const uint4*>(x + m * ldx);
    uint4 keep[kRowVecs];
    float a = 0.0f;
#pragma unroll
    for (int j = 0; j < kRowVecs; ++j) {
      const int64_t v = threadIdx.x + static_cast<int64_t>(j) * blockDim.x;
      if (v < nv) {
        keep[j] = __ldg(row + v);
        a = fmaxf(a, absmax8(keep[j]));
      }
    }
    for (int64_t v = threadIdx.x + static_cast<int64_t>(kRowVecs) * blockDim.x; v < nv; v += blockDim.x)
      a = fmaxf(a, absmax8(__ldg(row + v)));
    a = block_max(a, red);
    const float s = absmax_scale<QT>(a);
    if (threadIdx.x == 0) scale[m] = s;
    uint2* out = reinterpret_cast<uint2*>(q + m * ldq);
#pragma unroll
    for (int j = 0; j < kRowVecs; ++j) {
      const int64_t v = threadIdx.x + static_cast<int64_t>(j) * blockDim.x;
      if (v < nv) out[v] = encode8<QT>(keep[j], s);
    }
    for (int64_t v = threadIdx.x + static_cast<int64_t>(kRowVecs) * blockDim.x; v < nv; v += blockDim.x)
      out[v] = encode8<QT>(__ldg(row + v), s);
  }
}

// Tensor-wise weight quantization, pass 1: global absmax of W (as the bit
// pattern of a non-negative float, so an unsigned atomicMax orders it).
__global__ void __launch_bounds__(256) absmax_kernel(const uint4* __restrict__ w, int64_t nvec,
                                                     unsigned* __restrict__ amax_bits) {
  __shared__ float red[32];
  float a = 0.0f;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nvec;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    a = fmaxf(a, absmax8(__ldg(w + i)));
  a = block_max(a, red);
  if (threadIdx.x == 0) atomicMax(amax_bits, __float_as_uint(a));
}

// Pass 2: one scale for the whole tensor, codes for every element.
template <int QT>
__global__ void __launch_bounds__(256) quantize_tensor_kernel(const uint4* __restrict__ w, int64_t nvec,
                                                              const unsigned* __restrict__ amax_bits,
                                                              uint2* __restrict__ q, float* __restrict__ scale) {
  const float s = absmax_scale<QT>(__uint_as_float(*amax_bits));
  if (blockIdx.x == 0 && threadIdx.x == 0) scale[0] = s;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nvec;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    q[i] = encode8<QT>(__ldg(w + i), s);
}

// fp32 -> E4M3FN codes with the quantizers' conversion.
__global__ void e4m3_encode_kernel(const float* __restrict__ x, int64_t n, uint8_t* __restrict__ y) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    y[i] = static_cast<uint8_t>(cvt_e4m3x2(x[i], 0.0f) & 0xFFu);
}

// Bounded-wait self test: one thread waits on a barrier that nothing
// completes; the wait runs out after limit_ns and records kDevTimeout.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait(&bar, 0, &abort_flag, 0xFFu, limit_ns);
  }
}

}  // namespace w8a8
