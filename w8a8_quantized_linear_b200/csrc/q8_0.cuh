// q8_0.cuh - GGUF Q8_0 blocks (32 values -> f16 scale + 32 int8 codes =
// 34 bytes; entrenar 0.7.8 q8_0.rs) on the GPU, and the re-quantization of a
// Q8_0 weight to axis-wise int8 (OneTrainer wiki, GGUF A8 int).
//
// A 34-byte block is not 16-byte aligned, but 8 blocks are 272 = 17 * 16
// bytes: one warp handles such a group of 8 blocks, with 16-byte global
// accesses on the block side staged through 272 bytes of shared memory.
#pragma once
#include "device.cuh"
#include "quantize.cuh"

namespace w8a8 {

constexpr int kQ80Block = 32;
constexpr int kQ80Bytes = 34;
constexpr int kQ80Group = 8 * kQ80Bytes;   // 272 bytes, 16-byte aligned groups
constexpr int kQ80WarpsPerBlock = 8;

// Quantize: lane l of the warp holds values [8l, 8l+8) of the 256-value group,
// so block j of the group lives in lanes 4j..4j+3.
__global__ void __launch_bounds__(256) q8_0_quantize_kernel(const float* __restrict__ x, int64_t n,
                                                            uint8_t* __restrict__ blocks) {
  __shared__ __align__(16) uint8_t stage[kQ80WarpsPerBlock][kQ80Group];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* st = stage[warp];
  const int64_t ngroups = (n + 255) / 256;
  const int64_t nbytes = ((n + 31) / 32) * kQ80Bytes;
  for (int64_t g = blockIdx.x * static_cast<int64_t>(kQ80WarpsPerBlock) + warp; g < ngroups;
       g += static_cast<int64_t>(gridDim.x) * kQ80WarpsPerBlock) {
    const int64_t base = g * 256 + lane * 8;
    float v[8];
    if (base + 8 <= n) {
      const float4 p0 = __ldg(reinterpret_cast<const float4*>(x + base));
      const float4 p1 = __ldg(reinterpret_cast<const float4*>(x + base) + 1);
      v[0] = p0.x; v[1] = p0.y; v[2] = p0.z; v[3] = p0.w;
      v[4] = p1.x; v[5] = p1.y; v[6] = p1.z; v[7] = p1.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = (base + i < n) ? x[base + i] : 0.0f;   // zero padding
    }
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
    a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 2));
    const float scale = (a < 1e-10f) ? 1e-10f : __fdiv_rn(a, 127.0f);
    const int j = lane >> 2, part = lane & 3;
    uint8_t* blk = st + j * kQ80Bytes;
    if (part == 0) {
      const uint16_t d = __half_as_ushort(__float2half_rn(scale));
      blk[0] = static_cast<uint8_t>(d & 0xFFu);
      blk[1] = static_cast<uint8_t>(d >> 8);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float r = roundf(__fdiv_rn(v[i], scale));           // ties away from zero
      r = fminf(fmaxf(r, -128.0f), 127.0f);
      blk[2 + part * 8 + i] = static_cast<uint8_t>(static_cast<int8_t>(r));
    }
    __syncwarp();
    if (lane < kQ80Group / 16) {
      const int64_t off = g * kQ80Group + lane * 16;
      if (off + 16 <= nbytes) {
        *reinterpret_cast<uint4*>(blocks + off) = *reinterpret_cast<const uint4*>(st + lane * 16);
      } else {
        for (int b = 0; b < 16; ++b)
          if (off + b < nbytes) blocks[off + b] = st[lane * 16 + b];
      }
    }
    __syncwarp();
  }
}

// Dequantize: the 272-byte group is copied to shared memory with 16-byte
// loads, then lane l writes values [8l, 8l+8) = f16 scale * code.
__global__ void __launch_bounds__(256) q8_0_dequantize_kernel(const uint8_t* __restrict__ blocks, int64_t n,
                                                              float* __restrict__ y) {
  __shared__ __align__(16) uint8_t stage[kQ80WarpsPerBlock][kQ80Group];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* st = stage[warp];
  const int64_t ngroups = (n + 255) / 256;
  const int64_t nbytes = ((n + 31) / 32) * kQ80Bytes;
  for (int64_t g = blockIdx.x * static_cast<int64_t>(kQ80WarpsPerBlock) + warp; g < ngroups;
       g += static_cast<int64_t>(gridDim.x) * kQ80WarpsPerBlock) {
    if (lane < kQ80Group / 16) {
      const int64_t off = g * kQ80Group + lane * 16;
      if (off + 16 <= nbytes) {
        *reinterpret_cast<uint4*>(st + lane * 16) = __ldg(reinterpret_cast<const uint4*>(blocks + off));
      } else {
        for (int b = 0; b < 16; ++b) st[lane * 16 + b] = (off + b < nbytes) ? blocks[off + b] : 0;
      }
    }
    __syncwarp();
    const int j = lane >> 2, part = lane & 3;
    const uint8_t* blk = st + j * kQ80Bytes;
    const float d = __half2float(__ushort_as_half(static_cast<uint16_t>(blk[0] | (blk[1] << 8))));
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = d * static_cast<float>(static_cast<int8_t>(blk[2 + part * 8 + i]));
    const int64_t base = g * 256 + lane * 8;
    if (base + 8 <= n) {
      float4* o = reinterpret_cast<float4*>(y + base);
      o[0] = make_float4(v[0], v[1], v[2], v[3]);
      o[1] = make_float4(v[4], v[5], v[6], v[7]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (base + i < n) y[base + i] = v[i];
    }
    __syncwarp();
  }
}

// Q8_0 [N, K/32 blocks] -> int8 [N, K] + s [N]: one thread block per weight
// row.  The row's K/32 * 34 bytes are staged in shared memory; each value is
// dequantized exactly (f16 scale * code is exact in fp32), the row absmax
// gives s, and the codes are rounded half-to-even and clamped to +-127.
__global__ void __launch_bounds__(256) q8_0_to_axis_int8_kernel(const uint8_t* __restrict__ blocks, int64_t N,
                                                                int64_t K, int8_t* __restrict__ q,
                                                                float* __restrict__ scale) {
  extern __shared__ __align__(16) uint8_t rowbuf[];
  __shared__ float red[32];
  const int64_t row_bytes = (K / kQ80Block) * kQ80Bytes;
  const int64_t nchunk = K / 16;   // 16 values per chunk, half a block
  for (int64_t n = blockIdx.x; n < N; n += gridDim.x) {
    const uint8_t* src = blocks + n * row_bytes;
    __syncthreads();               // rowbuf reuse across rows
    if (((reinterpret_cast<uintptr_t>(src) | static_cast<uintptr_t>(row_bytes)) & 15) == 0) {
      for (int64_t i = threadIdx.x; i < row_bytes / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(rowbuf)[i] = __ldg(reinterpret_cast<const uint4*>(src) + i);
    } else {   // rows always start on an even byte: 2-byte copies
      for (int64_t i = threadIdx.x; i < row_bytes / 2; i += blockDim.x)
        reinterpret_cast<uint16_t*>(rowbuf)[i] = __ldg(reinterpret_cast<const uint16_t*>(src) + i);
    }
    __syncthreads();
    float a = 0.0f;
    for (int64_t c = threadIdx.x; c < nchunk; c += blockDim.x) {
      const uint8_t* blk = rowbuf + (c >> 1) * kQ80Bytes;
      const float d = __half2float(__ushort_as_half(static_cast<uint16_t>(blk[0] | (blk[1] << 8))));
      const uint8_t* codes = blk + 2 + (c & 1) * 16;
#pragma unroll
      for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(d * static_cast<float>(static_cast<int8_t>(codes[i]))));
    }
    a = block_max(a, red);
    const float s = (a < 1e-10f) ? 1e-10f : __fdiv_rn(a, 127.0f);
    if (threadIdx.x == 0) scale[n] = s;
    for (int64_t c = threadIdx.x; c < nchunk; c += blockDim.x) {
      const uint8_t* blk = rowbuf + (c >> 1) * kQ80Bytes;
      const float d = __half2float(__ushort_as_half(static_cast<uint16_t>(blk[0] | (blk[1] << 8))));
      const uint8_t* codes = blk + 2 + (c & 1) * 16;
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t acc = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const float deq = d * static_cast<float>(static_cast<int8_t>(codes[4 * i + b]));
          acc |= int8_code(__fdiv_rn(deq, s)) << (8 * b);
        }
        w[i] = acc;
      }
      *reinterpret_cast<uint4*>(q + n * K + c * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

}  // namespace w8a8
