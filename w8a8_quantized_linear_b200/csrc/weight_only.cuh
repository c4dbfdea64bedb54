// weight_only.cuh - the weight-only types of the OneTrainer wiki ("float8":
// tensor-wise e4m3 weights, and "GGUF"): the weight stays quantized in memory
// and is dequantized to the train data type (bf16) for each product, which
// then runs as a bf16 Linear on the tensor cores (gemm_pair_kernel /
// gemm_kernel with bf16 operands).  The GGUF dequantization is the Q8_0
// dequantizer with a bf16 output (q8_0.cuh).
#pragma once
#include "device.cuh"

namespace w8a8 {

// The e4m3 code in the top byte of `top` -> its value times 2^-120, exactly,
// without a conversion instruction: an arithmetic shift by 4 moves the
// exponent and mantissa bits (6..0 of the code) to fp32 bits 26..20 and
// copies the sign into bits 31..27; the mask keeps bit 31 and bits 26..20.
// The fp32 exponent field is then the code's 4-bit exponent e: for e > 0 the
// value is 2^(e-127) (1 + m/8) = 2^-120 * 2^(e-7) (1 + m/8), and for e = 0
// it is the fp32 subnormal m 2^-129 = 2^-120 * m 2^-9.  (The NaN codes
// 0x7F / 0xFF decode as a finite number; weight codes are never NaN.)
__device__ __forceinline__ float e4m3_top_byte_scaled(uint32_t top) {
  return __int_as_float((static_cast<int>(top) >> 4) & static_cast<int>(0x87F00000u));
}

// w[i] = bf16(e4m3_value(q[i]) * s): the value (exact, from the bits above
// times 2^120), one fp32 RN product with s, then bf16 RNE.  8 codes per
// thread and iteration: an 8-byte load and a 16-byte store, so that both
// are contiguous across the warp; n8 = n / 8.
__global__ void __launch_bounds__(256) dequant_e4m3_bf16_kernel(const uint2* __restrict__ q, int64_t n8,
                                                                const float* __restrict__ scale,
                                                                uint4* __restrict__ w) {
  griddep_launch();
  griddep_wait();   // the codes or the scale may be the previous kernel's output
  const float s = __ldg(scale);
  const float2 s2 = make_float2(s, s), up = make_float2(0x1p120f, 0x1p120f);
  for (int64_t i = blockIdx.x * 256ll + threadIdx.x; i < n8; i += static_cast<int64_t>(gridDim.x) * 256) {
    if (!in_bounds(i, n8, 0xB501)) break;
    const uint2 c = __ldg(q + i);
    const uint32_t cw[2] = {c.x, c.y};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float2 v01 = make_float2(e4m3_top_byte_scaled(cw[j] << 24), e4m3_top_byte_scaled(cw[j] << 16));
      const float2 v23 = make_float2(e4m3_top_byte_scaled(cw[j] << 8), e4m3_top_byte_scaled(cw[j]));
      const float2 a = __fmul2_rn(__fmul2_rn(v01, up), s2);   // the first product is exact
      const float2 b = __fmul2_rn(__fmul2_rn(v23, up), s2);
      o[2 * j] = pack_bf16x2(a.x, a.y);
      o[2 * j + 1] = pack_bf16x2(b.x, b.y);
    }
    w[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace w8a8
