// Exhaustive check of the refined quotient of the Q8_0 -> axis-wise
// re-quantization (q8_0.cuh, rq_block_codes): every value x = d q a Q8_0
// block can hold (f16 scale d, int8 code q: significand md * odd q with md in
// [1024, 2048) and odd q in [1, 127]; q = +-128 and even q share those
// significands) against every scale s = fl(a / QMAX) such values give (a of
// the same form) and the 1e-10 floor.  QMAX is the first argument: 127 (int8
// codes; binades holding x / s in [2^-3, 2^8)) or 448 (e4m3 codes; binades
// holding x / s in [2^-12, 2^9)).  With y = fl(1/s):
//     q0 = fl(x y),  r = fl(x - q0 s) (fma),  q1 = fl(q0 + r y) (fma)
// must equal fl(x / s), and so must the int8 code (RNE) and the e4m3 code
// (RNE-satfinite) taken from either.  Prints one line; exit 0 iff no mismatch.
#include <cstdint>
#include <cstdio>
#include <cuda_runtime.h>

#include <cstdlib>

__device__ unsigned long long g_bad_q = 0, g_bad_i8 = 0, g_bad_e4 = 0, g_checked = 0;

__device__ __forceinline__ unsigned e4m3_code(float v) {
  unsigned short c;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c) : "f"(0.0f), "f"(v));
  return c & 0xFFu;
}

__device__ __forceinline__ float norm1(float p) {   // a positive normal float scaled into [1, 2)
  return __uint_as_float((__float_as_uint(p) & 0x7FFFFFu) | 0x3F800000u);
}
__device__ __forceinline__ float product_significand(unsigned i) {   // i in [0, 65536)
  const unsigned md = 1024 + (i >> 6), oq = 2 * (i & 63) + 1;
  return norm1(static_cast<float>(md * oq));
}

__global__ void check(unsigned xbase, unsigned xcount, float qmax, int e_lo, int e_hi) {
  const unsigned si = blockIdx.x * blockDim.x + threadIdx.x;
  if (si > 65536) return;
  const float s = si == 65536 ? norm1(1e-10f) : norm1(__fdiv_rn(product_significand(si), qmax));
  const float y = __frcp_rn(s);
  unsigned long long bq = 0, bi = 0, be = 0, n = 0;
  for (unsigned xi = xbase; xi < xbase + xcount; ++xi) {
    const float p = product_significand(xi);
    for (int e = e_lo; e <= e_hi; ++e) {
      const float x = __fmul_rn(p, __uint_as_float(static_cast<unsigned>(127 + e) << 23));
      const float q0 = __fmul_rn(x, y);
      const float r = __fmaf_rn(-q0, s, x);
      const float q1 = __fmaf_rn(r, y, q0);
      const float qd = __fdiv_rn(x, s);
      ++n;
      bq += __float_as_uint(q1) != __float_as_uint(qd);
      bi += __float2int_rn(q1) != __float2int_rn(qd);
      be += e4m3_code(q1) != e4m3_code(qd);
    }
  }
  atomicAdd(&g_bad_q, bq);
  atomicAdd(&g_bad_i8, bi);
  atomicAdd(&g_bad_e4, be);
  atomicAdd(&g_checked, n);
}

int main(int argc, char** argv) {
  const int qmax = argc > 1 ? atoi(argv[1]) : 127;
  if (qmax != 127 && qmax != 448) {
    printf("QMAX must be 127 or 448\n");
    return 1;
  }
  const int e_lo = qmax == 127 ? -3 : -11, e_hi = qmax == 127 ? 7 : 8;
  for (unsigned x = 0; x < 65536; x += 4096) {
    check<<<(65537 + 255) / 256, 256>>>(x, 4096, static_cast<float>(qmax), e_lo, e_hi);
    const cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
      printf("CUDA error: %s\n", cudaGetErrorString(e));
      return 1;
    }
  }
  unsigned long long bq = 0, bi = 0, be = 0, n = 0;
  cudaMemcpyFromSymbol(&bq, g_bad_q, sizeof(bq));
  cudaMemcpyFromSymbol(&bi, g_bad_i8, sizeof(bi));
  cudaMemcpyFromSymbol(&be, g_bad_e4, sizeof(be));
  cudaMemcpyFromSymbol(&n, g_checked, sizeof(n));
  printf("checked %llu (s, x) pairs with QMAX %d: quotient mismatches %llu, int8 code mismatches %llu, "
         "e4m3 code mismatches %llu\n", n, qmax, bq, bi, be);
  return (bq || bi || be) ? 2 : 0;
}
