// Exhaustive check of the division-free quotient of the row quantizers
// (quantize.cuh, encode8): with y = fl(1/s),
//     q0 = fl(v y),  r = fl(v - q0 s) (fma),  q1 = fl(q0 + r y) (fma)
// must equal the IEEE quotient fl(v / s).  s runs over every fp32
// significand in [1, 2); v over every bf16 significand in each of the 23
// binades [2^-12, 2^11), i.e. every quotient the int8 (|v/s| <= 127) and
// e4m3 (|v/s| <= 448) codes depend on; scaling v and s by one power of two
// changes nothing away from under/overflow.  The int8 and e4m3 codes of q1
// and of fl(v / s) are compared as well.  Prints one line; exit 0 iff no
// mismatch.
#include <cstdint>
#include <cstdio>
#include <cuda_runtime.h>

__device__ unsigned long long g_bad_q = 0, g_bad_i8 = 0, g_bad_e4 = 0, g_checked = 0;

__device__ __forceinline__ unsigned e4m3_code(float x) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xFFu;
}

__global__ void check(unsigned base) {
  const unsigned ms = base + blockIdx.x * blockDim.x + threadIdx.x;
  if (ms >= (1u << 23)) return;
  const float s = __uint_as_float(0x3F800000u | ms);
  const float y = __frcp_rn(s);
  unsigned long long bq = 0, bi = 0, be = 0, n = 0;
  for (int e = -12; e <= 10; ++e) {
    for (unsigned mv = 0; mv < 128; ++mv) {
      const float v = __uint_as_float((static_cast<unsigned>(127 + e) << 23) | (mv << 16));
      const float q0 = __fmul_rn(v, y);
      const float r = __fmaf_rn(-q0, s, v);
      const float q1 = __fmaf_rn(r, y, q0);
      const float qd = __fdiv_rn(v, s);
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

int main() {
  for (unsigned base = 0; base < (1u << 23); base += (1u << 20)) {
    check<<<(1u << 20) / 256, 256>>>(base);
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
  printf("checked %llu (s, v) pairs: quotient mismatches %llu, int8 code mismatches %llu, e4m3 code mismatches %llu\n",
         n, bq, bi, be);
  return (bq || bi || be) ? 2 : 0;
}
