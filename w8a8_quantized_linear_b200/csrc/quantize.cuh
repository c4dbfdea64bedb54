// quantize.cuh - token-wise absmax calibration + quantization in one pass
// (the fused row calibrate-and-quantize of bitsandbytes #1401), and the
// tensor-wise weight quantizer.  Bandwidth-bound: 16-byte coalesced loads and
// stores, packed bf16x2 absmax, warp-shuffle reductions, no tensor cores.
#pragma once
#include "device.cuh"

namespace w8a8 {

constexpr int kRowVecs = 8;   // 16-byte vectors per thread kept in registers

template <int QT>
__device__ __forceinline__ float qmax_of() { return QT == 1 ? 448.0f : 127.0f; }

// absmax scale with the 1e-10 floor, IEEE fp32 division.
template <int QT>
__device__ __forceinline__ float absmax_scale(float a) {
  return (a < 1e-10f) ? 1e-10f : __fdiv_rn(a, qmax_of<QT>());
}

// Exact codes of fl(v / s) without a division in the common case.
//
// rcp = fl(1/s) is correctly rounded, so t = fl(v * rcp) lies within
// 3.0001 ulp (relative to |v / s|) of fl(v / s).
//
// int8: t is rounded to the nearest integer, ties to even, by adding
// 1.5 * 2^23 (an fp32 add rounds exactly there for |t| < 2^22); the low byte
// of the sum's bit pattern is then the two's-complement code.  The remainder
// d = t - rne(t) is exact; when |d| < 0.5 - 2^-14 no rounding boundary lies
// within 2^-14 > 3.0001 ulp * 127.5 of t, so fl(v / s) rounds to the same
// integer.  |v / s| <= 127 (1 + 2^-23) with the absmax scale, so no clamp is
// reached.  A group of values with any |d| at the margin is recomputed with
// IEEE divisions (the rare slow path).
//
// e4m3: the codes of t * (1 - 2^-21) and t * (1 + 2^-21) - the ends of a
// +-8 ulp interval that contains fl(v / s) - are compared; e4m3 rounding with
// saturation is monotonic, so when they agree they are the code of fl(v / s).
constexpr float kRneMagic = 12582912.0f;            // 1.5 * 2^23
constexpr float kNearHalf = 0.49993896484375f;      // 0.5 - 2^-14

__device__ __forceinline__ uint32_t rne_low_byte(float t, bool& near) {
  const float big = __fadd_rn(t, kRneMagic);
  const float d = __fsub_rn(t, __fsub_rn(big, kRneMagic));
  near |= fabsf(d) > kNearHalf;
  return __float_as_uint(big) & 0xFFu;
}
__device__ __forceinline__ uint32_t int8_code_exact(float v, float s) {   // RNE, clamp +-127
  int q = __float2int_rn(__fdiv_rn(v, s));
  q = max(-127, min(127, q));
  return static_cast<uint32_t>(q) & 0xFFu;
}
__device__ __forceinline__ uint32_t e4m3_code_exact(float v, float s) {
  return static_cast<uint32_t>(cvt_e4m3x2(__fdiv_rn(v, s), 0.0f)) & 0xFFu;
}
__device__ __forceinline__ uint32_t e4m3_code_fast(float t, bool& near) {
  const uint32_t pair = cvt_e4m3x2(__fmul_rn(t, 1.0f - 0x1p-21f), __fmul_rn(t, 1.0f + 0x1p-21f));
  near |= (pair & 0xFFu) != (pair >> 8);
  return pair & 0xFFu;
}

// 8 values -> 8 codes (one uint2), fast path with one exactness flag.
template <int QT>
__device__ __forceinline__ uint2 encode8f(const float (&v)[8], float s, float rcp) {
  bool near = false;
  uint32_t c[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float t = __fmul_rn(v[i], rcp);
    c[i] = (QT == 1) ? e4m3_code_fast(t, near) : rne_low_byte(t, near);
  }
  if (near) {
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = (QT == 1) ? e4m3_code_exact(v[i], s) : int8_code_exact(v[i], s);
  }
  return make_uint2(c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24), c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24));
}

// 8 bf16 (one uint4) -> 8 codes (one uint2).
template <int QT>
__device__ __forceinline__ uint2 encode8(uint4 w, float s, float rcp) {
  const float v[8] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y),
                      bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w)};
  return encode8f<QT>(v, s, rcp);
}

// The exact codes of 8 bf16 by IEEE division: the rare path of encode8_fast,
// kept out of line so that the hot loops stay small.
template <int QT>
__device__ __noinline__ uint2 encode8_exact(uint4 w, float s) {
  const float v[8] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y),
                      bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w)};
  uint32_t c[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) c[i] = (QT == 1) ? e4m3_code_exact(v[i], s) : int8_code_exact(v[i], s);
  return make_uint2(c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24), c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24));
}

// The same codes, four fp32 operations per value.  int8: the exact product
// x * rcp is rounded once, to an integer, by fma(x, rcp, 1.5 * 2^23) (ties
// to even), and its exact remainder d = fma(x, rcp, -rne) is rounded once.
// x * rcp lies within 2 ulp of fl(x / s), so |d| < 0.5 - 2^-14 proves that
// fl(x / s) rounds to the same integer; a group with any |d| at the margin
// takes the exact division.  e4m3: as encode8 (interval ends compared).
template <int QT>
__device__ __forceinline__ uint2 encode8_fast(uint4 w, float s, float rcp) {
  const float v[8] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y),
                      bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w)};
  uint32_t c[8];
  bool near = false;
  if constexpr (QT == 1) {
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const float t0 = __fmul_rn(v[i], rcp), t1 = __fmul_rn(v[i + 1], rcp);
      const uint32_t ca = cvt_e4m3x2(__fmul_rn(t0, 1.0f - 0x1p-21f), __fmul_rn(t1, 1.0f - 0x1p-21f));
      const uint32_t cb = cvt_e4m3x2(__fmul_rn(t0, 1.0f + 0x1p-21f), __fmul_rn(t1, 1.0f + 0x1p-21f));
      near |= ca != cb;
      c[i] = ca & 0xFFu;
      c[i + 1] = ca >> 8;
    }
  } else {
    float dmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float big = __fmaf_rn(v[i], rcp, kRneMagic);
      const float d = __fmaf_rn(v[i], rcp, -__fsub_rn(big, kRneMagic));
      dmax = fmaxf(dmax, fabsf(d));
      c[i] = __float_as_uint(big);
    }
    near = dmax > kNearHalf;
  }
  if (near) return encode8_exact<QT>(w, s);
  return make_uint2(prmt(prmt(c[0], c[1], 0x0040u), prmt(c[2], c[3], 0x0040u), 0x5410u),
                    prmt(prmt(c[4], c[5], 0x0040u), prmt(c[6], c[7], 0x0040u), 0x5410u));
}

// Packed absmax of 8 bf16 (finite inputs).
__device__ __forceinline__ __nv_bfloat162 absmax8_bf2(uint4 v, __nv_bfloat162 m) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) m = __hmax2(m, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&w[i])));
  return m;
}
__device__ __forceinline__ float bf2_max(__nv_bfloat162 m) {
  return fmaxf(__bfloat162float(m.x), __bfloat162float(m.y));
}
__device__ __forceinline__ __nv_bfloat162 bf2_zero() { return __floats2bfloat162_rn(0.0f, 0.0f); }

// Block-wide max; every thread gets the result.  red: >= 32 floats of smem.
__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = (blockDim.x + 31) >> 5;
  if (nw == 1) return v;
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
    __nv_bfloat162 mb = bf2_zero();
#pragma unroll
    for (int j = 0; j < kRowVecs; ++j) {
      const int64_t v = threadIdx.x + static_cast<int64_t>(j) * blockDim.x;
      if (v < nv) {
        keep[j] = __ldg(row + v);
        mb = absmax8_bf2(keep[j], mb);
      }
    }
    for (int64_t v = threadIdx.x + static_cast<int64_t>(kRowVecs) * blockDim.x; v < nv; v += blockDim.x)
      mb = absmax8_bf2(__ldg(row + v), mb);
    const float a = block_max(bf2_max(mb), red);
    const float s = absmax_scale<QT>(a);
    const float rcp = __frcp_rn(s);
    if (threadIdx.x == 0) scale[m] = s;
    uint2* out = reinterpret_cast<uint2*>(q + m * ldq);
#pragma unroll
    for (int j = 0; j < kRowVecs; ++j) {
      const int64_t v = threadIdx.x + static_cast<int64_t>(j) * blockDim.x;
      if (v < nv) out[v] = encode8<QT>(keep[j], s, rcp);
    }
    for (int64_t v = threadIdx.x + static_cast<int64_t>(kRowVecs) * blockDim.x; v < nv; v += blockDim.x)
      out[v] = encode8<QT>(__ldg(row + v), s, rcp);
  }
}

// Rows of up to kTeamVecs * 32 * TW 16-byte vectors: a team of TW warps per
// row, every lane holding up to kTeamVecs vectors of the row in registers
// (one pass over HBM).  Teams reduce the absmax with warp shuffles and, for
// TW > 1, a per-team named barrier over double-buffered shared slots.
constexpr int kTeamVecs = 8;
template <int QT, int TW>
__global__ void __launch_bounds__(256, 4) quantize_rows_team_kernel(const __nv_bfloat16* __restrict__ x, int64_t ldx,
                                                                 int64_t M, int64_t K, uint8_t* __restrict__ q,
                                                                 int64_t ldq, float* __restrict__ scale) {
  __shared__ float red[2][8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int team = warp / TW, tw = warp % TW;
  const int teams = (blockDim.x >> 5) / TW;
  const int tl = tw * 32 + lane;
  const int nv = static_cast<int>(K >> 3);
  int iter = 0;
  for (int64_t m = blockIdx.x * static_cast<int64_t>(teams) + team; m < M;
       m += static_cast<int64_t>(gridDim.x) * teams, ++iter) {
    const uint4* row = reinterpret_cast<const uint4*>(x + m * ldx);
    uint4 keep[kTeamVecs];
#pragma unroll
    for (int j = 0; j < kTeamVecs; ++j) {
      const int v = tl + j * (32 * TW);
      if (v < nv) keep[j] = __ldg(row + v);
    }
    __nv_bfloat162 mb = bf2_zero();
#pragma unroll
    for (int j = 0; j < kTeamVecs; ++j)
      if (tl + j * (32 * TW) < nv) mb = absmax8_bf2(keep[j], mb);
    float a = bf2_max(mb);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
    if constexpr (TW > 1) {
      if (lane == 0) red[iter & 1][warp] = a;
      asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(32 * TW) : "memory");
#pragma unroll
      for (int i = 0; i < TW; ++i) a = fmaxf(a, red[iter & 1][team * TW + i]);
    }
    const float s = absmax_scale<QT>(a);
    const float rcp = __frcp_rn(s);
    if (tl == 0) scale[m] = s;
    uint2* out = reinterpret_cast<uint2*>(q + m * ldq);
#pragma unroll
    for (int j = 0; j < kTeamVecs; ++j) {
      const int v = tl + j * (32 * TW);
      if (v < nv) out[v] = encode8_fast<QT>(keep[j], s, rcp);
    }
  }
}

// Tensor-wise weight quantization, pass 1: global absmax of W (as the bit
// pattern of a non-negative float, so an unsigned atomicMax orders it).
__global__ void __launch_bounds__(256) absmax_kernel(const uint4* __restrict__ w, int64_t nvec,
                                                     unsigned* __restrict__ amax_bits) {
  __shared__ float red[32];
  __nv_bfloat162 mb = bf2_zero();
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nvec;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    mb = absmax8_bf2(__ldg(w + i), mb);
  const float a = block_max(bf2_max(mb), red);
  if (threadIdx.x == 0) atomicMax(amax_bits, __float_as_uint(a));
}

// Pass 2: one scale for the whole tensor, codes for every element.
template <int QT>
__global__ void __launch_bounds__(256) quantize_tensor_kernel(const uint4* __restrict__ w, int64_t nvec,
                                                              const unsigned* __restrict__ amax_bits,
                                                              uint2* __restrict__ q, float* __restrict__ scale) {
  const float s = absmax_scale<QT>(__uint_as_float(*amax_bits));
  const float rcp = __frcp_rn(s);
  if (blockIdx.x == 0 && threadIdx.x == 0) scale[0] = s;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nvec;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    q[i] = encode8_fast<QT>(__ldg(w + i), s, rcp);
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
