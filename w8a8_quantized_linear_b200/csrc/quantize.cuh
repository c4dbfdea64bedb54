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

// Exact codes of fl(v / s) without a division and without a data-dependent
// branch.  With y = fl(1/s) (correctly rounded), the quotient is refined
// once (Markstein's correction step, P. Markstein, IBM J. Res. Dev. 34(1),
// 1990):
//     q0 = fl(v y),   r = fl(v - q0 s)  (one fma),   q1 = fl(q0 + r y)  (one fma)
// and q1 is the IEEE quotient fl(v / s) for every bf16 v: checked
// exhaustively on the GPU for every fp32 significand of s against every bf16
// significand of v over the 23 binades that hold |v / s| in [2^-13, 2^11)
// (tests/quotient_check.cu); the codes are invariant under scaling v and s by
// the same power of two, and smaller quotients give code 0 either way.
//   int8: fl(q1 + 1.5 * 2^23) rounds q1 to the nearest integer, ties to even
//         (an fp32 sum in [2^23, 2^24) has unit spacing); the low byte of its
//         bit pattern is the two's-complement code.  |v / s| <= 127 (1 +
//         2^-23) with the absmax scale, so no clamp is reached.
//   e4m3: the quotient goes through the RNE-satfinite conversion; its sign is
//         v's (fl(-0 / s) = -0 has code 0x80).
// Every step is an fp32 operation on pairs (the f32x2 forms of sm_100).
constexpr float kRneMagic = 12582912.0f;            // 1.5 * 2^23
constexpr float kNearHalf = 0.49993896484375f;      // 0.5 - 2^-14

// Remainder form of a division-free int8 rounding, for the Q8_0 quantizer
// (whose inputs are fp32, not bf16): t = fl(v * fl(1/s)) lies within 3.0001 ulp of
// fl(v / s); d = t - rne(t) is exact, and |d| < 0.5 - 2^-14 puts no rounding
// boundary between them, so the integer is right; otherwise `near` is set
// and the caller takes the IEEE division.
__device__ __forceinline__ uint32_t rne_low_byte(float t, bool& near) {
  const float big = __fadd_rn(t, kRneMagic);
  const float d = __fsub_rn(t, __fsub_rn(big, kRneMagic));
  near |= fabsf(d) > kNearHalf;
  return __float_as_uint(big) & 0xFFu;
}

// 8 bf16 (one uint4) -> 8 codes (one uint2); y = fl(1/s).
template <int QT>
__device__ __forceinline__ uint2 encode8(uint4 w, float s, float y) {
  const float2 v[4] = {make_float2(bf16_lo(w.x), bf16_hi(w.x)), make_float2(bf16_lo(w.y), bf16_hi(w.y)),
                       make_float2(bf16_lo(w.z), bf16_hi(w.z)), make_float2(bf16_lo(w.w), bf16_hi(w.w))};
  const float2 y2 = make_float2(y, y), ns2 = make_float2(-s, -s);
  float2 q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 q0 = __fmul2_rn(v[i], y2);
    const float2 r = __ffma2_rn(q0, ns2, v[i]);
    q[i] = __ffma2_rn(r, y2, q0);
  }
  if constexpr (QT == 1) {
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float lo = __uint_as_float((__float_as_uint(q[i].x) & 0x7FFFFFFFu) | (__float_as_uint(v[i].x) & 0x80000000u));
      const float hi = __uint_as_float((__float_as_uint(q[i].y) & 0x7FFFFFFFu) | (__float_as_uint(v[i].y) & 0x80000000u));
      c[i] = cvt_e4m3x2(lo, hi);
    }
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
  } else {
    const float2 mg = make_float2(kRneMagic, kRneMagic);
    uint32_t c[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 b = __fadd2_rn(q[i], mg);
      c[2 * i] = __float_as_uint(b.x);
      c[2 * i + 1] = __float_as_uint(b.y);
    }
    return make_uint2(prmt(prmt(c[0], c[1], 0x0040u), prmt(c[2], c[3], 0x0040u), 0x5410u),
                      prmt(prmt(c[4], c[5], 0x0040u), prmt(c[6], c[7], 0x0040u), 0x5410u));
  }
}

// Running absmax of packed bf16 pairs: max(|m|, |v|) per half (the sign bit
// of the result is junk; bf2_absmax_final clears it).  Finite inputs.
__device__ __forceinline__ uint32_t bf2_absmax(uint32_t m, uint32_t v) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(m), "r"(v));
  return d;
}
__device__ __forceinline__ uint32_t absmax8(uint4 v, uint32_t m) {
  return bf2_absmax(bf2_absmax(bf2_absmax(bf2_absmax(m, v.x), v.y), v.z), v.w);
}
__device__ __forceinline__ float bf2_absmax_final(uint32_t m) {
  return fmaxf(fabsf(bf16_lo(m)), fabsf(bf16_hi(m)));
}

// Optional side jobs of the row quantizers in a fused chain of Linears (the
// CHAIN instantiations; the others carry no code for them):
// zero_out [zero_n] is cleared (the next projection's row-absmax buffer, which
// its GEMM epilogue fills with atomicMax after this kernel has completed), and
// amax_in, when given, holds each row's absmax as fp32 bits (written by the
// producing GEMM's epilogue), so the row needs no reduction.
__device__ __forceinline__ void clear_words(uint32_t* zero_out, int64_t zero_n) {
  if (zero_out == nullptr) return;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < zero_n; i += stride)
    if (in_bounds(i, zero_n, 0xB006)) zero_out[i] = 0u;
}

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
template <int QT, bool CHAIN = false>
__global__ void __launch_bounds__(1024) quantize_rows_kernel(const __nv_bfloat16* __restrict__ x, int64_t ldx,
                                                             int64_t M, int64_t K, uint8_t* __restrict__ q,
                                                             int64_t ldq, float* __restrict__ scale,
                                                             const uint32_t* __restrict__ amax_in = nullptr,
                                                             uint32_t* __restrict__ zero_out = nullptr,
                                                             int64_t zero_n = 0) {
  __shared__ float red[32];
  // Wait first, then let the next kernel launch: a GEMM launched after this
  // quantizer may read its weight before its own wait, and that is safe only
  // once every kernel before this one (a weight producer among them) has
  // completed.
  griddep_wait();   // x may be the previous kernel's output
  griddep_launch();
  if constexpr (CHAIN) clear_words(zero_out, zero_n);
  const int64_t nv = K >> 3;
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    if (!in_bounds(m, M, 0xB001)) break;
    const uint4* row = reinterpret_cast<const uint4*>(x + m * ldx);
    uint4 keep[kRowVecs];
    uint32_t mb = 0;
#pragma unroll
    for (int j = 0; j < kRowVecs; ++j) {
      const int64_t v = threadIdx.x + static_cast<int64_t>(j) * blockDim.x;
      if (v < nv && in_bounds(v, nv, 0xB002)) {
        keep[j] = __ldg(row + v);
        mb = absmax8(keep[j], mb);
      }
    }
    for (int64_t v = threadIdx.x + static_cast<int64_t>(kRowVecs) * blockDim.x; v < nv; v += blockDim.x)
      if (in_bounds(v, nv, 0xB002)) mb = absmax8(__ldg(row + v), mb);
    const float a = (CHAIN && amax_in != nullptr) ? __uint_as_float(amax_in[m]) : block_max(bf2_absmax_final(mb), red);
    const float s = absmax_scale<QT>(a);
    const float rcp = __frcp_rn(s);
    if (threadIdx.x == 0) scale[m] = s;
    uint2* out = reinterpret_cast<uint2*>(q + m * ldq);
#pragma unroll
    for (int j = 0; j < kRowVecs; ++j) {
      const int64_t v = threadIdx.x + static_cast<int64_t>(j) * blockDim.x;
      if (v < nv && in_bounds(v, nv, 0xB002)) out[v] = encode8<QT>(keep[j], s, rcp);
    }
    for (int64_t v = threadIdx.x + static_cast<int64_t>(kRowVecs) * blockDim.x; v < nv; v += blockDim.x)
      if (in_bounds(v, nv, 0xB002)) out[v] = encode8<QT>(__ldg(row + v), s, rcp);
  }
}

// Rows of up to kTeamVecs * 32 * TW 16-byte vectors: a team of TW warps per
// row, every lane holding up to kTeamVecs vectors of the row in registers
// (one pass over HBM).  Teams reduce the absmax with warp shuffles and, for
// TW > 1, a per-team named barrier over double-buffered shared slots.
constexpr int kTeamVecs = 8;
template <int QT, int TW, bool CHAIN = false>
__global__ void __launch_bounds__(256, 4) quantize_rows_team_kernel(const __nv_bfloat16* __restrict__ x, int64_t ldx,
                                                                 int64_t M, int64_t K, uint8_t* __restrict__ q,
                                                                 int64_t ldq, float* __restrict__ scale,
                                                                 const uint32_t* __restrict__ amax_in = nullptr,
                                                                 uint32_t* __restrict__ zero_out = nullptr,
                                                                 int64_t zero_n = 0) {
  __shared__ float red[2][8];
  // Wait first, then let the next kernel launch: a GEMM launched after this
  // quantizer may read its weight before its own wait, and that is safe only
  // once every kernel before this one (a weight producer among them) has
  // completed.
  griddep_wait();   // x may be the previous kernel's output
  griddep_launch();
  if constexpr (CHAIN) clear_words(zero_out, zero_n);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int team = warp / TW, tw = warp % TW;
  const int teams = (blockDim.x >> 5) / TW;
  const int tl = tw * 32 + lane;
  const int nv = static_cast<int>(K >> 3);
  int iter = 0;
  for (int64_t m = blockIdx.x * static_cast<int64_t>(teams) + team; m < M;
       m += static_cast<int64_t>(gridDim.x) * teams, ++iter) {
    const bool row_ok = in_bounds(m, M, 0xB003);   // (a team-uniform test: no early exit before the barrier)
    const uint4* row = reinterpret_cast<const uint4*>(x + m * ldx);
    uint4 keep[kTeamVecs];
#pragma unroll
    for (int j = 0; j < kTeamVecs; ++j) {
      const int v = tl + j * (32 * TW);
      if (row_ok && v < nv && in_bounds(v, nv, 0xB004)) keep[j] = __ldg(row + v);
    }
    float a;
    if (CHAIN && amax_in != nullptr) {   // uniform over the kernel
      a = row_ok ? __uint_as_float(amax_in[m]) : 0.0f;
    } else {
      uint32_t mb = 0;
#pragma unroll
      for (int j = 0; j < kTeamVecs; ++j)
        if (tl + j * (32 * TW) < nv) mb = absmax8(keep[j], mb);
      a = bf2_absmax_final(mb);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
      if constexpr (TW > 1) {
        if (lane == 0) red[iter & 1][warp] = a;
        asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(32 * TW) : "memory");
#pragma unroll
        for (int i = 0; i < TW; ++i) a = fmaxf(a, red[iter & 1][team * TW + i]);
      }
    }
    const float s = absmax_scale<QT>(a);
    const float rcp = __frcp_rn(s);
    if (row_ok && tl == 0) scale[m] = s;
    uint2* out = reinterpret_cast<uint2*>(q + m * ldq);
#pragma unroll
    for (int j = 0; j < kTeamVecs; ++j) {
      const int v = tl + j * (32 * TW);
      if (row_ok && v < nv) out[v] = encode8<QT>(keep[j], s, rcp);
    }
  }
}

// 16-byte read-only loads with an L2 eviction priority (an L2 cache policy
// from createpolicy): the tensor-wise quantizer reads W twice, and marks
// its first pass's lines to stay in L2 and its second pass's to go first.
__device__ __forceinline__ uint4 ldg_policy(const uint4* p, uint64_t policy) {
  uint4 v;
  asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(policy));
  return v;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Tensor-wise weight quantization, pass 1: global absmax of W (as the bit
// pattern of a non-negative float, so an unsigned atomicMax orders it).
__global__ void __launch_bounds__(256) absmax_kernel(const uint4* __restrict__ w, int64_t nvec,
                                                     unsigned* __restrict__ amax_bits) {
  __shared__ float red[32];
  uint32_t mb = 0;
  const uint64_t keep = policy_evict_last();   // pass 2 reads W again
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nvec;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    if (in_bounds(i, nvec, 0xB005)) mb = absmax8(ldg_policy(w + i, keep), mb);
  const float a = block_max(bf2_absmax_final(mb), red);
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
  const uint64_t drop = policy_evict_first();   // W's last read
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nvec;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    if (in_bounds(i, nvec, 0xB005)) q[i] = encode8<QT>(ldg_policy(w + i, drop), s, rcp);
}

// fp32 -> E4M3FN codes with the quantizers' conversion.
__global__ void e4m3_encode_kernel(const float* __restrict__ x, int64_t n, uint8_t* __restrict__ y) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    y[i] = static_cast<uint8_t>(cvt_e4m3x2(x[i], 0.0f) & 0xFFu);
}

// Index-check self test: a check one past the end of an extent (no memory
// is touched): the debug build records kDevBounds at site 0xBFFF.
__global__ void selftest_bounds_kernel(int64_t extent) {
  if (!in_bounds(extent, extent, 0xBFFFu)) return;
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
