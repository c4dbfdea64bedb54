// q8_0.cuh - GGUF Q8_0 blocks (32 values -> f16 scale + 32 int8 codes =
// 34 bytes; entrenar 0.7.8 q8_0.rs) on the GPU, and the re-quantization of a
// Q8_0 weight to axis-wise int8 or e4m3 codes (OneTrainer wiki, GGUF A8 int
// and GGUF A8 float).  QT selects the target: 0 int8 (QMAX 127), 1 e4m3
// (QMAX 448).
//
// A 34-byte block is not 16-byte aligned, but 8 blocks are 272 = 17 * 16
// bytes.  A warp handles kQ80Unroll such groups of 8 blocks per iteration
// (1 KB of fp32 per group), with 16-byte global accesses on the block side
// staged through shared memory.
#pragma once
#include "device.cuh"
#include "quantize.cuh"

namespace w8a8 {

constexpr int kQ80Block = 32;
constexpr int kQ80Bytes = 34;
constexpr int kQ80Group = 8 * kQ80Bytes;          // 272 bytes = 17 x 16
constexpr int kQ80Unroll = 4;                     // groups per warp iteration
constexpr int kQ80Chunk = kQ80Unroll * kQ80Group; // 1088 bytes = 68 x 16
constexpr int kQ80WarpsPerBlock = 8;

// Q8_0 code of fl(v / scale): round half away from zero, clamp to [-128, 127]
// (Q8_0::quantize).  Fast path as for the W8A8 int8 codes (rne_low_byte):
// away from a tie half-away and half-even agree, and |v / scale| <= 127
// (1 + 2^-23) never reaches the clamp; groups with a value at the margin take
// the exact division with roundf.
__device__ __forceinline__ uint32_t q80_code_exact(float v, float scale) {
  const float r = fminf(fmaxf(roundf(__fdiv_rn(v, scale)), -128.0f), 127.0f);
  return static_cast<uint32_t>(static_cast<int>(r)) & 0xFFu;
}

// Quantize.  In group u of an iteration, lane l holds values [8l, 8l+8), so
// block j of the group lives in lanes 4j..4j+3.
__global__ void __launch_bounds__(256) q8_0_quantize_kernel(const float* __restrict__ x, int64_t n,
                                                            uint8_t* __restrict__ blocks) {
  __shared__ __align__(16) uint8_t stage[kQ80WarpsPerBlock][kQ80Chunk];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* st = stage[warp];
  const int64_t nchunks = (n + 256 * kQ80Unroll - 1) / (256 * kQ80Unroll);
  const int64_t nbytes = ((n + 31) / 32) * kQ80Bytes;
  for (int64_t c = blockIdx.x * static_cast<int64_t>(kQ80WarpsPerBlock) + warp; c < nchunks;
       c += static_cast<int64_t>(gridDim.x) * kQ80WarpsPerBlock) {
    float v[kQ80Unroll][8];
#pragma unroll
    for (int u = 0; u < kQ80Unroll; ++u) {
      const int64_t base = (c * kQ80Unroll + u) * 256 + lane * 8;
      if (base + 8 <= n && in_bounds(base + 7, n, 0xB401)) {
        const float4 p0 = __ldg(reinterpret_cast<const float4*>(x + base));
        const float4 p1 = __ldg(reinterpret_cast<const float4*>(x + base) + 1);
        v[u][0] = p0.x; v[u][1] = p0.y; v[u][2] = p0.z; v[u][3] = p0.w;
        v[u][4] = p1.x; v[u][5] = p1.y; v[u][6] = p1.z; v[u][7] = p1.w;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[u][i] = (base + i < n) ? x[base + i] : 0.0f;   // zero padding
      }
    }
    const int j = lane >> 2, part = lane & 3;
#pragma unroll
    for (int u = 0; u < kQ80Unroll; ++u) {
      float a = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[u][i]));
      a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 1));
      a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 2));
      const float scale = (a < 1e-10f) ? 1e-10f : __fdiv_rn(a, 127.0f);
      const float rcp = __frcp_rn(scale);
      uint16_t* blk = reinterpret_cast<uint16_t*>(st + u * kQ80Group + j * kQ80Bytes);   // 2-byte aligned
      if (part == 0) blk[0] = __half_as_ushort(__float2half_rn(scale));
      bool near = false;
      uint32_t c[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) c[i] = rne_low_byte(__fmul_rn(v[u][i], rcp), near);
      if (near) {
#pragma unroll
        for (int i = 0; i < 8; ++i) c[i] = q80_code_exact(v[u][i], scale);
      }
#pragma unroll
      for (int i = 0; i < 8; i += 2) blk[1 + part * 4 + i / 2] = static_cast<uint16_t>(c[i] | (c[i + 1] << 8));
    }
    __syncwarp();
    for (int i = lane; i < kQ80Chunk / 16; i += 32) {
      const int64_t off = c * kQ80Chunk + i * 16;
      if (off + 16 <= nbytes && in_bounds(off + 15, nbytes, 0xB401)) {
        *reinterpret_cast<uint4*>(blocks + off) = *reinterpret_cast<const uint4*>(st + i * 16);
      } else {
        for (int b = 0; b < 16; ++b)
          if (off + b < nbytes) blocks[off + b] = st[i * 16 + b];
      }
    }
    __syncwarp();
  }
}

// Dequantize: kQ80Unroll groups copied to shared memory with 16-byte loads,
// then in group u lane l writes values [8l, 8l+8) = f16 scale * code (exact
// in fp32).  BF16: the values rounded to bf16 (RNE), for the GGUF weight
// dequantized to the train data type (OneTrainer wiki, GGUF).
template <bool BF16>
__global__ void __launch_bounds__(256) q8_0_dequantize_kernel(const uint8_t* __restrict__ blocks, int64_t n,
                                                              void* __restrict__ yv) {
  griddep_launch();
  griddep_wait();   // the blocks may be the previous kernel's output, y its input
  __shared__ __align__(16) uint8_t stage[kQ80WarpsPerBlock][kQ80Chunk];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* st = stage[warp];
  const int64_t nchunks = (n + 256 * kQ80Unroll - 1) / (256 * kQ80Unroll);
  const int64_t nbytes = ((n + 31) / 32) * kQ80Bytes;
  for (int64_t c = blockIdx.x * static_cast<int64_t>(kQ80WarpsPerBlock) + warp; c < nchunks;
       c += static_cast<int64_t>(gridDim.x) * kQ80WarpsPerBlock) {
    for (int i = lane; i < kQ80Chunk / 16; i += 32) {
      const int64_t off = c * kQ80Chunk + i * 16;
      if (off + 16 <= nbytes && in_bounds(off + 15, nbytes, 0xB402)) {
        *reinterpret_cast<uint4*>(st + i * 16) = __ldg(reinterpret_cast<const uint4*>(blocks + off));
      } else {
        for (int b = 0; b < 16; ++b) st[i * 16 + b] = (off + b < nbytes) ? blocks[off + b] : 0;
      }
    }
    __syncwarp();
    const int j = lane >> 2, part = lane & 3;
#pragma unroll
    for (int u = 0; u < kQ80Unroll; ++u) {
      const uint16_t* blk = reinterpret_cast<const uint16_t*>(st + u * kQ80Group + j * kQ80Bytes);
      const float d = __half2float(__ushort_as_half(blk[0]));
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const uint16_t pair = blk[1 + part * 4 + i / 2];
        v[i] = d * static_cast<float>(static_cast<int8_t>(pair & 0xFF));
        v[i + 1] = d * static_cast<float>(static_cast<int8_t>(pair >> 8));
      }
      const int64_t base = (c * kQ80Unroll + u) * 256 + lane * 8;
      if constexpr (BF16) {
        __nv_bfloat16* y = static_cast<__nv_bfloat16*>(yv);
        if (base + 8 <= n && in_bounds(base + 7, n, 0xB402)) {
          *reinterpret_cast<uint4*>(y + base) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                                           pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (base + i < n) y[base + i] = __float2bfloat16_rn(v[i]);
        }
      } else {
        float* y = static_cast<float*>(yv);
        if (base + 8 <= n && in_bounds(base + 7, n, 0xB402)) {
          float4* o = reinterpret_cast<float4*>(y + base);
          o[0] = make_float4(v[0], v[1], v[2], v[3]);
          o[1] = make_float4(v[4], v[5], v[6], v[7]);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (base + i < n) y[base + i] = v[i];
        }
      }
    }
    __syncwarp();
  }
}

// Code of one dequantized value x = d q for the scale s (y = fl(1/s)), with
// the refined quotient of rq_block_codes below (exact for every value a Q8_0
// block can hold and every scale such values give).
template <int QT>
__device__ __forceinline__ uint32_t rq_code(float x, float s, float y) {
  const float q0 = __fmul_rn(x, y);
  const float q1 = __fmaf_rn(__fmaf_rn(-q0, s, x), y, q0);
  if constexpr (QT == 1) {
    const float v = __uint_as_float((__float_as_uint(q1) & 0x7FFFFFFFu) | (__float_as_uint(x) & 0x80000000u));
    return cvt_e4m3x2(v, 0.0f) & 0xFFu;
  } else {
    return __float_as_uint(__fadd_rn(q1, kRneMagic)) & 0xFFu;
  }
}

// Q8_0 [N, K/32 blocks] -> codes [N, K] + s [N]: one warp per weight row, for
// any K % 32 == 0.  The row's K/32 * 34 bytes are staged in the warp's shared
// memory; lane l takes blocks l, l+32, ...  Each value is dequantized exactly
// (f16 scale * code is exact in fp32), the row absmax gives s, and each value
// gets its code from rq_code.
constexpr int kRequantMaxWarps = 4;
template <int QT>
__global__ void __launch_bounds__(32 * kRequantMaxWarps) q8_0_to_axis_warp_kernel(const uint8_t* __restrict__ blocks,
                                                                               int64_t N, int64_t K,
                                                                               uint8_t* __restrict__ q,
                                                                               float* __restrict__ scale) {
  extern __shared__ __align__(16) uint8_t rowbuf_all[];
  griddep_launch();
  griddep_wait();   // the blocks may be the previous kernel's output, q and scale its input
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const int64_t nblk = K / kQ80Block;
  const int64_t row_bytes = nblk * kQ80Bytes;
  const int64_t row_stride = (row_bytes + 15) & ~int64_t(15);
  uint8_t* rowbuf = rowbuf_all + warp * row_stride;
  for (int64_t n = blockIdx.x * static_cast<int64_t>(nwarps) + warp; n < N;
       n += static_cast<int64_t>(gridDim.x) * nwarps) {
    if (!in_bounds(n, N, 0xB403)) break;   // warp-uniform
    const uint8_t* src = blocks + n * row_bytes;
    if (((reinterpret_cast<uintptr_t>(src) | static_cast<uintptr_t>(row_bytes)) & 15) == 0) {
      for (int64_t i = lane; i < row_bytes / 16; i += 32)
        reinterpret_cast<uint4*>(rowbuf)[i] = __ldg(reinterpret_cast<const uint4*>(src) + i);
    } else {   // rows always start on an even byte: 2-byte copies
      for (int64_t i = lane; i < row_bytes / 2; i += 32)
        reinterpret_cast<uint16_t*>(rowbuf)[i] = __ldg(reinterpret_cast<const uint16_t*>(src) + i);
    }
    __syncwarp();
    float a = 0.0f;
    for (int64_t b = lane; b < nblk; b += 32) {
      const uint16_t* blk = reinterpret_cast<const uint16_t*>(rowbuf + b * kQ80Bytes);
      const float d = fabsf(__half2float(__ushort_as_half(blk[0])));
      int cmax = 0;
#pragma unroll
      for (int i = 1; i <= 16; ++i) {
        const int pr = blk[i];
        cmax = max(cmax, max(abs(static_cast<int>(static_cast<int8_t>(pr & 0xFF))),
                             abs(static_cast<int>(static_cast<int8_t>(pr >> 8)))));
      }
      a = fmaxf(a, d * static_cast<float>(cmax));   // max |d * q| = |d| * max |q| (exact products)
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
    const float s = absmax_scale<QT>(a);
    const float rcp = __frcp_rn(s);
    if (lane == 0) scale[n] = s;
    for (int64_t b = lane; b < nblk; b += 32) {
      const uint16_t* blk = reinterpret_cast<const uint16_t*>(rowbuf + b * kQ80Bytes);
      const float d = __half2float(__ushort_as_half(blk[0]));
      uint32_t w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t p0 = blk[1 + 2 * i], p1 = blk[2 + 2 * i];
        uint32_t c = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int qv = static_cast<int8_t>(((j < 2 ? p0 : p1) >> (8 * (j & 1))) & 0xFFu);
          c |= rq_code<QT>(__fmul_rn(d, static_cast<float>(qv)), s, rcp) << (8 * j);
        }
        w[i] = c;
      }
      uint4* out = reinterpret_cast<uint4*>(q + n * K + b * kQ80Block);
      if (!in_bounds(n * K + b * kQ80Block + 31, N * K, 0xB404)) continue;
      out[0] = make_uint4(w[0], w[1], w[2], w[3]);
      out[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
    __syncwarp();
  }
}

// ----------------------------------------------------------------------------
// Q8_0 -> axis-wise codes for rows whose blocks fill whole 16-byte units
// (K % 256 == 0): a team of TW warps per row, thread t of the team taking
// blocks t, t + 32 TW, ...  Each team keeps its next S - 1 rows in flight
// into a ring of S shared-memory row buffers (cp.async) while it processes
// the current one; with S = 1 a row is loaded just before its turn and the
// other teams on the SM (up to 8 blocks) hide the latency.
//
// A block b starts at byte 34 b of the row, i.e. on a word boundary when b is
// even and 2 bytes past one when b is odd; its 34 bytes lie in the 9 words
// from word floor(34 b / 4), and prmt selects the f16 scale and the 32 codes
// from them.  Pass 1 takes max |q| of each block on sign-extended 16-bit
// pairs (max/min.s16x2); max |d q| = |d| max |q| exactly.  Pass 2 forms
// the codes with the refined quotient of rq_block_codes (no division, no
// data-dependent branch).
// ----------------------------------------------------------------------------
constexpr int kRqThreads = 256;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ uint32_t vmax_s16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.s16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t vmin_s16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("min.s16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

template <int TW>
__device__ __forceinline__ void team_sync(int team) {
  if constexpr (TW == 1) {
    __syncwarp();
  } else {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(32 * TW) : "memory");
  }
}

// The 9 words holding block b of a staged row.
__device__ __forceinline__ void rq_block_words(const uint8_t* row, int b, uint32_t (&w)[9]) {
  const uint32_t* p = reinterpret_cast<const uint32_t*>(row) + ((17 * b) >> 1);
#pragma unroll
  for (int i = 0; i < 9; ++i) w[i] = p[i];
}

// max |q| over the 32 codes of a block.  The codes fill words 1..8 of an odd
// block; for an even block they are the last two bytes of word 0, words
// 1..7 and the first two bytes of word 8, and one prmt joins the two halves.
// In a word [B3 B2 B1 B0] read as two signed 16-bit lanes, lane i is
// B(2i+1) * 256 + (B2i unsigned), so a lane's max / min carries the max / min
// of the upper bytes in its upper byte; the word shifted left by 8 bits puts
// B0 and B2 there.  Three-input s16x2 max / min over both forms cover all four
// bytes, and an arithmetic shift by 8 recovers the byte.
__device__ __forceinline__ int rq_block_maxabs(const uint32_t (&w)[9], bool odd) {
  uint32_t mx = 0x80008000u, mn = 0x7FFF7FFFu;
#pragma unroll
  for (int k = 1; k <= 8; ++k) {
    const uint32_t v = k < 8 ? w[k] : (odd ? w[8] : prmt(w[8], w[0], 0x7610u));
    const uint32_t v8 = v << 8;
    mx = vmax_s16x2(mx, vmax_s16x2(v, v8));
    mn = vmin_s16x2(mn, vmin_s16x2(v, v8));
  }
  const int hi = max(static_cast<int>(static_cast<int16_t>(mx & 0xFFFFu)), static_cast<int>(static_cast<int16_t>(mx >> 16))) >> 8;
  const int lo = min(static_cast<int>(static_cast<int16_t>(mn & 0xFFFFu)), static_cast<int>(static_cast<int16_t>(mn >> 16))) >> 8;
  return max(hi, -lo);
}

__device__ __forceinline__ float rq_block_scale(const uint32_t (&w)[9], bool odd) {
  return __half2float(__ushort_as_half(static_cast<uint16_t>(prmt(w[0], 0u, odd ? 0x4432u : 0x4410u))));
}

// 32 codes of a block -> 32 axis-wise codes (8 words).  Each value
// fl(d q) = d q is exact (an 11-bit by 8-bit product); its code is that of
// fl(d q / s), with the quotient refined from y = fl(1/s) as in the row
// quantizers (encode8): q0 = fl(x y), r = fl(x - q0 s), q1 = fl(q0 + r y) is
// the IEEE quotient for every value a Q8_0 block can hold and every scale
// s = fl(a / QMAX) such values give, for QMAX 127 and 448 (checked
// exhaustively on the GPU), so no value needs a division and no
// data-dependent branch is taken.  |x / s| <= QMAX (1 + 2^-23): int8 needs
// no clamp (RNE by the 1.5 * 2^23 sum), e4m3 saturates at 448 in the
// conversion, which takes x's sign (d q = -0 has code 0x80).
// The exact product is formed without converting the codes: with its sign
// bit flipped, code q is the byte u = q + 128, and the fp32 pattern
// 0x4B00uu00 is B = 2^23 + 256 u = K + 256 q with K = 2^23 + 2^15 (9
// significant bits, so K d is exact), hence x' = fl(B d - K d) = 256 d q
// exactly, in one fma.  The quotient is taken on x' with y / 256 and 256 s:
// every step of the refinement scales by 2^8 exactly, so q0 and q1 are the
// same numbers as for x, y and s.  x' keeps x's sign except for a zero value,
// where the fma gives +0: with d > 0 that is x's sign too, and blocks with
// d <= 0 (never written by a Q8_0 quantizer) take x = d q from its factors.
template <int QT, bool kPosScale>
__device__ __forceinline__ void rq_block_codes_impl(const uint32_t (&c)[8], float d, float s, float y,
                                                    uint32_t (&out)[8]) {
  constexpr float kK = 8421376.0f;   // 2^23 + 2^15
  constexpr float kBias = 8388736.0f;   // 2^23 + 128
  const float ys = y * 0.00390625f, ss = s * 256.0f;   // exact
  const float2 d2 = make_float2(d, d), y2 = make_float2(ys, ys), ns2 = make_float2(-ss, -ss);
  // int8: fl(q1 + 2^23 + 128) rounds q1 to the nearest integer, ties to
  // even (unit spacing in [2^23, 2^24), and 2^23 + 128 is even), leaving
  // code + 128 in the low byte
  const float2 nk2 = make_float2(-kK * d, -kK * d), mg = make_float2(kBias, kBias);
  const float2 nb2 = make_float2(-kBias, -kBias), d256 = make_float2(d * 256.0f, d * 256.0f);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    uint32_t b[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float2 x;
      if constexpr (kPosScale) {
        const float2 u = make_float2(__uint_as_float(prmt(c[k], 0x4B000000u, 0x7504u | ((2 * h) << 4))),
                                     __uint_as_float(prmt(c[k], 0x4B000000u, 0x7504u | ((2 * h + 1) << 4))));
        x = __ffma2_rn(u, d2, nk2);
      } else {
        const float2 u = make_float2(__uint_as_float(prmt(c[k], 0x4B000000u, 0x7540u | (2 * h))),
                                     __uint_as_float(prmt(c[k], 0x4B000000u, 0x7540u | (2 * h + 1))));
        x = __fmul2_rn(__fadd2_rn(u, nb2), d256);   // 256 (q d): +-0 as d q
      }
      const float2 q0 = __fmul2_rn(x, y2);
      const float2 r = __ffma2_rn(q0, ns2, x);
      if constexpr (QT == 1) {
        const float2 q1 = __ffma2_rn(r, y2, q0);
        if constexpr (kPosScale) {
          b[h] = cvt_e4m3x2(q1.x, q1.y);
        } else {
          const float lo = __uint_as_float((__float_as_uint(q1.x) & 0x7FFFFFFFu) | (__float_as_uint(x.x) & 0x80000000u));
          const float hi = __uint_as_float((__float_as_uint(q1.y) & 0x7FFFFFFFu) | (__float_as_uint(x.y) & 0x80000000u));
          b[h] = cvt_e4m3x2(lo, hi);
        }
      } else {
        const float2 q1 = __fadd2_rn(__ffma2_rn(r, y2, q0), mg);
        b[2 * h] = __float_as_uint(q1.x);
        b[2 * h + 1] = __float_as_uint(q1.y);
      }
    }
    if constexpr (QT == 1) {
      out[k] = prmt(b[0], b[1], 0x5410u);
    } else {
      // b = 0x4B000000 + (code + 128): integer multiply-adds put the four
      // bytes side by side (the multiples of 256 push 0x4B out of the word),
      // and flipping each byte's top bit gives the two's-complement codes
      out[k] = ((b[0] & 0xFFu) + b[1] * 256u + b[2] * 65536u + b[3] * 16777216u) ^ 0x80808080u;
    }
  }
}

template <int QT>
__device__ __forceinline__ void rq_block_codes(const uint32_t (&w)[9], bool odd, float d, float s, float y,
                                               uint32_t (&out)[8]) {
  const uint32_t csel = odd ? 0x7654u : 0x5432u;
  uint32_t c[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) c[k] = prmt(w[k], w[k + 1], csel) ^ 0x80808080u;
  if (QT == 0 || d > 0.0f) {   // int8 codes do not see the sign of a zero
    rq_block_codes_impl<QT, true>(c, d, s, y, out);
  } else {
    rq_block_codes_impl<QT, false>(c, d, s, y, out);
  }
}

template <int QT, int TW, int S>
__global__ void __launch_bounds__(kRqThreads) q8_0_to_axis_team_kernel(const uint8_t* __restrict__ blocks,
                                                                      int64_t N, int64_t K,
                                                                      uint8_t* __restrict__ q,
                                                                      float* __restrict__ scale) {
  extern __shared__ __align__(16) uint8_t rq_smem[];
  __shared__ float red[2][8];
  griddep_launch();
  griddep_wait();   // the blocks may be the previous kernel's output, q and scale its input
  constexpr int T = 32 * TW;
  constexpr int kTeams = kRqThreads / T;
  const int team = threadIdx.x / T, t = threadIdx.x % T;
  const int nblk = static_cast<int>(K >> 5);
  const int row_bytes = nblk * kQ80Bytes;   // a multiple of 16
  const int nvec = row_bytes >> 4;
  uint8_t* const buf = rq_smem + S * team * row_bytes;   // a ring of S row buffers per team
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kTeams;
  int64_t n = blockIdx.x * static_cast<int64_t>(kTeams) + team;
  auto fetch = [&](int64_t row, int slot) {   // one commit group per call, empty past the last row
    if (row < N) {
      const uint8_t* src = blocks + row * row_bytes;
      uint8_t* dst = buf + slot * row_bytes;
      for (int i = t; i < nvec; i += T) cp_async16(dst + 16 * i, src + 16 * i);
    }
    cp_async_commit();
  };
#pragma unroll
  for (int p = 0; p < S - 1; ++p) fetch(n + p * stride, p);
  for (int it = 0; n < N; n += stride, ++it) {
    const uint8_t* cur = buf + (it % S) * row_bytes;
    fetch(n + (S - 1) * stride, (it + S - 1) % S);
    cp_async_wait<S - 1>();   // this thread's copies of the current row have landed
    team_sync<TW>(team);      // ... and every other thread's
    float a = 0.0f;
#pragma unroll 1
    for (int b = t; b < nblk; b += T) {
      uint32_t w[9];
      rq_block_words(cur, b, w);
      const bool odd = b & 1;
      a = fmaxf(a, __fmul_rn(fabsf(rq_block_scale(w, odd)), static_cast<float>(rq_block_maxabs(w, odd))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
    if constexpr (TW > 1) {
      if ((t & 31) == 0) red[it & 1][threadIdx.x >> 5] = a;
      team_sync<TW>(team);
#pragma unroll
      for (int i = 0; i < TW; ++i) a = fmaxf(a, red[it & 1][team * TW + i]);
    }
    const float s = absmax_scale<QT>(a);
    const float rcp = __frcp_rn(s);
    if (t == 0) scale[n] = s;
#pragma unroll 1
    for (int b = t; b < nblk; b += T) {
      uint32_t w[9];
      rq_block_words(cur, b, w);
      const bool odd = b & 1;
      uint32_t o[8];
      rq_block_codes<QT>(w, odd, rq_block_scale(w, odd), s, rcp, o);
      uint4* dst = reinterpret_cast<uint4*>(q + n * K + 32 * static_cast<int64_t>(b));
      if (!in_bounds(n * K + 32 * static_cast<int64_t>(b) + 31, N * K, 0xB404)) continue;
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
    team_sync<TW>(team);   // this row's buffer is refilled on the next iteration
  }
  cp_async_wait<0>();
}

// The same computation for rows of at most HOLD * 32 * TW blocks: pass 1
// keeps each thread's blocks (9 words each) in registers, so a row buffer is
// free as soon as pass 1 has read it.  With S = 1 the next row's copy is
// issued then and overlaps the arithmetic of pass 2, which needs no shared
// memory; with S = 2 each team alternates between two row buffers and
// issues the next row's copy before pass 1 of the current one.  FULL: every
// row has exactly HOLD * 32 * TW blocks (no per-block bounds test).  NT
// threads per block.
template <int QT, int TW, int HOLD, int MINB = 1, int S = 1, bool FULL = false, int NT = kRqThreads>
__global__ void __launch_bounds__(NT, MINB) q8_0_to_axis_hold_kernel(const uint8_t* __restrict__ blocks,
                                                                            int64_t N, int64_t K,
                                                                            uint8_t* __restrict__ q,
                                                                            float* __restrict__ scale) {
  static_assert(S == 1 || S == 2, "one or two row buffers per team");
  extern __shared__ __align__(16) uint8_t rq_smem[];
  __shared__ float red[2][8];
  griddep_launch();
  griddep_wait();   // the blocks may be the previous kernel's output, q and scale its input
  constexpr int T = 32 * TW;
  static_assert(NT % T == 0 && NT <= 256, "whole teams, at most 8 warps");
  constexpr int kTeams = NT / T;
  const int team = threadIdx.x / T, t = threadIdx.x % T;
  const int nblk = static_cast<int>(K >> 5);
  const int row_bytes = nblk * kQ80Bytes;   // a multiple of 16
  const int nvec = row_bytes >> 4;
  uint8_t* const buf = rq_smem + S * team * row_bytes;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kTeams;
  int64_t n = blockIdx.x * static_cast<int64_t>(kTeams) + team;
  auto fetch = [&](int64_t row, int slot) {   // one commit group per call, empty past the last row
    if (row < N) {
      const uint8_t* src = blocks + row * row_bytes;
      uint8_t* dst = buf + slot * row_bytes;
      for (int i = t; i < nvec; i += T) cp_async16(dst + 16 * i, src + 16 * i);
    }
    cp_async_commit();
  };
  fetch(n, 0);
  for (int it = 0; n < N; n += stride, ++it) {
    const uint8_t* cur = buf + (S == 2 ? (it & 1) : 0) * row_bytes;
    if constexpr (S == 2) {
      fetch(n + stride, (it + 1) & 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    team_sync<TW>(team);   // the row has landed
    uint32_t w[HOLD][9];
    float a = 0.0f;
#pragma unroll
    for (int h = 0; h < HOLD; ++h) {
      const int b = t + h * T;
      if (FULL || b < nblk) {
        rq_block_words(cur, b, w[h]);
        const bool odd = b & 1;
        a = fmaxf(a, __fmul_rn(fabsf(rq_block_scale(w[h], odd)), static_cast<float>(rq_block_maxabs(w[h], odd))));
      }
    }
    team_sync<TW>(team);   // every thread has its words: the buffer may be refilled
    if constexpr (S == 1) fetch(n + stride, 0);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
    if constexpr (TW > 1) {
      if ((t & 31) == 0) red[it & 1][threadIdx.x >> 5] = a;
      team_sync<TW>(team);
#pragma unroll
      for (int i = 0; i < TW; ++i) a = fmaxf(a, red[it & 1][team * TW + i]);
    }
    const float s = absmax_scale<QT>(a);
    const float rcp = __frcp_rn(s);
    if (t == 0) scale[n] = s;
#pragma unroll
    for (int h = 0; h < HOLD; ++h) {
      const int b = t + h * T;
      if (FULL || b < nblk) {
        const bool odd = b & 1;
        uint32_t o[8];
        rq_block_codes<QT>(w[h], odd, rq_block_scale(w[h], odd), s, rcp, o);
        uint4* dst = reinterpret_cast<uint4*>(q + n * K + 32 * static_cast<int64_t>(b));
        if (!in_bounds(n * K + 32 * static_cast<int64_t>(b) + 31, N * K, 0xB404)) continue;
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
      }
    }
  }
  cp_async_wait<0>();
}

}  // namespace w8a8
