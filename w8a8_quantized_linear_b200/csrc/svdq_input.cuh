// svdq_input.cuh - the input side of the SVDQuant forward (OneTrainer PR
// #1034, "SVDQuant"; OneTrainer wiki "Quantization", SVDQuant paragraph) in
// one pass over X [M, K] bf16:
//   * the token-wise codes and scales of X, with the row quantizers'
//     arithmetic (row absmax, s = max(absmax, 1e-10) / QMAX, codes of
//     fl(x / s) by encode8), and
//   * the low-rank input T = bf16(X L1) [M, r] (L1 [K, r] bf16, fp32 sums,
//     one bf16 rounding).
// Both need all of a row, and together they are HBM-bound work: X is read
// once and the codes written once, while T is only 2 r flops per element of
// X.  So a CTA takes 32 rows, keeps them in shared memory for the whole
// kernel (row-major, rows padded by 16 bytes so that ldmatrix reads are free
// of bank conflicts; K up to kSiMaxK), and forms T with warp-level bf16 MMAs
// from shared memory while X lands:
//   warp 31      X: one bulk copy per row and 512-column chunk (1 KB
//                contiguous, chunk after chunk, a lane per row);
//   warp 30      L1 through a ring of [128 K rows x 32 ranks] blocks (ranks
//                past r zero-filled by the copy, 64-byte swizzle), its first
//                stages before any X copy; a copy instruction can block while
//                the copy engine is busy, so the ring is refilled by a thread
//                that issues no X copies;
//   warps 0-15   warp w takes rows 16 (w & 1) .. + 16 and k-step w >> 1 of
//                every 128-row L1 block: one m16n8k16 MMA per 8 ranks, and
//                the rows' absmax from the same A fragments;
//   all warps    then the eight k-groups' partial sums are added in a fixed
//                order and rounded once (T), the absmax gives the scales, and
//                the codes are encoded from shared memory, a warp per row,
//                consecutive lanes on consecutive 8-byte groups of codes.
// Every wait is bounded; the codes, scales and T land where the separate
// row quantizer and T product put them, so the GEMM after is unchanged.
#pragma once
#include "device.cuh"
#include "quantize.cuh"

namespace w8a8 {

constexpr int kSiRows = 32;                        // rows of X per CTA
constexpr int kSiKGroups = 8;                      // k-steps of an L1 block, one per MMA warp pair
constexpr int kSiMmaWarps = 2 * kSiKGroups;
constexpr int kSiWarps = 32;                       // all encode; the last two load first
constexpr int kSiThreads = 32 * kSiWarps;
constexpr int kSiXWarp = kSiWarps - 1;
constexpr int kSiL1Warp = kSiWarps - 2;
constexpr int kSiKC = 16 * kSiKGroups;             // L1 rows per ring stage
constexpr int kSiStages = 4;
constexpr int kSiL1Bytes = kSiKC * 64;             // 128 K rows x 32 bf16
constexpr int kSiXChunk = 512;                     // columns per X copy (1 KB)
constexpr int kSiMaxK = 3072;
constexpr int kSiMaxChunks = kSiMaxK / kSiXChunk;
constexpr int kSiAuxBytes = 1024;                  // barriers, row maxima, scales

// Row pitch in shared memory: 2K + 16 bytes, an odd number of 16-byte units
// (K is a multiple of 16), so the 8 rows of an ldmatrix read hit 8 distinct
// bank groups.  The L1 ring starts on the next 512-byte boundary (the
// 64-byte swizzle's period).
__host__ __device__ constexpr int si_pitch(int K) { return 2 * K + 16; }
__host__ __device__ constexpr int si_ring_offset(int K) { return (kSiRows * si_pitch(K) + 511) & ~511; }
__host__ __device__ constexpr size_t si_smem_bytes(int K) {
  return 1024 /*alignment slack*/ + static_cast<size_t>(si_ring_offset(K)) +
         static_cast<size_t>(kSiStages) * kSiL1Bytes + kSiAuxBytes;
}
static_assert(si_smem_bytes(kSiMaxK) <= 232448, "shared memory per block");
static_assert(kSiMaxK % kSiXChunk == 0, "whole chunks at the largest K");
static_assert(kSiRows == 32, "a producer lane per row");
static_assert(kSiKGroups * kSiRows * 32 * 4 <= kSiStages * kSiL1Bytes, "partial sums reuse the L1 ring");
static_assert((kSiMaxChunks + 2 * kSiStages) * 8 + 3 * kSiRows * 4 + 4 <= kSiAuxBytes, "aux area");

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// Column of the partial-sum array red[k-group][row][32] where rank column c
// of `row` is kept: c ^ (8 (row & 3) + ((row >> 2) & 1)).  An MMA warp's
// store of one accumulator element (rows r0 + lane / 4, columns 8 j + 2 (lane
// % 4) + e) then hits 32 distinct banks.
__device__ __forceinline__ int si_red_col(int row, int c) { return c ^ (8 * (row & 3) + ((row >> 2) & 1)); }

__device__ __forceinline__ void si_bar() {   // every warp of the block
  asm volatile("bar.sync 1, %0;" ::"n"(kSiThreads) : "memory");
}

// x: X [M, K] bf16 (rows of K elements, 16-byte aligned).
// tmL1: L1 [K, r] bf16 in [128 rows x 32 ranks] boxes, 64-byte swizzle.
// Grid: ceil(M / 32) CTAs of kSiThreads, si_smem_bytes(K) bytes, K <= kSiMaxK.
template <int QT>
__global__ void __launch_bounds__(kSiThreads, 1)
    svdq_input_kernel(const __nv_bfloat16* __restrict__ x, const __grid_constant__ CUtensorMap tmL1, int M, int K,
                      int r, uint8_t* __restrict__ q, float* __restrict__ scale, __nv_bfloat16* __restrict__ t) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* xs = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int pitch = si_pitch(K);
  const int nxc = (K + kSiXChunk - 1) / kSiXChunk;   // X chunks
  const int nc = (K + kSiKC - 1) / kSiKC;            // L1 blocks
  uint8_t* ring = xs + si_ring_offset(K);
  uint8_t* aux = ring + kSiStages * kSiL1Bytes;
  uint64_t* xfull = reinterpret_cast<uint64_t*>(aux);   // [kSiMaxChunks]
  uint64_t* full = xfull + kSiMaxChunks;                 // [kSiStages]
  uint64_t* empty = full + kSiStages;                    // [kSiStages]
  unsigned* amax = reinterpret_cast<unsigned*>(empty + kSiStages);   // [32] fp32 bits (non-negative)
  float* srow = reinterpret_cast<float*>(amax + kSiRows);           // [32]
  float* rrow = srow + kSiRows;                                      // [32] fl(1 / s)
  volatile int* abort = reinterpret_cast<volatile int*>(rrow + kSiRows);
  float* red = reinterpret_cast<float*>(ring);   // [8 k-groups][32 rows][32 ranks] once L1 is consumed

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kSiRows;
  if (threadIdx.x == 0) {
    for (int c = 0; c < nxc; ++c) mbar_init(&xfull[c], kSiRows);   // an arrival per row (lane)
    for (int s = 0; s < kSiStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kSiMmaWarps);
    }
    *abort = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < kSiRows) amax[threadIdx.x] = 0u;
  if (warp == kSiL1Warp && lane == 0) tma_prefetch_desc(&tmL1);
  __syncthreads();
  // Wait first, then let the next kernel launch (the rule of the row
  // quantizers: the GEMM after this kernel reads its weight before its own wait).
  griddep_wait();   // X may be the previous kernel's output
  griddep_launch();
  const uint64_t lim = g_wait_limit_ns;

  if (warp == kSiL1Warp) {
    const int first = nc < kSiStages ? nc : kSiStages;
    if (lane == 0)
      for (int c = 0; c < first; ++c) {
        mbar_arrive_expect_tx(&full[c], kSiL1Bytes);
        tma_load_2d(ring + c * kSiL1Bytes, &tmL1, &full[c], 0, c * kSiKC);
      }
    __syncwarp();
    asm volatile("bar.arrive 2, 64;" ::: "memory");   // the X copies may start
    if (lane == 0)
      for (int c = first; c < nc; ++c) {
        const int s = c % kSiStages;
        if (!mbar_wait(&empty[s], ((c / kSiStages) - 1) & 1, abort, 0xC601, lim)) break;
        mbar_arrive_expect_tx(&full[s], kSiL1Bytes);
        tma_load_2d(ring + s * kSiL1Bytes, &tmL1, &full[s], 0, c * kSiKC);
      }
    __syncwarp();
  } else if (warp == kSiXWarp) {
    // lane i copies row m0 + i, chunk after chunk (rows past M arrive empty),
    // once the first L1 stages are on their way
    asm volatile("bar.sync 2, 64;" ::: "memory");
    const int m = m0 + lane;
    const __nv_bfloat16* src = x + static_cast<int64_t>(m) * K;
    for (int c = 0; c < nxc; ++c) {
      const int c0 = c * kSiXChunk;
      const int cols = (K - c0) < kSiXChunk ? (K - c0) : kSiXChunk;
      if (m < M) {
        mbar_arrive_expect_tx(&xfull[c], static_cast<uint32_t>(cols) * 2);
        bulk_load(xs + lane * pitch + c0 * 2, src + c0, static_cast<uint32_t>(cols) * 2, &xfull[c]);
      } else {
        mbar_arrive(&xfull[c]);
      }
    }
  }
  if (warp < kSiMmaWarps) {
    // ---- T partial sums and row absmax, as the X chunks and L1 blocks land
    const int h = warp & 1, g = warp >> 1;
    const uint32_t xs_u = smem_u32(xs), ring_u = smem_u32(ring);
    const int arow = 16 * h + (lane & 15);                 // ldmatrix row of A (X rows of this m-tile)
    const uint32_t a_base = xs_u + arow * pitch + (lane >> 4) * 16;   // + k-step column * 2
    const int bk = g * 16 + (lane & 7) + (lane & 8);       // ldmatrix row of B (L1 row within the stage)
    const uint32_t bsw = static_cast<uint32_t>((bk >> 1) & 3);
    const uint32_t bnc = static_cast<uint32_t>(lane >> 4);
    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
    uint32_t mlo = 0, mhi = 0;   // bf16x2 running absmax of rows lane/4 and lane/4 + 8 of the m-tile
    int waited = -1;
    for (int c = 0; c < nc; ++c) {
      const int s = c % kSiStages;
      if (!mbar_wait(&full[s], (c / kSiStages) & 1, abort, 0xC602, lim)) break;
      const int kk = c * kSiKC + g * 16;   // first column of this warp's k-step
      if (kk < K) {
        const int xc = kk / kSiXChunk;
        if (xc != waited) {
          if (!mbar_wait(&xfull[xc], 0, abort, 0xC603, lim)) break;
          waited = xc;
        }
        uint32_t a[4];
        ldmatrix_x4(a, a_base + kk * 2);
        mlo = bf2_absmax(bf2_absmax(mlo, a[0]), a[2]);
        mhi = bf2_absmax(bf2_absmax(mhi, a[1]), a[3]);
        const uint32_t rb = ring_u + s * kSiL1Bytes + bk * 64;
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          uint32_t bb[4];
          ldmatrix_x4_trans(bb, rb + (((2 * p + bnc) ^ bsw) << 4));
          mma_bf16_m16n8k16(acc[2 * p], a, bb[0], bb[1]);
          mma_bf16_m16n8k16(acc[2 * p + 1], a, bb[2], bb[3]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    // (after a wait ran out, recorded in the status word, the sums are
    // incomplete and the outputs of this CTA are not meaningful)
    float alo = bf2_absmax_final(mlo), ahi = bf2_absmax_final(mhi);
    alo = fmaxf(alo, __shfl_xor_sync(0xFFFFFFFFu, alo, 1));
    alo = fmaxf(alo, __shfl_xor_sync(0xFFFFFFFFu, alo, 2));
    ahi = fmaxf(ahi, __shfl_xor_sync(0xFFFFFFFFu, ahi, 1));
    ahi = fmaxf(ahi, __shfl_xor_sync(0xFFFFFFFFu, ahi, 2));
    if ((lane & 3) == 0) {
      atomicMax(&amax[16 * h + (lane >> 2)], __float_as_uint(alo));
      atomicMax(&amax[16 * h + (lane >> 2) + 8], __float_as_uint(ahi));
    }
    si_bar();   // every MMA warp is past its last L1 block: the ring becomes `red`
    float* rg = red + g * (kSiRows * 32);
    const int r0 = 16 * h + (lane >> 2), c0 = 2 * (lane & 3);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      rg[r0 * 32 + si_red_col(r0, 8 * j + c0)] = acc[j][0];
      rg[r0 * 32 + si_red_col(r0, 8 * j + c0 + 1)] = acc[j][1];
      rg[(r0 + 8) * 32 + si_red_col(r0 + 8, 8 * j + c0)] = acc[j][2];
      rg[(r0 + 8) * 32 + si_red_col(r0 + 8, 8 * j + c0 + 1)] = acc[j][3];
    }
  } else {
    si_bar();   // (the MMA warps arrive above)
    if (warp == kSiMmaWarps) {
      // the row scales (every absmax is in), while the MMA warps store their sums
      const float sc = absmax_scale<QT>(__uint_as_float(amax[lane]));
      srow[lane] = sc;
      rrow[lane] = __frcp_rn(sc);
      const int m = m0 + lane;
      if (m < M && in_bounds(m, M, 0xB601)) scale[m] = sc;
    }
  }
  si_bar();
  if (threadIdx.x < kSiRows * 32 / 2) {
    // T: two ranks per thread, the k-groups' partial sums in order 0..7
    const int e = 2 * threadIdx.x;
    const int row = e >> 5, col = e & 31;
    const int p0 = row * 32 + si_red_col(row, col), p1 = row * 32 + si_red_col(row, col + 1);
    float v0 = 0.0f, v1 = 0.0f;
#pragma unroll
    for (int gg = 0; gg < kSiKGroups; ++gg) {
      v0 += red[gg * (kSiRows * 32) + p0];
      v1 += red[gg * (kSiRows * 32) + p1];
    }
    const int m = m0 + row;
    if (m < M && col < r && in_bounds(static_cast<int64_t>(m) * r + col + 1, static_cast<int64_t>(M) * r, 0xB602))
      *reinterpret_cast<uint32_t*>(t + static_cast<int64_t>(m) * r + col) = pack_bf16x2(v0, v1);
  }
  // ---- codes: warp w encodes row w from shared memory
  const int m = m0 + warp;
  if (m < M) {
    const int kv = K >> 3;   // 16-byte groups of the row
    const float sc = srow[warp], y = rrow[warp];
    const uint8_t* xr = xs + warp * pitch;
    uint2* out = reinterpret_cast<uint2*>(q + static_cast<int64_t>(m) * K);
#pragma unroll 4
    for (int cv = lane; cv < kv; cv += 32) {
      const uint4 w = *reinterpret_cast<const uint4*>(xr + cv * 16);
      if (in_bounds(cv, kv, 0xB603)) out[cv] = encode8<QT>(w, sc, y);
    }
  }
}

}  // namespace w8a8
