// gemm.cuh - 8-bit (and bf16) GEMM on the sm_100a tensor cores with the
// dequantizing epilogue fused.
//
//   D[m, n] = sum_k A[m, k] * B[n, k]       (B K-major: the forward, W[N,K])
//   D[m, n] = sum_k A[m, k] * B[k, n]       (B MN-major: the dgrad, W[N,K] read
//                                            with N as the contraction)
//
// One persistent CTA per SM, warp-specialized, 320 threads:
//   warp 0      TMA producer: A and B tiles into a ring of kStages shared-
//               memory stages (128-byte swizzle), completion on mbarriers;
//   warp 1      TMEM allocation; one thread issues tcgen05.mma (4 per stage)
//               into one of two TMEM accumulators and commits the stage back;
//   warps 2..9  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//               lanes 32*(w%4)..+31 = tile rows; the two warps of a lane
//               quarter take alternate 32-column chunks), scales / bias /
//               low-rank in fp32, bf16 stores.  Double buffering of the accumulator lets
//               the epilogue of tile i overlap the MMAs of tile i+1.
// Tile 128 x BN x 128 bytes of K per stage.  Every wait is bounded.
//
// Split-K (scale and plain epilogues): with ep.splits = S > 1 the work units are
// (tile, split) pairs, split s covering K blocks [s*nkb/S, (s+1)*nkb/S).  A
// unit writes its raw sums (int32, or fp32 bits for e4m3) for the tile's
// valid rows to ep.partial[s][m][n]; splitk_epilogue_kernel then adds the S
// partial sums in split order (a fixed order, so e4m3 results are
// reproducible; integer sums are exact in any order) and applies the
// epilogue.
#pragma once
#include "device.cuh"

namespace w8a8 {

constexpr int kBM = 128;
constexpr int kBKBytes = 128;

enum { kKindI8 = 0, kKindE4M3 = 1, kKindBF16 = 2 };
enum { kEpiScale = 0, kEpiLowRank = 1, kEpiPlain = 2, kEpiScaleT = 3 };

struct EpiParams {
  const float* s_row;            // [M] row (token) scales          (kEpiScale/LowRank)
  const float* s_col;            // [1] or [N] weight scale
  int s_col_axis;                // 1: s_col[n], 0: s_col[0]
  const __nv_bfloat16* bias;     // [N] or nullptr
  __nv_bfloat16* y;              // [M, ldy]
  int64_t ldy;
  int tma_store;                 // 1: Y goes out through the tmY tensor map (ldy % 8 == 0)
  const __nv_bfloat16* lr_t;     // T [M, r]                          (kEpiLowRank)
  const __nv_bfloat16* lr_l2;    // L2 [r, N]
  int r;
  int splits;                    // K splits per tile (>= 1; > 1 not with kEpiLowRank)
  uint32_t* partial;             // [splits, M, N] raw sums (splits > 1)
  int act;                       // kActNone / kActGelu / kActGeluTanh, applied last (kEpiScale)
  uint32_t* y_amax;              // [M] or null: atomicMax of max |y| per row (fp32 bits of the bf16 values)
  // 1: the weight (B, or A in the transposed form) may be read before
  // griddepcontrol.wait.  The host sets it only when the kernel just before
  // this GEMM on the stream is the row quantizer of the same call, which
  // waits for every earlier kernel before it lets this one launch and never
  // writes the weight; a weight that an earlier kernel wrote is then
  // complete.  0 (every other caller): nothing is read before the wait.
  int early_weights;
};

// Optional activation between two projections (the MLP's GELU): the exact
// form 0.5 v (1 + erf(v / sqrt 2)) or the tanh form 0.5 v (1 + tanh(sqrt(2/pi)
// (v + 0.044715 v^3))), on the fp32 epilogue value, before the bf16 rounding.
enum { kActNone = 0, kActGelu = 1, kActGeluTanh = 2 };
__device__ __forceinline__ float apply_act(float v, int act) {
  if (act == kActGelu) return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
  if (act == kActGeluTanh) return 0.5f * v * (1.0f + tanhf(0.79788456080286536f * (v + 0.044715f * v * v * v)));
  return v;
}

// Row absmax of bf16 outputs: max over |bf16| as 16-bit lanes (the magnitude
// bits order like the values), then one atomicMax on the fp32 bits (a
// non-negative float orders like its bit pattern).
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t m, uint32_t packed) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(m), "r"(packed & 0x7FFF7FFFu));
  return d;
}
__device__ __forceinline__ void row_amax_commit(uint32_t* y_amax, int64_t row, uint32_t m) {
  const uint32_t h = (m & 0xFFFFu) > (m >> 16) ? (m & 0xFFFFu) : (m >> 16);
  if (h != 0) atomicMax(y_amax + row, h << 16);
}

// Low-rank (SVDQuant) epilogue: ranks up to 32; the staged L2^T rows are
// kLowRankStride bf16 apart.
constexpr int kLowRankMaxRank = 32;
constexpr int kLowRankStride = 40;

template <int KIND, int BN, int EPI>
struct GemmCfg {
  static constexpr int kElem = (KIND == kKindBF16) ? 2 : 1;
  static constexpr int kBK = kBKBytes / kElem;            // K elements per stage
  static constexpr int kMmaK = 32 / kElem;                // K elements per MMA
  static constexpr int kABytes = kBM * kBKBytes;          // 16 KB
  static constexpr int kBBytes = BN * kBKBytes;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kLrBytes = (EPI == kEpiLowRank) ? BN * kLowRankStride * 2 : 0;   // L2^T tile (stage_l2t)
  static constexpr int kEpiWarps = 8;   // two per TMEM lane quarter, splitting the column chunks
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  // per epilogue warp, two 32 x 32 bf16 staging buffers for the TMA store
  // (in the transposed form a block is staged transposed)
  static constexpr int kOutBufBytes = 32 * 32 * 2;
  static constexpr int kOutBytes = kEpiWarps * 2 * kOutBufBytes;
  static constexpr int kFixedBytes = 1024 + ((kLrBytes + 1023) & ~1023) + kOutBytes + 256;
  static constexpr int kStagesFit = (232448 - kFixedBytes) / kStageBytes;
  // as many pipeline stages as the shared memory holds (4 for 128x256 tiles,
  // 8 for 128x64 tiles, whose CTAs must keep more bytes in flight), at most
  // 8, or 10 in the transposed form (a weight stream on few SMs)
  static constexpr int kMaxStages = (EPI == kEpiScaleT) ? 10 : 8;
  static constexpr int kStages = kStagesFit > kMaxStages ? kMaxStages : kStagesFit;
  static constexpr size_t kSmem = 1024 /*alignment slack*/ + static_cast<size_t>(kStages) * kStageBytes +
                                  ((kLrBytes + 1023) & ~1023) + kOutBytes + 256 /*barriers*/;
  static constexpr int kCtasPerSm = 1;
  static_assert(kSmem <= 232448, "shared memory per block");
};

// One epilogue warp's chunks of a 128-row x BN-column accumulator tile:
// the warp reads the 32 TMEM lanes of its quarter (rows m0 + 32 quarter +
// lane) for the 32-column chunks c = group, group + kGroups, ... at TMEM
// address tacc; y = bf16(((acc * s_x) * s_w) + bias), each step an fp32 RN
// operation, and with LR one more RN add of the fp32 low-rank sum read at
// TMEM address tlr; the warp's 32 x 32 bf16 block goes out through one of
// its two swizzled staging buffers (sOutWarp) with a TMA store, or directly
// when the row stride is not a multiple of 8.
template <int KIND, int EPI, int BN, int kGroups, bool kAxisOk, bool LR = false>
__device__ __forceinline__ void epilogue_scale_chunks(const EpiParams& ep, const CUtensorMap* tmY, uint32_t tacc, int m0,
                                                      int n0, int M, int N, int quarter, int group, int lane, float sx,
                                                      float sw0, uint8_t* sOutWarp, uint32_t& out_iter,
                                                      uint32_t tlr = 0) {
  const int row = m0 + quarter * 32 + lane;
  const bool row_ok = row < M;
  uint32_t amx = 0;   // this lane's row: max |y| over the tile's columns, as two bf16 lanes
  #pragma unroll 1
  for (int c = group; c < BN / 32; c += kGroups) {
    const int nc = n0 + c * 32;
    if (nc >= N) break;                       // warp-uniform
    const bool full_chunk = nc + 32 <= N;
    // Column parameters of the chunk, loaded before the TMEM load so that
    // their latency overlaps it: 16-byte vectors, the same addresses in
    // every lane (broadcast).
    float sw[32], bs[32];
    if constexpr (EPI != kEpiPlain) {
      if (kAxisOk && ep.s_col_axis) {
        if (full_chunk) {
  #pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const float4 f = __ldg(reinterpret_cast<const float4*>(ep.s_col + nc + j));
            sw[j] = f.x; sw[j + 1] = f.y; sw[j + 2] = f.z; sw[j + 3] = f.w;
          }
        } else {
  #pragma unroll
          for (int j = 0; j < 32; ++j) sw[j] = (nc + j < N) ? __ldg(ep.s_col + nc + j) : 0.0f;
        }
      }
    }
    {
      if (ep.bias != nullptr) {
        if (full_chunk) {
  #pragma unroll
          for (int j = 0; j < 32; j += 8) {
            const uint4 b = __ldg(reinterpret_cast<const uint4*>(ep.bias + nc + j));
            bs[j] = bf16_lo(b.x); bs[j + 1] = bf16_hi(b.x); bs[j + 2] = bf16_lo(b.y); bs[j + 3] = bf16_hi(b.y);
            bs[j + 4] = bf16_lo(b.z); bs[j + 5] = bf16_hi(b.z); bs[j + 6] = bf16_lo(b.w); bs[j + 7] = bf16_hi(b.w);
          }
        } else {
  #pragma unroll
          for (int j = 0; j < 32; ++j) bs[j] = (nc + j < N) ? __bfloat162float(ep.bias[nc + j]) : 0.0f;
        }
      }
    }
    uint32_t r[32];
    tmem_ld_x32(tacc + static_cast<uint32_t>(c * 32), r);
    uint32_t lr[LR ? 32 : 1];
    if constexpr (LR) tmem_ld_x32(tlr + static_cast<uint32_t>(c * 32), lr);
    tmem_ld_wait();
    float v[32];
  #pragma unroll
    for (int j = 0; j < 32; ++j) {
      float a = (KIND == kKindI8) ? __int2float_rn(static_cast<int>(r[j])) : __uint_as_float(r[j]);
      if constexpr (EPI != kEpiPlain) a = __fmul_rn(__fmul_rn(a, sx), (kAxisOk && ep.s_col_axis) ? sw[j] : sw0);
      if (ep.bias != nullptr) a = __fadd_rn(a, bs[j]);
      if constexpr (LR) a = __fadd_rn(a, __uint_as_float(lr[j]));
      v[j] = a;
    }
    if constexpr (EPI == kEpiScale && !LR) {
      if (ep.act != kActNone) {
  #pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = apply_act(v[j], ep.act);
      }
      if (ep.y_amax != nullptr) {
  #pragma unroll
        for (int j = 0; j < 32; j += 2) {
          // columns past N hold 0 (zero-filled operands, no bias there): no effect
          amx = bf16x2_absmax(amx, pack_bf16x2(v[j], v[j + 1]));
        }
      }
    }
    if (ep.tma_store) {
      // Stage the warp's 32 x 32 bf16 block in shared memory with the 64-byte
      // swizzle (16-byte unit j of row l at unit j ^ ((l >> 1) & 3)), then
      // one lane stores it with TMA; the box is clipped at M and N.
      uint8_t* buf = sOutWarp + (out_iter & 1) * (32 * 32 * 2);
      if (lane == 0) bulk_wait_read<1>();     // this buffer's previous store has read it
      __syncwarp();
  #pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint4 p;
        p.x = pack_bf16x2(v[8 * j], v[8 * j + 1]);
        p.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
        p.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
        p.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
        *reinterpret_cast<uint4*>(buf + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) = p;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && m0 + quarter * 32 < M) {   // skip blocks wholly below the last row
        tma_store_2d(tmY, buf, nc, m0 + quarter * 32);
        bulk_commit();
      }
      ++out_iter;
    } else if (row_ok && in_bounds(row, M, 0xB101) && in_bounds(nc, N, 0xB102)) {
      __nv_bfloat16* out = ep.y + static_cast<int64_t>(row) * ep.ldy + nc;
      if (nc + 32 <= N && (ep.ldy & 7) == 0) {
  #pragma unroll
        for (int j = 0; j < 32; j += 8) {
          uint4 p;
          p.x = pack_bf16x2(v[j], v[j + 1]);
          p.y = pack_bf16x2(v[j + 2], v[j + 3]);
          p.z = pack_bf16x2(v[j + 4], v[j + 5]);
          p.w = pack_bf16x2(v[j + 6], v[j + 7]);
          *reinterpret_cast<uint4*>(out + j) = p;
        }
      } else {
        for (int j = 0; j < 32; ++j)
          if (nc + j < N) out[j] = __float2bfloat16_rn(v[j]);
      }
    }
  }
  if constexpr (EPI == kEpiScale && !LR) {
    if (ep.y_amax != nullptr && row_ok) row_amax_commit(ep.y_amax, row, amx);
  }
}

// The SVDQuant low-rank epilogue.  L2^T of the tile's columns is staged in
// shared memory: sLr[n][k] = L2[k][n0 + n] (bf16), zero for k >= r or
// n0 + n >= N, rows kLowRankStride bf16 apart (32 ranks + 8 pad: no bank
// conflicts for the fragment loads).  The copy moves units of 8 columns of
// one rank: lane k of a warp takes rank k, so the transposing 2-byte stores
// of a warp hit 32 consecutive ranks (no bank conflicts); every load of a
// thread is issued before its first store (one round trip to L2, not one
// per unit).  `et` is the thread's index among the kEpiThreads epilogue
// threads.
template <int BN, int kEpiThreads>
__device__ __forceinline__ void stage_l2t(const EpiParams& ep, uint16_t* sLr, int n0, int N, int et) {
  static_assert(kEpiThreads % 32 == 0 && BN % 8 == 0, "whole warps, whole units");
  constexpr int kUnits = kLowRankMaxRank * BN / 8;
  constexpr int kPer = (kUnits + kEpiThreads - 1) / kEpiThreads;
  const bool vec = (N & 7) == 0;             // 16-byte aligned rows of L2
  uint4 v[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int i = et + u * kEpiThreads;
    const int k = i & 31, n = (i >> 5) * 8;
    v[u] = make_uint4(0u, 0u, 0u, 0u);
    if (i < kUnits && k < ep.r) {
      const __nv_bfloat16* src = ep.lr_l2 + static_cast<int64_t>(k) * N + n0 + n;
      if (vec && n0 + n + 8 <= N) {
        if (in_bounds(static_cast<int64_t>(k) * N + n0 + n + 7, static_cast<int64_t>(ep.r) * N, 0xB105))
          v[u] = __ldg(reinterpret_cast<const uint4*>(src));
      } else {
        uint32_t h[4] = {0u, 0u, 0u, 0u};
        for (int j = 0; j < 8; ++j)
          if (n0 + n + j < N && in_bounds(static_cast<int64_t>(k) * N + n0 + n + j, static_cast<int64_t>(ep.r) * N, 0xB105))
            h[j >> 1] |= static_cast<uint32_t>(__bfloat16_as_ushort(src[j])) << (16 * (j & 1));
        v[u] = make_uint4(h[0], h[1], h[2], h[3]);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int i = et + u * kEpiThreads;
    if (i < kUnits) {
      const int k = i & 31, n = (i >> 5) * 8;
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int j = 0; j < 8; ++j)
        sLr[(n + j) * kLowRankStride + k] = static_cast<uint16_t>(w[j >> 1] >> (16 * (j & 1)));
    }
  }
}

// One epilogue warp's part of a 128-row x BN tile with the low-rank term:
// y = bf16((((acc * s_x) * s_w) + bias) + lr), each step an fp32 RN
// operation, lr = T L2 for the element, computed on the tensor cores by
// warp-level bf16 MMAs from a zero accumulator (the MMA does not add an fp32
// C operand at full precision).  The accumulator is read with 16x256b loads,
// whose register layout is the m16n8 fragment layout of those MMAs, so each
// thread holds the int32 / fp32 sums of exactly the elements its lr
// fragments cover.  tacc: TMEM address of the accumulator buffer (column
// offset, lane 0); T rows come from ep.lr_t (global, [M, r]); sLr holds L2^T
// (stage_l2t); the warp's 32 x 32 blocks go out through its two staging
// buffers sOutWarp with TMA stores, or directly when ldy % 8 != 0.
template <int KIND, int BN, int kGroups>
__device__ __forceinline__ void epilogue_lowrank_tile(const EpiParams& ep, const CUtensorMap* tmY, uint32_t tacc, int m0,
                                                      int n0, int M, int N, int quarter, int group, int lane,
                                                      const uint16_t* sLr, uint8_t* sOutWarp, uint32_t& out_iter) {
  const int g = lane >> 2, tq = lane & 3;
  const int rbase = m0 + quarter * 32;
  const float sw0 = ep.s_col[0];    // the residual's tensor-wise scale
  uint32_t afr[2][2][4];            // T fragments [m16 tile][k16 step][4]
  float sxr[2][2];                  // s_x of rows g and g + 8 in each m16 tile
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int rr = rbase + mt * 16 + g + hh * 8;
      sxr[mt][hh] = rr < M ? ep.s_row[rr] : 0.0f;
    }
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int rr = rbase + mt * 16 + g + (q4 & 1) * 8;
        const int kk = ks * 16 + 2 * tq + (q4 >> 1) * 8;
        afr[mt][ks][q4] = (rr < M && kk < ep.r && in_bounds(static_cast<int64_t>(rr) * ep.r + kk,
                                                            static_cast<int64_t>(M) * ep.r, 0xB104))
                              ? *reinterpret_cast<const uint32_t*>(ep.lr_t + static_cast<int64_t>(rr) * ep.r + kk)
                              : 0u;
      }
    }
  }
  const int nks = (ep.r + 15) / 16;
#pragma unroll 1
  for (int c = group; c < BN / 32; c += kGroups) {
    const int nc = n0 + c * 32;
    if (nc >= N) break;                       // warp-uniform
    float bcol[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int n = nc + 8 * i + 2 * tq + u;
        bcol[i][u] = (ep.bias != nullptr && n < N) ? __bfloat162float(ep.bias[n]) : 0.0f;
      }
    }
    uint32_t rfr[2][16];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
      tmem_ld_16x256b_x4(tacc + (static_cast<uint32_t>(quarter * 32 + mt * 16) << 16) + static_cast<uint32_t>(c * 32),
                         rfr[mt]);
    tmem_ld_wait();
    uint8_t* buf = sOutWarp + (out_iter & 1) * (32 * 32 * 2);
    if (ep.tma_store) {
      if (lane == 0) bulk_wait_read<1>();
      __syncwarp();
    }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float lr[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        const uint16_t* brow = sLr + (c * 32 + 8 * i + g) * kLowRankStride + 2 * tq;
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          if (ks < nks)
            mma_bf16_m16n8k16(lr, afr[mt][ks], *reinterpret_cast<const uint32_t*>(brow + ks * 16),
                              *reinterpret_cast<const uint32_t*>(brow + ks * 16 + 8));
        }
        float d[4];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          float a = (KIND == kKindI8) ? __int2float_rn(static_cast<int>(rfr[mt][4 * i + q4]))
                                      : __uint_as_float(rfr[mt][4 * i + q4]);
          a = __fmul_rn(__fmul_rn(a, sxr[mt][q4 >> 1]), sw0);
          if (ep.bias != nullptr) a = __fadd_rn(a, bcol[i][q4 & 1]);
          d[q4] = __fadd_rn(a, lr[q4]);
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int rl = mt * 16 + g + hh * 8;            // row within the warp's 32-row block
          if (ep.tma_store) {
            *reinterpret_cast<uint32_t*>(buf + rl * 64 + ((i ^ ((rl >> 1) & 3)) << 4) + 4 * tq) =
                pack_bf16x2(d[2 * hh], d[2 * hh + 1]);
          } else {   // row stride not a 16-byte multiple: guarded 2-byte stores
            const int rr = rbase + rl, n = nc + 8 * i + 2 * tq;
            if (rr < M && in_bounds(rr, M, 0xB101)) {
              __nv_bfloat16* out = ep.y + static_cast<int64_t>(rr) * ep.ldy;
              if (n < N) out[n] = __float2bfloat16_rn(d[2 * hh]);
              if (n + 1 < N) out[n + 1] = __float2bfloat16_rn(d[2 * hh + 1]);
            }
          }
        }
      }
    }
    if (ep.tma_store) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && rbase < M) {
        tma_store_2d(tmY, buf, nc, rbase);
        bulk_commit();
      }
      ++out_iter;
    }
  }
}

template <int KIND, bool B_MN, int BN, int EPI>
__global__ void __launch_bounds__(GemmCfg<KIND, BN, EPI>::kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmY, int M, int N, int Kc, EpiParams ep) {
  using C = GemmCfg<KIND, BN, EPI>;
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "tile N");
  static_assert(!B_MN || (BN * C::kElem) % 128 == 0, "MN-major B needs whole 128-byte blocks");
  constexpr uint32_t kIdesc = idesc<KIND>(kBM, BN, B_MN);
  constexpr int kEpiThreads = 32 * C::kEpiWarps;
  constexpr bool kAxisOk = (EPI == kEpiScale);   // per-column weight scales (the low-rank path is tensor-wise)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int kStages = C::kStages;
  uint8_t* sA = smem;                                        // kStages x kABytes
  uint8_t* sB = smem + kStages * C::kABytes;                 // kStages x kBBytes
  uint16_t* sLr = reinterpret_cast<uint16_t*>(smem + kStages * C::kStageBytes);   // L2^T [BN][kLowRankStride] bf16
  uint8_t* sOut = smem + kStages * C::kStageBytes + ((C::kLrBytes + 1023) & ~1023);   // epilogue staging
  uint8_t* tail = sOut + C::kOutBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* teardown = tempty + 2;
  uint64_t* lr_ready = teardown + 1;
  uint64_t* lr_done = lr_ready + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lr_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t limit = g_wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], C::kEpiWarps);   // one arrival per epilogue warp
    }
    mbar_init(teardown, 1);
    mbar_init(lr_ready, kEpiThreads);
    mbar_init(lr_done, kEpiThreads);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (ep.tma_store) tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_launch();   // the next kernel may set itself up while this one runs

  const int tiles_m = (M + kBM - 1) / kBM;
  const int tiles_n = (N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int num_kb = (Kc + C::kBK - 1) / C::kBK;
  // the host keeps 1 <= splits <= num_kb, so every unit has at least one K block
  const int splits = (EPI != kEpiLowRank) ? ep.splits : 1;
  const int num_units = num_tiles * splits;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_phase = 0;   // per-stage bits, for teardown
      bool ok = true;
      auto load_b = [&](int st, int kb, int n0) {
        uint8_t* b = sB + st * C::kBBytes;
        if constexpr (!B_MN) {
          tma_load_2d(b, &tmB, &full[st], kb * C::kBK, n0);
        } else {
#pragma unroll
          for (int j = 0; j < BN * C::kElem / 128; ++j)
            tma_load_2d(b + j * (C::kBK * 128), &tmB, &full[st], n0 + j * (128 / C::kElem), kb * C::kBK);
        }
      };
      // With ep.early_weights the weight tiles of the first unit's first
      // stages are requested before waiting for the previous kernel (the
      // same call's row quantizer, which never writes them); the activation
      // codes it may be producing are read after the wait.  The weight is B,
      // or A in the transposed form (kEpiScaleT).
      constexpr bool kWeightA = (EPI == kEpiScaleT);
      int pre = 0;
      if (ep.early_weights && static_cast<int>(blockIdx.x) < num_units) {
        const int tile = blockIdx.x / splits, split = blockIdx.x - tile * splits;
        const int kb0 = split * num_kb / splits, kb1 = (split + 1) * num_kb / splits;
        pre = (kb1 - kb0) < kStages ? (kb1 - kb0) : kStages;
        for (int i = 0; i < pre; ++i) {
          mbar_arrive_expect_tx(&full[i], C::kStageBytes);
          if constexpr (kWeightA)
            tma_load_2d(sA + i * C::kABytes, &tmA, &full[i], (kb0 + i) * C::kBK, (tile % tiles_m) * kBM);
          else
            load_b(i, kb0 + i, (tile / tiles_m) * BN);
          issued |= 1u << i;
        }
      }
      griddep_wait();
      for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
        const int tile = u / splits, split = u - tile * splits;
        const int m0 = (tile % tiles_m) * kBM, n0 = (tile / tiles_m) * BN;
        const int kb0 = split * num_kb / splits, kb1 = (split + 1) * num_kb / splits;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, 0x100u | stage, limit)) { ok = false; break; }
          if (pre > 0) {
            --pre;   // this stage's weight tile and byte count are in flight already
          } else {
            mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
            if constexpr (kWeightA)
              tma_load_2d(sA + stage * C::kABytes, &tmA, &full[stage], kb * C::kBK, m0);
            else
              load_b(stage, kb, n0);
          }
          if constexpr (kWeightA)
            load_b(stage, kb, n0);
          else
            tma_load_2d(sA + stage * C::kABytes, &tmA, &full[stage], kb * C::kBK, m0);
          issued |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      // Teardown: every copy this thread started has landed before the block
      // can exit (a no-op on the normal path, where the MMAs consumed them).
      for (int s = 0; s < kStages; ++s)
        if (issued & (1u << s)) mbar_wait(&full[s], (issued_phase >> s) & 1u, nullptr, 0x180u | s, limit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
        const int split = u % splits;
        const int kb0 = split * num_kb / splits, kb1 = (split + 1) * num_kb / splits;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, 0x200u | acc, limit)) break;
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, 0x300u | stage, limit)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * C::kABytes);
          const uint32_t b_base = smem_u32(sB + stage * C::kBBytes);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = sdesc_sw128(a_base + k * 32, 16, 1024);
            const uint64_t bd = B_MN ? sdesc_sw128(b_base + k * (C::kMmaK * 128), C::kBK * 128, 1024)
                                     : sdesc_sw128(b_base + k * 32, 16, 1024);
            tc_mma<KIND>(d, ad, bd, kIdesc, (kb > kb0 || k > 0) ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      // Teardown: all MMAs issued by this thread have completed.
      tc_commit(teardown);
      mbar_wait(teardown, 0, nullptr, 0x380u, limit);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    griddep_wait();                               // row scales come from the previous kernel
    const int e = warp - 2;                       // epilogue warp index
    const int quarter = warp & 3;                 // TMEM lanes this warp may read
    const int group = e >> 2;                     // column-chunk interleave
    constexpr int kGroups = C::kEpiWarps / 4;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    int acc = 0;
    uint32_t acc_phase = 0;
    int local = 0;
    uint32_t out_iter = 0;
    for (int u = blockIdx.x; u < num_units; u += gridDim.x, ++local) {
      const int tile = u / splits, split = u - tile * splits;
      const int m0 = (tile % tiles_m) * kBM, n0 = (tile / tiles_m) * BN;
      if constexpr (EPI == kEpiLowRank) {
        // Every epilogue thread is done with the previous tile's L2^T before it
        // is overwritten.
        if (local > 0 && !__all_sync(0xFFFFFFFFu, mbar_wait(lr_done, (local - 1) & 1, abort_flag, 0x500u, limit)))
          break;
        stage_l2t<BN, kEpiThreads>(ep, sLr, n0, N, threadIdx.x - 64);
        mbar_arrive(lr_ready);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(lr_ready, local & 1, abort_flag, 0x600u, limit))) break;
      }
      // Transposed form: the token scales of this warp's first chunk, the
      // weight row's scale and its bias are loaded before the wait, so that
      // their latency overlaps the MMAs.
      float sx_first[32];
      float swr = 0.0f, br = 0.0f;
      if constexpr (EPI == kEpiScaleT) {
        const int nc = n0 + group * 32;
        if (nc + 32 <= N) {
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const float4 f = __ldg(reinterpret_cast<const float4*>(ep.s_row + nc + j));
            sx_first[j] = f.x; sx_first[j + 1] = f.y; sx_first[j + 2] = f.z; sx_first[j + 3] = f.w;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) sx_first[j] = (nc + j < N) ? __ldg(ep.s_row + nc + j) : 0.0f;
        }
        const int row = m0 + quarter * 32 + lane;   // n
        if (row < M) {
          swr = ep.s_col_axis ? __ldg(ep.s_col + row) : __ldg(ep.s_col);
          if (ep.bias != nullptr) br = __bfloat162float(ep.bias[row]);
        }
      }
      // Every lane polls; the warp then agrees (and reconverges) before the
      // warp-collective tcgen05.ld, also when the wait ran out.
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&tfull[acc], acc_phase, abort_flag, 0x400u | acc, limit))) break;
      tc_fence_after();
      if constexpr (EPI == kEpiLowRank) {
        epilogue_lowrank_tile<KIND, BN, kGroups>(ep, &tmY, tmem + static_cast<uint32_t>(acc * BN), m0, n0, M, N,
                                                 quarter, group, lane, sLr, sOut + e * 2 * C::kOutBufBytes, out_iter);
      } else if constexpr (EPI == kEpiScaleT) {
        // Transposed product (few tokens): the kernel's rows are weight rows n
        // (A = the weight codes) and its columns tokens m (B = the activation
        // codes), so a lane holds y[m, n] for one n and the chunk's 32 m.
        // y[m, n] = bf16(((acc * s_x[m]) * s_w[n or 0]) + bias[n]) - the fp32
        // steps of the other epilogues - is stored for each m, 32 lanes
        // writing 32 consecutive n; split partial sums go to partial[split][m][n].
        const int row = m0 + quarter * 32 + lane;   // n
        const bool row_ok = row < M;
  #pragma unroll 1
        for (int c = group; c < BN / 32; c += kGroups) {
          const int nc = n0 + c * 32;               // first token of the chunk
          if (nc >= N) break;                       // warp-uniform
          float sxc[32];
          if (c == group) {
  #pragma unroll
            for (int j = 0; j < 32; ++j) sxc[j] = sx_first[j];
          } else {
  #pragma unroll
            for (int j = 0; j < 32; ++j) sxc[j] = (nc + j < N) ? __ldg(ep.s_row + nc + j) : 0.0f;
          }
          uint32_t r[32];
          tmem_ld_x32(tmem + lane_base + static_cast<uint32_t>(acc * BN + c * 32), r);
          tmem_ld_wait();
          if (row_ok) {
            if (splits > 1) {
              uint32_t* pcol = ep.partial + static_cast<int64_t>(split) * N * M + row;
              for (int j = 0; j < 32; ++j)
                if (nc + j < N && in_bounds((static_cast<int64_t>(split) * N + nc + j) * M + row,
                                            static_cast<int64_t>(splits) * N * M, 0xB103))
                  pcol[static_cast<int64_t>(nc + j) * M] = r[j];
            } else if (!ep.tma_store) {
              for (int j = 0; j < 32; ++j) {
                if (nc + j < N && in_bounds(static_cast<int64_t>(nc + j) * ep.ldy + row,
                                            static_cast<int64_t>(N) * ep.ldy, 0xB106)) {
                  float a = (KIND == kKindI8) ? __int2float_rn(static_cast<int>(r[j])) : __uint_as_float(r[j]);
                  a = __fmul_rn(__fmul_rn(a, sxc[j]), swr);
                  if (ep.bias != nullptr) a = __fadd_rn(a, br);
                  ep.y[static_cast<int64_t>(nc + j) * ep.ldy + row] = __float2bfloat16_rn(a);
                }
              }
            }
          }
          if (splits == 1 && ep.tma_store) {
            // the 32 tokens x 32 weight rows block, staged transposed (token j's
            // 64-byte row, this lane's column, 64-byte swizzle) and stored by
            // TMA; rows and columns past the output are clipped by the copy
            uint8_t* buf = sOut + e * 2 * C::kOutBufBytes + (out_iter & 1) * C::kOutBufBytes;
            if (lane == 0) bulk_wait_read<1>();   // this buffer's previous store has read it
            __syncwarp();
  #pragma unroll
            for (int j = 0; j < 32; ++j) {
              float a = (KIND == kKindI8) ? __int2float_rn(static_cast<int>(r[j])) : __uint_as_float(r[j]);
              a = __fmul_rn(__fmul_rn(a, sxc[j]), swr);
              if (ep.bias != nullptr) a = __fadd_rn(a, br);
              const uint32_t chunk = static_cast<uint32_t>(lane >> 3) ^ static_cast<uint32_t>((j >> 1) & 3);
              *reinterpret_cast<__nv_bfloat16*>(buf + j * 64 + (chunk << 4) + (lane & 7) * 2) = __float2bfloat16_rn(a);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmY, buf, m0 + quarter * 32, nc);
              bulk_commit();
            }
            ++out_iter;
          }
        }
      } else {
        const int row = m0 + quarter * 32 + lane;
        const bool row_ok = row < M;
        float sx = 1.0f;
        if constexpr (EPI != kEpiPlain) sx = row_ok ? ep.s_row[row] : 0.0f;
        const float sw0 = (EPI != kEpiPlain && !ep.s_col_axis) ? ep.s_col[0] : 1.0f;
        const bool vec_partial = (N & 3) == 0;      // partial rows are 16-byte aligned
        bool write_out = true;
        if (splits > 1) {
          // This unit's raw sums -> partial[split][row][n] (valid rows only).
          uint32_t* prow = ep.partial + (static_cast<int64_t>(split) * M + (row_ok ? row : 0)) * N;
  #pragma unroll 1
          for (int c = group; c < BN / 32; c += kGroups) {
            const int nc = n0 + c * 32;
            if (nc >= N) break;                     // warp-uniform
            uint32_t r[32];
            tmem_ld_x32(tmem + lane_base + static_cast<uint32_t>(acc * BN + c * 32), r);
            tmem_ld_wait();
            if (row_ok && in_bounds((static_cast<int64_t>(split) * M + row) * N + nc, static_cast<int64_t>(splits) * M * N,
                                    0xB103)) {
              if (vec_partial && nc + 32 <= N) {
  #pragma unroll
                for (int j = 0; j < 32; j += 4)
                  *reinterpret_cast<uint4*>(prow + nc + j) = make_uint4(r[j], r[j + 1], r[j + 2], r[j + 3]);
              } else {
                for (int j = 0; j < 32; ++j)
                  if (nc + j < N) prow[nc + j] = r[j];
              }
            }
          }
          write_out = false;   // splitk_epilogue_kernel finishes the tile
        }
        if (write_out)
          epilogue_scale_chunks<KIND, EPI, BN, kGroups, kAxisOk>(ep, &tmY, tmem + lane_base + static_cast<uint32_t>(acc * BN),
                                                                 m0, n0, M, N, quarter, group, lane, sx, sw0,
                                                                 sOut + e * 2 * C::kOutBufBytes, out_iter);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if constexpr (EPI == kEpiLowRank) mbar_arrive(lr_done);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    // the staging buffers must outlive the stores that read them
    if (ep.tma_store && lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Finish a split-K product:  y[m, n] = bf16( ((sum_s partial[s][m][n]) * s_x[m]) * s_w[n or 0] + bias[n] ),
// the partial sums added in split order and every other step the fp32 RN
// operation of the fused epilogue, so the result equals the unsplit one
// (int8) or is reproducible (e4m3).  KIND = kKindBF16 is the plain form:
// y = bf16(sum_s partial (+ bias[n])), fp32 sums in split order, no scales.
// 8 columns per thread: N % 8 == 0, y contiguous [M, N].
template <int KIND>
__global__ void __launch_bounds__(256) splitk_epilogue_kernel(const uint32_t* __restrict__ partial, int splits,
                                                              int64_t M, int64_t N, const float* __restrict__ s_row,
                                                              const float* __restrict__ s_col, int axis,
                                                              const __nv_bfloat16* __restrict__ bias,
                                                              __nv_bfloat16* __restrict__ y, int act = kActNone,
                                                              uint32_t* __restrict__ y_amax = nullptr) {
  griddep_launch();
  griddep_wait();   // the partial sums come from the GEMM just before
  const int64_t n8 = N >> 3;
  const int64_t total = M * n8;
  const int64_t plane = M * N;
  for (int64_t i = blockIdx.x * 256ll + threadIdx.x; i < total; i += static_cast<int64_t>(gridDim.x) * 256) {
    const int64_t m = i / n8, n = (i - m * n8) * 8;
    if (!in_bounds(m, M, 0xB107) || !in_bounds(n + 7, N, 0xB107)) continue;
    const uint4* p = reinterpret_cast<const uint4*>(partial + m * N + n);
    uint4 lo = __ldcg(p), hi = __ldcg(p + 1);
    uint32_t r[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll 4
    for (int sp = 1; sp < splits; ++sp) {
      const uint4* q = reinterpret_cast<const uint4*>(partial + sp * plane + m * N + n);
      lo = __ldcg(q);
      hi = __ldcg(q + 1);
      const uint32_t t[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
      for (int j = 0; j < 8; ++j)
        r[j] = (KIND == kKindI8) ? r[j] + t[j] : __float_as_uint(__fadd_rn(__uint_as_float(r[j]), __uint_as_float(t[j])));
    }
    if constexpr (KIND == kKindBF16) {
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(r[j]);
      if (bias != nullptr) {
        const uint4 b = __ldg(reinterpret_cast<const uint4*>(bias + n));
        v[0] = __fadd_rn(v[0], bf16_lo(b.x)); v[1] = __fadd_rn(v[1], bf16_hi(b.x));
        v[2] = __fadd_rn(v[2], bf16_lo(b.y)); v[3] = __fadd_rn(v[3], bf16_hi(b.y));
        v[4] = __fadd_rn(v[4], bf16_lo(b.z)); v[5] = __fadd_rn(v[5], bf16_hi(b.z));
        v[6] = __fadd_rn(v[6], bf16_lo(b.w)); v[7] = __fadd_rn(v[7], bf16_hi(b.w));
      }
      *reinterpret_cast<uint4*>(y + m * N + n) =
          make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
      continue;
    }
    const float sx = s_row[m];
    float sw[8], bs[8];
    if (axis) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(s_col + n));
      const float4 b = __ldg(reinterpret_cast<const float4*>(s_col + n) + 1);
      sw[0] = a.x; sw[1] = a.y; sw[2] = a.z; sw[3] = a.w; sw[4] = b.x; sw[5] = b.y; sw[6] = b.z; sw[7] = b.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) sw[j] = s_col[0];
    }
    if (bias != nullptr) {
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(bias + n));
      bs[0] = bf16_lo(b.x); bs[1] = bf16_hi(b.x); bs[2] = bf16_lo(b.y); bs[3] = bf16_hi(b.y);
      bs[4] = bf16_lo(b.z); bs[5] = bf16_hi(b.z); bs[6] = bf16_lo(b.w); bs[7] = bf16_hi(b.w);
    }
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float a = (KIND == kKindI8) ? __int2float_rn(static_cast<int>(r[j])) : __uint_as_float(r[j]);
      a = __fmul_rn(__fmul_rn(a, sx), sw[j]);
      if (bias != nullptr) a = __fadd_rn(a, bs[j]);
      v[j] = (act != kActNone) ? apply_act(a, act) : a;
    }
    const uint4 out = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                 pack_bf16x2(v[6], v[7]));
    *reinterpret_cast<uint4*>(y + m * N + n) = out;
    if (y_amax != nullptr)
      row_amax_commit(y_amax, m, bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(0u, out.x), out.y), out.z), out.w));
  }
}

}  // namespace w8a8
