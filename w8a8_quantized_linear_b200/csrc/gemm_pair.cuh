// gemm_pair.cuh - the 8-bit GEMM with the scale epilogue on CTA pairs: a
// cluster of two CTAs on two SMs computes a 256 x 256 tile with one
// tcgen05.mma.cta_group::2 stream (M = 256: 128 rows in each CTA's shared
// memory and TMEM; B split along N, 128 rows or columns in each CTA).  Per
// SM this moves 32 KB per 128-byte K step instead of the 48 KB of the
// single-SM 128 x 256 tile, for the same MMA work.
//
//   D[m, n] = sum_k A[m, k] * B[n, k]    (B K-major: the forward)
//   D[m, n] = sum_k A[m, k] * B[k, n]    (B MN-major: the dgrad)
//
// Roles per CTA (320 threads), as in gemm_kernel:
//   warp 0      TMA producer: this CTA's A rows and B half into its own stage
//               ring; the bytes of both CTAs complete on the even CTA's
//               `full` barrier, whose one arrival (with the byte count of
//               both) comes from the even CTA's producer;
//   warp 1      TMEM (cta_group::2 allocation in both CTAs); in the even CTA
//               one thread issues the pair's MMAs and commits each stage to
//               the `empty` barriers of both CTAs, each finished tile to the
//               `tfull` barriers of both;
//   warps 2..9  epilogue on this CTA's 128 rows x 256 columns (the code of
//               gemm_kernel), releasing the accumulator on the even CTA's
//               `tempty` barrier (16 warps arrive per tile).
// Two TMEM buffers of 256 columns: a tile's epilogue overlaps the next
// tile's MMAs.  At the end the two CTAs hand over (bounded waits) before
// TMEM is freed: the odd CTA's epilogue is done, the even CTA's MMAs have
// completed.  Every wait is bounded; no TMA multicast.
//
// LR, the SVDQuant form, y = bf16((((acc s_x) s_w) + bias) + T L2): the
// low-rank product is a bf16 tensor-core MMA of the pair (M = 256, K = 16 per
// instruction, r <= 32 padded to whole steps) written into the SAME TMEM
// buffer as the tile's int32 / fp32 sums once the epilogue has read them, in
// two halves of the tile's columns (N = 128 each):
//   1. the epilogue warps read the sums of columns [128 h, 128 h + 128) and
//      keep the fp32 values ((acc s_x) s_w) + bias in registers (64 per thread);
//   2. they hand those TMEM columns back (`lrreq`); warp 10 of the even CTA,
//      whose one thread issues only these products, multiplies the tile's T
//      rows [128 per CTA x r] by L2 columns [r x 64 per CTA] into them, from
//      zero, and commits `lrfull` (a thread's commit tracks the MMAs that
//      thread issued, and the two issuers write different TMEM buffers, so
//      the main MMA thread keeps its plain waits).  Each CTA's L2 tile holds
//      columns [64 rank, +64) and [128 + 64 rank, +64) of the pair tile, so
//      that half h of the pair MMA (64 columns from each CTA) lands exactly on
//      TMEM columns [128 h, 128 h + 128);
//   3. the epilogue reads the fp32 low-rank sums, adds them with one RN add
//      and stores bf16; then the next half.
// T and L2 come in by TMA once per tile (r zero-filled).  So the low-rank term
// costs two small MMAs per tile on the tensor pipe, and the double buffering
// of the plain kernel is kept.
#pragma once
#include "gemm.cuh"

namespace w8a8 {

template <int KIND, bool LR>
struct PairCfg {
  static constexpr int kBN = 256;                  // pair tile N (each CTA holds 128 rows or columns of B)
  static constexpr int kBHalf = kBN / 2;
  static constexpr int kBK = kBKBytes / (KIND == kKindBF16 ? 2 : 1);   // K elements per 128-byte stage row
  static constexpr int kABytes = kBM * kBKBytes;   // 16 KB: this CTA's 128 rows of A
  static constexpr int kBBytes = kBHalf * kBKBytes;   // 16 KB: this CTA's half of B
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = LR ? 5 : 6;
  static constexpr int kTmemCols = 512;            // two buffers of 256 columns
  static constexpr int kTBytes = LR ? kBM * 128 : 0;       // T tile: 128 rows x 64 bf16 (r zero-padded)
  static constexpr int kL2Bytes = LR ? 2 * 32 * 128 : 0;   // L2 tile: 32 rows x 128 bf16 (two 64-column boxes)
  static constexpr int kEpiWarps = 8;
  static constexpr int kThreads = 64 + 32 * kEpiWarps + (LR ? 32 : 0);   // LR: warp 10 issues the low-rank MMAs
  static constexpr int kOutBufBytes = 32 * 32 * 2;
  static constexpr int kOutBytes = kEpiWarps * 2 * kOutBufBytes;
  static constexpr size_t kSmem =
      1024 + static_cast<size_t>(kStages) * kStageBytes + kTBytes + kL2Bytes + kOutBytes + 256;
  static_assert(kSmem <= 232448, "shared memory per block");
};

// One epilogue warp's staged TMA store of a 32 x 32 bf16 block (rows
// rbase.., columns nc..) from fp32 values v (this lane's row), through one
// of its two 64-byte-swizzled staging buffers; or direct stores when the
// output row stride is not a multiple of 8.
__device__ __forceinline__ void store_block_bf16(const EpiParams& ep, const CUtensorMap* tmY, const float (&v)[32],
                                                 int rbase, int nc, int M, int N, int lane, uint8_t* sOutWarp,
                                                 uint32_t& out_iter) {
  if (ep.tma_store) {
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
    if (lane == 0 && rbase < M) {
      tma_store_2d(tmY, buf, nc, rbase);
      bulk_commit();
    }
    ++out_iter;
  } else if (rbase + lane < M && in_bounds(rbase + lane, M, 0xB201) && in_bounds(nc, N, 0xB201)) {
    __nv_bfloat16* out = ep.y + static_cast<int64_t>(rbase + lane) * ep.ldy + nc;
    for (int j = 0; j < 32; ++j)
      if (nc + j < N) out[j] = __float2bfloat16_rn(v[j]);
  }
}

template <int KIND, bool B_MN, bool LR = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<KIND, LR>::kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmT,
                     const __grid_constant__ CUtensorMap tmL2, int M, int N, int Kc, EpiParams ep) {
  using C = PairCfg<KIND, LR>;
  static_assert(KIND != kKindBF16 || !LR, "bf16 operands: no low-rank branch");
  // bf16 operands (the weight-only Linear): y = bf16(acc (+ bias)), no scales
  constexpr int kEpi = (KIND == kKindBF16) ? kEpiPlain : kEpiScale;
  constexpr int BN = C::kBN;
  constexpr uint32_t kIdesc = idesc<KIND>(2 * kBM, BN, B_MN);
  constexpr uint32_t kIdescLr = idesc<kKindBF16>(2 * kBM, BN / 2, true);   // T K-major, L2 MN-major, half the columns
  constexpr int kStages = C::kStages;
  constexpr int kGroups = C::kEpiWarps / 4;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                                  // kStages x 16 KB
  uint8_t* sB = smem + kStages * C::kABytes;           // kStages x kBBytes
  uint8_t* sT = smem + kStages * C::kStageBytes;       // LR: 16 KB
  uint8_t* sL2 = sT + C::kTBytes;                      // LR: 8 KB
  uint8_t* sOut = sL2 + C::kL2Bytes;                   // epilogue staging
  uint64_t* full = reinterpret_cast<uint64_t*>(sOut + C::kOutBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* teardown = tempty + 2;
  uint64_t* handover = teardown + 1;
  uint64_t* lrreq = handover + 1;                      // LR [buffer][half]: the epilogue read those sums (even CTA's)
  uint64_t* lrfull = lrreq + 4;                        // LR [buffer][half]: the low-rank sums are there
  uint64_t* tlfull = lrfull + 4;                       // LR: the tile's T and L2 landed (even CTA's)
  uint64_t* tlempty = tlfull + 1;                      // LR: the low-rank MMAs read them
  uint64_t* lrdrain = tlempty + 1;                     // LR: the low-rank issuer's MMAs completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lrdrain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();   // 0: issues the MMAs
  const bool leader = rank == 0;
  const uint64_t limit = g_wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * C::kEpiWarps);   // the epilogue warps of both CTAs
      for (int h = 0; h < 2; ++h) {
        mbar_init(&lrreq[2 * a + h], 2 * C::kEpiWarps);
        mbar_init(&lrfull[2 * a + h], 1);
      }
    }
    mbar_init(teardown, 1);
    mbar_init(handover, 1);
    mbar_init(tlfull, 1);
    mbar_init(tlempty, 1);
    mbar_init(lrdrain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (ep.tma_store) tma_prefetch_desc(&tmY);
    if constexpr (LR) {
      tma_prefetch_desc(&tmT);
      tma_prefetch_desc(&tmL2);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();   // both CTAs' barriers exist before either reaches the other's
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_launch();

  const int tiles_m = (M + 2 * kBM - 1) / (2 * kBM);
  const int tiles_n = (N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int num_kb = (Kc + C::kBK - 1) / C::kBK;
  const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_phase = 0;
      uint32_t tl_phase = 0;
      bool tl_issued = false;
      bool ok = true;
      griddep_wait();
      for (int tile = pair; ok && tile < num_tiles; tile += num_pairs) {
        const int m0 = (tile % tiles_m) * (2 * kBM) + static_cast<int>(rank) * kBM;
        const int nh = (tile / tiles_m) * BN + static_cast<int>(rank) * C::kBHalf;   // this CTA's half of B
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, 0x100u | stage, limit)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::kStageBytes);
          const uint32_t fb = mapa_shared(&full[stage], 0);   // the even CTA's full[stage]
          tma_load_2d_pair(sA + stage * C::kABytes, &tmA, fb, kb * C::kBK, m0);
          if constexpr (!B_MN) {
            tma_load_2d_pair(sB + stage * C::kBBytes, &tmB, fb, kb * C::kBK, nh);
          } else if constexpr (KIND != kKindBF16) {
            tma_load_2d_pair(sB + stage * C::kBBytes, &tmB, fb, nh, kb * C::kBK);
          } else {
            // bf16 MN-major: this CTA's 128 columns are two 128-byte atoms of
            // 64 columns, each [64 K rows][128 B]
            tma_load_2d_pair(sB + stage * C::kBBytes, &tmB, fb, nh, kb * C::kBK);
            tma_load_2d_pair(sB + stage * C::kBBytes + C::kBK * 128, &tmB, fb, nh + 64, kb * C::kBK);
          }
          issued |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if constexpr (LR) {
          // This tile's T rows and L2 columns, once the previous tile's
          // low-rank MMAs have read the buffers.
          if (ok && !mbar_wait(tlempty, tl_phase ^ 1u, abort_flag, 0x700u, limit)) ok = false;
          if (ok) {
            if (leader) mbar_arrive_expect_tx(tlfull, 2 * (C::kTBytes + C::kL2Bytes));
            const uint32_t lb = mapa_shared(tlfull, 0);
            const int n0 = (tile / tiles_m) * BN + static_cast<int>(rank) * 64;
            tma_load_2d_pair(sT, &tmT, lb, 0, m0);
            tma_load_2d_pair(sL2, &tmL2, lb, n0, 0);                 // half 0 of the low-rank product
            tma_load_2d_pair(sL2 + 32 * 128, &tmL2, lb, n0 + 128, 0);  // half 1
            tl_issued = true;
            tl_phase ^= 1u;
          }
        }
      }
      // Teardown (even CTA): every stage filled has completed.  The odd
      // CTA's copies complete on the even CTA's barriers; the hand-over at
      // the end keeps it resident until the MMAs have read them.
      if (leader) {
        for (int s = 0; s < kStages; ++s)
          if (issued & (1u << s)) mbar_wait(&full[s], (issued_phase >> s) & 1u, nullptr, 0x180u | s, limit);
        if (LR && tl_issued) mbar_wait(tlfull, tl_phase ^ 1u, nullptr, 0x780u, limit);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (leader && lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < num_tiles; tile += num_pairs) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, 0x200u | acc, limit)) break;
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(acc * 256);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, 0x300u | stage, limit)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * C::kABytes);
          const uint32_t b_base = smem_u32(sB + stage * C::kBBytes);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = sdesc_sw128(a_base + k * 32, 16, 1024);
            // MN-major B: an MMA's K rows (32 codes or 16 bf16) are rows of
            // 128 bytes; bf16 atoms of 64 columns lie kBK rows apart (LBO)
            const uint64_t bd = !B_MN ? sdesc_sw128(b_base + k * 32, 16, 1024)
                                : (KIND == kKindBF16 ? sdesc_sw128(b_base + k * (16 * 128), C::kBK * 128, 1024)
                                                     : sdesc_sw128(b_base + k * (32 * 128), 16, 1024));
            tc_mma_pair<KIND>(d, ad, bd, kIdesc, (kb > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair_mc(&tfull[acc], 0x3);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      tc_commit_pair(teardown);
      mbar_wait(teardown, 0, nullptr, 0x380u, limit);
    }
  } else if (LR && warp == 2 + C::kEpiWarps) {
    // ------------------------------------------------------------ low-rank MMA issuer (even CTA)
    if (leader && lane == 0) {
      // tile t's two halves (columns 0-127, 128-255 of TMEM buffer t % 2), in order
      int t = 0;
      for (int tile = pair; tile < num_tiles; tile += num_pairs, ++t) {
        const int b = t & 1;
        bool ok = true;
        for (int h = 0; ok && h < 2; ++h) {
          if (!mbar_wait(&lrreq[2 * b + h], static_cast<uint32_t>(t >> 1) & 1u, abort_flag, 0x880u | (2 * b + h), limit) ||
              (h == 0 && !mbar_wait(tlfull, static_cast<uint32_t>(t) & 1u, abort_flag, 0x800u, limit))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + static_cast<uint32_t>(b * 256 + h * 128);
          const uint32_t t_base = smem_u32(sT), l_base = smem_u32(sL2 + h * (32 * 128));
          const int nks = (ep.r + 15) / 16;
          for (int k = 0; k < nks; ++k)
            tc_mma_pair<kKindBF16>(d, sdesc_sw128(t_base + k * 32, 16, 1024),
                                   sdesc_sw128(l_base + k * (16 * 128), 32 * 128, 1024), kIdescLr, k > 0 ? 1u : 0u);
          if (h == 1) tc_commit_pair_mc(tlempty, 0x3);
          tc_commit_pair_mc(&lrfull[2 * b + h], 0x3);
        }
        if (!ok) break;
      }
      // Teardown: every low-rank MMA issued by this thread has completed.
      tc_commit_pair(lrdrain);
      mbar_wait(lrdrain, 0, nullptr, 0x8C0u, limit);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    griddep_wait();
    const int e = warp - 2;
    const int quarter = warp & 3;
    const int group = e >> 2;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t out_iter = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs) {
      const int m0 = (tile % tiles_m) * (2 * kBM) + static_cast<int>(rank) * kBM;
      const int n0 = (tile / tiles_m) * BN;
      // the row's scales are loaded before the wait, so that their latency
      // overlaps it
      const int row = m0 + quarter * 32 + lane;
      float sx = 1.0f, sw0 = 1.0f;
      if constexpr (kEpi != kEpiPlain) {
        sx = row < M ? ep.s_row[row] : 0.0f;
        sw0 = ep.s_col_axis ? 1.0f : ep.s_col[0];
      }
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&tfull[acc], acc_phase, abort_flag, 0x400u | acc, limit))) break;
      tc_fence_after();
      const uint32_t tacc = tmem + lane_base + static_cast<uint32_t>(acc * 256);
      if constexpr (!LR) {
        epilogue_scale_chunks<KIND, kEpi, BN, kGroups, true>(ep, &tmY, tacc, m0, n0, M, N, quarter, group, lane, sx,
                                                             sw0, sOut + e * 2 * C::kOutBufBytes, out_iter);
      } else {
        // per half h of the columns, this warp's chunks c = group + kGroups i
        // (i = 0, 1) of the half: v = ((acc s_x) s_w) + bias, hand the TMEM
        // columns back, then y = bf16(v + lr), one RN add
        constexpr int kHalfChunks = BN / 64 / kGroups;
        bool ok = true;
#pragma unroll 1
        for (int h = 0; ok && h < 2; ++h) {
          // both chunks' TMEM loads in flight before one wait
          float v[kHalfChunks][32];
          {
            uint32_t r[kHalfChunks][32];
#pragma unroll
            for (int i = 0; i < kHalfChunks; ++i)
              tmem_ld_x32(tacc + static_cast<uint32_t>((h * (BN / 64) + group + kGroups * i) * 32), r[i]);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < kHalfChunks; ++i) {
              const int nc = n0 + (h * (BN / 64) + group + kGroups * i) * 32;
              float bs[32];
              if (ep.bias != nullptr) {
                if (nc + 32 <= N) {
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
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                float a = (KIND == kKindI8) ? __int2float_rn(static_cast<int>(r[i][j])) : __uint_as_float(r[i][j]);
                a = __fmul_rn(__fmul_rn(a, sx), sw0);
                if (ep.bias != nullptr) a = __fadd_rn(a, bs[j]);
                v[i][j] = a;
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(mapa_shared(&lrreq[2 * acc + h], 0));
          ok = __all_sync(0xFFFFFFFFu, mbar_wait(&lrfull[2 * acc + h], acc_phase, abort_flag, 0x480u | (2 * acc + h), limit));
          if (!ok) break;
          tc_fence_after();
          {
            uint32_t r[kHalfChunks][32];
#pragma unroll
            for (int i = 0; i < kHalfChunks; ++i)
              tmem_ld_x32(tacc + static_cast<uint32_t>((h * (BN / 64) + group + kGroups * i) * 32), r[i]);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < kHalfChunks; ++i) {
              const int nc = n0 + (h * (BN / 64) + group + kGroups * i) * 32;
              if (nc < N) {                           // warp-uniform
#pragma unroll
                for (int j = 0; j < 32; ++j) v[i][j] = __fadd_rn(v[i][j], __uint_as_float(r[i][j]));
                store_block_bf16(ep, &tmY, v[i], m0 + quarter * 32, nc, M, N, lane, sOut + e * 2 * C::kOutBufBytes,
                                 out_iter);
              }
            }
          }
        }
        if (!ok) break;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(&tempty[acc], 0));   // the even CTA's barrier
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (ep.tma_store && lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  // Hand-over: the odd CTA reports that its epilogue is done; the even CTA
  // (whose MMAs have completed) answers; then both free the pair's TMEM.
  if (warp == 1) {
    if (lane == 0) {
      if (!leader) {
        mbar_arrive_cluster(mapa_shared(handover, 0));
        mbar_wait(handover, 0, nullptr, 0x600u, limit);
      } else {
        mbar_wait(handover, 0, nullptr, 0x600u, limit);
        mbar_arrive_cluster(mapa_shared(handover, 1));
      }
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::kTmemCols);
  }
}

}  // namespace w8a8
