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
// At the end the two CTAs hand over (bounded waits) before TMEM is freed:
// the odd CTA's epilogue is done, the even CTA's MMAs have completed.
// Every wait is bounded; no TMA multicast.
#pragma once
#include "gemm.cuh"

namespace w8a8 {

// LR: the SVDQuant form.  TMEM holds one buffer of the int32 sums (256
// columns) and the fp32 low-rank sums T L2 (256 columns), so the epilogue
// of a tile does not overlap the next tile's MMAs; the stage ring is one
// stage shorter to make room for the T and L2 tiles.  Per tile, after the
// int8 MMAs, bf16 MMAs (r <= 32 in K steps of 16) multiply the tile's T
// [128 rows x r per CTA] by its L2 [r x 128 columns per CTA], both brought
// in by TMA once per tile (r padded to 64 columns and 32 rows by the TMA
// zero fill).
template <int KIND, bool LR>
struct PairCfg {
  static constexpr int kBN = 256;                  // pair tile N (each CTA holds 128 rows or columns of B)
  static constexpr int kBHalf = kBN / 2;
  static constexpr int kBK = kBKBytes / (KIND == kKindBF16 ? 2 : 1);   // K elements per 128-byte stage row
  static constexpr int kABytes = kBM * kBKBytes;   // 16 KB: this CTA's 128 rows of A
  static constexpr int kBBytes = kBHalf * kBKBytes;   // 16 KB: this CTA's half of B
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = LR ? 5 : 6;
  static constexpr int kAccBufs = LR ? 1 : 2;      // TMEM buffers of 256 columns (+ 256 low-rank with LR)
  static constexpr int kTmemCols = 512;
  static constexpr int kTBytes = LR ? kBM * 128 : 0;       // T tile: 128 rows x 64 bf16 (r zero-padded)
  static constexpr int kL2Bytes = LR ? 2 * 32 * 128 : 0;   // L2 tile: 32 rows x 128 bf16 (two 64-column boxes)
  static constexpr int kEpiWarps = 8;
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  static constexpr int kOutBufBytes = 32 * 32 * 2;
  static constexpr int kOutBytes = kEpiWarps * 2 * kOutBufBytes;
  static constexpr size_t kSmem =
      1024 + static_cast<size_t>(kStages) * kStageBytes + kTBytes + kL2Bytes + kOutBytes + 256;
  static_assert(kSmem <= 232448, "shared memory per block");
};

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
  constexpr uint32_t kIdescLr = idesc<kKindBF16>(2 * kBM, BN, true);   // T K-major, L2 MN-major
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
  uint64_t* lrfull = handover + 1;                     // LR: T and L2 tiles landed (even CTA's)
  uint64_t* lrempty = lrfull + 1;                      // LR: the low-rank MMAs read them
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lrempty + 1);
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
    }
    mbar_init(teardown, 1);
    mbar_init(handover, 1);
    mbar_init(lrfull, 1);
    mbar_init(lrempty, 1);
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
      uint32_t lr_phase = 0;
      bool lr_issued = false;
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
          // low-rank MMAs have read the buffers (long done by now: they ran
          // before this tile's first MMA).
          if (ok && !mbar_wait(lrempty, lr_phase ^ 1u, abort_flag, 0x700u, limit)) ok = false;
          if (ok) {
            if (leader) mbar_arrive_expect_tx(lrfull, 2 * (C::kTBytes + C::kL2Bytes));
            const uint32_t lb = mapa_shared(lrfull, 0);
            tma_load_2d_pair(sT, &tmT, lb, 0, m0);
            tma_load_2d_pair(sL2, &tmL2, lb, nh, 0);
            tma_load_2d_pair(sL2 + 32 * 128, &tmL2, lb, nh + 64, 0);
            lr_issued = true;
            lr_phase ^= 1u;
          }
        }
      }
      // Teardown (even CTA): every stage filled has completed.  The odd
      // CTA's copies complete on the even CTA's barriers; the hand-over at
      // the end keeps it resident until the MMAs have read them.
      if (leader) {
        for (int s = 0; s < kStages; ++s)
          if (issued & (1u << s)) mbar_wait(&full[s], (issued_phase >> s) & 1u, nullptr, 0x180u | s, limit);
        if (LR && lr_issued) mbar_wait(lrfull, lr_phase ^ 1u, nullptr, 0x780u, limit);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (leader && lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0, lr_phase = 0;
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
        if constexpr (LR) {
          // T L2 into the buffer's second 128 columns, from zero, fp32
          if (!mbar_wait(lrfull, lr_phase, abort_flag, 0x800u, limit)) break;
          tc_fence_after();
          const uint32_t t_base = smem_u32(sT), l_base = smem_u32(sL2);
          const int nks = (ep.r + 15) / 16;
          for (int k = 0; k < nks; ++k)
            tc_mma_pair<kKindBF16>(d + BN, sdesc_sw128(t_base + k * 32, 16, 1024),
                                   sdesc_sw128(l_base + k * (16 * 128), 32 * 128, 1024), kIdescLr, k > 0 ? 1u : 0u);
          tc_commit_pair_mc(lrempty, 0x3);
          lr_phase ^= 1u;
        }
        tc_commit_pair_mc(&tfull[acc], 0x3);
        if (++acc == C::kAccBufs) { acc = 0; acc_phase ^= 1u; }
      }
      tc_commit_pair(teardown);
      mbar_wait(teardown, 0, nullptr, 0x380u, limit);
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
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&tfull[acc], acc_phase, abort_flag, 0x400u | acc, limit))) break;
      tc_fence_after();
      const int row = m0 + quarter * 32 + lane;
      float sx = 1.0f, sw0 = 1.0f;
      if constexpr (kEpi != kEpiPlain) {
        sx = row < M ? ep.s_row[row] : 0.0f;
        sw0 = ep.s_col_axis ? 1.0f : ep.s_col[0];
      }
      const uint32_t tacc = tmem + lane_base + static_cast<uint32_t>(acc * 256);
      epilogue_scale_chunks<KIND, kEpi, BN, kGroups, !LR, LR>(ep, &tmY, tacc, m0, n0, M, N, quarter, group, lane,
                                                                    sx, sw0, sOut + e * 2 * C::kOutBufBytes, out_iter,
                                                                    tacc + BN);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(&tempty[acc], 0));   // the even CTA's barrier
      if (++acc == C::kAccBufs) { acc = 0; acc_phase ^= 1u; }
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
