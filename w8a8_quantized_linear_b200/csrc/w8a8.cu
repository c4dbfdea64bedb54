// w8a8.cu - the C ABI of libw8a8.so (declared in include/w8a8.h): argument
// checks, workspace layout, TMA tensor maps and kernel launches.  One
// translation unit holds every kernel, so the device status word and the
// wait limit are single per-device symbols without relocatable device code.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>

#include <nvtx3/nvToolsExt.h>

#include "w8a8.h"
#include "device.cuh"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "quantize.cuh"
#include "q8_0.cuh"
#include "gemv.cuh"
#include "weight_only.cuh"
#include "svdq_input.cuh"

namespace w8a8 {
namespace {

thread_local std::string t_last_error;

w8a8_status fail(w8a8_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
w8a8_status fail(w8a8_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return st;
}

w8a8_status cuda_fail(cudaError_t e, const char* what) {
  return fail(W8A8_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int64_t round_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

constexpr int kMaxDevices = 64;

// Compute capability 10.0 check and SM count, cached per device.
struct DeviceInfo {
  std::atomic<int> state{0};   // 0 unknown, 1 ok, 2 unsupported
  int sms = 0;
};
DeviceInfo g_dev[kMaxDevices];

w8a8_status current_device(int* dev_out, int* sms_out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(W8A8_ERR_UNSUPPORTED_DEVICE, "no CUDA device: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(W8A8_ERR_UNSUPPORTED_DEVICE, "device index %d out of range", dev);
  DeviceInfo& di = g_dev[dev];
  int st = di.state.load(std::memory_order_acquire);
  if (st == 0) {
    int major = 0, minor = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    di.sms = sms;
    st = (major == 10 && minor == 0) ? 1 : 2;
    di.state.store(st, std::memory_order_release);
  }
  if (st != 1) return fail(W8A8_ERR_UNSUPPORTED_DEVICE, "device %d is not compute capability 10.0 (sm_100a)", dev);
  if (dev_out) *dev_out = dev;
  if (sms_out) *sms_out = di.sms;
  return W8A8_OK;
}

// ---------------------------------------------------------------- TMA maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D row-major tensor [outer, inner] with `row_bytes` between rows, copied in
// boxes of [box_outer, box_inner] elements with the given swizzle (128-byte
// for the operand tiles, 64-byte for the epilogue's output blocks).
w8a8_status make_map(CUtensorMap* map, CUtensorMapDataType dt, int elem, const void* base, int64_t inner,
                     int64_t outer, int64_t row_bytes, int box_inner, int box_outer,
                     CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(W8A8_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  if (inner * elem > row_bytes || (row_bytes & 15) != 0 || !aligned16(base))
    return fail(W8A8_ERR_MISALIGNED, "tensor map: base/stride not 16-byte aligned");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(W8A8_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return W8A8_OK;
}

// ---------------------------------------------------------------- launches
template <typename Kernel>
cudaError_t set_smem_once(Kernel k, size_t bytes, int dev, std::atomic<uint64_t>& mask) {
  const uint64_t bit = 1ull << dev;
  if (mask.load(std::memory_order_acquire) & bit) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess) mask.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Launch with programmatic stream serialization: the kernel may start (and
// run up to its griddep_wait) while the previous kernel on the stream
// finishes.  The kernels launched this way are the row quantizers, the GEMMs,
// the split-K epilogue, the few-token product, the Q8_0 re-quantization and
// the dequantizers; each waits before touching memory that the previous
// kernel may write or read.  The single exception, the single-SM GEMM's
// weight prefetch, is enabled only where the kernel before it is the same
// call's row quantizer (EpiParams::early_weights), which waits for all
// earlier work before it lets the GEMM launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Output tensor map for the epilogue's TMA stores: bf16 [M, ldy] in 32 x 32
// boxes with the 64-byte swizzle.  Used only when ldy % 8 == 0 (16-byte row
// stride); otherwise the epilogue stores directly and the map is not read.
w8a8_status make_out_map(CUtensorMap* map, EpiParams* ep, int64_t M, int64_t N) {
  ep->tma_store = (ep->ldy % 8) == 0 ? 1 : 0;
  if (!ep->tma_store) {
    std::memset(map, 0, sizeof(*map));
    return W8A8_OK;
  }
  return make_map(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ep->y, N, M, ep->ldy * 2, 32, 32,
                  CU_TENSOR_MAP_SWIZZLE_64B);
}

template <int KIND, bool B_MN, int BN, int EPI>
w8a8_status launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, int64_t M, int64_t N, int64_t Kc,
                        EpiParams ep, cudaStream_t st) {
  alignas(64) CUtensorMap ty;
  // the transposed form's rows are y's columns (weight rows) and its columns
  // y's rows (tokens)
  w8a8_status ms = (EPI == kEpiScaleT) ? make_out_map(&ty, &ep, N, M) : make_out_map(&ty, &ep, M, N);
  if (ms != W8A8_OK) return ms;
  using C = GemmCfg<KIND, BN, EPI>;
  static std::atomic<uint64_t> smem_set{0};
  int dev = 0, sms = 0;
  w8a8_status s = current_device(&dev, &sms);
  if (s != W8A8_OK) return s;
  auto kern = gemm_kernel<KIND, B_MN, BN, EPI>;
  cudaError_t e = set_smem_once(kern, C::kSmem, dev, smem_set);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemm)");
  if (ep.splits < 1) ep.splits = 1;
  const int64_t units = ((M + kBM - 1) / kBM) * ((N + BN - 1) / BN) * ep.splits;
  const int64_t slots = static_cast<int64_t>(sms) * C::kCtasPerSm;
  const int grid = static_cast<int>(units < slots ? units : slots);
  e = launch_pdl(kern, dim3(grid), dim3(C::kThreads), C::kSmem, st, ta, tb, ty, static_cast<int>(M),
                 static_cast<int>(N), static_cast<int>(Kc), ep);
  return e == cudaSuccess ? W8A8_OK : cuda_fail(e, "gemm launch");
}

// The CTA-pair GEMM (256-row tiles, clusters of two), persistent over tile
// pairs.  tt / tl2: the T and L2 maps of the low-rank form (LR), unused
// otherwise.
template <int KIND, bool B_MN, bool LR = false>
w8a8_status launch_gemm_pair(const CUtensorMap& ta, const CUtensorMap& tb, int64_t M, int64_t N, int64_t Kc,
                             EpiParams ep, cudaStream_t st, const CUtensorMap* tt = nullptr,
                             const CUtensorMap* tl2 = nullptr) {
  alignas(64) CUtensorMap ty, tz;
  w8a8_status ms = make_out_map(&ty, &ep, M, N);
  if (ms != W8A8_OK) return ms;
  std::memset(&tz, 0, sizeof(tz));
  using C = PairCfg<KIND, LR>;
  static std::atomic<uint64_t> smem_set{0};
  int dev = 0, sms = 0;
  w8a8_status s = current_device(&dev, &sms);
  if (s != W8A8_OK) return s;
  auto kern = gemm_pair_kernel<KIND, B_MN, LR>;
  cudaError_t e = set_smem_once(kern, C::kSmem, dev, smem_set);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemm pair)");
  const int64_t tiles = ((M + 2 * kBM - 1) / (2 * kBM)) * ((N + C::kBN - 1) / C::kBN);
  const int64_t pairs = sms / 2;
  const int grid = static_cast<int>(2 * (tiles < pairs ? tiles : pairs));
  ep.splits = 1;
  e = launch_pdl(kern, dim3(grid), dim3(C::kThreads), C::kSmem, st, ta, tb, ty, LR ? *tt : tz, LR ? *tl2 : tz,
                 static_cast<int>(M), static_cast<int>(N), static_cast<int>(Kc), ep);
  return e == cudaSuccess ? W8A8_OK : cuda_fail(e, "gemm pair launch");
}

// The few-token int8 forward in one launch (gemv.cuh): M <= kGemvUseRows,
// K <= kGemvMaxK; each block quantizes the M rows itself.
w8a8_status launch_gemv(const void* x, int64_t M, int64_t N, int64_t K, const void* wq, const float* sw, int axis,
                        const void* bias, void* y, cudaStream_t st) {
  int dev = 0, sms = 0;
  w8a8_status s = current_device(&dev, &sms);
  if (s != W8A8_OK) return s;
  static std::atomic<uint64_t> smem_set[kGemvMaxRows] = {};
  const size_t smem = static_cast<size_t>(M * K);
  // up to 4 blocks per SM (as shared memory allows) keep the weight stream's
  // loads in flight
  int64_t per_sm = static_cast<int64_t>(200 * 1024) / static_cast<int64_t>(smem + 1024);
  per_sm = per_sm < 1 ? 1 : (per_sm > 4 ? 4 : per_sm);
  int64_t grid = (N + kGemvThreads / 32 - 1) / (kGemvThreads / 32);
  if (grid > per_sm * sms) grid = per_sm * sms;
  const auto* xp = static_cast<const __nv_bfloat16*>(x);
  const auto* wp = static_cast<const int8_t*>(wq);
  const auto* bp = static_cast<const __nv_bfloat16*>(bias);
  auto* yp = static_cast<__nv_bfloat16*>(y);
  cudaError_t e = cudaSuccess;
#define W8A8_GEMV(MM)                                                                                            \
  case MM:                                                                                                       \
    e = set_smem_once(gemv_int8_kernel<MM>, static_cast<size_t>(MM) * kGemvMaxK, dev, smem_set[MM - 1]);         \
    if (e == cudaSuccess)                                                                                        \
      e = launch_pdl(gemv_int8_kernel<MM>, dim3(static_cast<unsigned>(grid)), dim3(kGemvThreads), smem, st, xp, K, \
                     static_cast<int>(N), static_cast<int>(K), wp, sw, axis, bp, yp);                            \
    break;
  switch (M) {
    W8A8_GEMV(1) W8A8_GEMV(2)
    default: return fail(W8A8_ERR_UNSUPPORTED_SHAPE, "gemv rows");
  }
#undef W8A8_GEMV
  return e == cudaSuccess ? W8A8_OK : cuda_fail(e, "gemv launch");
}

// Products with at least this many rows (and no split) run on CTA pairs.
constexpr int64_t kPairMinRows = 512;

w8a8_status launch_quantize_rows(const void* x, int64_t ldx, int64_t M, int64_t K, int qt, void* q, int64_t ldq,
                                 float* s, cudaStream_t st, const uint32_t* amax_in = nullptr,
                                 uint32_t* zero_out = nullptr, int64_t zero_n = 0) {
  const auto* xp = static_cast<const __nv_bfloat16*>(x);
  auto* qp = static_cast<uint8_t*>(q);
  const int64_t nv = K / 8;
  const bool chain = amax_in != nullptr || zero_out != nullptr;
  const int64_t tw = (nv + 32 * kTeamVecs - 1) / (32 * kTeamVecs);   // warps per row
  if (tw <= 8) {
    int team_w = 1;
    while (team_w < tw) team_w *= 2;
    const int64_t teams = 8 / team_w;
    const int grid = static_cast<int>((M + teams - 1) / teams < (1 << 20) ? (M + teams - 1) / teams : (1 << 20));
    cudaError_t e = cudaSuccess;
#define W8A8_TEAM_LAUNCH(QT, TW)                                                                                    \
  e = chain ? launch_pdl(quantize_rows_team_kernel<QT, TW, true>, dim3(grid), dim3(256), 0, st, xp, ldx, M, K, qp, ldq, \
                         s, amax_in, zero_out, zero_n)                                                                \
            : launch_pdl(quantize_rows_team_kernel<QT, TW, false>, dim3(grid), dim3(256), 0, st, xp, ldx, M, K, qp,     \
                         ldq, s, amax_in, zero_out, zero_n)
    if (qt == W8A8_E4M3) {
      switch (team_w) {
        case 1: W8A8_TEAM_LAUNCH(1, 1); break;
        case 2: W8A8_TEAM_LAUNCH(1, 2); break;
        case 4: W8A8_TEAM_LAUNCH(1, 4); break;
        default: W8A8_TEAM_LAUNCH(1, 8); break;
      }
    } else {
      switch (team_w) {
        case 1: W8A8_TEAM_LAUNCH(0, 1); break;
        case 2: W8A8_TEAM_LAUNCH(0, 2); break;
        case 4: W8A8_TEAM_LAUNCH(0, 4); break;
        default: W8A8_TEAM_LAUNCH(0, 8); break;
      }
    }
#undef W8A8_TEAM_LAUNCH
    return e == cudaSuccess ? W8A8_OK : cuda_fail(e, "quantize_rows launch");
  } else {
    int64_t t = (nv + kRowVecs - 1) / kRowVecs;
    t = round_up(t, 32);
    if (t < 32) t = 32;
    if (t > 1024) t = 1024;
    const int grid = static_cast<int>(M < (1 << 20) ? M : (1 << 20));
    const dim3 gd(grid), bd(static_cast<unsigned>(t));
    const cudaError_t e =
        (qt == W8A8_E4M3)
            ? (chain ? launch_pdl(quantize_rows_kernel<1, true>, gd, bd, 0, st, xp, ldx, M, K, qp, ldq, s, amax_in,
                                  zero_out, zero_n)
                     : launch_pdl(quantize_rows_kernel<1, false>, gd, bd, 0, st, xp, ldx, M, K, qp, ldq, s, amax_in,
                                  zero_out, zero_n))
            : (chain ? launch_pdl(quantize_rows_kernel<0, true>, gd, bd, 0, st, xp, ldx, M, K, qp, ldq, s, amax_in,
                                  zero_out, zero_n)
                     : launch_pdl(quantize_rows_kernel<0, false>, gd, bd, 0, st, xp, ldx, M, K, qp, ldq, s, amax_in,
                                  zero_out, zero_n));
    return e == cudaSuccess ? W8A8_OK : cuda_fail(e, "quantize_rows launch");
  }
}

// Workspace carving: each piece starts on a 256-byte boundary.
struct Carve {
  uint8_t* base;
  size_t off = 0;
  explicit Carve(void* b) : base(static_cast<uint8_t*>(b)) {}
  void* take(size_t bytes) {
    void* p = base ? base + off : nullptr;
    off += static_cast<size_t>(round_up(static_cast<int64_t>(bytes), 256));
    return p;
  }
};

// Split-K for int8 GEMMs with few output tiles (few tokens): when the tiles
// fill at most half of a B200's 148 SMs, the contraction is split, at least
// 4 K blocks (512 codes) per split and at most 16 splits; the partial sums
// [S, M, Nout] go to the workspace and splitk_epilogue_kernel finishes them
// (Nout % 8 == 0).  Integer partial sums add up exactly, so the result is the
// unsplit one bit for bit.  e4m3 products are never split: the tensor cores'
// fp32 accumulation order would change, and with it the rounding.  The count
// depends on the shape alone (the workspace size covers the int8 case for
// both formats), so workspace sizes do not depend on the device.
constexpr int64_t kSplitSms = 148;
int choose_splits(int64_t M, int64_t Nout, int64_t Kc) {
  const int64_t tiles = ((M + kBM - 1) / kBM) * ((Nout + 255) / 256);
  const int64_t num_kb = (Kc + kBKBytes - 1) / kBKBytes;
  if (tiles <= 0 || tiles * 2 > kSplitSms || (Nout % 8) != 0) return 1;
  int64_t s = kSplitSms / tiles;
  if (s > num_kb / 4) s = num_kb / 4;
  if (s > 16) s = 16;
  return s < 2 ? 1 : static_cast<int>(s);
}

// The transposed forward for few tokens (M <= kSwapMaxRows): the weight is
// the 128-row MMA operand A and the tokens the N side (64 or 128 columns), so
// no MMA rows are padding and each stage is mostly weight bytes.
constexpr int64_t kSwapMaxRows = 128;
bool use_swap(int64_t M) { return M >= 1 && M <= kSwapMaxRows; }
int swap_bn(int64_t M) { return M <= 64 ? 64 : 128; }
int choose_splits_t(int64_t M, int64_t Nout, int64_t Kc) {
  const int64_t tiles = ((Nout + kBM - 1) / kBM) * ((M + swap_bn(M) - 1) / swap_bn(M));
  const int64_t num_kb = (Kc + kBKBytes - 1) / kBKBytes;
  if (tiles <= 0 || tiles * 2 > kSplitSms || (Nout % 8) != 0) return 1;
  int64_t s = kSplitSms / tiles;
  if (s > num_kb / 4) s = num_kb / 4;
  if (s > 16) s = 16;
  return s < 2 ? 1 : static_cast<int>(s);
}

// Workspace of a linear call: codes [M, ld] and row scales [M], then, when
// the GEMM is split, the partial sums [S, M, Nout] (for a forward with few
// tokens, room for either layout's split count).
struct LinearWs {
  size_t bytes;
  int splits;
};
LinearWs linear_ws(int64_t M, int64_t ld, int64_t Nout, bool fwd = false) {
  int sp = choose_splits(M, Nout, ld);
  if (fwd && use_swap(M) && choose_splits_t(M, Nout, ld) > sp) sp = choose_splits_t(M, Nout, ld);
  LinearWs w{0, sp};
  Carve c(nullptr);
  c.take(static_cast<size_t>(M * ld));
  c.take(static_cast<size_t>(M) * 4);
  if (w.splits > 1) c.take(static_cast<size_t>(w.splits) * static_cast<size_t>(M) * static_cast<size_t>(Nout) * 4);
  w.bytes = c.off;
  return w;
}
size_t ws_linear(int64_t M, int64_t ld, int64_t Nout, bool fwd = false) { return linear_ws(M, ld, Nout, fwd).bytes; }

// The split-K part of a carved workspace.
struct SplitWs {
  int splits = 1;
  uint32_t* partial = nullptr;
};
SplitWs carve_split(Carve& c, int64_t M, int64_t Nout, const LinearWs& w, int qt) {
  SplitWs sk;
  if (w.splits > 1 && qt == W8A8_INT8) {
    sk.splits = w.splits;
    sk.partial = static_cast<uint32_t*>(
        c.take(static_cast<size_t>(w.splits) * static_cast<size_t>(M) * static_cast<size_t>(Nout) * 4));
  }
  return sk;
}

// The finishing kernel of a split product (after the GEMM on the stream).
w8a8_status launch_splitk_epilogue(int qt, const SplitWs& sk, int64_t M, int64_t Nout, const float* sx,
                                   const float* sw, int axis, const void* bias, void* y, cudaStream_t st,
                                   int act = kActNone, uint32_t* y_amax = nullptr) {
  int sms = 0;
  w8a8_status s = current_device(nullptr, &sms);
  if (s != W8A8_OK) return s;
  int64_t grid = (M * (Nout / 8) + 255) / 256;
  if (grid > 8 * static_cast<int64_t>(sms)) grid = 8 * static_cast<int64_t>(sms);
  const auto* b = static_cast<const __nv_bfloat16*>(bias);
  auto* yp = static_cast<__nv_bfloat16*>(y);
  const uint32_t* part = sk.partial;
  const cudaError_t e =
      (qt == W8A8_E4M3)
          ? launch_pdl(splitk_epilogue_kernel<kKindE4M3>, dim3(static_cast<unsigned>(grid)), dim3(256), 0, st, part,
                       sk.splits, M, Nout, sx, sw, axis, b, yp, act, y_amax)
          : launch_pdl(splitk_epilogue_kernel<kKindI8>, dim3(static_cast<unsigned>(grid)), dim3(256), 0, st, part,
                       sk.splits, M, Nout, sx, sw, axis, b, yp, act, y_amax);
  return e == cudaSuccess ? W8A8_OK : cuda_fail(e, "split-K epilogue launch");
}

// Split count of the SVDQuant low-rank input T = X L1 (a bf16 product with
// r <= 32 columns: one output tile per 128 rows), as choose_splits with
// 64-element K blocks.
int t_splits(int64_t M, int64_t K) {
  const int64_t tiles = (M + kBM - 1) / kBM;
  const int64_t num_kb = (K + 63) / 64;
  if (tiles * 2 > kSplitSms) return 1;
  int64_t s = kSplitSms / tiles;
  if (s > num_kb / 4) s = num_kb / 4;
  if (s > 16) s = 16;
  return s < 2 ? 1 : static_cast<int>(s);
}
// Workspace of svdq_linear_fwd: codes [M, K], row scales [M], T [M, r]
// bf16, then T's split-K partial sums [S, M, r] fp32 when split (rows longer
// than the one-pass input kernel takes).
size_t ws_svdq(int64_t M, int64_t K, int r) {
  Carve c(nullptr);
  c.take(static_cast<size_t>(M * K));
  c.take(static_cast<size_t>(M) * 4);
  c.take(static_cast<size_t>(M) * r * 2);
  const int s = K <= kSiMaxK ? 1 : t_splits(M, K);
  if (s > 1) c.take(static_cast<size_t>(s) * static_cast<size_t>(M) * static_cast<size_t>(r) * 4);
  return c.off;
}

bool valid_qt(int qt) { return qt == W8A8_INT8 || qt == W8A8_E4M3; }
bool valid_g(int g) { return g == W8A8_TENSOR || g == W8A8_AXIS; }

CUtensorMapDataType code_type() { return CU_TENSOR_MAP_DATA_TYPE_UINT8; }

// GEMM on codes.  fwd: A = xq [M, lda] K-major, B = wq [N, K] K-major.
// sk: split-K workspace (partial sums), or null for an unsplit product.
// early_weights: the kernel just before on the stream is this call's row
// quantizer, so the single-SM GEMM may fetch weight tiles before its wait
// (EpiParams::early_weights); false when the caller launched nothing before.
w8a8_status gemm_fwd(const void* xq, int64_t lda, const float* sx, int64_t M, int64_t N, int64_t K, int qt,
                     const void* wq, const float* sw, int g, const void* bias, void* y, cudaStream_t st,
                     const SplitWs* sk = nullptr, int act = kActNone, uint32_t* y_amax = nullptr,
                     bool early_weights = false) {
  alignas(64) CUtensorMap ta, tb;
  w8a8_status s = make_map(&ta, code_type(), 1, xq, K, M, lda, kBKBytes, kBM);
  if (s != W8A8_OK) return s;
  s = make_map(&tb, code_type(), 1, wq, K, N, K, kBKBytes, 256);
  if (s != W8A8_OK) return s;
  EpiParams ep{};
  ep.s_row = sx;
  ep.s_col = sw;
  ep.s_col_axis = (g == W8A8_AXIS);
  ep.bias = static_cast<const __nv_bfloat16*>(bias);
  ep.y = static_cast<__nv_bfloat16*>(y);
  ep.ldy = N;
  ep.splits = 1;
  ep.act = act;
  ep.y_amax = y_amax;
  ep.early_weights = early_weights ? 1 : 0;
  if (sk != nullptr && sk->splits > 1) {
    ep.splits = sk->splits;
    ep.partial = sk->partial;
  }
  if (use_swap(M) && act == kActNone && y_amax == nullptr) {
    // transposed: A = the weight [N, K], B = the codes [M, K]; the kernel's
    // rows are n and its columns m; split count chosen for this layout (the
    // workspace has room for it)
    if (ep.splits > 1) ep.splits = choose_splits_t(M, N, K);
    const int bn = swap_bn(M);
    if ((s = make_map(&ta, code_type(), 1, wq, K, N, K, kBKBytes, kBM)) != W8A8_OK) return s;
    if ((s = make_map(&tb, code_type(), 1, xq, K, M, lda, kBKBytes, bn)) != W8A8_OK) return s;
    if (bn == 64)
      s = (qt == W8A8_E4M3) ? launch_gemm<kKindE4M3, false, 64, kEpiScaleT>(ta, tb, N, M, K, ep, st)
                            : launch_gemm<kKindI8, false, 64, kEpiScaleT>(ta, tb, N, M, K, ep, st);
    else
      s = (qt == W8A8_E4M3) ? launch_gemm<kKindE4M3, false, 128, kEpiScaleT>(ta, tb, N, M, K, ep, st)
                            : launch_gemm<kKindI8, false, 128, kEpiScaleT>(ta, tb, N, M, K, ep, st);
    if (s != W8A8_OK || ep.splits == 1) return s;
    SplitWs skt = *sk;
    skt.splits = ep.splits;
    return launch_splitk_epilogue(qt, skt, M, N, sx, sw, g == W8A8_AXIS, bias, y, st);
  }
  if (ep.splits == 1 && M >= kPairMinRows) {
    // B in halves of 128 rows, one per CTA of the pair
    if ((s = make_map(&tb, code_type(), 1, wq, K, N, K, kBKBytes, 128)) != W8A8_OK) return s;
    return (qt == W8A8_E4M3) ? launch_gemm_pair<kKindE4M3, false>(ta, tb, M, N, K, ep, st)
                             : launch_gemm_pair<kKindI8, false>(ta, tb, M, N, K, ep, st);
  }
  s = (qt == W8A8_E4M3) ? launch_gemm<kKindE4M3, false, 256, kEpiScale>(ta, tb, M, N, K, ep, st)
                        : launch_gemm<kKindI8, false, 256, kEpiScale>(ta, tb, M, N, K, ep, st);
  if (s != W8A8_OK || ep.splits == 1) return s;
  return launch_splitk_epilogue(qt, *sk, M, N, sx, sw, g == W8A8_AXIS, bias, y, st, act, y_amax);
}

// dgrad: A = dyq [M, lda] (contraction N), B = wq [N, K] read MN-major.
// early_weights as for gemm_fwd.
w8a8_status gemm_dgrad(const void* dyq, int64_t lda, const float* sdy, int64_t M, int64_t N, int64_t K, int qt,
                       const void* wq, const float* sw, void* dx, cudaStream_t st, const SplitWs* sk = nullptr,
                       bool early_weights = false) {
  alignas(64) CUtensorMap ta, tb;
  w8a8_status s = make_map(&ta, code_type(), 1, dyq, N, M, lda, kBKBytes, kBM);
  if (s != W8A8_OK) return s;
  s = make_map(&tb, code_type(), 1, wq, K, N, K, 128, kBKBytes);
  if (s != W8A8_OK) return s;
  EpiParams ep{};
  ep.s_row = sdy;
  ep.s_col = sw;
  ep.s_col_axis = 0;
  ep.y = static_cast<__nv_bfloat16*>(dx);
  ep.ldy = K;
  ep.splits = 1;
  ep.early_weights = early_weights ? 1 : 0;
  if (sk != nullptr && sk->splits > 1) {
    ep.splits = sk->splits;
    ep.partial = sk->partial;
  }
  if (ep.splits == 1 && M >= kPairMinRows)
    return (qt == W8A8_E4M3) ? launch_gemm_pair<kKindE4M3, true>(ta, tb, M, K, N, ep, st)
                             : launch_gemm_pair<kKindI8, true>(ta, tb, M, K, N, ep, st);
  s = (qt == W8A8_E4M3) ? launch_gemm<kKindE4M3, true, 256, kEpiScale>(ta, tb, M, K, N, ep, st)
                        : launch_gemm<kKindI8, true, 256, kEpiScale>(ta, tb, M, K, N, ep, st);
  if (s != W8A8_OK || ep.splits == 1) return s;
  return launch_splitk_epilogue(qt, *sk, M, K, sdy, sw, 0, nullptr, dx, st);
}

// ---------------------------------------------------------------------------
// The bf16 Linear of the weight-only types (OneTrainer wiki, float8 and GGUF:
// the weight dequantized to the train data type): y = bf16(X W^T (+ bias)),
// fp32 sums on the tensor cores (kind::f16), split along K (fp32 partial sums
// added in split order) when the output makes few tiles.
int bf16_splits(int64_t M, int64_t N, int64_t K) {
  const int64_t tiles = ((M + kBM - 1) / kBM) * ((N + 255) / 256);
  const int64_t num_kb = (K + 63) / 64;
  if (tiles <= 0 || tiles * 2 > kSplitSms || (N % 8) != 0) return 1;
  int64_t s = kSplitSms / tiles;
  if (s > num_kb / 4) s = num_kb / 4;
  if (s > 16) s = 16;
  return s < 2 ? 1 : static_cast<int>(s);
}
size_t split_bytes(int s, int64_t M, int64_t N) {
  return s > 1 ? static_cast<size_t>(s) * static_cast<size_t>(M) * static_cast<size_t>(N) * 4 : 0;
}
// Workspace of bf16_linear_fwd (partial sums only) and of the weight-only
// forwards (the dequantized weight [N, K] bf16, then the partial sums).
size_t ws_bf16(int64_t M, int64_t N, int64_t K) {
  Carve c(nullptr);
  const size_t p = split_bytes(bf16_splits(M, N, K), M, N);
  if (p) c.take(p);
  return c.off;
}
size_t ws_bf16_dgrad(int64_t M, int64_t N, int64_t K) {
  Carve c(nullptr);
  const size_t p = split_bytes(bf16_splits(M, K, N), M, K);
  if (p) c.take(p);
  return c.off;
}
size_t ws_weight_only_dgrad(int64_t M, int64_t N, int64_t K) {
  Carve c(nullptr);
  c.take(static_cast<size_t>(N) * static_cast<size_t>(K) * 2);
  const size_t p = split_bytes(bf16_splits(M, K, N), M, K);
  if (p) c.take(p);
  return c.off;
}
size_t ws_weight_only(int64_t M, int64_t N, int64_t K) {
  Carve c(nullptr);
  c.take(static_cast<size_t>(N) * static_cast<size_t>(K) * 2);
  const size_t p = split_bytes(bf16_splits(M, N, K), M, N);
  if (p) c.take(p);
  return c.off;
}

// fwd: y [M, N] = x [M, K] w[N, K]^T (+ bias).  dgrad (B_MN): y [M, K] =
// x [M, N] w [N, K], the weight read MN-major (its rows are the
// contraction); Nout = K, Kc = N.
template <bool DGRAD>
w8a8_status gemm_bf16_t(const void* x, int64_t M, int64_t N, int64_t K, const void* w, const void* bias, void* y,
                        Carve& c, cudaStream_t st) {
  const int64_t nout = DGRAD ? K : N, kc = DGRAD ? N : K;
  const int splits = bf16_splits(M, nout, kc);
  alignas(64) CUtensorMap ta, tb;
  w8a8_status s = make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, kc, M, kc * 2, 64, kBM);
  if (s != W8A8_OK) return s;
  EpiParams ep{};
  ep.bias = static_cast<const __nv_bfloat16*>(bias);
  ep.y = static_cast<__nv_bfloat16*>(y);
  ep.ldy = nout;
  ep.splits = 1;
  if (splits == 1 && M >= kPairMinRows) {
    if (DGRAD)
      s = make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w, K, N, K * 2, 64, 64);
    else
      s = make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w, K, N, K * 2, 64, 128);
    if (s != W8A8_OK) return s;
    return launch_gemm_pair<kKindBF16, DGRAD>(ta, tb, M, nout, kc, ep, st);
  }
  if (DGRAD)
    s = make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w, K, N, K * 2, 64, 64);
  else
    s = make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w, K, N, K * 2, 64, 256);
  if (s != W8A8_OK) return s;
  if (splits > 1) {
    ep.splits = splits;
    ep.partial = static_cast<uint32_t*>(c.take(split_bytes(splits, M, nout)));
  }
  if ((s = launch_gemm<kKindBF16, DGRAD, 256, kEpiPlain>(ta, tb, M, nout, kc, ep, st)) != W8A8_OK || splits == 1)
    return s;
  int sms = 0;
  if ((s = current_device(nullptr, &sms)) != W8A8_OK) return s;
  int64_t grid = (M * (nout / 8) + 255) / 256;
  if (grid > 8 * static_cast<int64_t>(sms)) grid = 8 * static_cast<int64_t>(sms);
  const uint32_t* part = ep.partial;
  const cudaError_t e =
      launch_pdl(splitk_epilogue_kernel<kKindBF16>, dim3(static_cast<unsigned>(grid)), dim3(256), 0, st, part, splits, M,
                 nout, static_cast<const float*>(nullptr), static_cast<const float*>(nullptr), 0, ep.bias, ep.y,
                 static_cast<int>(kActNone), static_cast<uint32_t*>(nullptr));
  return e == cudaSuccess ? W8A8_OK : cuda_fail(e, "split-K epilogue launch");
}
w8a8_status gemm_bf16(const void* x, int64_t M, int64_t N, int64_t K, const void* w, const void* bias, void* y,
                      Carve& c, cudaStream_t st) {
  return gemm_bf16_t<false>(x, M, N, K, w, bias, y, c, st);
}

// Q8_0 -> fp32 (BF16 = false) or bf16 values.
template <bool BF16>
w8a8_status launch_q8_0_dequant(const void* blocks, int64_t n, void* y, cudaStream_t st) {
  int sms = 0;
  w8a8_status s = current_device(nullptr, &sms);
  if (s != W8A8_OK) return s;
  const int64_t chunks = (n + 256 * kQ80Unroll - 1) / (256 * kQ80Unroll);
  int64_t grid = (chunks + kQ80WarpsPerBlock - 1) / kQ80WarpsPerBlock;
  if (grid > 16 * sms) grid = 16 * sms;
  const cudaError_t e = launch_pdl(q8_0_dequantize_kernel<BF16>, dim3(static_cast<int>(grid)), dim3(256), 0, st,
                                   static_cast<const uint8_t*>(blocks), n, y);
  return e == cudaSuccess ? W8A8_OK : cuda_fail(e, "q8_0 dequantize launch");
}

// e4m3 codes -> bf16(value * scale), n % 16 == 0.
w8a8_status launch_dequant_e4m3(const void* q, int64_t n, const float* scale, void* w, cudaStream_t st) {
  int sms = 0;
  w8a8_status s = current_device(nullptr, &sms);
  if (s != W8A8_OK) return s;
  const int64_t n8 = n / 8;
  int64_t grid = (n8 + 255) / 256;
  if (grid > 8 * static_cast<int64_t>(sms)) grid = 8 * static_cast<int64_t>(sms);
  const cudaError_t e = launch_pdl(dequant_e4m3_bf16_kernel, dim3(static_cast<int>(grid)), dim3(256), 0, st,
                                   static_cast<const uint2*>(q), n8, scale, static_cast<uint4*>(w));
  return e == cudaSuccess ? W8A8_OK : cuda_fail(e, "e4m3 dequantize launch");
}

#define W8A8_CHECK(cond, status, ...) \
  do {                                \
    if (!(cond)) return fail(status, __VA_ARGS__); \
  } while (0)

w8a8_status check_k(int64_t K, const char* name) {
  if (K < 16 || (K % 16) != 0)
    return fail(W8A8_ERR_UNSUPPORTED_SHAPE, "%s = %lld: need >= 16 and a multiple of 16", name,
                static_cast<long long>(K));
  if (K > (1ll << 30)) return fail(W8A8_ERR_UNSUPPORTED_SHAPE, "%s too large", name);
  return W8A8_OK;
}

// Scratch of w8a8_linear_fwd_noalloc: activation codes at offset 0, row
// scales at offset W8A8_NOALLOC_MAX_CODES (both 256-byte aligned).  Host code
// only sees a stand-in for this symbol; its device address comes from
// cudaGetSymbolAddress with the device current.
static __device__ __align__(256) uint8_t g_noalloc_scratch[W8A8_NOALLOC_SCRATCH_BYTES];

// The address belongs to the module instance of one CUDA context, so it is
// cached per context: keyed on the context's process-unique id
// (cuCtxGetId), which no later context reuses - after cudaDeviceReset, or
// under another context on the same device, the first call looks the
// address up again.  The lookup allocates nothing.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
struct NoallocSlot {
  unsigned long long ctx_id = 0;   // 0: empty (context ids start at 1)
  void* addr = nullptr;
};
constexpr int kNoallocSlots = 16;
std::mutex g_noalloc_mu;
NoallocSlot g_noalloc_slot[kNoallocSlots];
int g_noalloc_next = 0;

template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion(name, &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

w8a8_status current_ctx_id(unsigned long long* id) {
  static CtxGetCurrentFn get_ctx = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_ctx || !get_id) return fail(W8A8_ERR_CUDA, "cuCtxGetCurrent / cuCtxGetId unavailable");
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return fail(W8A8_ERR_CUDA, "no current CUDA context");
  if (get_id(ctx, id) != CUDA_SUCCESS) return fail(W8A8_ERR_CUDA, "cuCtxGetId failed");
  return W8A8_OK;
}

w8a8_status noalloc_scratch(void** out) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  unsigned long long id = 0;
  if (current_ctx_id(&id) != W8A8_OK) {
    // no context is current yet: the symbol lookup below makes the device's
    // primary context current, then the id is taken again
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
    w8a8_status st = current_ctx_id(&id);
    if (st != W8A8_OK) return st;
  }
  for (const NoallocSlot& sl : g_noalloc_slot)
    if (sl.ctx_id == id) {
      *out = sl.addr;
      return W8A8_OK;
    }
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
  g_noalloc_slot[g_noalloc_next] = NoallocSlot{id, p};
  g_noalloc_next = (g_noalloc_next + 1) % kNoallocSlots;
  *out = p;
  return W8A8_OK;
}

}  // namespace
}  // namespace w8a8

using namespace w8a8;

// The few-token e4m3 forward (gemv.cuh): M <= kGemvE4m3MaxRows and the M
// activation rows (fp32, K rounded up to 512) within kGemvE4m3SmemBytes.
static bool gemv_e4m3_fits(int64_t M, int64_t K) {
  return M >= 1 && M <= kGemvE4m3MaxRows && M * ((K + 511) / 512) * 512 * 4 <= kGemvE4m3SmemBytes;
}
static w8a8_status launch_gemv_e4m3(const void* x, int64_t M, int64_t N, int64_t K, const void* wq, const float* sw,
                                    int axis, const void* bias, void* y, cudaStream_t st) {
  int dev = 0, sms = 0;
  w8a8_status s = current_device(&dev, &sms);
  if (s != W8A8_OK) return s;
  static std::atomic<uint64_t> smem_set[kGemvE4m3MaxRows] = {};
  const size_t smem = static_cast<size_t>(M * ((K + 511) / 512) * 512 * 2);   // f16 activations
  const int64_t reg_cap = M == 1 ? 4 : (M == 2 ? 3 : 2);   // gemv_e4m3_min_blocks
  int64_t per_sm = static_cast<int64_t>(200 * 1024) / static_cast<int64_t>(smem + 1024);
  per_sm = per_sm < 1 ? 1 : (per_sm > reg_cap ? reg_cap : per_sm);
  int64_t grid = (N + kGemvThreads / 32 - 1) / (kGemvThreads / 32);
  if (grid > per_sm * sms) grid = per_sm * sms;
  const auto* xp = static_cast<const __nv_bfloat16*>(x);
  const auto* wp = static_cast<const uint8_t*>(wq);
  const auto* bp = static_cast<const __nv_bfloat16*>(bias);
  auto* yp = static_cast<__nv_bfloat16*>(y);
  cudaError_t e = cudaSuccess;
#define W8A8_GEMV_E4(MM)                                                                                          \
  case MM:                                                                                                        \
    e = set_smem_once(gemv_e4m3_kernel<MM>, kGemvE4m3SmemBytes, dev, smem_set[MM - 1]);                           \
    if (e == cudaSuccess)                                                                                         \
      e = launch_pdl(gemv_e4m3_kernel<MM>, dim3(static_cast<unsigned>(grid)), dim3(kGemvThreads), smem, st, xp, K, \
                     static_cast<int>(N), static_cast<int>(K), wp, sw, axis, bp, yp);                             \
    break;
  switch (M) {
    W8A8_GEMV_E4(1)
    default: return fail(W8A8_ERR_UNSUPPORTED_SHAPE, "gemv rows");
  }
#undef W8A8_GEMV_E4
  return e == cudaSuccess ? W8A8_OK : cuda_fail(e, "gemv launch");
}

// Q8_0 -> axis-wise codes of type QT (0 int8, 1 e4m3).
template <int QT>
static w8a8_status requant_axis(const void* blocks, int64_t N, int64_t K, uint8_t* q, float* scale,
                                w8a8_stream_t stream, const char* name) {
  W8A8_CHECK(N >= 1, W8A8_ERR_UNSUPPORTED_SHAPE, "N < 1");
  W8A8_CHECK(K >= 32 && K % 32 == 0 && K <= 131072, W8A8_ERR_UNSUPPORTED_SHAPE,
             "K must be a multiple of 32 in [32, 131072]");
  W8A8_CHECK(blocks && q && scale, W8A8_ERR_INVALID_ARG, "null pointer");
  W8A8_CHECK(aligned16(blocks) && aligned16(q) && aligned16(scale), W8A8_ERR_MISALIGNED,
             "pointers must be 16-byte aligned");
  int dev = 0, sms = 0;
  w8a8_status st = current_device(&dev, &sms);
  if (st != W8A8_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const auto* bp = static_cast<const uint8_t*>(blocks);
  const int64_t nblk = K / 32;
  if (K % 256 == 0 && nblk <= 8 * 96) {
    // rows of whole 16-byte units and at most 3 blocks per thread of a team
    // of TW warps: blocks held in registers between the two passes, one row
    // per team
    constexpr int kBufs = 1, kCtasPerSm = 16;   // row buffers per team; grid cap per SM
    // 128 threads per block (8 blocks per SM) for teams of 1 and 4 warps:
    // finer blocks leave less of the last wave idle than 256-thread blocks,
    // whose slot is held until the slowest of their rows is done (measured:
    // 12288 x 3072 16.4 -> 15.7 us, 3072 x 12288 18.4 -> 17.8 us; teams of 2
    // warps were slower that way, 4096 x 4096 9.8 -> 12.6 us)
    constexpr int kNtSmall = 128;
    int tw = 1;
    while (tw * 96 < nblk) tw *= 2;
    const int nt = (tw == 1 || tw == 4) ? kNtSmall : kRqThreads;
    const int teams = nt / 32 / tw;               // rows per block
    const size_t smem = static_cast<size_t>(kBufs * teams) * static_cast<size_t>(nblk * 34);
    int64_t grid = (N + teams - 1) / teams;
    if (grid > kCtasPerSm * static_cast<int64_t>(sms) * (256 / nt)) grid = kCtasPerSm * static_cast<int64_t>(sms) * (256 / nt);
    static std::atomic<uint64_t> hold_smem_set[8] = {};
    cudaError_t e = cudaSuccess;
    const bool full = nblk == 96 * tw;   // every thread holds exactly 3 blocks
#define W8A8_RQ_HOLD(TW, F, IDX, NT)                                                                       \
  e = set_smem_once(q8_0_to_axis_hold_kernel<QT, TW, 3, 1024 / NT, kBufs, F, NT>, 64 * 1024, dev,           \
                    hold_smem_set[IDX]);                                                                   \
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(requant)");                             \
  e = launch_pdl(q8_0_to_axis_hold_kernel<QT, TW, 3, 1024 / NT, kBufs, F, NT>, dim3(static_cast<int>(grid)), dim3(NT), \
                 smem, cs, bp, N, K, q, scale)
    switch (tw) {
      case 1: if (full) { W8A8_RQ_HOLD(1, true, 4, kNtSmall); } else { W8A8_RQ_HOLD(1, false, 0, kNtSmall); } break;
      case 2: if (full) { W8A8_RQ_HOLD(2, true, 5, kRqThreads); } else { W8A8_RQ_HOLD(2, false, 1, kRqThreads); } break;
      case 4: if (full) { W8A8_RQ_HOLD(4, true, 6, kNtSmall); } else { W8A8_RQ_HOLD(4, false, 2, kNtSmall); } break;
      default: if (full) { W8A8_RQ_HOLD(8, true, 7, kRqThreads); } else { W8A8_RQ_HOLD(8, false, 3, kRqThreads); } break;
    }
#undef W8A8_RQ_HOLD
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess ? W8A8_OK : cuda_fail(e, name);
  }
  if (K % 256 == 0) {
    // rows of whole 16-byte units: a team of TW warps per row (at least 3
    // blocks per thread), one row buffer per team and up to 8 blocks per SM
    // (more warps in flight beat a deeper prefetch ring here)
    int tw = 1;
    while (tw < 8 && tw * 2 * 96 <= nblk) tw *= 2;
    const size_t smem = static_cast<size_t>(8 / tw) * static_cast<size_t>(nblk * 34);
    if (smem <= 200 * 1024) {
      int per_sm = static_cast<int>((220 * 1024) / (smem + 1024));
      per_sm = per_sm < 1 ? 1 : (per_sm > 8 ? 8 : per_sm);
      int64_t grid = (N + (8 / tw) - 1) / (8 / tw);
      if (grid > static_cast<int64_t>(per_sm) * sms) grid = static_cast<int64_t>(per_sm) * sms;
      static std::atomic<uint64_t> team_smem_set[4] = {};
      cudaError_t e = cudaSuccess;
#define W8A8_RQ_TEAM(TW, IDX)                                                                              \
  e = set_smem_once(q8_0_to_axis_team_kernel<QT, TW, 1>, 200 * 1024, dev, team_smem_set[IDX]);             \
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(requant)");                             \
  e = launch_pdl(q8_0_to_axis_team_kernel<QT, TW, 1>, dim3(static_cast<int>(grid)), dim3(kRqThreads), smem, cs, bp, N, \
                 K, q, scale)
      switch (tw) {
        case 1: W8A8_RQ_TEAM(1, 0); break;
        case 2: W8A8_RQ_TEAM(2, 1); break;
        case 4: W8A8_RQ_TEAM(4, 2); break;
        default: W8A8_RQ_TEAM(8, 3); break;
      }
#undef W8A8_RQ_TEAM
      if (e == cudaSuccess) e = cudaGetLastError();
      return e == cudaSuccess ? W8A8_OK : cuda_fail(e, name);
    }
  }
  // other rows: one warp per row; each warp stages its row (rounded to 16 bytes) in shared memory
  const size_t row_stride = (static_cast<size_t>(K / 32) * 34 + 15) & ~static_cast<size_t>(15);
  int warps = static_cast<int>((200 * 1024) / row_stride);
  warps = warps < 1 ? 1 : (warps > kRequantMaxWarps ? kRequantMaxWarps : warps);
  const size_t smem = row_stride * warps;
  static std::atomic<uint64_t> smem_set{0};
  cudaError_t e = set_smem_once(q8_0_to_axis_warp_kernel<QT>, 200 * 1024, dev, smem_set);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(requant)");
  int64_t grid = (N + warps - 1) / warps;
  if (grid > 32 * sms) grid = 32 * sms;
  e = launch_pdl(q8_0_to_axis_warp_kernel<QT>, dim3(static_cast<int>(grid)), dim3(32 * warps), smem, cs, bp, N, K, q,
                 scale);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? W8A8_OK : cuda_fail(e, name);
}

// SVDQuant forward with residual codes of type QT (int8 or e4m3).
template <int QT>
static w8a8_status svdq_fwd_impl(const void* x, int64_t M, int64_t N, int64_t K, const void* rq, const float* r_scale,
                                 int r, const void* l1, const void* l2, const void* bias, void* y, void* ws,
                                 size_t ws_bytes, w8a8_stream_t stream) {
  constexpr int kKind = (QT == W8A8_E4M3) ? kKindE4M3 : kKindI8;
  W8A8_CHECK(M >= 0 && N >= 1 && M < (1ll << 31) && N < (1ll << 31), W8A8_ERR_UNSUPPORTED_SHAPE, "bad M/N");
  w8a8_status st = check_k(K, "K");
  if (st != W8A8_OK) return st;
  W8A8_CHECK(r >= 8 && r <= 32 && r % 8 == 0, W8A8_ERR_UNSUPPORTED_SHAPE, "rank r must be 8, 16, 24 or 32");
  if (M == 0) return W8A8_OK;
  W8A8_CHECK(x && rq && r_scale && l1 && l2 && y, W8A8_ERR_INVALID_ARG, "null pointer");
  W8A8_CHECK(aligned16(x) && aligned16(rq) && aligned16(r_scale) && aligned16(l1) && aligned16(l2) && aligned16(y) &&
                 (bias == nullptr || aligned16(bias)),
             W8A8_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  W8A8_CHECK(ws != nullptr && ws_bytes >= ws_svdq(M, K, r), W8A8_ERR_WORKSPACE,
             "workspace too small: need %zu bytes", ws_svdq(M, K, r));
  W8A8_CHECK(aligned16(ws), W8A8_ERR_MISALIGNED, "workspace must be 16-byte aligned");
  if ((st = current_device(nullptr, nullptr)) != W8A8_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Carve c(ws);
  void* xq = c.take(static_cast<size_t>(M * K));
  float* sx = static_cast<float*>(c.take(static_cast<size_t>(M) * 4));
  auto* t = static_cast<__nv_bfloat16*>(c.take(static_cast<size_t>(M) * r * 2));
  const bool one_pass = K <= kSiMaxK;   // 32 rows fit in one CTA's shared memory
  const int tsplit = one_pass ? 1 : t_splits(M, K);
  SplitWs tsk;
  if (tsplit > 1) {
    tsk.splits = tsplit;
    tsk.partial = static_cast<uint32_t*>(
        c.take(static_cast<size_t>(tsplit) * static_cast<size_t>(M) * static_cast<size_t>(r) * 4));
  }
  if (one_pass) {
    // codes, scales and T = bf16(X L1) in one pass over X
    alignas(64) CUtensorMap tl1;
    if ((st = make_map(&tl1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, l1, r, K, static_cast<int64_t>(r) * 2, 32, kSiKC,
                       CU_TENSOR_MAP_SWIZZLE_64B)) != W8A8_OK)
      return st;
    static std::atomic<uint64_t> si_smem_set{0};
    int dev = 0;
    if ((st = current_device(&dev, nullptr)) != W8A8_OK) return st;
    auto kern = svdq_input_kernel<QT>;
    cudaError_t e = set_smem_once(kern, si_smem_bytes(kSiMaxK), dev, si_smem_set);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(svdq_input)");
    e = launch_pdl(kern, dim3(static_cast<unsigned>((M + kSiRows - 1) / kSiRows)), dim3(kSiThreads),
                   si_smem_bytes(static_cast<int>(K)), s, static_cast<const __nv_bfloat16*>(x), tl1,
                   static_cast<int>(M), static_cast<int>(K), r, static_cast<uint8_t*>(xq), sx, t);
    if (e != cudaSuccess) return cuda_fail(e, "svdq input launch");
  } else {
    // longer rows: the row quantizer, then T = bf16(X L1) as a bf16 tensor-core GEMM, L1
    // [K, r] read MN-major, split along K when the rows make few tiles (fp32
    // partial sums, added in split order, then one bf16 rounding)
    if ((st = launch_quantize_rows(x, K, M, K, QT, xq, K, sx, s)) != W8A8_OK) return st;
    alignas(64) CUtensorMap ta, tb;
    if ((st = make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, K, M, K * 2, 64, kBM)) != W8A8_OK) return st;
    if ((st = make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, l1, r, K, static_cast<int64_t>(r) * 2, 64, 64)) !=
        W8A8_OK)
      return st;
    EpiParams ep{};
    ep.y = t;
    ep.ldy = r;
    ep.splits = tsk.splits;
    ep.partial = tsk.partial;
    ep.early_weights = 1;   // L1 is read early: the kernel just before is this call's row quantizer
    if ((st = launch_gemm<kKindBF16, true, 64, kEpiPlain>(ta, tb, M, r, K, ep, s)) != W8A8_OK) return st;
    if (tsk.splits > 1) {
      int sms = 0;
      if ((st = current_device(nullptr, &sms)) != W8A8_OK) return st;
      int64_t grid = (M * (r / 8) + 255) / 256;
      if (grid > 8 * static_cast<int64_t>(sms)) grid = 8 * static_cast<int64_t>(sms);
      const uint32_t* part = tsk.partial;
      const cudaError_t e = launch_pdl(splitk_epilogue_kernel<kKindBF16>, dim3(static_cast<unsigned>(grid)), dim3(256), 0,
                                       s, part, tsk.splits, M, static_cast<int64_t>(r), static_cast<const float*>(nullptr),
                                       static_cast<const float*>(nullptr), 0, static_cast<const __nv_bfloat16*>(nullptr),
                                       t, static_cast<int>(kActNone), static_cast<uint32_t*>(nullptr));
      if (e != cudaSuccess) return cuda_fail(e, "split-K epilogue launch");
    }
  }
  alignas(64) CUtensorMap ta, tb;
  if ((st = make_map(&ta, code_type(), 1, xq, K, M, K, kBKBytes, kBM)) != W8A8_OK) return st;
  const bool pair = M >= kPairMinRows && (N % 8) == 0;   // L2 rows must be 16-byte multiples for its tensor map
  if ((st = make_map(&tb, code_type(), 1, rq, K, N, K, kBKBytes, pair ? 128 : 256)) != W8A8_OK) return st;
  EpiParams ep{};
  ep.s_row = sx;
  ep.s_col = r_scale;
  ep.s_col_axis = 0;
  ep.bias = static_cast<const __nv_bfloat16*>(bias);
  ep.y = static_cast<__nv_bfloat16*>(y);
  ep.ldy = N;
  ep.lr_t = t;
  ep.lr_l2 = static_cast<const __nv_bfloat16*>(l2);
  ep.r = r;
  // Rq is read early by the single-SM kernel: the kernels since this call's
  // first kernel (which waits for all earlier work before it lets the next
  // one launch) write only the codes, scales, T and T's partial sums
  ep.early_weights = 1;
  if (pair) {
    // T [M, r] and L2 [r, N] tiles for the tensor-core low-rank product:
    // 64 bf16 (128 bytes) wide, r zero-padded by the copy
    alignas(64) CUtensorMap tt, tl2;
    if ((st = make_map(&tt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, t, r, M, static_cast<int64_t>(r) * 2, 64, kBM)) !=
        W8A8_OK)
      return st;
    if ((st = make_map(&tl2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, l2, N, r, N * 2, 64, 32)) != W8A8_OK) return st;
    return launch_gemm_pair<kKind, false, true>(ta, tb, M, N, K, ep, s, &tt, &tl2);
  }
  return launch_gemm<kKind, false, 256, kEpiLowRank>(ta, tb, M, N, K, ep, s);
}

// Tracing: every compute call of the C ABI is one NVTX range named after the
// call (its launches nest inside it in a profiler's timeline).  The NVTX
// header is inert until a profiling tool injects itself, so an untraced run
// pays one predictable branch per call.
struct TraceRange {
  explicit TraceRange(const char* name) { nvtxRangePushA(name); }
  ~TraceRange() { nvtxRangePop(); }
  TraceRange(const TraceRange&) = delete;
  TraceRange& operator=(const TraceRange&) = delete;
};
#define W8A8_TRACE() const TraceRange w8a8_trace_range_(__func__)

extern "C" {

const char* w8a8_last_error(void) { return t_last_error.c_str(); }

size_t q8_0_bytes(int64_t n) { return n <= 0 ? 0 : static_cast<size_t>((n + 31) / 32) * 34; }

size_t w8a8_workspace_bytes(int op, int64_t M, int64_t N, int64_t K, int r) {
  if (M < 0 || N < 0 || K < 0) return 0;
  switch (op) {
    case W8A8_OP_LINEAR_FWD: return ws_linear(M, K, N, true);
    case W8A8_OP_LINEAR_DGRAD: return ws_linear(M, round_up(N, 16), K);
    case W8A8_OP_SVDQ_FWD: return ws_svdq(M, K, r);
    case W8A8_OP_QUANTIZE_WEIGHT: return 256;
    case W8A8_OP_BF16_FWD: return ws_bf16(M, N, K);
    case W8A8_OP_WEIGHT_ONLY_FWD: return ws_weight_only(M, N, K);
    case W8A8_OP_BF16_DGRAD: return ws_bf16_dgrad(M, N, K);
    case W8A8_OP_WEIGHT_ONLY_DGRAD: return ws_weight_only_dgrad(M, N, K);
    default: return 0;
  }
}

w8a8_status w8a8_quantize_rows(const void* x, int64_t M, int64_t K, int64_t ldx, w8a8_qtype qt, void* q,
                               int64_t ldq, float* s, w8a8_stream_t stream) {
  W8A8_TRACE();
  W8A8_CHECK(valid_qt(qt), W8A8_ERR_INVALID_ARG, "invalid qtype %d", static_cast<int>(qt));
  W8A8_CHECK(M >= 0, W8A8_ERR_UNSUPPORTED_SHAPE, "M < 0");
  w8a8_status st = check_k(K, "K");
  if (st != W8A8_OK) return st;
  W8A8_CHECK(ldx >= K && ldx % 8 == 0, W8A8_ERR_MISALIGNED, "ldx must be >= K and a multiple of 8");
  W8A8_CHECK(ldq >= K && ldq % 16 == 0, W8A8_ERR_MISALIGNED, "ldq must be >= K and a multiple of 16");
  if (M == 0) return W8A8_OK;   // empty tensors may carry null pointers
  W8A8_CHECK(x && q && s, W8A8_ERR_INVALID_ARG, "null pointer");
  W8A8_CHECK(aligned16(x) && aligned16(q) && aligned16(s), W8A8_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  if ((st = current_device(nullptr, nullptr)) != W8A8_OK) return st;
  return launch_quantize_rows(x, ldx, M, K, qt, q, ldq, s, reinterpret_cast<cudaStream_t>(stream));
}

w8a8_status w8a8_quantize_weight(const void* w, int64_t N, int64_t K, w8a8_qtype qt, w8a8_wgran g, void* q,
                                 float* scale, void* ws, size_t ws_bytes, w8a8_stream_t stream) {
  W8A8_TRACE();
  W8A8_CHECK(valid_qt(qt) && valid_g(g), W8A8_ERR_INVALID_ARG, "invalid qtype/granularity");
  W8A8_CHECK(N >= 1, W8A8_ERR_UNSUPPORTED_SHAPE, "N < 1");
  w8a8_status st = check_k(K, "K");
  if (st != W8A8_OK) return st;
  W8A8_CHECK(w && q && scale, W8A8_ERR_INVALID_ARG, "null pointer");
  W8A8_CHECK(aligned16(w) && aligned16(q) && aligned16(scale), W8A8_ERR_MISALIGNED,
             "pointers must be 16-byte aligned");
  if (g == W8A8_TENSOR) {
    W8A8_CHECK(ws != nullptr && ws_bytes >= 256, W8A8_ERR_WORKSPACE, "tensor-wise quantization needs 256 B workspace");
    W8A8_CHECK(aligned16(ws), W8A8_ERR_MISALIGNED, "workspace must be 16-byte aligned");
  }
  int sms = 0;
  if ((st = current_device(nullptr, &sms)) != W8A8_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (g == W8A8_AXIS) return launch_quantize_rows(w, K, N, K, qt, q, K, scale, s);
  const int64_t nvec = N * K / 8;
  unsigned* amax = static_cast<unsigned*>(ws);
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(unsigned), s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  int64_t blocks = (nvec + 255) / 256;
  if (blocks > 8 * sms) blocks = 8 * sms;
  absmax_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(static_cast<const uint4*>(w), nvec, amax);
  if (qt == W8A8_E4M3)
    quantize_tensor_kernel<1><<<static_cast<int>(blocks), 256, 0, s>>>(static_cast<const uint4*>(w), nvec, amax,
                                                                       static_cast<uint2*>(q), scale);
  else
    quantize_tensor_kernel<0><<<static_cast<int>(blocks), 256, 0, s>>>(static_cast<const uint4*>(w), nvec, amax,
                                                                       static_cast<uint2*>(q), scale);
  e = cudaGetLastError();
  return e == cudaSuccess ? W8A8_OK : cuda_fail(e, "quantize_weight launch");
}

w8a8_status q8_0_quantize(const float* x, int64_t n, void* blocks, w8a8_stream_t stream) {
  W8A8_TRACE();
  W8A8_CHECK(n >= 0, W8A8_ERR_UNSUPPORTED_SHAPE, "n < 0");
  if (n == 0) return W8A8_OK;
  W8A8_CHECK(x && blocks, W8A8_ERR_INVALID_ARG, "null pointer");
  W8A8_CHECK(aligned16(x) && aligned16(blocks), W8A8_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  int sms = 0;
  w8a8_status st = current_device(nullptr, &sms);
  if (st != W8A8_OK) return st;
  const int64_t chunks = (n + 256 * kQ80Unroll - 1) / (256 * kQ80Unroll);
  int64_t grid = (chunks + kQ80WarpsPerBlock - 1) / kQ80WarpsPerBlock;
  if (grid > 16 * sms) grid = 16 * sms;
  q8_0_quantize_kernel<<<static_cast<int>(grid), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      x, n, static_cast<uint8_t*>(blocks));
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W8A8_OK : cuda_fail(e, "q8_0_quantize launch");
}

w8a8_status q8_0_dequantize(const void* blocks, int64_t n, float* y, w8a8_stream_t stream) {
  W8A8_TRACE();
  W8A8_CHECK(n >= 0, W8A8_ERR_UNSUPPORTED_SHAPE, "n < 0");
  if (n == 0) return W8A8_OK;
  W8A8_CHECK(y && blocks, W8A8_ERR_INVALID_ARG, "null pointer");
  W8A8_CHECK(aligned16(y) && aligned16(blocks), W8A8_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  return launch_q8_0_dequant<false>(blocks, n, y, reinterpret_cast<cudaStream_t>(stream));
}

w8a8_status q8_0_dequantize_bf16(const void* blocks, int64_t n, void* y, w8a8_stream_t stream) {
  W8A8_TRACE();
  W8A8_CHECK(n >= 0, W8A8_ERR_UNSUPPORTED_SHAPE, "n < 0");
  if (n == 0) return W8A8_OK;
  W8A8_CHECK(y && blocks, W8A8_ERR_INVALID_ARG, "null pointer");
  W8A8_CHECK(aligned16(y) && aligned16(blocks), W8A8_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  return launch_q8_0_dequant<true>(blocks, n, y, reinterpret_cast<cudaStream_t>(stream));
}

w8a8_status w8a8_dequantize_e4m3_bf16(const void* q, int64_t n, const float* scale, void* w,
                                      w8a8_stream_t stream) {
  W8A8_TRACE();
  W8A8_CHECK(n >= 0 && n % 16 == 0, W8A8_ERR_UNSUPPORTED_SHAPE, "n must be a non-negative multiple of 16");
  if (n == 0) return W8A8_OK;
  W8A8_CHECK(q && scale && w, W8A8_ERR_INVALID_ARG, "null pointer");
  W8A8_CHECK(aligned16(q) && aligned16(scale) && aligned16(w), W8A8_ERR_MISALIGNED,
             "pointers must be 16-byte aligned");
  return launch_dequant_e4m3(q, n, scale, w, reinterpret_cast<cudaStream_t>(stream));
}

// Shared argument checks of the bf16-Linear entry points.
static w8a8_status check_bf16_linear(const void* x, int64_t M, int64_t N, int64_t K, const void* w, const void* bias,
                                     const void* y, const void* ws, size_t ws_bytes, size_t need,
                                     bool need_scale = false, const void* scale = nullptr) {
  W8A8_CHECK(M >= 0 && N >= 1 && M < (1ll << 31) && N < (1ll << 31), W8A8_ERR_UNSUPPORTED_SHAPE, "bad M/N");
  w8a8_status st = check_k(K, "K");
  if (st != W8A8_OK) return st;
  if (M == 0) return W8A8_OK;
  W8A8_CHECK(x && w && y && (!need_scale || scale), W8A8_ERR_INVALID_ARG, "null pointer");
  W8A8_CHECK(aligned16(x) && aligned16(w) && aligned16(y) && (bias == nullptr || aligned16(bias)) &&
                 (!need_scale || aligned16(scale)),
             W8A8_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  W8A8_CHECK(need == 0 || (ws != nullptr && ws_bytes >= need), W8A8_ERR_WORKSPACE, "workspace too small: need %zu bytes",
             need);
  W8A8_CHECK(ws == nullptr || aligned16(ws), W8A8_ERR_MISALIGNED, "workspace must be 16-byte aligned");
  return current_device(nullptr, nullptr);
}

w8a8_status bf16_linear_fwd(const void* x, int64_t M, int64_t N, int64_t K, const void* w, const void* bias, void* y,
                            void* ws, size_t ws_bytes, w8a8_stream_t stream) {
  W8A8_TRACE();
  w8a8_status st = check_bf16_linear(x, M, N, K, w, bias, y, ws, ws_bytes, M > 0 ? ws_bf16(M, N, K) : 0);
  if (st != W8A8_OK || M == 0) return st;
  Carve c(ws);
  return gemm_bf16(x, M, N, K, w, bias, y, c, reinterpret_cast<cudaStream_t>(stream));
}

w8a8_status float8_linear_fwd(const void* x, int64_t M, int64_t N, int64_t K, const void* wq, const float* w_scale,
                              const void* bias, void* y, void* ws, size_t ws_bytes, w8a8_stream_t stream) {
  W8A8_TRACE();
  w8a8_status st = check_bf16_linear(x, M, N, K, wq, bias, y, ws, ws_bytes, M > 0 ? ws_weight_only(M, N, K) : 0,
                                     true, w_scale);
  if (st != W8A8_OK || M == 0) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Carve c(ws);
  void* wb = c.take(static_cast<size_t>(N) * static_cast<size_t>(K) * 2);
  if ((st = launch_dequant_e4m3(wq, N * K, w_scale, wb, s)) != W8A8_OK) return st;
  return gemm_bf16(x, M, N, K, wb, bias, y, c, s);
}

// dgrad argument checks: dy [M, N] (N % 8 == 0: 16-byte rows), dx [M, K].
static w8a8_status check_bf16_dgrad(const void* dy, int64_t M, int64_t N, int64_t K, const void* w, const void* dx,
                                    const void* ws, size_t ws_bytes, size_t need, bool need_scale = false,
                                    const void* scale = nullptr) {
  W8A8_CHECK(N >= 8 && N % 8 == 0, W8A8_ERR_UNSUPPORTED_SHAPE, "N must be a multiple of 8 (16-byte dY rows)");
  return check_bf16_linear(dy, M, N, K, w, nullptr, dx, ws, ws_bytes, need, need_scale, scale);
}

w8a8_status bf16_linear_dgrad(const void* dy, int64_t M, int64_t N, int64_t K, const void* w, void* dx, void* ws,
                              size_t ws_bytes, w8a8_stream_t stream) {
  W8A8_TRACE();
  w8a8_status st = check_bf16_dgrad(dy, M, N, K, w, dx, ws, ws_bytes, M > 0 ? ws_bf16_dgrad(M, N, K) : 0);
  if (st != W8A8_OK || M == 0) return st;
  Carve c(ws);
  return gemm_bf16_t<true>(dy, M, N, K, w, nullptr, dx, c, reinterpret_cast<cudaStream_t>(stream));
}

w8a8_status float8_linear_dgrad(const void* dy, int64_t M, int64_t N, int64_t K, const void* wq,
                                const float* w_scale, void* dx, void* ws, size_t ws_bytes, w8a8_stream_t stream) {
  W8A8_TRACE();
  w8a8_status st = check_bf16_dgrad(dy, M, N, K, wq, dx, ws, ws_bytes, M > 0 ? ws_weight_only_dgrad(M, N, K) : 0,
                                    true, w_scale);
  if (st != W8A8_OK || M == 0) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Carve c(ws);
  void* wb = c.take(static_cast<size_t>(N) * static_cast<size_t>(K) * 2);
  if ((st = launch_dequant_e4m3(wq, N * K, w_scale, wb, s)) != W8A8_OK) return st;
  return gemm_bf16_t<true>(dy, M, N, K, wb, nullptr, dx, c, s);
}

w8a8_status gguf_linear_dgrad(const void* dy, int64_t M, int64_t N, int64_t K, const void* blocks, void* dx, void* ws,
                              size_t ws_bytes, w8a8_stream_t stream) {
  W8A8_TRACE();
  w8a8_status st = check_bf16_dgrad(dy, M, N, K, blocks, dx, ws, ws_bytes, M > 0 ? ws_weight_only_dgrad(M, N, K) : 0);
  if (st != W8A8_OK || M == 0) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Carve c(ws);
  void* wb = c.take(static_cast<size_t>(N) * static_cast<size_t>(K) * 2);
  if ((st = launch_q8_0_dequant<true>(blocks, N * K, wb, s)) != W8A8_OK) return st;
  return gemm_bf16_t<true>(dy, M, N, K, wb, nullptr, dx, c, s);
}

w8a8_status gguf_linear_fwd(const void* x, int64_t M, int64_t N, int64_t K, const void* blocks, const void* bias,
                            void* y, void* ws, size_t ws_bytes, w8a8_stream_t stream) {
  W8A8_TRACE();
  w8a8_status st = check_bf16_linear(x, M, N, K, blocks, bias, y, ws, ws_bytes, M > 0 ? ws_weight_only(M, N, K) : 0);
  if (st != W8A8_OK || M == 0) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Carve c(ws);
  void* wb = c.take(static_cast<size_t>(N) * static_cast<size_t>(K) * 2);
  if ((st = launch_q8_0_dequant<true>(blocks, N * K, wb, s)) != W8A8_OK) return st;
  return gemm_bf16(x, M, N, K, wb, bias, y, c, s);
}

w8a8_status q8_0_to_axis_int8(const void* blocks, int64_t N, int64_t K, int8_t* q, float* scale,
                              w8a8_stream_t stream) {
  W8A8_TRACE();
  return requant_axis<0>(blocks, N, K, reinterpret_cast<uint8_t*>(q), scale, stream, "q8_0_to_axis_int8 launch");
}

w8a8_status q8_0_to_axis_e4m3(const void* blocks, int64_t N, int64_t K, uint8_t* q, float* scale,
                              w8a8_stream_t stream) {
  W8A8_TRACE();
  return requant_axis<1>(blocks, N, K, q, scale, stream, "q8_0_to_axis_e4m3 launch");
}

w8a8_status w8a8_qgemm_fwd(const void* xq, int64_t ldq, const float* sx, int64_t M, int64_t N, int64_t K,
                           w8a8_qtype qt, const void* wq, const float* sw, w8a8_wgran g, const void* bias, void* y,
                           w8a8_stream_t stream) {
  W8A8_TRACE();
  W8A8_CHECK(valid_qt(qt) && valid_g(g), W8A8_ERR_INVALID_ARG, "invalid qtype/granularity");
  W8A8_CHECK(M >= 0 && N >= 1 && M < (1ll << 31) && N < (1ll << 31), W8A8_ERR_UNSUPPORTED_SHAPE, "bad M/N");
  w8a8_status st = check_k(K, "K");
  if (st != W8A8_OK) return st;
  W8A8_CHECK(ldq >= K && ldq % 16 == 0, W8A8_ERR_MISALIGNED, "ldq must be >= K and a multiple of 16");
  if (M == 0) return W8A8_OK;
  W8A8_CHECK(xq && sx && wq && sw && y, W8A8_ERR_INVALID_ARG, "null pointer");
  W8A8_CHECK(aligned16(xq) && aligned16(sx) && aligned16(wq) && aligned16(sw) && aligned16(y) &&
                 (bias == nullptr || aligned16(bias)),
             W8A8_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  if ((st = current_device(nullptr, nullptr)) != W8A8_OK) return st;
  return gemm_fwd(xq, ldq, sx, M, N, K, qt, wq, sw, g, bias, y, reinterpret_cast<cudaStream_t>(stream));
}

w8a8_status w8a8_qgemm_dgrad(const void* dyq, int64_t ldq, const float* sdy, int64_t M, int64_t N, int64_t K,
                             w8a8_qtype qt, const void* wq, const float* sw, void* dx, w8a8_stream_t stream) {
  W8A8_TRACE();
  W8A8_CHECK(valid_qt(qt), W8A8_ERR_INVALID_ARG, "invalid qtype");
  W8A8_CHECK(M >= 0 && M < (1ll << 31), W8A8_ERR_UNSUPPORTED_SHAPE, "bad M");
  w8a8_status st = check_k(K, "K");
  if (st != W8A8_OK) return st;
  if ((st = check_k(N, "N")) != W8A8_OK) return st;
  W8A8_CHECK(ldq >= N && ldq % 16 == 0, W8A8_ERR_MISALIGNED, "ldq must be >= N and a multiple of 16");
  if (M == 0) return W8A8_OK;
  W8A8_CHECK(dyq && sdy && wq && sw && dx, W8A8_ERR_INVALID_ARG, "null pointer");
  W8A8_CHECK(aligned16(dyq) && aligned16(sdy) && aligned16(wq) && aligned16(sw) && aligned16(dx),
             W8A8_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  if ((st = current_device(nullptr, nullptr)) != W8A8_OK) return st;
  return gemm_dgrad(dyq, ldq, sdy, M, N, K, qt, wq, sw, dx, reinterpret_cast<cudaStream_t>(stream));
}

w8a8_status w8a8_linear_fwd(const void* x, int64_t M, int64_t N, int64_t K, w8a8_qtype qt, const void* wq,
                            const float* sw, w8a8_wgran g, const void* bias, void* y, void* ws, size_t ws_bytes,
                            w8a8_stream_t stream) {
  W8A8_TRACE();
  return w8a8_linear_fwd_ex(x, M, N, K, qt, wq, sw, g, bias, W8A8_ACT_NONE, nullptr, nullptr, y, ws, ws_bytes, stream);
}

w8a8_status w8a8_linear_fwd_ex(const void* x, int64_t M, int64_t N, int64_t K, w8a8_qtype qt, const void* wq,
                               const float* sw, w8a8_wgran g, const void* bias, w8a8_act act, const uint32_t* x_amax,
                               uint32_t* y_amax, void* y, void* ws, size_t ws_bytes, w8a8_stream_t stream) {
  W8A8_TRACE();
  W8A8_CHECK(valid_qt(qt) && valid_g(g), W8A8_ERR_INVALID_ARG, "invalid qtype/granularity");
  W8A8_CHECK(act == W8A8_ACT_NONE || act == W8A8_ACT_GELU || act == W8A8_ACT_GELU_TANH, W8A8_ERR_INVALID_ARG,
             "invalid activation %d", static_cast<int>(act));
  W8A8_CHECK(M >= 0 && N >= 1 && M < (1ll << 31) && N < (1ll << 31), W8A8_ERR_UNSUPPORTED_SHAPE, "bad M/N");
  w8a8_status st = check_k(K, "K");
  if (st != W8A8_OK) return st;
  if (M == 0) return W8A8_OK;   // empty tensors may carry null pointers
  W8A8_CHECK(x && wq && sw && y, W8A8_ERR_INVALID_ARG, "null pointer");
  W8A8_CHECK(aligned16(x) && aligned16(wq) && aligned16(sw) && aligned16(y) && (bias == nullptr || aligned16(bias)) &&
                 (x_amax == nullptr || aligned16(x_amax)) && (y_amax == nullptr || aligned16(y_amax)),
             W8A8_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  W8A8_CHECK(x_amax == nullptr || y_amax == nullptr || x_amax != y_amax, W8A8_ERR_INVALID_ARG,
             "x_amax and y_amax must be different buffers");
  const LinearWs lw = linear_ws(M, K, N, true);
  W8A8_CHECK(ws != nullptr && ws_bytes >= lw.bytes, W8A8_ERR_WORKSPACE, "workspace too small: need %zu bytes",
             lw.bytes);
  W8A8_CHECK(aligned16(ws), W8A8_ERR_MISALIGNED, "workspace must be 16-byte aligned");
  if ((st = current_device(nullptr, nullptr)) != W8A8_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool plain = act == W8A8_ACT_NONE && x_amax == nullptr && y_amax == nullptr;
  // A few tokens: one weight-streaming launch on the CUDA cores.  Measured
  // at N = 12288, K = 3072 against quantize + the transposed tensor-core
  // GEMM (about 13.5-14 us from 3 to 64 rows): int8 wins for 1 and 2 rows
  // (9.5 / 11.5 us; 13.9 at 3, 16.8 at 4), e4m3 (decoded in fp32) for one
  // row only (13.5 us).
  if (plain && qt == W8A8_INT8 && M <= kGemvUseRows && K <= kGemvMaxK)
    return launch_gemv(x, M, N, K, wq, sw, g == W8A8_AXIS, bias, y, s);
  if (plain && qt == W8A8_E4M3 && M == 1 && gemv_e4m3_fits(M, K))
    return launch_gemv_e4m3(x, M, N, K, wq, sw, g == W8A8_AXIS, bias, y, s);
  Carve c(ws);
  void* xq = c.take(static_cast<size_t>(M * K));
  float* sx = static_cast<float*>(c.take(static_cast<size_t>(M) * 4));
  const SplitWs sk = carve_split(c, M, N, lw, qt);
  // the quantizer clears y_amax; the GEMM's epilogue runs after it completes
  if ((st = launch_quantize_rows(x, K, M, K, qt, xq, K, sx, s, x_amax, y_amax, y_amax ? M : 0)) != W8A8_OK) return st;
  return gemm_fwd(xq, K, sx, M, N, K, qt, wq, sw, g, bias, y, s, &sk, static_cast<int>(act), y_amax,
                  /*early_weights=*/true);
}

w8a8_status w8a8_linear_fwd_noalloc(const void* x, int64_t M, int64_t N, int64_t K, w8a8_qtype qt, const void* wq,
                                    const float* sw, w8a8_wgran g, const void* bias, void* y, w8a8_stream_t stream) {
  W8A8_TRACE();
  W8A8_CHECK(valid_qt(qt) && valid_g(g), W8A8_ERR_INVALID_ARG, "invalid qtype/granularity");
  W8A8_CHECK(M >= 0 && N >= 1 && M < (1ll << 31) && N < (1ll << 31), W8A8_ERR_UNSUPPORTED_SHAPE, "bad M/N");
  w8a8_status st = check_k(K, "K");
  if (st != W8A8_OK) return st;
  if (M == 0) return W8A8_OK;
  W8A8_CHECK(M <= W8A8_NOALLOC_MAX_ROWS && static_cast<uint64_t>(M) * static_cast<uint64_t>(K) <= W8A8_NOALLOC_MAX_CODES,
             W8A8_ERR_WORKSPACE,
             "w8a8_linear_fwd_noalloc: M=%lld, M*K=%lld exceed the built-in scratch (M <= %lld, M*K <= %llu); "
             "use w8a8_linear_fwd with a workspace",
             static_cast<long long>(M), static_cast<long long>(M * K), static_cast<long long>(W8A8_NOALLOC_MAX_ROWS),
             static_cast<unsigned long long>(W8A8_NOALLOC_MAX_CODES));
  W8A8_CHECK(x && wq && sw && y, W8A8_ERR_INVALID_ARG, "null pointer");
  W8A8_CHECK(aligned16(x) && aligned16(wq) && aligned16(sw) && aligned16(y) && (bias == nullptr || aligned16(bias)),
             W8A8_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  if ((st = current_device(nullptr, nullptr)) != W8A8_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The few-token kernels need no scratch: the same dispatch as
  // w8a8_linear_fwd, so that both compute the same bits.
  if (qt == W8A8_INT8 && M <= kGemvUseRows && K <= kGemvMaxK)
    return launch_gemv(x, M, N, K, wq, sw, g == W8A8_AXIS, bias, y, s);
  if (qt == W8A8_E4M3 && M == 1 && gemv_e4m3_fits(M, K))
    return launch_gemv_e4m3(x, M, N, K, wq, sw, g == W8A8_AXIS, bias, y, s);
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != W8A8_OK) return st;
  void* xq = scratch;
  float* sx = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + W8A8_NOALLOC_MAX_CODES);
  if ((st = launch_quantize_rows(x, K, M, K, qt, xq, K, sx, s)) != W8A8_OK) return st;
  return gemm_fwd(xq, K, sx, M, N, K, qt, wq, sw, g, bias, y, s, nullptr, kActNone, nullptr, /*early_weights=*/true);
}

w8a8_status w8a8_linear_dgrad(const void* dy, int64_t M, int64_t N, int64_t K, w8a8_qtype qt, const void* wq,
                              const float* sw, w8a8_wgran g, void* dx, void* ws, size_t ws_bytes,
                              w8a8_stream_t stream) {
  W8A8_TRACE();
  W8A8_CHECK(valid_qt(qt) && valid_g(g), W8A8_ERR_INVALID_ARG, "invalid qtype/granularity");
  W8A8_CHECK(g == W8A8_TENSOR, W8A8_ERR_INVALID_ARG, "dgrad reads a tensor-wise weight scale");
  W8A8_CHECK(M >= 0 && M < (1ll << 31), W8A8_ERR_UNSUPPORTED_SHAPE, "bad M");
  w8a8_status st = check_k(K, "K");
  if (st != W8A8_OK) return st;
  if ((st = check_k(N, "N")) != W8A8_OK) return st;
  if (M == 0) return W8A8_OK;
  W8A8_CHECK(dy && wq && sw && dx, W8A8_ERR_INVALID_ARG, "null pointer");
  W8A8_CHECK(aligned16(dy) && aligned16(wq) && aligned16(sw) && aligned16(dx), W8A8_ERR_MISALIGNED,
             "pointers must be 16-byte aligned");
  const LinearWs lw = linear_ws(M, N, K);
  W8A8_CHECK(ws != nullptr && ws_bytes >= lw.bytes, W8A8_ERR_WORKSPACE, "workspace too small: need %zu bytes",
             lw.bytes);
  W8A8_CHECK(aligned16(ws), W8A8_ERR_MISALIGNED, "workspace must be 16-byte aligned");
  if ((st = current_device(nullptr, nullptr)) != W8A8_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Carve c(ws);
  void* dyq = c.take(static_cast<size_t>(M * N));
  float* sdy = static_cast<float*>(c.take(static_cast<size_t>(M) * 4));
  const SplitWs sk = carve_split(c, M, K, lw, qt);
  if ((st = launch_quantize_rows(dy, N, M, N, qt, dyq, N, sdy, s)) != W8A8_OK) return st;
  return gemm_dgrad(dyq, N, sdy, M, N, K, qt, wq, sw, dx, s, &sk, /*early_weights=*/true);
}

w8a8_status svdq_linear_fwd(const void* x, int64_t M, int64_t N, int64_t K, const void* rq, const float* r_scale,
                            int r, const void* l1, const void* l2, const void* bias, void* y, void* ws,
                            size_t ws_bytes, w8a8_stream_t stream) {
  W8A8_TRACE();
  return svdq_fwd_impl<W8A8_INT8>(x, M, N, K, rq, r_scale, r, l1, l2, bias, y, ws, ws_bytes, stream);
}

w8a8_status svdq_linear_fwd_e4m3(const void* x, int64_t M, int64_t N, int64_t K, const void* rq,
                                 const float* r_scale, int r, const void* l1, const void* l2, const void* bias,
                                 void* y, void* ws, size_t ws_bytes, w8a8_stream_t stream) {
  W8A8_TRACE();
  return svdq_fwd_impl<W8A8_E4M3>(x, M, N, K, rq, r_scale, r, l1, l2, bias, y, ws, ws_bytes, stream);
}

w8a8_status w8a8_device_status(w8a8_stream_t stream, int reset) {
  w8a8_status st = current_device(nullptr, nullptr);
  if (st != W8A8_OK) return st;
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned v = 0, site = 0;
  if ((e = cudaMemcpyFromSymbol(&v, g_status, sizeof(v))) != cudaSuccess) return cuda_fail(e, "read status");
  cudaMemcpyFromSymbol(&site, g_status_site, sizeof(site));
  if (reset) {
    const unsigned z = 0;
    cudaMemcpyToSymbol(g_status, &z, sizeof(z));
    cudaMemcpyToSymbol(g_status_site, &z, sizeof(z));
  }
  if (v == kDevOk) return W8A8_OK;
  if (v == kDevTimeout) return fail(W8A8_ERR_DEVICE_TIMEOUT, "device wait ran out (site 0x%x)", site);
  if (v == kDevBounds) return fail(W8A8_ERR_DEVICE_BOUNDS, "device index check failed (site 0x%x)", site);
  return fail(W8A8_ERR_CUDA, "device status %u (site 0x%x)", v, site);
}

w8a8_status w8a8_set_wait_limit_ns(uint64_t limit_ns) {
  w8a8_status st = current_device(nullptr, nullptr);
  if (st != W8A8_OK) return st;
  W8A8_CHECK(limit_ns > 0, W8A8_ERR_INVALID_ARG, "limit must be > 0");
  unsigned long long v = limit_ns;
  cudaError_t e = cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v));
  return e == cudaSuccess ? W8A8_OK : cuda_fail(e, "set wait limit");
}

w8a8_status w8a8_selftest_wait(uint64_t limit_ns, w8a8_stream_t stream) {
  W8A8_TRACE();
  W8A8_CHECK(limit_ns > 0 && limit_ns <= 10000000000ull, W8A8_ERR_INVALID_ARG, "limit must be in (0, 10 s]");
  w8a8_status st = current_device(nullptr, nullptr);
  if (st != W8A8_OK) return st;
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W8A8_OK : cuda_fail(e, "selftest launch");
}

w8a8_status w8a8_selftest_bounds(w8a8_stream_t stream) {
  W8A8_TRACE();
  w8a8_status st = current_device(nullptr, nullptr);
  if (st != W8A8_OK) return st;
  selftest_bounds_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(1024);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W8A8_OK : cuda_fail(e, "selftest launch");
}

int w8a8_debug_checks(void) { return W8A8_DEBUG_CHECKS; }

w8a8_status w8a8_e4m3_encode(const float* x, int64_t n, uint8_t* y, w8a8_stream_t stream) {
  W8A8_TRACE();
  W8A8_CHECK(n >= 0, W8A8_ERR_UNSUPPORTED_SHAPE, "n < 0");
  if (n == 0) return W8A8_OK;
  W8A8_CHECK(x && y, W8A8_ERR_INVALID_ARG, "null pointer");
  W8A8_CHECK(aligned16(x) && aligned16(y), W8A8_ERR_MISALIGNED, "pointers must be 16-byte aligned");
  int sms = 0;
  w8a8_status st = current_device(nullptr, &sms);
  if (st != W8A8_OK) return st;
  int64_t grid = (n + 255) / 256;
  if (grid > 16 * sms) grid = 16 * sms;
  e4m3_encode_kernel<<<static_cast<int>(grid), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, n, y);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W8A8_OK : cuda_fail(e, "e4m3 encode launch");
}

}  // extern "C"
