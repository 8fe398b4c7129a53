// qlin.cu -- the C ABI declared in include/qlin.h (single translation unit:
// the kernels of prep.cuh and gemm.cuh are instantiated and launched here).
//
// Host side of every entry point: validate arguments, carve the caller's
// workspace, build the TMA tensor maps, and enqueue kernels on the caller's
// stream. No device memory is allocated or freed and no stream is
// synchronised inside a forward.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "../../include/qlin.h"
#include "common.cuh"
#include "gemm.cuh"
#include "gemm_w4a8.cuh"
#include "gemm_cvt.cuh"
#include "prep.cuh"

using namespace qlin;

namespace {

thread_local char g_err[512] = "";

qlin_status fail(qlin_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

qlin_status ok() {
  g_err[0] = '\0';
  return QLIN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

constexpr int64_t kMaxK = 32768;

qlin_status check_cuda(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return fail(QLIN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return QLIN_OK;
}

// ---- per-device facts (SM count, sm_100 check), cached ------------------
struct DeviceInfo {
  int sms = 0;
  bool sm100 = false;
  // set once per kernel instantiation; host threads may race to set it, and
  // setting a function attribute twice is harmless
  std::atomic<bool> gemm_attr_set[64] = {};
};
std::mutex g_dev_mu;
DeviceInfo g_dev[16];

qlin_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) return fail(QLIN_ERR_CUDA, "cudaGetDevice failed");
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.sms == 0) {
    cudaDeviceProp prop;
    qlin_status s = check_cuda(cudaGetDeviceProperties(&prop, dev), "cudaGetDeviceProperties");
    if (s != QLIN_OK) return s;
    d.sms = prop.multiProcessorCount;
    d.sm100 = (prop.major == 10 && prop.minor == 0);
  }
  if (!d.sm100) return fail(QLIN_ERR_UNSUPPORTED, "libqlin needs an sm_100 (B200) device");
  *out = &d;
  return QLIN_OK;
}

// ---- TMA descriptors -----------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

qlin_status get_encode(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  std::call_once(g_encode_once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  if (!g_encode) return fail(QLIN_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  *fn = g_encode;
  return QLIN_OK;
}

// 8-bit row-major [rows, K] matrix, box of box_rows x 128 bytes, 128B swizzle.
qlin_status make_tmap_k128(CUtensorMap* m, const void* base, int64_t rows, int64_t K, int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  qlin_status s = get_encode(&enc);
  if (s != QLIN_OK) return s;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(GEMM_BK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(QLIN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return QLIN_OK;
}

// 16-bit row-major Y [M, N] for the GEMM's TMA stores: box 16 columns x 32
// rows, 32-byte swizzle (the epilogue writes its staging boxes in that layout).
qlin_status make_tmap_y16(CUtensorMap* m, void* Y, int64_t M, int64_t N) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  qlin_status s = get_encode(&enc);
  if (s != QLIN_OK) return s;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(N * 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(GEMM_CW), 32u};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, Y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(QLIN_ERR_CUDA, "cuTensorMapEncodeTiled (Y) failed (%d)", static_cast<int>(r));
  return QLIN_OK;
}

// ---- GEMM launch ------------------------------------------------------------
// Tile width: 128 x 256 tiles (4 stages) unless the problem has too few of
// them to fill the SMs; then 128 x 128 tiles (6 stages), whose MMAs move
// twice the operand bytes per MAC and are counted at 75% (measured: the
// text-encoder gate projection, 192 wide tiles in two waves, ran as fast as
// with 384 narrow ones in three; its down projection, 64 wide tiles, gained
// a quarter from 128 narrow ones). The int8 GEMMs with a workspace may run
// 128 x 256 tiles under stream-K instead, when the last wave of whole tiles
// would leave many SMs idle.
qlin_status make_tmap_bytes(CUtensorMap* m, const void* base, int64_t rows, int64_t row_bytes, int box_inner,
                            int box_rows, CUtensorMapSwizzle sw, int64_t stride_bytes = 0);
static_assert(kMaxK == OUTL_MAX_K, "the streaming pass keeps a bitmap of up to kMaxK columns in shared memory");
static_assert(OUTL_CODES == GEMM_CORR_K, "the prep's compact outlier codes feed the GEMM's correction MMA");

template <int KIND, int EPI, typename TOut, int BN, int STAGES>
qlin_status launch_gemm_bn(const CUtensorMap& ta, const void* B, EpiParams ep, const CUtensorMap& ty,
                           DeviceInfo* d, cudaStream_t st, int attr_slot, int grid_ctas = 0) {
  qlin_status s;
  CUtensorMap tb, txc, twc, txo, two;
  if ((s = make_tmap_k128(&tb, B, ep.N, ep.K, BN)) != QLIN_OK) return s;
  std::memset(&txc, 0, sizeof(txc));
  std::memset(&twc, 0, sizeof(twc));
  std::memset(&txo, 0, sizeof(txo));
  std::memset(&two, 0, sizeof(two));
  if constexpr (EPI == EPI_INT8_OUTLIER || EPI == EPI_INT8_OUTLIER_I32) {
    // -Xq[:,O] [M,32] and Wq[:,O] [N,32] for the correction MMA (32B swizzle)
    if ((s = make_tmap_bytes(&txc, ep.XqO, ep.M, GEMM_CORR_K, GEMM_CORR_K, GEMM_BM, CU_TENSOR_MAP_SWIZZLE_32B)) != QLIN_OK)
      return s;
    if ((s = make_tmap_bytes(&twc, ep.WqO, ep.N, GEMM_CORR_K, GEMM_CORR_K, BN, CU_TENSOR_MAP_SWIZZLE_32B)) != QLIN_OK)
      return s;
  }
  if constexpr (EPI == EPI_INT8_OUTLIER && BN == 128) {
    // X_O [M,16] and W_O [N,16] (16-bit, first 16 of ostride columns, zero
    // past the count) for the fp outlier MMA (32B swizzle)
    constexpr int FB = GEMM_OUTL_STAGED * 2;
    if ((s = make_tmap_bytes(&txo, ep.X_O, ep.M, FB, FB, GEMM_BM, CU_TENSOR_MAP_SWIZZLE_32B, 2 * ep.ostride)) !=
        QLIN_OK)
      return s;
    if ((s = make_tmap_bytes(&two, ep.W_O, ep.N, FB, FB, BN, CU_TENSOR_MAP_SWIZZLE_32B, 2 * ep.ostride)) != QLIN_OK)
      return s;
  }
  auto kern = k_gemm<KIND, EPI, TOut, BN, STAGES>;
  constexpr int smem = GemmSmem<BN, STAGES>::TOTAL;
  static_assert(smem <= 227 * 1024, "k_gemm shared memory");
  if (!d->gemm_attr_set[attr_slot].load(std::memory_order_acquire)) {
    // the kernel's warpgroups trade registers with setmaxnreg: the launch
    // register count must leave enough in the block's pool for the split
    cudaFuncAttributes fa{};
    s = check_cuda(cudaFuncGetAttributes(&fa, kern), "cudaFuncGetAttributes");
    if (s != QLIN_OK) return s;
    if (fa.numRegs < GEMM_REGS_MIN_LAUNCH || fa.numRegs > GEMM_REGS_HIGH)
      return fail(QLIN_ERR_UNSUPPORTED, "k_gemm was built with %d registers per thread; the register split needs %d..%d",
                  fa.numRegs, GEMM_REGS_MIN_LAUNCH, GEMM_REGS_HIGH);
    s = check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
                   "cudaFuncSetAttribute");
    if (s != QLIN_OK) return s;
    d->gemm_attr_set[attr_slot].store(true, std::memory_order_release);
  }
  const int64_t tiles = ((ep.M + GEMM_BM - 1) / GEMM_BM) * ((ep.N + BN - 1) / BN);
  const int grid = grid_ctas > 0 ? grid_ctas : static_cast<int>(tiles < d->sms ? tiles : d->sms);
  // programmatic dependent launch: the CTAs may start (barrier set-up, TMEM
  // allocation) while the kernel before them finishes; they wait for it with
  // griddepcontrol.wait before touching its outputs
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(GEMM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return check_cuda(cudaLaunchKernelEx(&cfg, kern, ta, tb, ty, txc, twc, txo, two, ep), "k_gemm launch");
}

// Work schedule of the int8 GEMMs (qlin_set_gemm_schedule): 0 automatic,
// 1 whole tiles only, 2 stream-K wherever the workspace has partial slots.
std::atomic<int> g_gemm_schedule{0};

// Tile width and schedule. Costs are in k-blocks of 128 x 256 main loop on the
// busiest SM. Tile width: whole 128 x 256 tiles take ceil(tiles / SMs) * KB,
// whole 128 x 128 tiles ceil(tiles / SMs) * KB * 2/3 (half the work at 75% of
// the rate). Stream-K (int8 with a workspace; sk_cap = the CTAs its partial
// slots serve, 0: none) keeps all but the last two waves of whole tiles and
// cuts the rest into equal ranges: it pays when the main loop, not the
// epilogue, bounds a tile (each CTA still runs an epilogue per tile it
// finishes, GEMM_EPI_KB each, and its ranges add up to two more).
template <int KIND, int EPI, typename TOut>
qlin_status launch_gemm(const void* A, const void* B, EpiParams ep, cudaStream_t st, int attr_slot,
                        int sk_cap = 0) {
  DeviceInfo* d;
  qlin_status s = device_info(&d);
  if (s != QLIN_OK) return s;
  CUtensorMap ta, ty;
  if ((s = make_tmap_k128(&ta, A, ep.M, ep.K, GEMM_BM)) != QLIN_OK) return s;
  std::memset(&ty, 0, sizeof(ty));
  ep.tma_y = 0;
  // 16-bit Y goes out through TMA when its rows are 16-byte multiples and it is 16-byte aligned
  constexpr bool y16 = EPI != EPI_I32 && EPI != EPI_INT8_OUTLIER_I32;
  if (y16 && ep.N % 8 == 0 && aligned16(ep.Y)) {
    if ((s = make_tmap_y16(&ty, ep.Y, ep.M, ep.N)) != QLIN_OK) return s;
    ep.tma_y = 1;
  }
  const int64_t mt = (ep.M + GEMM_BM - 1) / GEMM_BM;
  const int64_t sms = d->sms;
  const int64_t kb = (ep.K + GEMM_BK - 1) / GEMM_BK;
  const int64_t t256 = mt * ((ep.N + 255) / 256), t128 = mt * ((ep.N + 127) / 128);
  const double dp256 = static_cast<double>((t256 + sms - 1) / sms * kb);
  const double dp128 = static_cast<double>((t128 + sms - 1) / sms * kb) * (2.0 / 3.0);
  ep.sk = 0;
  ep.sk_dp_tiles = 0;
  // tile bands pay when A and B do not fit in L2 together (measured: the
  // 2048^2 block linears, 59-240 MB of operands, gained 2-24%; the 1024^2 up
  // projection, 51 MB, and the FP8 QKV, 41 MB, lost 1-2% to them)
  ep.group_m = (ep.M + ep.N) * ep.K > (int64_t{56} << 20) ? GEMM_GROUP_M : 0;
  const int mode = g_gemm_schedule.load(std::memory_order_relaxed);
  if constexpr (KIND == 0 || KIND == 1) {
    const int64_t G0 = std::min<int64_t>(sms, sk_cap);
    if (G0 >= 2 && mode != 1 && ep.sk_count != nullptr && ep.sk_part != nullptr) {
      const int64_t W = t256 / G0;                      // whole waves
      const int64_t dp_tiles = W >= 1 ? (W - 1) * G0 : 0;
      const int64_t tail = (t256 - dp_tiles) * kb;      // iterations cut into ranges
      const int64_t G = W >= 1 ? G0 : std::min<int64_t>(G0, tail / (mode == 2 ? 1 : GEMM_SK_MIN_ITERS));
      if (G >= 2) {
        const int64_t per = (tail + G - 1) / G;
        const int64_t segs = (per + kb - 1) / kb + 1;   // a cut tail, whole tiles, a cut head
        const double main = static_cast<double>((W >= 1 ? (W - 1) * kb : 0) + per + GEMM_SK_COST_KB);
        const double epi = (static_cast<double>(W >= 1 ? W - 1 : 0) + segs - 0.5) * GEMM_EPI_KB;
        const double dpc256 = static_cast<double>((t256 + sms - 1) / sms) * std::max<double>(kb, GEMM_EPI_KB);
        const double dpc128 =
            static_cast<double>((t128 + sms - 1) / sms) * std::max<double>(kb * (2.0 / 3.0), GEMM_EPI_KB / 2.0);
        if (mode == 2 || std::max(main, epi) < 0.95 * std::min(dpc256, dpc128)) {
          ep.sk = 1;
          ep.sk_dp_tiles = static_cast<int>(dp_tiles);
          // kind::f8f6f4 takes its counters from the caller's scratch: clear
          // them here, only when tiles are cut (the int8 prepare stage clears
          // its own); the kernel leaves them zero
          if constexpr (KIND == 1) {
            const qlin_status z = check_cuda(
                cudaMemsetAsync(ep.sk_count, 0, sizeof(int32_t) * GEMM_EPI_GROUPS * static_cast<size_t>(t256), st),
                "cudaMemsetAsync");
            if (z != QLIN_OK) return z;
          }
          return launch_gemm_bn<KIND, EPI, TOut, 256, 4>(ta, B, ep, ty, d, st, 2 * attr_slot, static_cast<int>(G));
        }
      }
    }
  }
  if (dp128 < dp256)
    return launch_gemm_bn<KIND, EPI, TOut, 128, 6>(ta, B, ep, ty, d, st, 2 * attr_slot + 1);
  return launch_gemm_bn<KIND, EPI, TOut, 256, 4>(ta, B, ep, ty, d, st, 2 * attr_slot);
}

// ---- row quantiser dispatch ---------------------------------------------------
template <typename T, int V, int CODE, bool SBF16, bool OUTL>
qlin_status launch_prep_v(const void* X, const PrepArgs& a, int sms, cudaStream_t st) {
  auto kern = k_prep_rows<T, V, CODE, SBF16, OUTL>;
  const size_t smem = static_cast<size_t>(PF_DEPTH) * V * RQ_THREADS * 16;
  static std::atomic<bool> attr_set[16] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 16 && !attr_set[dev].load(std::memory_order_acquire)) {
    qlin_status s0 = check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024),
                                "cudaFuncSetAttribute");
    if (s0 != QLIN_OK) return s0;
    attr_set[dev].store(true, std::memory_order_release);
  }
  int per_sm = 0;
  qlin_status s = check_cuda(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, RQ_THREADS, smem),
                             "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
  if (s != QLIN_OK) return s;
  if (per_sm < 1) return fail(QLIN_ERR_UNSUPPORTED, "row quantiser does not fit on an SM");
  const int units = RQ_WARPS / a.rw;
  const int64_t want = (a.M + units - 1) / units;
  const int64_t cap = static_cast<int64_t>(per_sm) * sms;
  const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(RQ_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  // LLM.int8: a programmatic dependent of k_ws_reset, which zeroes the row
  // counter and the bitmap this pass uses (it waits for it before using them)
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = OUTL ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return check_cuda(cudaLaunchKernelEx(&cfg, kern, static_cast<const T*>(X), a), "k_prep_rows launch");
}

template <typename T, int CODE, bool SBF16, bool OUTL>
qlin_status launch_prep(const void* X, PrepArgs a, cudaStream_t st) {
  if (a.M == 0) return QLIN_OK;
  DeviceInfo* d;
  qlin_status s = device_info(&d);
  if (s != QLIN_OK) return s;
  const int64_t KV = a.K / 8;
  int rw = 1;   // warps per row: the smallest power of two giving <= 6 vectors per lane
  while (rw < 8 && (KV + 32 * rw - 1) / (32 * rw) > 6) rw *= 2;
  a.rw = rw;
  const int64_t per = (KV + 32 * rw - 1) / (32 * rw);
  if (per <= 2) return launch_prep_v<T, 2, CODE, SBF16, OUTL>(X, a, d->sms, st);
  if (per <= 4) return launch_prep_v<T, 4, CODE, SBF16, OUTL>(X, a, d->sms, st);
  if (per <= 6) return launch_prep_v<T, 6, CODE, SBF16, OUTL>(X, a, d->sms, st);
  if (per <= 8) return launch_prep_v<T, 8, CODE, SBF16, OUTL>(X, a, d->sms, st);
  return launch_prep_v<T, 16, CODE, SBF16, OUTL>(X, a, d->sms, st);
}

// Largest 16-bit |x| pattern (of T) whose value is <= thr (thr > 0 finite):
// |x| > thr exactly when the pattern of |x| exceeds it.
template <typename T>
uint32_t threshold_bits(float thr) {
  auto val = [](uint32_t p) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value) return __bfloat162float(__ushort_as_bfloat16(static_cast<unsigned short>(p)));
    else return __half2float(__ushort_as_half(static_cast<unsigned short>(p)));
  };
  const uint32_t top = std::is_same<T, __nv_bfloat16>::value ? 0x7F7Fu : 0x7BFFu;   // largest finite
  if (val(top) <= thr) return top;
  uint32_t lo = 0, hi = top;   // val(lo) <= thr < val(hi)
  while (hi - lo > 1) {
    const uint32_t mid = (lo + hi) / 2;
    if (val(mid) <= thr) lo = mid;
    else hi = mid;
  }
  return lo;
}

// Row quantiser without outlier handling (weights, FP8 dynamic activations,
// int8 activations with the decomposition off).
template <typename T, int CODE, bool SBF16>
qlin_status launch_rowquant(const void* X, int64_t rows, int64_t K, uint8_t* Q, float* s32, uint16_t* sbf,
                            cudaStream_t st) {
  PrepArgs a{};
  a.M = rows; a.K = K; a.Q = Q; a.s_f32 = s32; a.s_bf16 = sbf;
  return launch_prep<T, CODE, SBF16, false>(X, a, st);
}

// ---- LLM.int8 workspace layout -----------------------------------------------
struct Int8Ws {
  uint32_t* hdr;      // the per-call header, zeroed by k_ws_reset: count, flags, sk_count
  int32_t* count;     // [1]
  uint32_t* flags;    // [NW]
  int32_t* O;         // [K]
  float* s_x;         // [M]
  uint16_t* amax;     // [M] pass-1 absmax patterns of the prep kernel
  int8_t* Xq;         // [M,K]
  uint16_t* X_O;      // [M,ostride]
  uint16_t* W_O;      // [N,ostride]
  int8_t* XqO;        // [M,OUTL_CODES]
  int8_t* WqO;        // [N,OUTL_CODES]
  int32_t* sk_count;  // [128x256 tiles][GEMM_EPI_GROUPS] stream-K arrival counters
  int32_t* sk_part;   // [sk_ctas * 2][128 * 256] stream-K partial accumulators
  int sk_ctas;        // CTAs the partial slots serve
  int64_t ostride;
  int64_t hdr_words;  // 32-bit words of the header
  size_t total;
};

// Stream-K capacity of a GEMM: min(GEMM_SK_MAX_CTAS, iterations of its
// 128 x 256 tiles) CTAs.
int64_t sk_tiles(int64_t M, int64_t N) { return ((M + GEMM_BM - 1) / GEMM_BM) * ((N + GEMM_SK_BN - 1) / GEMM_SK_BN); }
int sk_capacity(int64_t M, int64_t N, int64_t K) {
  const int64_t T = sk_tiles(M, N) * ((K + GEMM_BK - 1) / GEMM_BK);
  return static_cast<int>(T < GEMM_SK_MAX_CTAS ? T : GEMM_SK_MAX_CTAS);
}

// Scratch of the FP8 GEMM: the stream-K arrival counters (zeroed by every
// call, left zero by the kernel) and the fp32 partial slots, two per CTA.
struct Fp8GemmWs {
  int32_t* sk_count;
  int32_t* sk_part;
  int sk_ctas;
  int64_t nctr;
  size_t total;
};
Fp8GemmWs fp8_gemm_layout(void* base, int64_t M, int64_t N, int64_t K) {
  Fp8GemmWs w{};
  uint8_t* p = static_cast<uint8_t*>(base);
  w.nctr = GEMM_EPI_GROUPS * sk_tiles(M, N);
  w.sk_ctas = sk_capacity(M, N, K);
  const size_t ctr_bytes = static_cast<size_t>(round_up(4 * w.nctr, 256));
  w.sk_count = p ? reinterpret_cast<int32_t*>(p) : nullptr;
  w.sk_part = p ? reinterpret_cast<int32_t*>(p + ctr_bytes) : nullptr;
  w.total = ctr_bytes + static_cast<size_t>(2 * w.sk_ctas) * GEMM_BM * GEMM_SK_BN * sizeof(int32_t);
  return w;
}

// with_sk: room for the stream-K arrival counters and partial slots (the
// GEMM then may run stream-K); without it the GEMM takes whole tiles only.
Int8Ws int8_layout(void* base, int64_t M, int64_t N, int64_t K, bool with_gemm_parts, bool with_sk = true) {
  Int8Ws w{};
  uint8_t* p = static_cast<uint8_t*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* r = p ? p + off : nullptr;
    off = static_cast<size_t>(round_up(static_cast<int64_t>(off + bytes), 256));
    return r;
  };
  const int64_t NW = (K + 31) / 32;
  const int64_t nctr = with_gemm_parts && with_sk ? GEMM_EPI_GROUPS * sk_tiles(M, N) : 0;
  // header: [reserved, count, reserved, reserved], flags [NW], sk_count [nctr]
  uint8_t* hdr = take(16 + 4 * NW + 4 * nctr);
  w.hdr = reinterpret_cast<uint32_t*>(hdr);
  w.count = reinterpret_cast<int32_t*>(hdr ? hdr + 4 : nullptr);
  w.flags = reinterpret_cast<uint32_t*>(hdr ? hdr + 16 : nullptr);
  w.sk_count = reinterpret_cast<int32_t*>(hdr && nctr > 0 ? hdr + 16 + 4 * NW : nullptr);
  w.hdr_words = 4 + NW + nctr;
  w.O = reinterpret_cast<int32_t*>(take(4 * K));
  w.ostride = round_up(K, 8);
  w.amax = reinterpret_cast<uint16_t*>(take(2 * M));
  if (with_gemm_parts) {
    w.s_x = reinterpret_cast<float*>(take(4 * M));
    w.Xq = reinterpret_cast<int8_t*>(take(static_cast<size_t>(M * K)));
    w.X_O = reinterpret_cast<uint16_t*>(take(static_cast<size_t>(2 * M * w.ostride)));
    w.W_O = reinterpret_cast<uint16_t*>(take(static_cast<size_t>(2 * N * w.ostride)));
    w.XqO = reinterpret_cast<int8_t*>(take(static_cast<size_t>(M * OUTL_CODES)));
    w.WqO = reinterpret_cast<int8_t*>(take(static_cast<size_t>(N * OUTL_CODES)));
    w.sk_ctas = with_sk ? sk_capacity(M, N, K) : 0;
    w.sk_part = with_sk ? reinterpret_cast<int32_t*>(
                              take(static_cast<size_t>(2 * w.sk_ctas) * GEMM_BM * GEMM_SK_BN * sizeof(int32_t)))
                        : nullptr;
  }
  w.total = off;
  return w;
}

bool decomposition_on(float thr) { return thr > 0.0f && !std::isinf(thr); }

// The finishing kernel of the LLM.int8 prepare stage (a programmatic
// dependent of the streaming pass).
template <typename T>
qlin_status launch_finish(const void* X, const FinishArgs& f, int sms, cudaStream_t st) {
  const int64_t NW = (f.K + 31) / 32;
  cudaLaunchConfig_t cfg{};
  // one wave (two CTAs per SM): the kernel is a few dependent round trips long
  cfg.gridDim = dim3(static_cast<unsigned>(2 * sms));
  cfg.blockDim = dim3(FIN_THREADS);
  cfg.dynamicSmemBytes = static_cast<size_t>(8 * NW);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return check_cuda(cudaLaunchKernelEx(&cfg, k_outlier_finish<T>, static_cast<const T*>(X), f),
                    "k_outlier_finish launch");
}

// The LLM.int8 prepare stage: k_ws_reset (zeroed header), the streaming pass
// (codes, scales, outlier bitmap) and, with the decomposition on,
// k_outlier_finish (outlier list, X_O, XqO, requantised rows, W_O, WqO); each
// a programmatic dependent of the one before.
template <typename T>
qlin_status int8_prep_impl(const void* X, int64_t M, int64_t K, float thr, const Int8Ws& w, int8_t* Xq, float* s_x,
                           uint16_t* X_O, int64_t ostride, cudaStream_t st,
                           WoGather wo = WoGather{nullptr, nullptr, 0, nullptr, nullptr, nullptr}) {
  DeviceInfo* d;
  qlin_status s = device_info(&d);
  if (s != QLIN_OK) return s;
  const int64_t rgrid = std::min<int64_t>(16, (w.hdr_words + 255) / 256);
  k_ws_reset<<<static_cast<unsigned>(rgrid), 256, 0, st>>>(w.hdr, w.hdr_words);
  s = check_cuda(cudaGetLastError(), "k_ws_reset launch");
  if (s != QLIN_OK) return s;
  if (M == 0) return QLIN_OK;
  if (decomposition_on(thr)) {
    PrepArgs a{};
    a.M = M; a.K = K; a.thr = thr; a.thr_bits = threshold_bits<T>(thr);
    a.Q = reinterpret_cast<uint8_t*>(Xq); a.s_f32 = s_x; a.amax_bits = w.amax;
    a.flags = w.flags;
    s = launch_prep<T, 0, false, true>(X, a, st);
    if (s != QLIN_OK) return s;
    FinishArgs f{};
    f.M = M; f.K = K; f.thr_bits = a.thr_bits; f.flags = w.flags; f.O = w.O; f.count = w.count;
    f.amax_bits = w.amax; f.s_x = s_x; f.Q = reinterpret_cast<uint8_t*>(Xq); f.X_O = X_O; f.ostride = ostride;
    f.XqO = w.XqO; f.wo = wo;
    return launch_finish<T>(X, f, d->sms, st);
  }
  return launch_rowquant<T, 0, false>(X, M, K, reinterpret_cast<uint8_t*>(Xq), s_x, nullptr, st);
}

qlin_status check_common(const void* X, qlin_dtype dt, int64_t M, int64_t K, int64_t N) {
  if (dt != QLIN_F16 && dt != QLIN_BF16) return fail(QLIN_ERR_INVALID_ARG, "dtype must be QLIN_F16 or QLIN_BF16");
  if (M < 0 || N < 0 || K < 0) return fail(QLIN_ERR_INVALID_ARG, "negative size");
  if (K == 0 || K % 16 != 0) return fail(QLIN_ERR_ALIGNMENT, "K must be a positive multiple of 16 (got %lld)",
                                         static_cast<long long>(K));
  if (K > kMaxK) return fail(QLIN_ERR_UNSUPPORTED, "K = %lld exceeds %lld", static_cast<long long>(K),
                             static_cast<long long>(kMaxK));
  if (X == nullptr && M > 0) return fail(QLIN_ERR_INVALID_ARG, "X is NULL");
  if (!aligned16(X)) return fail(QLIN_ERR_ALIGNMENT, "X is not 16-byte aligned");
  return QLIN_OK;
}

// The two stages of the LLM.int8 forward on a workspace already carved
// (arguments validated by the caller).
qlin_status int8_outlier_prepare_ws(const void* X, qlin_dtype xdt, int64_t M, int64_t K, const int8_t* Wq,
                                    const float* w_scale, int64_t N, float threshold, const Int8Ws& w,
                                    cudaStream_t st) {
  const WoGather wo{Wq, w_scale, N, w.O, w.W_O, w.WqO};
  return xdt == QLIN_BF16
             ? int8_prep_impl<__nv_bfloat16>(X, M, K, threshold, w, w.Xq, w.s_x, w.X_O, w.ostride, st, wo)
             : int8_prep_impl<__half>(X, M, K, threshold, w, w.Xq, w.s_x, w.X_O, w.ostride, st, wo);
}

qlin_status int8_outlier_gemm_ws(qlin_dtype xdt, int64_t M, int64_t K, const int8_t* Wq, const float* w_scale,
                                 int64_t N, const void* bias, void* Y, const Int8Ws& w, cudaStream_t st) {
  EpiParams ep{};
  ep.M = M; ep.N = N; ep.K = K; ep.Y = Y;
  ep.s_x = w.s_x; ep.s_w = w_scale; ep.bias = static_cast<const uint16_t*>(bias);
  ep.count = w.count; ep.X_O = w.X_O; ep.W_O = w.W_O; ep.ostride = w.ostride;
  ep.Xq = w.Xq; ep.Wq = Wq; ep.O = w.O; ep.XqO = w.XqO; ep.WqO = w.WqO;
  ep.sk_count = w.sk_count; ep.sk_part = w.sk_part;
  if (xdt == QLIN_BF16) return launch_gemm<0, EPI_INT8_OUTLIER, __nv_bfloat16>(w.Xq, Wq, ep, st, 1, w.sk_ctas);
  return launch_gemm<0, EPI_INT8_OUTLIER, __half>(w.Xq, Wq, ep, st, 2, w.sk_ctas);
}

#define QLIN_TRY(...)                  \
  do {                                 \
    qlin_status _s = (__VA_ARGS__);    \
    if (_s != QLIN_OK) return _s;      \
  } while (0)

#define QLIN_REQ_PTR(p, name)                                                          \
  do {                                                                                 \
    if ((p) == nullptr) return fail(QLIN_ERR_INVALID_ARG, "%s is NULL", name);         \
    if (!aligned16(p)) return fail(QLIN_ERR_ALIGNMENT, "%s is not 16-byte aligned", name); \
  } while (0)

}  // namespace

// =============================================================================
// C ABI
// =============================================================================
extern "C" {

int qlin_version(void) { return 100; }

const char* qlin_last_error_string(void) { return g_err; }

size_t qlin_workspace_bytes(qlin_op op, int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K <= 0) return 0;
  switch (op) {
    case QLIN_OP_INT8_OUTLIER:
      return int8_layout(nullptr, M, N, K, true).total;
    case QLIN_OP_INT8_PREP:
      return int8_layout(nullptr, M, N, K, false).total;
    case QLIN_OP_FP8:
      return static_cast<size_t>(round_up(M * K, 256) + round_up(4 * M, 256)) +
             fp8_gemm_layout(nullptr, M, N, K).total;
    case QLIN_OP_FP8_GEMM:
      return fp8_gemm_layout(nullptr, M, N, K).total;
    case QLIN_OP_W4A8:
      return static_cast<size_t>(round_up(M * K, 256) + round_up(4 * M, 256));
    case QLIN_OP_QUANTIZE_WEIGHT:
      return 256;
    case QLIN_OP_INT8_BLOCK:
      return static_cast<size_t>(round_up(2 * M * K, 256) + round_up(4 * M, 256));
    default:
      return 0;
  }
}

qlin_status qlin_get_device_status(int32_t* status, int reset) {
  if (!status) return fail(QLIN_ERR_INVALID_ARG, "status is NULL");
  QLIN_TRY(check_cuda(cudaDeviceSynchronize(), "cudaDeviceSynchronize"));
  int v = 0;
  QLIN_TRY(check_cuda(cudaMemcpyFromSymbol(&v, qlin::g_status, sizeof(int)), "cudaMemcpyFromSymbol"));
  *status = v;
  if (reset) {
    const int z = 0;
    QLIN_TRY(check_cuda(cudaMemcpyToSymbol(qlin::g_status, &z, sizeof(int)), "cudaMemcpyToSymbol"));
  }
  return ok();
}

qlin_status qlin_debug_inject_wait_timeout(int on) {
  const int v = on ? 1 : 0;
  QLIN_TRY(check_cuda(cudaMemcpyToSymbol(qlin::g_inject_wait_timeout, &v, sizeof(v)), "cudaMemcpyToSymbol"));
  return ok();
}

qlin_status qlin_set_gemm_schedule(int mode) {
  if (mode < 0 || mode > 2) return fail(QLIN_ERR_INVALID_ARG, "schedule mode must be 0, 1 or 2 (got %d)", mode);
  g_gemm_schedule.store(mode, std::memory_order_relaxed);
  return ok();
}

qlin_status qlin_set_wait_timeout_ns(uint64_t ns) {
  const unsigned long long v = ns;
  QLIN_TRY(check_cuda(cudaMemcpyToSymbol(qlin::g_wait_timeout_ns, &v, sizeof(v)), "cudaMemcpyToSymbol"));
  return ok();
}

qlin_status qlin_quantize_weight(const void* W, qlin_dtype wdt, int64_t N, int64_t K, qlin_wmode mode, void* Wq,
                                 void* w_scale, void* workspace, size_t ws_bytes, void* stream) {
  QLIN_TRY(check_common(W, wdt, N, K, 0));
  if (mode == QLIN_W_INT4_G128 && K % 128 != 0) return fail(QLIN_ERR_ALIGNMENT, "int4 format needs K % 128 == 0");
  if (mode == QLIN_W_INT8_BLOCK32 && K % 32 != 0)
    return fail(QLIN_ERR_ALIGNMENT, "block-scaled int8 needs K % 32 == 0");
  if (mode == QLIN_W_NVFP4 && K % 64 != 0) return fail(QLIN_ERR_ALIGNMENT, "NVFP4 format needs K % 64 == 0");
  if (N == 0) return ok();
  QLIN_REQ_PTR(Wq, "Wq");
  QLIN_REQ_PTR(w_scale, "w_scale");
  DeviceInfo* d;
  QLIN_TRY(device_info(&d));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool bf = (wdt == QLIN_BF16);
  const int64_t nvec = N * K / 8;
  switch (mode) {
    case QLIN_W_INT8_ROW:
      QLIN_TRY(bf ? launch_rowquant<__nv_bfloat16, 0, false>(W, N, K, static_cast<uint8_t*>(Wq),
                                                              static_cast<float*>(w_scale), nullptr, st)
                  : launch_rowquant<__half, 0, false>(W, N, K, static_cast<uint8_t*>(Wq), static_cast<float*>(w_scale),
                                                      nullptr, st));
      return ok();
    case QLIN_W_FP8_CHANNEL:
      QLIN_TRY(bf ? launch_rowquant<__nv_bfloat16, 1, true>(W, N, K, static_cast<uint8_t*>(Wq), nullptr,
                                                             static_cast<uint16_t*>(w_scale), st)
                  : launch_rowquant<__half, 1, true>(W, N, K, static_cast<uint8_t*>(Wq), nullptr,
                                                     static_cast<uint16_t*>(w_scale), st));
      return ok();
    case QLIN_W_FP8_TENSOR: {
      if (workspace == nullptr || ws_bytes < qlin_workspace_bytes(QLIN_OP_QUANTIZE_WEIGHT, 0, N, K))
        return fail(QLIN_ERR_WORKSPACE, "workspace too small");
      QLIN_REQ_PTR(workspace, "workspace");
      uint32_t* amax = static_cast<uint32_t*>(workspace);
      QLIN_TRY(check_cuda(cudaMemsetAsync(amax, 0, 4, st), "cudaMemsetAsync"));
      const int grid = d->sms * 4;
      if (bf) {
        k_absmax<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(W), nvec, amax);
        k_fp8_tensor_quant<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(W), nvec, amax,
                                                                static_cast<uint8_t*>(Wq),
                                                                static_cast<float*>(w_scale));
      } else {
        k_absmax<__half><<<grid, 256, 0, st>>>(static_cast<const __half*>(W), nvec, amax);
        k_fp8_tensor_quant<__half><<<grid, 256, 0, st>>>(static_cast<const __half*>(W), nvec, amax,
                                                         static_cast<uint8_t*>(Wq), static_cast<float*>(w_scale));
      }
      QLIN_TRY(check_cuda(cudaGetLastError(), "fp8 tensor quant launch"));
      return ok();
    }
    case QLIN_W_INT4_G128: {
      const int64_t warps = N * (K / 128);
      const int64_t blocks = (warps * 32 + 255) / 256;
      if (bf)
        k_int4_group_quant<__nv_bfloat16><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
            static_cast<const __nv_bfloat16*>(W), N, K, static_cast<uint8_t*>(Wq), static_cast<float*>(w_scale));
      else
        k_int4_group_quant<__half><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
            static_cast<const __half*>(W), N, K, static_cast<uint8_t*>(Wq), static_cast<float*>(w_scale));
      QLIN_TRY(check_cuda(cudaGetLastError(), "int4 quant launch"));
      return ok();
    }
    case QLIN_W_INT8_BLOCK32: {
      const int64_t blocks = N * (K / 32);
      const int64_t want = (blocks + 255) / 256, cap = static_cast<int64_t>(d->sms) * 16;
      const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
      if (bf)
        k_int8_block_quant<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(W), N, K,
                                                                static_cast<int8_t*>(Wq), static_cast<float*>(w_scale));
      else
        k_int8_block_quant<__half><<<grid, 256, 0, st>>>(static_cast<const __half*>(W), N, K, static_cast<int8_t*>(Wq),
                                                         static_cast<float*>(w_scale));
      QLIN_TRY(check_cuda(cudaGetLastError(), "int8 block quant launch"));
      return ok();
    }
    case QLIN_W_NVFP4: {
      if (workspace == nullptr || ws_bytes < qlin_workspace_bytes(QLIN_OP_QUANTIZE_WEIGHT, 0, N, K))
        return fail(QLIN_ERR_WORKSPACE, "workspace too small");
      QLIN_REQ_PTR(workspace, "workspace");
      if (!aligned16(w_scale)) return fail(QLIN_ERR_ALIGNMENT, "w_scale is not 16-byte aligned");
      uint32_t* amax = static_cast<uint32_t*>(workspace);
      uint8_t* sb = static_cast<uint8_t*>(w_scale);
      float* s_t = reinterpret_cast<float*>(sb + round_up(N * K / 16, 16));
      QLIN_TRY(check_cuda(cudaMemsetAsync(amax, 0, 4, st), "cudaMemsetAsync"));
      const int grid = d->sms * 4;
      const int64_t threads = N * (K / 32);
      const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
      if (bf) {
        k_absmax<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(W), nvec, amax);
        k_nvfp4_quant<__nv_bfloat16><<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(W), N, K, amax,
                                                            static_cast<uint8_t*>(Wq), sb, s_t);
      } else {
        k_absmax<__half><<<grid, 256, 0, st>>>(static_cast<const __half*>(W), nvec, amax);
        k_nvfp4_quant<__half><<<blocks, 256, 0, st>>>(static_cast<const __half*>(W), N, K, amax,
                                                     static_cast<uint8_t*>(Wq), sb, s_t);
      }
      QLIN_TRY(check_cuda(cudaGetLastError(), "nvfp4 quant launch"));
      return ok();
    }
    default:
      return fail(QLIN_ERR_INVALID_ARG, "unknown weight mode %d", static_cast<int>(mode));
  }
}

qlin_status qlin_calibrate_input_scale(const void* X, qlin_dtype xdt, int64_t M, int64_t K, float* x_scale,
                                       void* workspace, size_t ws_bytes, void* stream) {
  QLIN_TRY(check_common(X, xdt, M, K, 0));
  QLIN_REQ_PTR(x_scale, "x_scale");
  if (workspace == nullptr || ws_bytes < qlin_workspace_bytes(QLIN_OP_QUANTIZE_WEIGHT, M, 0, K))
    return fail(QLIN_ERR_WORKSPACE, "workspace too small");
  QLIN_REQ_PTR(workspace, "workspace");
  DeviceInfo* d;
  QLIN_TRY(device_info(&d));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* amax = static_cast<uint32_t*>(workspace);
  QLIN_TRY(check_cuda(cudaMemsetAsync(amax, 0, 4, st), "cudaMemsetAsync"));
  const int64_t nvec = M * K / 8;
  if (nvec > 0) {
    if (xdt == QLIN_BF16)
      k_absmax<__nv_bfloat16><<<d->sms * 4, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(X), nvec, amax);
    else
      k_absmax<__half><<<d->sms * 4, 256, 0, st>>>(static_cast<const __half*>(X), nvec, amax);
  }
  k_scale_from_absmax<<<1, 1, 0, st>>>(amax, 448.0f, x_scale);
  QLIN_TRY(check_cuda(cudaGetLastError(), "calibration launch"));
  return ok();
}

qlin_status qlin_int8_prep(const void* X, qlin_dtype xdt, int64_t M, int64_t K, float threshold, int8_t* Xq,
                           float* s_x, uint32_t* flags, int32_t* O, int32_t* count, void* X_O, int64_t ostride,
                           void* workspace, size_t ws_bytes, void* stream) {
  QLIN_TRY(check_common(X, xdt, M, K, 0));
  QLIN_REQ_PTR(Xq, "Xq");
  QLIN_REQ_PTR(s_x, "s_x");
  QLIN_REQ_PTR(flags, "flags");
  QLIN_REQ_PTR(O, "O");
  QLIN_REQ_PTR(count, "count");
  QLIN_REQ_PTR(X_O, "X_O");
  if (ostride < round_up(K, 8) || ostride % 8 != 0)
    return fail(QLIN_ERR_INVALID_ARG, "ostride must be a multiple of 8 and >= round_up(K, 8)");
  if (workspace == nullptr || ws_bytes < qlin_workspace_bytes(QLIN_OP_INT8_PREP, M, 0, K))
    return fail(QLIN_ERR_WORKSPACE, "workspace too small");
  QLIN_REQ_PTR(workspace, "workspace");
  DeviceInfo* d;
  QLIN_TRY(device_info(&d));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Int8Ws w = int8_layout(workspace, M, 0, K, false);
  QLIN_TRY(xdt == QLIN_BF16
               ? int8_prep_impl<__nv_bfloat16>(X, M, K, threshold, w, Xq, s_x, static_cast<uint16_t*>(X_O), ostride,
                                               st)
               : int8_prep_impl<__half>(X, M, K, threshold, w, Xq, s_x, static_cast<uint16_t*>(X_O), ostride, st));
  if (decomposition_on(threshold) && M > 0) {
    // the prep leaves the sub-threshold codes of outlier columns in place (the
    // GEMM masks them); this export returns the decomposed Xq with them at 0
    const int64_t want = (M + 7) / 8, cap = static_cast<int64_t>(d->sms) * 8;
    k_zero_outlier_cols<<<static_cast<unsigned>(want < cap ? want : cap), 256, 0, st>>>(Xq, M, K, w.O, w.count);
    QLIN_TRY(check_cuda(cudaGetLastError(), "k_zero_outlier_cols launch"));
  }
  const int64_t NW = (K + 31) / 32;
  QLIN_TRY(check_cuda(cudaMemcpyAsync(flags, w.flags, 4 * NW, cudaMemcpyDeviceToDevice, st), "copy flags"));
  QLIN_TRY(check_cuda(cudaMemcpyAsync(count, w.count, 4, cudaMemcpyDeviceToDevice, st), "copy count"));
  QLIN_TRY(check_cuda(cudaMemcpyAsync(O, w.O, 4 * K, cudaMemcpyDeviceToDevice, st), "copy O"));
  return ok();
}

qlin_status qlin_outlier_weights(const int8_t* Wq, const float* w_scale, int64_t N, int64_t K, const int32_t* O,
                                 const int32_t* count, qlin_dtype dt, void* W_O, int64_t ostride, void* stream) {
  if (dt != QLIN_F16 && dt != QLIN_BF16) return fail(QLIN_ERR_INVALID_ARG, "bad dtype");
  if (N < 0 || K <= 0) return fail(QLIN_ERR_INVALID_ARG, "bad sizes");
  if (N == 0) return ok();
  QLIN_REQ_PTR(Wq, "Wq");
  QLIN_REQ_PTR(w_scale, "w_scale");
  QLIN_REQ_PTR(O, "O");
  QLIN_REQ_PTR(count, "count");
  QLIN_REQ_PTR(W_O, "W_O");
  if (ostride < round_up(K, 8) || ostride % 8 != 0) return fail(QLIN_ERR_INVALID_ARG, "bad ostride");
  DeviceInfo* d;
  QLIN_TRY(device_info(&d));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == QLIN_BF16)
    k_gather_wo<__nv_bfloat16><<<d->sms * 4, 256, 0, st>>>(Wq, w_scale, N, K, O, count,
                                                           static_cast<uint16_t*>(W_O), ostride);
  else
    k_gather_wo<__half><<<d->sms * 4, 256, 0, st>>>(Wq, w_scale, N, K, O, count, static_cast<uint16_t*>(W_O),
                                                    ostride);
  QLIN_TRY(check_cuda(cudaGetLastError(), "k_gather_wo launch"));
  return ok();
}

qlin_status qlin_int8_gemm_i32(const int8_t* Xq, const int8_t* Wq, int64_t M, int64_t N, int64_t K, int32_t* C,
                               void* stream) {
  if (M < 0 || N < 0) return fail(QLIN_ERR_INVALID_ARG, "negative size");
  if (K <= 0 || K % 16 != 0) return fail(QLIN_ERR_ALIGNMENT, "K must be a positive multiple of 16");
  if (K > kMaxK) return fail(QLIN_ERR_UNSUPPORTED, "K too large");
  if (M == 0 || N == 0) return ok();
  QLIN_REQ_PTR(Xq, "Xq");
  QLIN_REQ_PTR(Wq, "Wq");
  QLIN_REQ_PTR(C, "C");
  EpiParams ep{};
  ep.M = M; ep.N = N; ep.K = K; ep.Y = C;
  QLIN_TRY((launch_gemm<0, EPI_I32, __nv_bfloat16>(Xq, Wq, ep, static_cast<cudaStream_t>(stream), 0)));
  return ok();
}

qlin_status qlin_int8_outlier_prepare(const void* X, qlin_dtype xdt, int64_t M, int64_t K, const int8_t* Wq,
                                      const float* w_scale, int64_t N, float threshold, void* workspace,
                                      size_t ws_bytes, void* stream) {
  QLIN_TRY(check_common(X, xdt, M, K, N));
  if (M == 0 || N == 0) return ok();
  QLIN_REQ_PTR(Wq, "Wq");
  QLIN_REQ_PTR(w_scale, "w_scale");
  if (workspace == nullptr || ws_bytes < qlin_workspace_bytes(QLIN_OP_INT8_OUTLIER, M, N, K))
    return fail(QLIN_ERR_WORKSPACE, "workspace too small (need %zu bytes)",
                qlin_workspace_bytes(QLIN_OP_INT8_OUTLIER, M, N, K));
  QLIN_REQ_PTR(workspace, "workspace");
  DeviceInfo* d;
  QLIN_TRY(device_info(&d));
  QLIN_TRY(int8_outlier_prepare_ws(X, xdt, M, K, Wq, w_scale, N, threshold, int8_layout(workspace, M, N, K, true),
                                   static_cast<cudaStream_t>(stream)));
  return ok();
}

qlin_status qlin_int8_outlier_gemm(qlin_dtype xdt, int64_t M, int64_t K, const int8_t* Wq, const float* w_scale,
                                   int64_t N, const void* bias, void* Y, void* workspace, size_t ws_bytes,
                                   void* stream) {
  if (xdt != QLIN_F16 && xdt != QLIN_BF16) return fail(QLIN_ERR_INVALID_ARG, "bad dtype");
  if (M < 0 || N < 0) return fail(QLIN_ERR_INVALID_ARG, "negative size");
  if (K <= 0 || K % 16 != 0) return fail(QLIN_ERR_ALIGNMENT, "K must be a positive multiple of 16");
  if (K > kMaxK) return fail(QLIN_ERR_UNSUPPORTED, "K too large");
  if (M == 0 || N == 0) return ok();
  QLIN_REQ_PTR(Wq, "Wq");
  QLIN_REQ_PTR(w_scale, "w_scale");
  QLIN_REQ_PTR(Y, "Y");
  if (bias != nullptr && !aligned16(bias)) return fail(QLIN_ERR_ALIGNMENT, "bias is not 16-byte aligned");
  if (workspace == nullptr || ws_bytes < qlin_workspace_bytes(QLIN_OP_INT8_OUTLIER, M, N, K))
    return fail(QLIN_ERR_WORKSPACE, "workspace too small");
  QLIN_REQ_PTR(workspace, "workspace");
  QLIN_TRY(int8_outlier_gemm_ws(xdt, M, K, Wq, w_scale, N, bias, Y, int8_layout(workspace, M, N, K, true),
                                static_cast<cudaStream_t>(stream)));
  return ok();
}

qlin_status qlin_int8_outlier_gemm_i32(int64_t M, int64_t K, const int8_t* Wq, int64_t N, int32_t* C,
                                       void* workspace, size_t ws_bytes, void* stream) {
  if (M < 0 || N < 0) return fail(QLIN_ERR_INVALID_ARG, "negative size");
  if (K <= 0 || K % 16 != 0) return fail(QLIN_ERR_ALIGNMENT, "K must be a positive multiple of 16");
  if (K > kMaxK) return fail(QLIN_ERR_UNSUPPORTED, "K too large");
  if (M == 0 || N == 0) return ok();
  QLIN_REQ_PTR(Wq, "Wq");
  QLIN_REQ_PTR(C, "C");
  if (workspace == nullptr || ws_bytes < qlin_workspace_bytes(QLIN_OP_INT8_OUTLIER, M, N, K))
    return fail(QLIN_ERR_WORKSPACE, "workspace too small");
  QLIN_REQ_PTR(workspace, "workspace");
  Int8Ws w = int8_layout(workspace, M, N, K, true);
  EpiParams ep{};
  ep.M = M; ep.N = N; ep.K = K; ep.Y = C;
  ep.count = w.count; ep.Xq = w.Xq; ep.Wq = Wq; ep.O = w.O; ep.XqO = w.XqO; ep.WqO = w.WqO;
  ep.sk_count = w.sk_count; ep.sk_part = w.sk_part;
  QLIN_TRY((launch_gemm<0, EPI_INT8_OUTLIER_I32, __nv_bfloat16>(w.Xq, Wq, ep, static_cast<cudaStream_t>(stream), 7,
                                                                 w.sk_ctas)));
  return ok();
}

qlin_status qlin_int8_outlier_forward(const void* X, qlin_dtype xdt, int64_t M, int64_t K, const int8_t* Wq,
                                      const float* w_scale, int64_t N, float threshold, const void* bias, void* Y,
                                      void* workspace, size_t ws_bytes, void* stream) {
  QLIN_TRY(check_common(X, xdt, M, K, N));
  if (M == 0 || N == 0) return ok();
  QLIN_REQ_PTR(Y, "Y");
  if (bias != nullptr && !aligned16(bias)) return fail(QLIN_ERR_ALIGNMENT, "bias is not 16-byte aligned");
  QLIN_TRY(qlin_int8_outlier_prepare(X, xdt, M, K, Wq, w_scale, N, threshold, workspace, ws_bytes, stream));
  return qlin_int8_outlier_gemm(xdt, M, K, Wq, w_scale, N, bias, Y, workspace, ws_bytes, stream);
}

qlin_status qlin_e4m3_encode_f32(const float* t, uint8_t* codes, int64_t n, void* stream) {
  if (n < 0) return fail(QLIN_ERR_INVALID_ARG, "negative size");
  if (n == 0) return ok();
  QLIN_REQ_PTR(t, "t");
  QLIN_REQ_PTR(codes, "codes");
  DeviceInfo* d;
  QLIN_TRY(device_info(&d));
  const int64_t want = (n + 511) / 512, cap = static_cast<int64_t>(d->sms) * 16;
  k_e4m3_encode<<<static_cast<unsigned>(want < cap ? want : cap), 256, 0, static_cast<cudaStream_t>(stream)>>>(t, codes, n);
  return check_cuda(cudaGetLastError(), "k_e4m3_encode launch");
}

qlin_status qlin_fp8_prep(const void* X, qlin_dtype xdt, int64_t M, int64_t K, const float* x_scale, uint8_t* Xq,
                          float* s_x, void* stream) {
  QLIN_TRY(check_common(X, xdt, M, K, 0));
  if (M == 0) return ok();
  QLIN_REQ_PTR(Xq, "Xq");
  DeviceInfo* d;
  QLIN_TRY(device_info(&d));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool bf = (xdt == QLIN_BF16);
  if (x_scale != nullptr) {
    QLIN_REQ_PTR(x_scale, "x_scale");
    const int64_t nvec = M * K / 8;
    if (bf) k_fp8_static<__nv_bfloat16><<<d->sms * 8, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(X), nvec,
                                                                    x_scale, Xq);
    else k_fp8_static<__half><<<d->sms * 8, 256, 0, st>>>(static_cast<const __half*>(X), nvec, x_scale, Xq);
    return check_cuda(cudaGetLastError(), "k_fp8_static launch") == QLIN_OK ? ok() : QLIN_ERR_CUDA;
  }
  QLIN_REQ_PTR(s_x, "s_x");
  QLIN_TRY(bf ? launch_rowquant<__nv_bfloat16, 1, false>(X, M, K, Xq, s_x, nullptr, st)
              : launch_rowquant<__half, 1, false>(X, M, K, Xq, s_x, nullptr, st));
  return ok();
}

qlin_status qlin_fp8_gemm(qlin_dtype xdt, int64_t M, int64_t K, const uint8_t* Xq, const float* s_x,
                          const uint8_t* Wq, const void* w_scale, qlin_wmode wmode, int64_t N, const float* x_scale,
                          const void* bias, void* Y, void* workspace, size_t ws_bytes, void* stream) {
  if (xdt != QLIN_F16 && xdt != QLIN_BF16) return fail(QLIN_ERR_INVALID_ARG, "bad dtype");
  if (wmode != QLIN_W_FP8_TENSOR && wmode != QLIN_W_FP8_CHANNEL)
    return fail(QLIN_ERR_INVALID_ARG, "wmode must be QLIN_W_FP8_TENSOR or QLIN_W_FP8_CHANNEL");
  if (M < 0 || N < 0) return fail(QLIN_ERR_INVALID_ARG, "negative size");
  if (K <= 0 || K % 16 != 0) return fail(QLIN_ERR_ALIGNMENT, "K must be a positive multiple of 16");
  if (K > kMaxK) return fail(QLIN_ERR_UNSUPPORTED, "K too large");
  if (M == 0 || N == 0) return ok();
  QLIN_REQ_PTR(Xq, "Xq");
  QLIN_REQ_PTR(Wq, "Wq");
  QLIN_REQ_PTR(w_scale, "w_scale");
  QLIN_REQ_PTR(Y, "Y");
  if (bias != nullptr && !aligned16(bias)) return fail(QLIN_ERR_ALIGNMENT, "bias is not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  EpiParams ep{};
  ep.M = M; ep.N = N; ep.K = K; ep.Y = Y;
  ep.bias = static_cast<const uint16_t*>(bias);
  const bool bf = (xdt == QLIN_BF16);
  if (wmode == QLIN_W_FP8_TENSOR) {
    if (x_scale == nullptr) return fail(QLIN_ERR_UNSUPPORTED, "per-tensor weight scales need a static x_scale");
    QLIN_REQ_PTR(x_scale, "x_scale");
  } else {
    if (x_scale != nullptr)
      return fail(QLIN_ERR_UNSUPPORTED, "per-channel weight scales go with dynamic per-token activations");
    QLIN_REQ_PTR(s_x, "s_x");
  }
  // with scratch: stream-K may cut tiles across CTAs (fp32 partials, summed
  // in a fixed order); launch_gemm clears the arrival counters when it does
  int sk_cap = 0;
  if (workspace != nullptr) {
    const Fp8GemmWs w = fp8_gemm_layout(workspace, M, N, K);
    if (ws_bytes < w.total) return fail(QLIN_ERR_WORKSPACE, "workspace too small");
    if (!aligned16(workspace)) return fail(QLIN_ERR_ALIGNMENT, "workspace is not 16-byte aligned");
    ep.sk_count = w.sk_count;
    ep.sk_part = w.sk_part;
    sk_cap = w.sk_ctas;
  }
  if (wmode == QLIN_W_FP8_TENSOR) {
    ep.x_scale = x_scale;
    ep.w_scale = static_cast<const float*>(w_scale);
    if (bf) QLIN_TRY((launch_gemm<1, EPI_FP8_TENSOR, __nv_bfloat16>(Xq, Wq, ep, st, 3, sk_cap)));
    else QLIN_TRY((launch_gemm<1, EPI_FP8_TENSOR, __half>(Xq, Wq, ep, st, 4, sk_cap)));
  } else {
    ep.s_x = s_x;
    ep.s_w_bf16 = static_cast<const uint16_t*>(w_scale);
    if (bf) QLIN_TRY((launch_gemm<1, EPI_FP8_ROWCOL, __nv_bfloat16>(Xq, Wq, ep, st, 5, sk_cap)));
    else QLIN_TRY((launch_gemm<1, EPI_FP8_ROWCOL, __half>(Xq, Wq, ep, st, 6, sk_cap)));
  }
  return ok();
}

qlin_status qlin_fp8_forward(const void* X, qlin_dtype xdt, int64_t M, int64_t K, const uint8_t* Wq,
                             const void* w_scale, qlin_wmode wmode, int64_t N, const float* x_scale, const void* bias,
                             void* Y, void* workspace, size_t ws_bytes, void* stream) {
  QLIN_TRY(check_common(X, xdt, M, K, N));
  if (wmode != QLIN_W_FP8_TENSOR && wmode != QLIN_W_FP8_CHANNEL)
    return fail(QLIN_ERR_INVALID_ARG, "wmode must be QLIN_W_FP8_TENSOR or QLIN_W_FP8_CHANNEL");
  if (wmode == QLIN_W_FP8_TENSOR && x_scale == nullptr)
    return fail(QLIN_ERR_UNSUPPORTED, "per-tensor weight scales need a static x_scale");
  if (wmode == QLIN_W_FP8_CHANNEL && x_scale != nullptr)
    return fail(QLIN_ERR_UNSUPPORTED, "per-channel weight scales go with dynamic per-token activations (x_scale NULL)");
  if (M == 0 || N == 0) return ok();
  if (workspace == nullptr || ws_bytes < qlin_workspace_bytes(QLIN_OP_FP8, M, N, K))
    return fail(QLIN_ERR_WORKSPACE, "workspace too small");
  QLIN_REQ_PTR(workspace, "workspace");
  uint8_t* Xq = static_cast<uint8_t*>(workspace);
  float* s_x = reinterpret_cast<float*>(Xq + round_up(M * K, 256));
  uint8_t* scratch = Xq + round_up(M * K, 256) + round_up(4 * M, 256);
  QLIN_TRY(qlin_fp8_prep(X, xdt, M, K, x_scale, Xq, s_x, stream));
  return qlin_fp8_gemm(xdt, M, K, Xq, s_x, Wq, w_scale, wmode, N, x_scale, bias, Y, scratch,
                       fp8_gemm_layout(nullptr, M, N, K).total, stream);
}

// Unquantised 16-bit linear: the tcgen05 GEMM with kind::f16 operands (the
// tiles hold 64 elements of K, 128 bytes, per stage) and a bias epilogue.
qlin_status qlin_fp_linear_forward(const void* X, qlin_dtype xdt, int64_t M, int64_t K, const void* W, int64_t N,
                                   const void* bias, void* Y, void* stream) {
  QLIN_TRY(check_common(X, xdt, M, K, N));
  if (M == 0 || N == 0) return ok();
  QLIN_REQ_PTR(W, "W");
  QLIN_REQ_PTR(Y, "Y");
  if (bias != nullptr && !aligned16(bias)) return fail(QLIN_ERR_ALIGNMENT, "bias is not 16-byte aligned");
  EpiParams ep{};
  ep.M = M; ep.N = N; ep.K = 2 * K; ep.Y = Y;
  ep.bias = static_cast<const uint16_t*>(bias);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (xdt == QLIN_BF16) QLIN_TRY((launch_gemm<2, EPI_F16, __nv_bfloat16>(X, W, ep, st, 8)));
  else QLIN_TRY((launch_gemm<2, EPI_F16, __half>(X, W, ep, st, 9)));
  return ok();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// W4A8
// ---------------------------------------------------------------------------
namespace {

// A 2-D byte tensor [rows, row_bytes] (row pitch stride_bytes, or row_bytes when 0).
qlin_status make_tmap_bytes(CUtensorMap* m, const void* base, int64_t rows, int64_t row_bytes, int box_inner,
                            int box_rows, CUtensorMapSwizzle sw, int64_t stride_bytes) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  qlin_status s = get_encode(&enc);
  if (s != QLIN_OK) return s;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(stride_bytes > 0 ? stride_bytes : row_bytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(QLIN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return QLIN_OK;
}

template <typename TOut, bool DBG = false>
qlin_status launch_w4a8(const int8_t* Xq, const uint8_t* Wq4, const W4Params& wp, cudaStream_t st) {
  DeviceInfo* d;
  qlin_status s = device_info(&d);
  if (s != QLIN_OK) return s;
  CUtensorMap ta, tb;
  if ((s = make_tmap_bytes(&ta, Xq, wp.M, wp.K, W4_G, W4_BM, CU_TENSOR_MAP_SWIZZLE_128B)) != QLIN_OK) return s;
  if ((s = make_tmap_bytes(&tb, Wq4, wp.N, wp.K / 2, W4_G / 2, W4_BN, CU_TENSOR_MAP_SWIZZLE_NONE)) != QLIN_OK)
    return s;
  auto kern = k_gemm_w4a8<TOut, DBG>;
  static std::atomic<bool> attr_set[16] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 16 && !attr_set[dev].load(std::memory_order_acquire)) {
    // the warpgroups trade registers with setmaxnreg: the launch register
    // count must leave enough in the block's pool for the split
    cudaFuncAttributes fa{};
    s = check_cuda(cudaFuncGetAttributes(&fa, kern), "cudaFuncGetAttributes");
    if (s != QLIN_OK) return s;
    if (fa.numRegs < W4_REGS_MIN_LAUNCH || fa.numRegs > W4_REGS_HIGH)
      return fail(QLIN_ERR_UNSUPPORTED, "k_gemm_w4a8 was built with %d registers per thread; the register split needs %d..%d",
                  fa.numRegs, W4_REGS_MIN_LAUNCH, W4_REGS_HIGH);
    s = check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, W4Smem::TOTAL),
                   "cudaFuncSetAttribute");
    if (s != QLIN_OK) return s;
    attr_set[dev].store(true, std::memory_order_release);
  }
  const int64_t tiles = ((wp.M + W4_BM - 1) / W4_BM) * ((wp.N + W4_BN - 1) / W4_BN);
  const int grid = static_cast<int>(tiles < d->sms ? tiles : d->sms);
  kern<<<grid, W4_THREADS, W4Smem::TOTAL, st>>>(ta, tb, wp);
  return check_cuda(cudaGetLastError(), "k_gemm_w4a8 launch");
}

qlin_status check_w4(const void* Xq, const void* Wq4, const float* w_scale, int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0) return fail(QLIN_ERR_INVALID_ARG, "negative size");
  if (K <= 0 || K % W4_G != 0) return fail(QLIN_ERR_ALIGNMENT, "W4A8 needs K a positive multiple of 128");
  if (K > kMaxK) return fail(QLIN_ERR_UNSUPPORTED, "K too large");
  if (M == 0 || N == 0) return QLIN_OK;
  QLIN_REQ_PTR(Xq, "Xq");
  QLIN_REQ_PTR(Wq4, "Wq4");
  QLIN_REQ_PTR(w_scale, "w_scale");
  return QLIN_OK;
}

}  // namespace

extern "C" {

qlin_status qlin_w4a8_gemm(qlin_dtype xdt, int64_t M, int64_t K, const int8_t* Xq, const float* s_x,
                           const uint8_t* Wq4, const float* w_scale, int64_t N, const void* bias, void* Y,
                           void* stream) {
  if (xdt != QLIN_F16 && xdt != QLIN_BF16) return fail(QLIN_ERR_INVALID_ARG, "bad dtype");
  QLIN_TRY(check_w4(Xq, Wq4, w_scale, M, N, K));
  if (M == 0 || N == 0) return ok();
  QLIN_REQ_PTR(s_x, "s_x");
  QLIN_REQ_PTR(Y, "Y");
  if (bias != nullptr && !aligned16(bias)) return fail(QLIN_ERR_ALIGNMENT, "bias is not 16-byte aligned");
  W4Params wp{};
  wp.M = M; wp.N = N; wp.K = K; wp.Y = Y; wp.s_x = s_x; wp.s_w = w_scale;
  wp.bias = static_cast<const uint16_t*>(bias); wp.dbg = nullptr; wp.dbg_group = -1;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (xdt == QLIN_BF16) QLIN_TRY(launch_w4a8<__nv_bfloat16>(Xq, Wq4, wp, st));
  else QLIN_TRY(launch_w4a8<__half>(Xq, Wq4, wp, st));
  return ok();
}

qlin_status qlin_w4a8_group_i32(const int8_t* Xq, const uint8_t* Wq4, int64_t M, int64_t N, int64_t K, int group,
                                int32_t* C, void* stream) {
  if (M < 0 || N < 0) return fail(QLIN_ERR_INVALID_ARG, "negative size");
  if (K <= 0 || K % W4_G != 0) return fail(QLIN_ERR_ALIGNMENT, "W4A8 needs K a positive multiple of 128");
  if (K > kMaxK) return fail(QLIN_ERR_UNSUPPORTED, "K too large");
  if (group < 0 || group >= K / W4_G) return fail(QLIN_ERR_INVALID_ARG, "group out of range");
  if (M == 0 || N == 0) return ok();
  QLIN_REQ_PTR(Xq, "Xq");
  QLIN_REQ_PTR(Wq4, "Wq4");
  QLIN_REQ_PTR(C, "C");
  W4Params wp{};
  wp.M = M; wp.N = N; wp.K = K; wp.Y = nullptr; wp.s_x = nullptr; wp.s_w = nullptr; wp.bias = nullptr;
  wp.dbg = C; wp.dbg_group = group;
  QLIN_TRY((launch_w4a8<__nv_bfloat16, true>(Xq, Wq4, wp, static_cast<cudaStream_t>(stream))));
  return ok();
}

qlin_status qlin_w4a8_prep(const void* X, qlin_dtype xdt, int64_t M, int64_t K, int8_t* Xq, float* s_x,
                           void* stream) {
  QLIN_TRY(check_common(X, xdt, M, K, 0));
  if (M == 0) return ok();
  QLIN_REQ_PTR(Xq, "Xq");
  QLIN_REQ_PTR(s_x, "s_x");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (xdt == QLIN_BF16)
    return launch_rowquant<__nv_bfloat16, 0, false>(X, M, K, reinterpret_cast<uint8_t*>(Xq), s_x, nullptr, st);
  return launch_rowquant<__half, 0, false>(X, M, K, reinterpret_cast<uint8_t*>(Xq), s_x, nullptr, st);
}

qlin_status qlin_w4a8_forward(const void* X, qlin_dtype xdt, int64_t M, int64_t K, const uint8_t* Wq4,
                              const float* w_scale, int64_t N, const void* bias, void* Y, void* workspace,
                              size_t ws_bytes, void* stream) {
  QLIN_TRY(check_common(X, xdt, M, K, N));
  if (K % W4_G != 0) return fail(QLIN_ERR_ALIGNMENT, "W4A8 needs K a multiple of 128");
  if (M == 0 || N == 0) return ok();
  if (workspace == nullptr || ws_bytes < qlin_workspace_bytes(QLIN_OP_W4A8, M, N, K))
    return fail(QLIN_ERR_WORKSPACE, "workspace too small");
  QLIN_REQ_PTR(workspace, "workspace");
  int8_t* Xq = static_cast<int8_t*>(workspace);
  float* s_x = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + round_up(M * K, 256));
  QLIN_TRY(qlin_w4a8_prep(X, xdt, M, K, Xq, s_x, stream));
  return qlin_w4a8_gemm(xdt, M, K, Xq, s_x, Wq4, w_scale, N, bias, Y, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Weight-only FP8
// ---------------------------------------------------------------------------
namespace {

template <int FMT, typename TOut>
qlin_status launch_cvt(const void* A, const void* Wq, const Wo8Params& wp, cudaStream_t st) {
  DeviceInfo* d;
  qlin_status s = device_info(&d);
  if (s != QLIN_OK) return s;
  CUtensorMap ta, tb;
  if ((s = make_tmap_k128(&ta, A, wp.M, 2 * wp.K, WO8_BM)) != QLIN_OK) return s;
  if ((s = make_tmap_bytes(&tb, Wq, wp.N, FMT == 2 ? wp.K / 2 : wp.K, FMT == 2 ? WO8_BK / 2 : WO8_BK, WO8_BN,
                           CU_TENSOR_MAP_SWIZZLE_NONE)) != QLIN_OK)
    return s;
  auto kern = k_gemm_cvt<FMT, TOut>;
  static std::atomic<bool> attr_set[16] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 16 && !attr_set[dev].load(std::memory_order_acquire)) {
    s = check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Wo8Smem::TOTAL),
                   "cudaFuncSetAttribute");
    if (s != QLIN_OK) return s;
    attr_set[dev].store(true, std::memory_order_release);
  }
  const int64_t tiles = ((wp.M + WO8_BM - 1) / WO8_BM) * ((wp.N + WO8_BN - 1) / WO8_BN);
  const int grid = static_cast<int>(tiles < d->sms ? tiles : d->sms);
  kern<<<grid, WO8_THREADS, Wo8Smem::TOTAL, st>>>(ta, tb, wp);
  return check_cuda(cudaGetLastError(), "k_gemm_cvt launch");
}

}  // namespace

extern "C" qlin_status qlin_fp8_weight_only_forward(const void* X, qlin_dtype xdt, int64_t M, int64_t K,
                                                    const uint8_t* Wq, const void* w_scale, int64_t N,
                                                    const void* bias, void* Y, void* stream) {
  QLIN_TRY(check_common(X, xdt, M, K, N));
  if (xdt != QLIN_BF16)
    return fail(QLIN_ERR_UNSUPPORTED, "weight-only FP8 takes bf16 activations (the weight dequantises to bf16)");
  if (M == 0 || N == 0) return ok();
  QLIN_REQ_PTR(Wq, "Wq");
  QLIN_REQ_PTR(w_scale, "w_scale");
  QLIN_REQ_PTR(Y, "Y");
  if (bias != nullptr && !aligned16(bias)) return fail(QLIN_ERR_ALIGNMENT, "bias is not 16-byte aligned");
  Wo8Params wp{};
  wp.M = M; wp.N = N; wp.K = K; wp.Y = Y;
  wp.s_w = static_cast<const uint16_t*>(w_scale);
  wp.bias = static_cast<const uint16_t*>(bias);
  QLIN_TRY((launch_cvt<0, __nv_bfloat16>(X, Wq, wp, static_cast<cudaStream_t>(stream))));
  return ok();
}

extern "C" qlin_status qlin_nvfp4_weight_only_forward(const void* X, qlin_dtype xdt, int64_t M, int64_t K,
                                                      const uint8_t* Wq, const void* w_scale, int64_t N,
                                                      const void* bias, void* Y, void* stream) {
  QLIN_TRY(check_common(X, xdt, M, K, N));
  if (xdt != QLIN_BF16)
    return fail(QLIN_ERR_UNSUPPORTED, "NVFP4 weight-only takes bf16 activations (the weight dequantises to bf16)");
  if (K % 64 != 0) return fail(QLIN_ERR_ALIGNMENT, "NVFP4 format needs K % 64 == 0");
  if (M == 0 || N == 0) return ok();
  QLIN_REQ_PTR(Wq, "Wq");
  QLIN_REQ_PTR(w_scale, "w_scale");
  QLIN_REQ_PTR(Y, "Y");
  if (!aligned16(w_scale)) return fail(QLIN_ERR_ALIGNMENT, "w_scale is not 16-byte aligned");
  if (bias != nullptr && !aligned16(bias)) return fail(QLIN_ERR_ALIGNMENT, "bias is not 16-byte aligned");
  Wo8Params wp{};
  wp.M = M; wp.N = N; wp.K = K; wp.Y = Y;
  wp.s_b4 = static_cast<const uint8_t*>(w_scale);
  wp.s_t = reinterpret_cast<const float*>(static_cast<const uint8_t*>(w_scale) + round_up(N * K / 16, 16));
  wp.bias = static_cast<const uint16_t*>(bias);
  QLIN_TRY((launch_cvt<2, __nv_bfloat16>(X, Wq, wp, static_cast<cudaStream_t>(stream))));
  return ok();
}

extern "C" qlin_status qlin_int8_block_prep(const void* X, qlin_dtype xdt, int64_t M, int64_t K, void* Xq16,
                                            float* s_x, void* stream) {
  QLIN_TRY(check_common(X, xdt, M, K, 0));
  if (M == 0) return ok();
  QLIN_REQ_PTR(Xq16, "Xq16");
  QLIN_REQ_PTR(s_x, "s_x");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (xdt == QLIN_BF16)
    return launch_rowquant<__nv_bfloat16, 2, false>(X, M, K, static_cast<uint8_t*>(Xq16), s_x, nullptr, st);
  return launch_rowquant<__half, 2, false>(X, M, K, static_cast<uint8_t*>(Xq16), s_x, nullptr, st);
}

extern "C" qlin_status qlin_int8_block_forward(const void* X, qlin_dtype xdt, int64_t M, int64_t K, const int8_t* Wq,
                                               const float* w_scale, int64_t N, const void* bias, void* Y,
                                               void* workspace, size_t ws_bytes, void* stream) {
  QLIN_TRY(check_common(X, xdt, M, K, N));
  if (K % 32 != 0) return fail(QLIN_ERR_ALIGNMENT, "block-scaled int8 needs K a multiple of 32");
  if (M == 0 || N == 0) return ok();
  QLIN_REQ_PTR(Wq, "Wq");
  QLIN_REQ_PTR(w_scale, "w_scale");
  QLIN_REQ_PTR(Y, "Y");
  if (bias != nullptr && !aligned16(bias)) return fail(QLIN_ERR_ALIGNMENT, "bias is not 16-byte aligned");
  if (workspace == nullptr || ws_bytes < qlin_workspace_bytes(QLIN_OP_INT8_BLOCK, M, N, K))
    return fail(QLIN_ERR_WORKSPACE, "workspace too small");
  QLIN_REQ_PTR(workspace, "workspace");
  uint8_t* Xq16 = static_cast<uint8_t*>(workspace);
  float* s_x = reinterpret_cast<float*>(Xq16 + round_up(2 * M * K, 256));
  QLIN_TRY(qlin_int8_block_prep(X, xdt, M, K, Xq16, s_x, stream));
  Wo8Params wp{};
  wp.M = M; wp.N = N; wp.K = K; wp.Y = Y;
  wp.s_wb = w_scale; wp.s_x = s_x;
  wp.bias = static_cast<const uint16_t*>(bias);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (xdt == QLIN_BF16) QLIN_TRY((launch_cvt<1, __nv_bfloat16>(Xq16, Wq, wp, st)));
  else QLIN_TRY((launch_cvt<1, __half>(Xq16, Wq, wp, st)));
  return ok();
}


// ---------------------------------------------------------------------------
// LLM.int8 forward without caller-provided scratch.
//
// Some callers cannot allocate device memory at the point where they run the
// layer: a plugin whose host framework owns every allocation and gives the
// plugin no allocator, or a latency-critical path where a cudaMalloc (which
// may synchronise the device) is not acceptable. For them the scratch of the
// LLM.int8 forward lives in this file-scope device array, created with the
// module: every GPU that loads the library holds these bytes until the
// process exits. All calls share it, and it keeps the previous call's
// contents; the prepare stage clears the parts that must start at zero
// (barrier counter, outlier count, outlier bitmap) on the stream of each
// call, so calls that are ordered on one stream are correct, while calls
// that may overlap on the GPU (other streams, other host threads) race on it.
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_noalloc_scratch[QLIN_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[16] = {};

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (in host code the array's name is only a host-side stand-in).
qlin_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) return fail(QLIN_ERR_CUDA, "cudaGetDevice failed");
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(QLIN_ERR_CUDA, "cudaGetSymbolAddress(no-alloc scratch): %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return QLIN_OK;
}

// Bytes of built-in scratch the forward needs: the LLM.int8 workspace layout
// without the stream-K arrival counters and partial slots.
size_t noalloc_scratch_needed(int64_t M, int64_t N, int64_t K) {
  return int8_layout(nullptr, M, N, K, true, false).total;
}
}  // namespace

extern "C" qlin_status qlin_int8_outlier_forward_noalloc(const void* X, qlin_dtype xdt, int64_t M, int64_t K,
                                                         const int8_t* Wq, const float* w_scale, int64_t N,
                                                         float threshold, const void* bias, void* Y, void* stream) {
  QLIN_TRY(check_common(X, xdt, M, K, N));
  if (M == 0 || N == 0) return ok();
  // the built-in scratch holds the forward's layout without the stream-K
  // partial slots (the GEMM then takes whole tiles, the same results)
  const size_t need = noalloc_scratch_needed(M, N, K);
  if (need > static_cast<size_t>(QLIN_NOALLOC_SCRATCH_BYTES))
    return fail(QLIN_ERR_UNSUPPORTED,
                "qlin_int8_outlier_forward_noalloc: M=%lld N=%lld K=%lld needs %zu bytes of scratch, more than the "
                "%lld bytes of its built-in array; use qlin_int8_outlier_forward with a workspace",
                static_cast<long long>(M), static_cast<long long>(N), static_cast<long long>(K), need,
                static_cast<long long>(QLIN_NOALLOC_SCRATCH_BYTES));
  QLIN_REQ_PTR(Y, "Y");
  QLIN_REQ_PTR(Wq, "Wq");
  QLIN_REQ_PTR(w_scale, "w_scale");
  if (bias != nullptr && !aligned16(bias)) return fail(QLIN_ERR_ALIGNMENT, "bias is not 16-byte aligned");
  DeviceInfo* d;
  QLIN_TRY(device_info(&d));
  void* ws = nullptr;
  QLIN_TRY(noalloc_scratch(&ws));
  const Int8Ws w = int8_layout(ws, M, N, K, true, false);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  QLIN_TRY(int8_outlier_prepare_ws(X, xdt, M, K, Wq, w_scale, N, threshold, w, st));
  QLIN_TRY(int8_outlier_gemm_ws(xdt, M, K, Wq, w_scale, N, bias, Y, w, st));
  return ok();
}



