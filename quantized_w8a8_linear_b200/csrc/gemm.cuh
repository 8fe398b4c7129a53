// gemm.cuh -- persistent, warp-specialised tcgen05 GEMM for sm_100a.
//
//   C[M,N] = A[M,K] B[N,K]^T, A and B 8-bit (int8 -> int32 with kind::i8, or
//   E4M3 -> fp32 with kind::f8f6f4), both K-major in global memory.
//
// Roles (one CTA per SM, 6 warps):
//   warp 0      TMA producer: 128x128-byte A tiles and BNx128-byte B tiles,
//               128B-swizzled, into a STAGES-deep shared-memory ring;
//   warp 1      MMA issuer: allocates all 512 TMEM columns (two BN-column
//               accumulators), issues 4 UMMAs (K = 32 each) per stage and
//               commits stage release / accumulator-ready to mbarriers;
//   warps 2-5   epilogue: tcgen05.ld of their 32-lane quarter, fused dequant
//               (row x column scales), the floating-point outlier part of
//               LLM.int8 as a rank-|O| update on CUDA cores, bias, rounding,
//               and the store of Y. The second accumulator lets the epilogue
//               of tile t overlap the main loop of tile t+1.
// Tiles are handed out round-robin (tile = blockIdx.x + i * gridDim.x) with
// the M index fastest, so CTAs running together share the same weight tile.
// Out-of-range rows and K columns are zero-filled by TMA; stores are
// predicated on M and N.
#pragma once
#include "common.cuh"

namespace qlin {

enum EpiKind { EPI_I32 = 0, EPI_INT8_OUTLIER = 1, EPI_FP8_TENSOR = 2, EPI_FP8_ROWCOL = 3 };

constexpr int GEMM_BM = 128;
constexpr int GEMM_BK = 128;                 // bytes (= elements) per stage along K
constexpr int GEMM_EPI_WARPS = 4;
constexpr int GEMM_THREADS = 64 + 32 * GEMM_EPI_WARPS;

struct EpiParams {
  int64_t M, N, K;
  void* Y;                    // [M,N]: int32 (EPI_I32) or 16-bit output dtype
  const float* s_x;           // [M] per-token scale
  const float* s_w;           // [N] fp32 per-channel weight scale
  const uint16_t* s_w_bf16;   // [N] bf16 per-channel weight scale
  const float* x_scale;       // static per-tensor input scale (device scalar)
  const float* w_scale;       // per-tensor weight scale (device scalar)
  const uint16_t* bias;       // [N] output dtype, nullable
  const int32_t* count;       // number of outlier columns (device)
  const uint16_t* X_O;        // [M, ostride] outlier activations
  const uint16_t* W_O;        // [N, ostride] dequantised outlier weights
  int64_t ostride;
};

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr int A_BYTES = GEMM_BM * GEMM_BK;
  static constexpr int B_BYTES = BN * GEMM_BK;
  static constexpr int TILE_BYTES = STAGES * (A_BYTES + B_BYTES);
  static constexpr int BAR_BYTES = 8 * (2 * STAGES + 4 + 1) + 16;
  static constexpr int TOTAL = 1024 + TILE_BYTES + BAR_BYTES;   // 1024: alignment slack
};

// 32 consecutive fp32 column values starting at n0 (0 past N).
__device__ __forceinline__ void load_cols_f32(const float* p, int64_t n0, int64_t N, bool full, float (&o)[32]) {
  if (full) {
    const float4* q = reinterpret_cast<const float4*>(p + n0);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 v = __ldg(q + i);
      o[4 * i] = v.x; o[4 * i + 1] = v.y; o[4 * i + 2] = v.z; o[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) o[j] = (n0 + j < N) ? __ldg(p + n0 + j) : 0.0f;
  }
}

// 32 consecutive 16-bit column values (as float) starting at n0 (0 past N).
template <typename T>
__device__ __forceinline__ void load_cols_h(const uint16_t* p, int64_t n0, int64_t N, bool full, float (&o)[32]) {
  if (full) {
    const uint4* q = reinterpret_cast<const uint4*>(p + n0);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint16_t h[8];
      unpack8(__ldg(q + i), h);
#pragma unroll
      for (int e = 0; e < 8; ++e) o[8 * i + e] = to_f<T>(h[e]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) o[j] = (n0 + j < N) ? to_f<T>(__ldg(p + n0 + j)) : 0.0f;
  }
}

template <typename TOut, int EPI>
__device__ __forceinline__ void epilogue_chunk(const EpiParams& p, const uint32_t (&r)[32], int64_t row,
                                               int64_t n0, float sx, float alpha, int cnt) {
  const int64_t N = p.N;
  const bool full = (n0 + 32 <= N);
  if constexpr (EPI == EPI_I32) {
    int32_t* y = reinterpret_cast<int32_t*>(p.Y) + row * N + n0;
    if (full && (N & 3) == 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        reinterpret_cast<int4*>(y)[i] = make_int4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (n0 + j < N) y[j] = static_cast<int32_t>(r[j]);
    }
  } else {
    float acc[32];
    float cs[32];
    if constexpr (EPI == EPI_INT8_OUTLIER) {
      load_cols_f32(p.s_w, n0, N, full, cs);
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] = static_cast<float>(static_cast<int32_t>(r[j])) * (sx * cs[j]);
      // floating-point outlier part: F[row, n] = sum_o X_O[row, o] * W_O[n, o]
      for (int o0 = 0; o0 < cnt; o0 += 8) {
        uint16_t xh[8];
        unpack8(*reinterpret_cast<const uint4*>(p.X_O + row * p.ostride + o0), xh);
        float xo[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) xo[e] = to_f<TOut>(xh[e]);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (full || n0 + j < N) {
            uint16_t wh[8];
            unpack8(__ldg(reinterpret_cast<const uint4*>(p.W_O + (n0 + j) * p.ostride + o0)), wh);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[j] = fmaf(xo[e], to_f<TOut>(wh[e]), acc[j]);
          }
        }
      }
    } else if constexpr (EPI == EPI_FP8_TENSOR) {
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] = __uint_as_float(r[j]) * alpha;
    } else {  // EPI_FP8_ROWCOL
      load_cols_h<__nv_bfloat16>(p.s_w_bf16, n0, N, full, cs);
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] = __uint_as_float(r[j]) * (sx * cs[j]);
    }
    if (p.bias != nullptr) {
      load_cols_h<TOut>(p.bias, n0, N, full, cs);
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] += cs[j];
    }
    uint16_t* y = reinterpret_cast<uint16_t*>(p.Y) + row * N + n0;
    if (full && (N & 7) == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 v;
        v.x = pack2<TOut>(acc[8 * i + 0], acc[8 * i + 1]);
        v.y = pack2<TOut>(acc[8 * i + 2], acc[8 * i + 3]);
        v.z = pack2<TOut>(acc[8 * i + 4], acc[8 * i + 5]);
        v.w = pack2<TOut>(acc[8 * i + 6], acc[8 * i + 7]);
        reinterpret_cast<uint4*>(y)[i] = v;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (n0 + j < N) y[j] = from_f<TOut>(acc[j]);
    }
  }
}

template <int KIND, int EPI, typename TOut, int BN, int STAGES>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const EpiParams p) {
  using L = GemmSmem<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * L::A_BYTES;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + L::TILE_BYTES);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* tfull_bar = empty_bar + STAGES;     // [2]
  uint64_t* tempty_bar = tfull_bar + 2;         // [2]
  uint64_t* drain_bar = tempty_bar + 2;         // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t M = p.M, N = p.N, K = p.K;
  const int num_m = static_cast<int>((M + GEMM_BM - 1) / GEMM_BM);
  const int num_n = static_cast<int>((N + BN - 1) / BN);
  const int num_tiles = num_m * num_n;
  const int num_kb = static_cast<int>((K + GEMM_BK - 1) / GEMM_BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], GEMM_EPI_WARPS);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;   // bit s: stage s has a load in flight that nobody consumed yet
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        const int mb = tile % num_m, nb = tile / num_m;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_bar[stage], L::A_BYTES + L::B_BYTES);
          tma_load_2d(sA + stage * L::A_BYTES, &tmA, &full_bar[stage], kb * GEMM_BK, mb * GEMM_BM);
          tma_load_2d(sB + stage * L::B_BYTES, &tmB, &full_bar[stage], kb * GEMM_BK, nb * BN);
          issued |= 1u << stage;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // aborted: wait (bounded) for the copies still in flight before the CTA exits
        for (int i = 0; i < STAGES; ++i) {
          if (--stage < 0) { stage = STAGES - 1; phase ^= 1u; }
          if (issued & (1u << stage)) {
            const uint32_t a = smem_u32(&full_bar[stage]);
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(a, phase) && globaltimer() - t0 < g_wait_timeout_ns) {}
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = KIND == 0 ? idesc_i8(GEMM_BM, BN) : idesc_e4m3(GEMM_BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = sdesc_k128(smem_u32(sA + stage * L::A_BYTES));
          const uint64_t bdesc = sdesc_k128(smem_u32(sB + stage * L::B_BYTES));
#pragma unroll
          for (int k = 0; k < GEMM_BK / 32; ++k)
            umma<KIND>(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc, (kb | k) != 0 ? 1u : 0u);
          umma_commit(&empty_bar[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull_bar[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      // every MMA this thread issued has completed before TMEM is released
      umma_commit(drain_bar);
      const uint32_t a = smem_u32(drain_bar);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(a, 0) && globaltimer() - t0 < g_wait_timeout_ns) {}
    }
  } else {
    // ---------------- epilogue ----------------
    const int q = warp & 3;   // TMEM lane quarter this warp may access
    int cnt = 0;
    float alpha = 0.0f;
    if constexpr (EPI == EPI_INT8_OUTLIER) cnt = *p.count;
    if constexpr (EPI == EPI_FP8_TENSOR) alpha = __ldg(p.x_scale) * __ldg(p.w_scale);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int mb = tile % num_m, nb = tile / num_m;
      if (!mbar_wait(&tfull_bar[acc], acc_phase, abort_flag)) break;
      tc_fence_after();
      const int64_t row = static_cast<int64_t>(mb) * GEMM_BM + q * 32 + lane;
      const bool row_ok = row < M;
      float sx = 0.0f;
      if constexpr (EPI == EPI_INT8_OUTLIER || EPI == EPI_FP8_ROWCOL) sx = row_ok ? __ldg(p.s_x + row) : 0.0f;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(t_row + static_cast<uint32_t>(c * 32), r);
        tmem_ld_wait();
        const int64_t n0 = static_cast<int64_t>(nb) * BN + c * 32;
        if (row_ok && n0 < N) epilogue_chunk<TOut, EPI>(p, r, row, n0, sx, alpha, cnt);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * BN);
  }
}

}  // namespace qlin
