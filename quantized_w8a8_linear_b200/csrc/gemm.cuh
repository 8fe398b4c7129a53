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

// EPI_INT8_OUTLIER_I32: the int32 accumulator of the LLM.int8 path after the
// outlier-column correction, written out (parity export of the same kernel).
enum EpiKind { EPI_I32 = 0, EPI_INT8_OUTLIER = 1, EPI_FP8_TENSOR = 2, EPI_FP8_ROWCOL = 3, EPI_INT8_OUTLIER_I32 = 4 };

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
  // LLM.int8: the int8 operands and the outlier columns. The A operand may
  // hold non-zero codes in outlier columns; the epilogue subtracts their
  // exact int32 contribution sum_o Xq[m,O[o]] * Wq[n,O[o]] from the accumulator.
  const int8_t* Xq;           // [M,K]
  const int8_t* Wq;           // [N,K]
  const int32_t* O;           // [K] ascending outlier columns, first *count valid
};

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr int A_BYTES = GEMM_BM * GEMM_BK;
  static constexpr int B_BYTES = BN * GEMM_BK;
  static constexpr int TILE_BYTES = STAGES * (A_BYTES + B_BYTES);
  static constexpr int EPI_BYTES = static_cast<int>(sizeof(float) * 2 * BN + sizeof(uint32_t) * (16 + 8) * BN);
  static constexpr int BAR_BYTES = 8 * (2 * STAGES + 4 + 2) + 16;
  static constexpr int TOTAL = 1024 + TILE_BYTES + EPI_BYTES + BAR_BYTES;   // 1024: alignment slack
};

// Per-tile epilogue data staged in shared memory by the epilogue warps:
// column scales, bias, and (LLM.int8) the tile's slice of the dequantised
// outlier weight columns, up to 32 outliers as packed 16-bit pairs, and the
// int8 weight codes of those columns, 4 to a word. All lanes of a warp read
// the same word (a broadcast), so there are no bank conflicts.
template <int BN>
struct EpiStage {
  float sw[BN];
  float bias[BN];
  uint32_t wo[BN][16];
  uint32_t wq[BN][8];
};

// Four int8 codes of row `base` at outlier columns O[o0..o0+3] packed into a
// word (0 beyond cnt).
__device__ __forceinline__ uint32_t gather_codes4(const int8_t* __restrict__ base, const int32_t* __restrict__ O,
                                                  int o0, int cnt) {
  uint32_t w = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    if (o0 + e < cnt) w |= static_cast<uint32_t>(static_cast<uint8_t>(__ldg(base + __ldg(O + o0 + e)))) << (8 * e);
  return w;
}


template <typename TOut, int EPI, int BN>
__device__ __forceinline__ void epi_stage(const EpiParams& p, EpiStage<BN>& es, int64_t n_base, int et, int cn,
                                          int cnt) {
  for (int j = et; j < BN; j += 32 * GEMM_EPI_WARPS) {
    const int64_t n = n_base + j;
    float sw = 0.0f, b = 0.0f;
    if (n < p.N) {
      if constexpr (EPI == EPI_INT8_OUTLIER) sw = __ldg(p.s_w + n);
      if constexpr (EPI == EPI_FP8_ROWCOL) sw = to_f<__nv_bfloat16>(__ldg(p.s_w_bf16 + n));
      if (p.bias != nullptr) b = to_f<TOut>(__ldg(p.bias + n));
    }
    es.sw[j] = sw;
    es.bias[j] = b;
  }
  if (cn > 0 && EPI == EPI_INT8_OUTLIER) {
    const int nq = cn / 8;   // 16-byte quads of 8 outlier values per column
    for (int idx = et; idx < BN * nq; idx += 32 * GEMM_EPI_WARPS) {
      const int j = idx / nq, qd = idx - j * nq;
      const int64_t n = n_base + j;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (n < p.N && qd * 8 < cnt) v = __ldg(reinterpret_cast<const uint4*>(p.W_O + n * p.ostride + qd * 8));
      *reinterpret_cast<uint4*>(&es.wo[j][qd * 4]) = v;
    }
  }
  if (cn > 0) {
    const int nw = cn / 4;
    for (int idx = et; idx < BN * nw; idx += 32 * GEMM_EPI_WARPS) {
      const int j = idx / nw, w = idx - j * nw;
      const int64_t n = n_base + j;
      es.wq[j][w] = n < p.N ? gather_codes4(p.Wq + n * p.K, p.O, 4 * w, cnt) : 0u;
    }
  }
}

// CW outputs (16-bit pairs, the lower column in the low half) to Y[row, n0..].
template <int CW>
__device__ __forceinline__ void store_chunk(const EpiParams& p, const uint32_t (&out)[CW / 2], int64_t row,
                                            int64_t n0) {
  const int64_t N = p.N;
  uint16_t* y = reinterpret_cast<uint16_t*>(p.Y) + row * N + n0;
  if (n0 + CW <= N && (N & 7) == 0) {
#pragma unroll
    for (int i = 0; i < CW / 8; ++i)
      reinterpret_cast<uint4*>(y)[i] = make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
  } else {
#pragma unroll
    for (int j = 0; j < CW; ++j)
      if (n0 + j < N) y[j] = static_cast<uint16_t>(out[j >> 1] >> (16 * (j & 1)));
  }
}

// LLM.int8 accumulator of (row, n) without the outlier columns:
// acc - sum_o Xq[row,O[o]] * Wq[n,O[o]], exact in int32. xq: the row's codes
// in the outlier columns, 4 to a word; the weight codes come from the stage
// (CN > 0) or from global memory (CN < 0).
template <int CN, int BN, int NXQ>
__device__ __forceinline__ int32_t corrected(const EpiParams& p, const EpiStage<BN>& es, const uint32_t (&xq)[NXQ],
                                             uint32_t acc, int64_t row, int64_t n, int jj, int cnt) {
  int32_t c32 = static_cast<int32_t>(acc);
  if constexpr (CN > 0) {
#pragma unroll
    for (int w = 0; w < CN / 4; ++w) c32 -= __dp4a(static_cast<int>(xq[w]), static_cast<int>(es.wq[jj][w]), 0);
  }
  if constexpr (CN < 0) {
    if (n < p.N)
      for (int o = 0; o < cnt; ++o) {
        const int k = __ldg(p.O + o);
        c32 -= static_cast<int32_t>(__ldg(p.Xq + row * p.K + k)) * static_cast<int32_t>(__ldg(p.Wq + n * p.K + k));
      }
  }
  return c32;
}

// One accumulator tile, one thread per row: TMEM -> registers in chunks of
// CW columns (32; 16 where the outlier operands take the registers), then
// y = acc * scales (+ outlier part) + bias -> Y.
// CN: outlier columns handled from shared memory (0, 8, 16 or 32; a bucket
// >= the count, zero-padded); CN < 0: more than 32 outliers, the weight
// columns are read from global memory (correct for any count, not fast).
template <typename TOut, int EPI, int BN, int CN>
__device__ __forceinline__ void epi_tile(const EpiParams& p, const EpiStage<BN>& es, uint32_t t_row, int64_t row,
                                         bool row_ok, int64_t n_base, float sx, float alpha, int cnt) {
  constexpr int NX = CN > 0 ? CN : 1;
  float xo[NX];
  uint32_t xq[(NX + 3) / 4];   // this row's codes in the outlier columns, 4 to a word
#pragma unroll
  for (int i = 0; i < NX; ++i) xo[i] = 0.0f;
#pragma unroll
  for (int i = 0; i < (NX + 3) / 4; ++i) xq[i] = 0u;
  if constexpr (CN > 0) {
#pragma unroll
    for (int w = 0; w < CN / 4; ++w)
      if (row_ok && 4 * w < cnt) xq[w] = gather_codes4(p.Xq + row * p.K, p.O, 4 * w, cnt);
#pragma unroll
    for (int qd = 0; qd < CN / 8; ++qd) {
      if (EPI == EPI_INT8_OUTLIER && row_ok && qd * 8 < cnt) {
        uint16_t h[8];
        unpack8(*reinterpret_cast<const uint4*>(p.X_O + row * p.ostride + qd * 8), h);
#pragma unroll
        for (int e = 0; e < 8; ++e) xo[qd * 8 + e] = to_f<TOut>(h[e]);
      }
    }
  }
  constexpr int CW = (CN == 32 || CN < 0) ? 16 : 32;
#pragma unroll 1
  for (int c = 0; c < BN / CW; ++c) {
    uint32_t r[CW];
    __syncwarp();
    tmem_ld(t_row + static_cast<uint32_t>(c * CW), r);
    tmem_ld_wait();
    const int64_t n0 = n_base + c * CW;
    if (row_ok && n0 < p.N) {
      if constexpr (EPI == EPI_I32 || EPI == EPI_INT8_OUTLIER_I32) {
        if constexpr (EPI == EPI_INT8_OUTLIER_I32) {
#pragma unroll
          for (int j = 0; j < CW; ++j)
            r[j] = static_cast<uint32_t>(corrected<CN>(p, es, xq, r[j], row, n0 + j, c * CW + j, cnt));
        }
        int32_t* y = reinterpret_cast<int32_t*>(p.Y) + row * p.N + n0;
        if (n0 + CW <= p.N && (p.N & 3) == 0) {
#pragma unroll
          for (int i = 0; i < CW / 4; ++i)
            reinterpret_cast<int4*>(y)[i] = make_int4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < CW; ++j)
            if (n0 + j < p.N) y[j] = static_cast<int32_t>(r[j]);
        }
      } else {
        uint32_t out[CW / 2];   // the chunk's outputs as packed 16-bit pairs
        float prev = 0.0f;
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          const int jj = c * CW + j;
          float a;
          if constexpr (EPI == EPI_INT8_OUTLIER)
            a = static_cast<float>(corrected<CN>(p, es, xq, r[j], row, n0 + j, jj, cnt)) * (sx * es.sw[jj]);
          else if constexpr (EPI == EPI_FP8_TENSOR) a = __uint_as_float(r[j]) * alpha;
          else a = __uint_as_float(r[j]) * (sx * es.sw[jj]);
          if constexpr (CN > 0) {
#pragma unroll
            for (int qd = 0; qd < CN / 8; ++qd) {
              uint16_t h[8];
              unpack8(*reinterpret_cast<const uint4*>(&es.wo[jj][qd * 4]), h);
#pragma unroll
              for (int e = 0; e < 8; ++e) a = fmaf(xo[qd * 8 + e], to_f<TOut>(h[e]), a);
            }
          }
          if constexpr (CN < 0) {
            for (int o0 = 0; o0 < cnt; o0 += 8) {
              uint16_t xh[8], wh[8];
              unpack8(*reinterpret_cast<const uint4*>(p.X_O + row * p.ostride + o0), xh);
              if (n0 + j < p.N) {
                unpack8(__ldg(reinterpret_cast<const uint4*>(p.W_O + (n0 + j) * p.ostride + o0)), wh);
#pragma unroll
                for (int e = 0; e < 8; ++e) a = fmaf(to_f<TOut>(xh[e]), to_f<TOut>(wh[e]), a);
              }
            }
          }
          a += es.bias[jj];
          if (j & 1) out[j >> 1] = pack2<TOut>(prev, a);
          else prev = a;
        }
        store_chunk<CW>(p, out, row, n0);
      }
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
  EpiStage<BN>& es = *reinterpret_cast<EpiStage<BN>*>(smem + L::TILE_BYTES);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + L::TILE_BYTES + L::EPI_BYTES);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* tfull_bar = empty_bar + STAGES;     // [2]
  uint64_t* tempty_bar = tfull_bar + 2;         // [2]
  uint64_t* drain_bar = tempty_bar + 2;         // [1]
  uint64_t* epi_mbar = drain_bar + 1;           // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epi_mbar + 1);
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
    mbar_init(epi_mbar, 32 * GEMM_EPI_WARPS);
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
    const int et = threadIdx.x - 64;
    int cnt = 0;
    float alpha = 0.0f;
    if constexpr (EPI == EPI_INT8_OUTLIER || EPI == EPI_INT8_OUTLIER_I32) cnt = *p.count;
    if constexpr (EPI == EPI_FP8_TENSOR) alpha = __ldg(p.x_scale) * __ldg(p.w_scale);
    const int cn = cnt == 0 ? 0 : cnt <= 8 ? 8 : cnt <= 16 ? 16 : cnt <= 32 ? 32 : -1;
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t bar_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int mb = tile % num_m, nb = tile / num_m;
      const int64_t n_base = static_cast<int64_t>(nb) * BN;
      if constexpr (EPI != EPI_I32) {
        // the previous tile's readers are done with the staging area
        if (!epi_bar(epi_mbar, bar_phase, abort_flag)) break;
        epi_stage<TOut, EPI, BN>(p, es, n_base, et, cn, cnt);
        if (!epi_bar(epi_mbar, bar_phase, abort_flag)) break;
      }
      if (!mbar_wait(&tfull_bar[acc], acc_phase, abort_flag)) break;
      tc_fence_after();
      const int64_t row = static_cast<int64_t>(mb) * GEMM_BM + q * 32 + lane;
      const bool row_ok = row < M;
      float sx = 0.0f;
      if constexpr (EPI == EPI_INT8_OUTLIER || EPI == EPI_FP8_ROWCOL) sx = row_ok ? __ldg(p.s_x + row) : 0.0f;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
      if constexpr (EPI == EPI_INT8_OUTLIER || EPI == EPI_INT8_OUTLIER_I32) {
        if (cn == 0) epi_tile<TOut, EPI, BN, 0>(p, es, t_row, row, row_ok, n_base, sx, alpha, cnt);
        else if (cn == 8) epi_tile<TOut, EPI, BN, 8>(p, es, t_row, row, row_ok, n_base, sx, alpha, cnt);
        else if (cn == 16) epi_tile<TOut, EPI, BN, 16>(p, es, t_row, row, row_ok, n_base, sx, alpha, cnt);
        else if (cn == 32) epi_tile<TOut, EPI, BN, 32>(p, es, t_row, row, row_ok, n_base, sx, alpha, cnt);
        else epi_tile<TOut, EPI, BN, -1>(p, es, t_row, row, row_ok, n_base, sx, alpha, cnt);
      } else {
        epi_tile<TOut, EPI, BN, 0>(p, es, t_row, row, row_ok, n_base, sx, alpha, cnt);
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
