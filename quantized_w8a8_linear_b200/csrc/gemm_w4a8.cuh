// gemm_w4a8.cuh -- W4A8 GEMM for sm_100a: int4 per-group weights (group 128
// along K, fp32 scales) with per-token int8 activations (Qwen-Image-fni8
// page, "Format"):
//
//   C_g[i,j] = sum_{k in group g} Xq[i,k] * Wq4[j,k]          (int32, exact)
//   Y[i,j]   = dtype( s_x[i] * sum_g s_w[j,g] * C_g[i,j] + bias[j] )
//
// Roles (one CTA per SM, 16 warps, persistent over 128x128 output tiles):
//   warp 0       TMA producer: the int8 A tile (128 x 128 B) and the packed
//                int4 B tile (128 rows x 64 B) of one group per stage;
//   warp 1       MMA issuer: TMEM holds four 128-column int32 group
//                accumulators; each group is 4 x tcgen05.mma kind::i8 (K=32)
//                into a fresh accumulator;
//   warps 2-3,   converters: unpack the int4 B tile to int8 in the 128-byte
//   12-13        swizzled K-major layout the MMA reads (the same layout TMA
//                writes), then hand the stage to the MMA;
//   warps 14-15  idle;
//   warps 4-11   promotion + epilogue, two warps per 32-lane TMEM quarter,
//                each with 64 columns: per group, int32 -> fp32 (exact: |C_g|
//                <= 128*127*7 < 2^22) and sum += s_w[j,g] * C_g in registers
//                (packed f32x2 arithmetic); the next group's accumulator is
//                read from TMEM while this one is promoted, and an accumulator
//                is handed back to the MMA as soon as it has been read;
//                after the last group, y = s_x[i] * sum + bias -> Y.
// All waits are bounded (common.cuh).
#pragma once
#include "common.cuh"

namespace qlin {

constexpr int W4_BM = 128, W4_BN = 128, W4_G = 128;   // tile rows, tile columns, group (= K per stage)
constexpr int W4_STAGES = 4;
constexpr int W4_CONV_WARPS = 4, W4_PROMO_WARPS = 8;
constexpr int W4_THREADS = 512;   // 16 warps: 4 warpgroups (see the role list above)
constexpr int W4_ACC = 4;                             // TMEM group accumulators (4 x 128 columns)
constexpr int W4_SWIN = 32;                           // groups per staged window of weight scales
// Register split (setmaxnreg): warpgroups 0 and 3 (producer, MMA, converters)
// drop to W4_REGS_LOW, the promotion warpgroups 1 and 2 rise to W4_REGS_HIGH.
// It fits the block's pool when 2 * 128 (R - LOW) >= 256 (HIGH - R) for the
// launch count R.
constexpr int W4_REGS_LOW = 40;
constexpr int W4_REGS_HIGH = 216;
constexpr int W4_REGS_MIN_LAUNCH = 128;
static_assert(2 * 128 * (W4_REGS_MIN_LAUNCH - W4_REGS_LOW) >= 256 * (W4_REGS_HIGH - W4_REGS_MIN_LAUNCH),
              "register split must fit the launch pool");

struct W4Params {
  int64_t M, N, K;
  void* Y;                    // [M,N] output dtype
  const float* s_x;           // [M]
  const float* s_w;           // [N, K/128] (nullptr: int32 export mode)
  const uint16_t* bias;       // [N] nullable
  int32_t* dbg;               // [M,N] int32 partials of group dbg_group (parity export), or nullptr
  int dbg_group;
};

struct W4Smem {
  static constexpr int A_BYTES = W4_BM * W4_G;            // 16 KB int8
  static constexpr int BP_BYTES = W4_BN * W4_G / 2;       // 8 KB packed int4
  static constexpr int BU_BYTES = W4_BN * W4_G;           // 16 KB unpacked int8 (swizzled)
  static constexpr int STAGE_BYTES = A_BYTES + BP_BYTES + BU_BYTES;
  static constexpr int SW_BYTES = 4 * W4_SWIN * W4_BN;    // 16 KB weight-scale window
  static constexpr int BAR_BYTES = 8 * (3 * W4_STAGES + 2 * W4_ACC + 2) + 16;
  static constexpr int TOTAL = 1024 + W4_STAGES * STAGE_BYTES + SW_BYTES + BAR_BYTES;
};

// 32 signed int4 (16 packed bytes, even k in the low nibble) -> 32 int8.
// Per byte: 0x80 | (nibble ^ 8) is 0x80 + (t + 8) for the nibble's value t,
// so subtracting 8 borrows from no neighbour and leaves 0x80 + t, and
// flipping bit 7 gives t in two's complement.
__device__ __forceinline__ uint32_t sext_nibbles(uint32_t nib4) {   // four nibbles in the low halves of 4 bytes
  return ((((nib4 & 0x0F0F0F0Fu) ^ 0x88888888u) - 0x08080808u) ^ 0x80808080u);
}
__device__ __forceinline__ void unpack_int4x32(const uint4& p, uint4& lo16, uint4& hi16) {
  const uint32_t w[4] = {p.x, p.y, p.z, p.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t l = sext_nibbles(w[i]);        // even k
    const uint32_t h = sext_nibbles(w[i] >> 4);   // odd k
    o[2 * i] = __byte_perm(l, h, 0x5140);
    o[2 * i + 1] = __byte_perm(l, h, 0x7362);
  }
  lo16 = make_uint4(o[0], o[1], o[2], o[3]);
  hi16 = make_uint4(o[4], o[5], o[6], o[7]);
}

template <typename TOut>
__global__ void __launch_bounds__(W4_THREADS, 1)
    k_gemm_w4a8(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const W4Params p) {
  using L = W4Smem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // per stage: [A 16 KB | unpacked B 16 KB | packed B 8 KB] (A and unpacked B 1024-aligned)
  auto sA = [&](int s) { return smem + s * L::STAGE_BYTES; };
  auto sBu = [&](int s) { return smem + s * L::STAGE_BYTES + L::A_BYTES; };
  auto sBp = [&](int s) { return smem + s * L::STAGE_BYTES + L::A_BYTES + L::BU_BYTES; };
  float* s_win = reinterpret_cast<float*>(smem + W4_STAGES * L::STAGE_BYTES);   // [W4_SWIN][W4_BN]
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + W4_STAGES * L::STAGE_BYTES + L::SW_BYTES);
  uint64_t* conv_bar = full_bar + W4_STAGES;
  uint64_t* empty_bar = conv_bar + W4_STAGES;
  uint64_t* gfull_bar = empty_bar + W4_STAGES;
  uint64_t* gempty_bar = gfull_bar + W4_ACC;
  uint64_t* drain_bar = gempty_bar + W4_ACC;
  uint64_t* promo_bar = drain_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(promo_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t M = p.M, N = p.N, K = p.K;
  const int num_m = static_cast<int>((M + W4_BM - 1) / W4_BM);
  const int num_n = static_cast<int>((N + W4_BN - 1) / W4_BN);
  const int num_tiles = num_m * num_n;
  const int G = static_cast<int>(K / W4_G);

  if (threadIdx.x == 0) {
    for (int s = 0; s < W4_STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&conv_bar[s], W4_CONV_WARPS);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < W4_ACC; ++b) {
      mbar_init(&gfull_bar[b], 1);
      mbar_init(&gempty_bar[b], W4_PROMO_WARPS);
    }
    mbar_init(drain_bar, 1);
    mbar_init(promo_bar, 32 * W4_PROMO_WARPS);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 32 * 16);   // 512 columns
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4 || warp >= 12) {
  setmaxnreg_dec<W4_REGS_LOW>();
  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        const int mb = tile % num_m, nb = tile / num_m;
        for (int g = 0; g < G; ++g) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_bar[stage], L::A_BYTES + L::BP_BYTES);
          tma_load_2d(sA(stage), &tmA, &full_bar[stage], g * W4_G, mb * W4_BM);
          tma_load_2d(sBp(stage), &tmB, &full_bar[stage], g * (W4_G / 2), nb * W4_BN);
          issued |= 1u << stage;
          if (++stage == W4_STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        for (int i = 0; i < W4_STAGES; ++i) {
          if (--stage < 0) { stage = W4_STAGES - 1; phase ^= 1u; }
          if (issued & (1u << stage)) {
            const uint32_t a = smem_u32(&full_bar[stage]);
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(a, phase) && globaltimer() - t0 < drain_limit_ns()) {}
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = idesc_i8(W4_BM, W4_BN);
      int stage = 0;
      uint32_t phase = 0;
      int buf = 0;
      uint32_t buf_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        for (int g = 0; g < G; ++g) {
          if (!mbar_wait(&gempty_bar[buf], buf_phase ^ 1u, abort_flag)) { ok = false; break; }
          if (!mbar_wait(&conv_bar[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * W4_BN);
          const uint64_t adesc = sdesc_k128(smem_u32(sA(stage)));
          const uint64_t bdesc = sdesc_k128(smem_u32(sBu(stage)));
#pragma unroll
          for (int k = 0; k < W4_G / 32; ++k) umma<0>(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc, k != 0 ? 1u : 0u);
          umma_commit(&empty_bar[stage]);
          umma_commit(&gfull_bar[buf]);
          if (++stage == W4_STAGES) { stage = 0; phase ^= 1u; }
          if (++buf == W4_ACC) { buf = 0; buf_phase ^= 1u; }
        }
      }
      umma_commit(drain_bar);
      const uint32_t a = smem_u32(drain_bar);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(a, 0) && globaltimer() - t0 < drain_limit_ns()) {}
    }
  } else if (warp == 2 || warp == 3 || warp == 12 || warp == 13) {
    // ---------------- converters: packed int4 -> swizzled int8 ----------------
    const int ct = warp < 4 ? threadIdx.x - 64 : threadIdx.x - 384 + 64;   // 0..127
    int stage = 0;
    uint32_t phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      bool ok = true;
      for (int g = 0; g < G; ++g) {
        if (!mbar_wait(&full_bar[stage], phase, abort_flag)) { ok = false; break; }
        const uint4* src = reinterpret_cast<const uint4*>(sBp(stage));
        uint8_t* dst = sBu(stage);
#pragma unroll
        for (int i = 0; i < (L::BP_BYTES / 16) / (32 * W4_CONV_WARPS); ++i) {
          const int c = ct + i * 32 * W4_CONV_WARPS;   // 16-byte chunk of the packed tile
          const int r = c >> 2, part = c & 3;          // row, quarter of the row's 64 packed bytes
          uint4 lo, hi;
          unpack_int4x32(src[c], lo, hi);
          // row r's 128 int8 bytes: 16-byte chunk ch lives at chunk (ch ^ (r & 7)) of the row
          *reinterpret_cast<uint4*>(dst + r * 128 + (((2 * part) ^ (r & 7)) << 4)) = lo;
          *reinterpret_cast<uint4*>(dst + r * 128 + (((2 * part + 1) ^ (r & 7)) << 4)) = hi;
        }
        fence_proxy_async_smem();   // generic writes -> read by the tensor core (async proxy)
        __syncwarp();
        if (lane == 0) mbar_arrive(&conv_bar[stage]);
        if (++stage == W4_STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
  }
  } else {
    setmaxnreg_inc<W4_REGS_HIGH>();
    // ---------------- promotion + epilogue ----------------
    const int pw = warp - 4;                     // 0..7
    const int q = warp & 3;                      // TMEM lane quarter
    const int c0 = (pw >> 2) * 64;               // this warp's first column of the tile
    const int pt = threadIdx.x - 128;            // 0..255
    int buf = 0;
    uint32_t buf_phase = 0, bar_phase = 0;
    bool ok = true;
    // TMEM address of this warp's lane quarter, columns c0 + 32h of accumulator buffer b
    auto taddr = [&](int b, int h) {
      return tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(b * W4_BN + c0 + 32 * h);
    };
    uint32_t ra0[32], ra1[32], rb0[32], rb1[32];   // two groups' 64 columns (halves 0 and 1)
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      const int mb = tile % num_m, nb = tile / num_m;
      const int64_t n_base = static_cast<int64_t>(nb) * W4_BN;
      const int64_t row = static_cast<int64_t>(mb) * W4_BM + q * 32 + lane;
      const bool row_ok = row < M;
      unsigned long long acc[32];   // 64 fp32 sums as pairs
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] = 0ull;
      // acc[16h..16h+15] += s_w[., g] * float(C_g) for half h of the warp's columns
      auto promote = [&](int g, int h, const uint32_t (&r)[32]) {
        const float2* sw = reinterpret_cast<const float2*>(s_win + (g % W4_SWIN) * W4_BN + c0 + 32 * h);
        // int32 -> fp32: |C| < 2^22, so C + 1.5*2^23 is exact as a float and subtracting gives C
        const unsigned long long magic = f32x2_of(__float_as_uint(-12582912.0f), __float_as_uint(-12582912.0f));
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const unsigned long long c =
              add_f32x2(f32x2_of(static_cast<uint32_t>(static_cast<int32_t>(r[2 * j]) + 0x4B400000),
                                 static_cast<uint32_t>(static_cast<int32_t>(r[2 * j + 1]) + 0x4B400000)),
                        magic);
          const float2 s2 = sw[j];
          acc[16 * h + j] = fma_f32x2(f32x2_of(__float_as_uint(s2.x), __float_as_uint(s2.y)), c, acc[16 * h + j]);
        }
        if (p.dbg != nullptr && g == p.dbg_group && row_ok) {
          for (int j = 0; j < 32; ++j) {
            const int64_t n = n_base + c0 + 32 * h + j;
            if (n < N) p.dbg[row * N + n] = static_cast<int32_t>(r[j]);
          }
        }
      };
      // Groups alternate between register sets a and b: group g+1's loads are
      // issued right after group g's have landed and fly while g is promoted
      // (tcgen05.wait::ld waits for all of a thread's loads, so the overlap is
      // one group deep). An accumulator goes back to the MMA once it is read.
      auto fetch = [&](uint32_t (&r0)[32], uint32_t (&r1)[32]) -> bool {
        if (!mbar_wait(&gfull_bar[buf], buf_phase, abort_flag)) return false;
        tc_fence_after();
        __syncwarp();
        tmem_ld32(taddr(buf, 0), r0);
        tmem_ld32(taddr(buf, 1), r1);
        return true;
      };
      auto landed = [&](uint32_t (&r0)[32], uint32_t (&r1)[32]) {
        __syncwarp();
        tmem_wait_regs32(r0);
        tmem_wait_regs32(r1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&gempty_bar[buf]);
        if (++buf == W4_ACC) { buf = 0; buf_phase ^= 1u; }
      };
      static_assert(W4_SWIN % 2 == 0, "scale windows start on even groups (register set a)");
      if (!fetch(ra0, ra1)) { ok = false; break; }
      for (int g = 0; g < G; g += 2) {
        if (g % W4_SWIN == 0) {
          // stage the weight scales of groups [g, g + W4_SWIN) for the tile's columns
          if (!epi_bar(promo_bar, bar_phase, abort_flag)) { ok = false; break; }
          for (int idx = pt; idx < W4_SWIN * W4_BN; idx += 32 * W4_PROMO_WARPS) {
            const int gg = idx / W4_BN, j = idx - gg * W4_BN;
            const int64_t n = n_base + j;
            s_win[idx] = (p.s_w != nullptr && n < N && g + gg < G) ? __ldg(p.s_w + n * G + g + gg) : 0.0f;
          }
          if (!epi_bar(promo_bar, bar_phase, abort_flag)) { ok = false; break; }
        }
        landed(ra0, ra1);
        if (g + 1 < G && !fetch(rb0, rb1)) { ok = false; break; }
        promote(g, 0, ra0);
        promote(g, 1, ra1);
        if (g + 1 >= G) break;
        landed(rb0, rb1);
        if (g + 2 < G && !fetch(ra0, ra1)) { ok = false; break; }
        promote(g + 1, 0, rb0);
        promote(g + 1, 1, rb1);
      }
      if (!ok) {
        tmem_ld_wait();   // no TMEM load of this warp is left in flight when the CTA winds down
        break;
      }
      if (row_ok && p.dbg == nullptr) {
        const float sx = __ldg(p.s_x + row);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int64_t n0 = n_base + c0 + 32 * h;
          if (n0 >= N) continue;
          float y[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int64_t n = n0 + j;
            const float b = (p.bias != nullptr && n < N) ? to_f<TOut>(__ldg(p.bias + n)) : 0.0f;
            const unsigned long long a2 = acc[16 * h + j / 2];
            const float a = __uint_as_float(static_cast<uint32_t>((j & 1) ? (a2 >> 32) : a2));
            y[j] = sx * a + b;
          }
          uint16_t* yp = reinterpret_cast<uint16_t*>(p.Y) + row * N + n0;
          if (n0 + 32 <= N && (N & 7) == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint4 v;
              v.x = pack2<TOut>(y[8 * i + 0], y[8 * i + 1]);
              v.y = pack2<TOut>(y[8 * i + 2], y[8 * i + 3]);
              v.z = pack2<TOut>(y[8 * i + 4], y[8 * i + 5]);
              v.w = pack2<TOut>(y[8 * i + 6], y[8 * i + 7]);
              reinterpret_cast<uint4*>(yp)[i] = v;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n0 + j < N) yp[j] = from_f<TOut>(y[j]);
          }
        }
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 32 * 16);
  }
}

}  // namespace qlin
