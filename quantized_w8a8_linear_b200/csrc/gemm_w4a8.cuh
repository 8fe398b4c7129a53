// gemm_w4a8.cuh -- W4A8 GEMM for sm_100a: int4 per-group weights (group 128
// along K, fp32 scales) with per-token int8 activations (Qwen-Image-fni8
// page, "Format"):
//
//   C_g[i,j] = sum_{k in group g} Xq[i,k] * Wq4[j,k]          (int32, exact)
//   Y[i,j]   = dtype( s_x[i] * sum_g s_w[j,g] * C_g[i,j] + bias[j] )
//
// Roles (one CTA per SM, 20 warps, persistent over tiles of 256 tokens x 128
// output columns):
//   warp 0       TMA producer: the int8 activation tile (256 x 128 B) and the
//                packed int4 weight tile (128 rows x 64 B) of one group per
//                stage;
//   warp 1       MMA issuer: TMEM holds two 256-column int32 group
//                accumulators; each group is 4 x tcgen05.mma kind::i8
//                (M = 128, N = 256, K = 32) into a fresh accumulator. The MMA
//                computes the transposed tile
//                C_g^T = Wq4 Xq^T (the unpacked weight tile is the A operand):
//                TMEM lane = output column j, TMEM column = token i, so a
//                thread of the promotion holds one output column and needs one
//                weight scale per group;
//   warps 2-3    converters: unpack the int4 weight tile to int8 in the
//                128-byte swizzled K-major layout the MMA reads (the same
//                layout TMA writes), into one of three unpacked tiles (a ring
//                of its own, so a TMA stage holds only what TMA writes), then
//                hand it to the MMA; one unpacked tile serves 256 tokens;
//   warps 4-19   promotion + epilogue, four warps per 32-lane TMEM quarter
//                (32 output columns), each with 64 tokens: per group, int32 ->
//                fp32 and sum += s_w[j,g] * C_g in registers (packed f32x2
//                arithmetic, one scale per thread); after the last group,
//                y = s_x[i] * sum + bias[j] -> Y.
//
// The weights reach the MMA as 16 t (unpacking is two masks and a shift per
// word, see unpack_int4x32), so the MMA computes 16 C_g, exactly.
// int32 -> fp32: the promotion adds the bits 0x4B400000 (1.5 * 2^23 as an
// fp32) to each accumulator word. |16 C_g| <= 16*128*127*7 < 2^21, so the sum
// read as an fp32 f is exactly 1.5 * 2^23 + 16 C_g, and one packed fma
// f * 2^-4 - 1.5 * 2^19 gives C_g exactly (the product is exact and so is the
// integer difference). An accumulator goes back to the MMA as soon as its
// last chunk is in registers, before that chunk is promoted.
// All waits are bounded (common.cuh).
#pragma once
#include "common.cuh"

namespace qlin {

constexpr int W4_BM = 256, W4_BN = 128, W4_G = 128;   // tokens per tile, output columns per tile, group (= K per stage)
constexpr int W4_STAGES = 4;                          // TMA stages: activations + packed weights
constexpr int W4_URING = 3;                           // unpacked weight tiles (converter -> MMA)
constexpr int W4_CONV_WARPS = 2, W4_PROMO_WARPS = 16;
constexpr int W4_PT = W4_BM / 4;                      // tokens per promotion warp
constexpr int W4_THREADS = 640;   // 20 warps: 5 warpgroups (see the role list above)
constexpr int W4_ACC = 2;                             // TMEM group accumulators (2 x 256 columns)
constexpr int W4_SWIN = 32;                           // groups per staged window of weight scales
constexpr uint32_t W4_SEED = 0x4B400000u;             // fp32 bits of 1.5 * 2^23, added to each accumulator word
// Register split (setmaxnreg): warpgroup 0 (producer, MMA, converters) drops
// to W4_REGS_LOW, the promotion warpgroups 1-4 rise to W4_REGS_HIGH. It fits
// the block's pool when 128 (R - LOW) >= 512 (HIGH - R) for the launch count R.
constexpr int W4_REGS_LOW = 32;
constexpr int W4_REGS_HIGH = 112;
constexpr int W4_REGS_MIN_LAUNCH = 96;
static_assert(128 * (W4_REGS_MIN_LAUNCH - W4_REGS_LOW) >= 512 * (W4_REGS_HIGH - W4_REGS_MIN_LAUNCH),
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
  static constexpr int A_BYTES = W4_BM * W4_G;            // 32 KB int8
  static constexpr int BP_BYTES = W4_BN * W4_G / 2;       // 8 KB packed int4
  static constexpr int BU_BYTES = W4_BN * W4_G;           // 16 KB unpacked int8 (swizzled)
  static constexpr int STAGE_BYTES = A_BYTES + BP_BYTES;   // one TMA stage
  static constexpr int SW_BYTES = 4 * W4_SWIN * W4_BN;    // 16 KB weight-scale window
  static constexpr int SX_BYTES = 4 * W4_BM;              // the tile's token scales
  static constexpr int BAR_BYTES = 8 * (2 * W4_STAGES + 2 * W4_URING + 2 * W4_ACC + 2) + 16;
  static constexpr int TOTAL =
      1024 + W4_STAGES * STAGE_BYTES + W4_URING * BU_BYTES + SW_BYTES + SX_BYTES + BAR_BYTES;
};

// 32 int4 codes t (16 packed bytes; byte b holds element b of the block in
// its low nibble and element b + 16 in its high nibble) -> 32 int8 bytes
// holding 16 t: a nibble moved to the top half of a byte, with the low half
// cleared, is the int8 16 t (its sign bit is the byte's). Elements 0..15 go to
// lo16, 16..31 to hi16.
__device__ __forceinline__ void unpack_int4x32(const uint4& p, uint4& lo16, uint4& hi16) {
  lo16 = make_uint4((p.x << 4) & 0xF0F0F0F0u, (p.y << 4) & 0xF0F0F0F0u, (p.z << 4) & 0xF0F0F0F0u,
                    (p.w << 4) & 0xF0F0F0F0u);
  hi16 = make_uint4(p.x & 0xF0F0F0F0u, p.y & 0xF0F0F0F0u, p.z & 0xF0F0F0F0u, p.w & 0xF0F0F0F0u);
}

// 32 lanes x 8 consecutive 32-bit columns into registers, and the wait naming them
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait8(uint32_t (&r)[8]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7])
               :
               : "memory");
}

// fma.rn.f32x2 on the pair {lo, hi} built inside the instruction's own asm
// block (a register-pair move), and the two halves of a pair read back the
// same way.
__device__ __forceinline__ unsigned long long fma2_pk(uint32_t lo, uint32_t hi, unsigned long long b,
                                                      unsigned long long c) {
  unsigned long long d;
  asm("{\n\t.reg .b64 t;\n\tmov.b64 t, {%1, %2};\n\tfma.rn.f32x2 %0, t, %3, %4;\n\t}"
      : "=l"(d)
      : "r"(lo), "r"(hi), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ void split2(unsigned long long v, float& lo, float& hi) {
  uint32_t a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(a), "=r"(b) : "l"(v));
  lo = __uint_as_float(a);
  hi = __uint_as_float(b);
}

// DBG: parity export (int32 partials of group p.dbg_group into p.dbg, no Y)
template <typename TOut, bool DBG>
__global__ void __launch_bounds__(W4_THREADS, 1)
    k_gemm_w4a8(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const W4Params p) {
  using L = W4Smem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // TMA stage s: [activations 32 KB | packed weights 8 KB]; then the ring of
  // unpacked weight tiles, 16 KB each (all 1024-aligned)
  auto sA = [&](int s) { return smem + s * L::STAGE_BYTES; };
  auto sBp = [&](int s) { return smem + s * L::STAGE_BYTES + L::A_BYTES; };
  auto sBu = [&](int u) { return smem + W4_STAGES * L::STAGE_BYTES + u * L::BU_BYTES; };
  uint8_t* tail = smem + W4_STAGES * L::STAGE_BYTES + W4_URING * L::BU_BYTES;
  float* s_win = reinterpret_cast<float*>(tail);   // [W4_SWIN][W4_BN]
  float* s_xt = s_win + W4_SWIN * W4_BN;           // [W4_BM]
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(tail + L::SW_BYTES + L::SX_BYTES);
  uint64_t* empty_bar = full_bar + W4_STAGES;
  uint64_t* ufull_bar = empty_bar + W4_STAGES;     // unpacked tile u written (converters)
  uint64_t* uempty_bar = ufull_bar + W4_URING;     // unpacked tile u read (MMA commit)
  uint64_t* gfull_bar = uempty_bar + W4_URING;
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
      mbar_init(&empty_bar[s], 1);
    }
    for (int u = 0; u < W4_URING; ++u) {
      mbar_init(&ufull_bar[u], W4_CONV_WARPS);
      mbar_init(&uempty_bar[u], 1);
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

  if (warp < 4) {
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
      constexpr uint32_t idesc = idesc_i8(W4_BN, W4_BM);   // M = output columns, N = tokens
      int stage = 0, u = 0;
      uint32_t phase = 0, uphase = 0;
      int buf = 0;
      uint32_t buf_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        for (int g = 0; g < G; ++g) {
          // the u-th use of an accumulator waits for its u-th release (the first is at start-up)
          if (!mbar_wait(&gempty_bar[buf], buf_phase, abort_flag)) { ok = false; break; }
          if (!mbar_wait(&full_bar[stage], phase, abort_flag)) { ok = false; break; }
          if (!mbar_wait(&ufull_bar[u], uphase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * W4_BM);
          // A = the unpacked weight tile (rows j), B = the activation tile (rows i)
          const uint64_t adesc = sdesc_k128(smem_u32(sBu(u)));
          const uint64_t bdesc = sdesc_k128(smem_u32(sA(stage)));
#pragma unroll
          for (int k = 0; k < W4_G / 32; ++k) umma<0>(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc, k != 0 ? 1u : 0u);
          umma_commit(&empty_bar[stage]);
          umma_commit(&uempty_bar[u]);
          umma_commit(&gfull_bar[buf]);
          if (++stage == W4_STAGES) { stage = 0; phase ^= 1u; }
          if (++u == W4_URING) { u = 0; uphase ^= 1u; }
          if (++buf == W4_ACC) { buf = 0; buf_phase ^= 1u; }
        }
      }
      umma_commit(drain_bar);
      const uint32_t a = smem_u32(drain_bar);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(a, 0) && globaltimer() - t0 < drain_limit_ns()) {}
    }
  } else {
    // ---------------- converters: packed int4 -> swizzled int8 ----------------
    const int ct = threadIdx.x - 64;   // 0..63
    int stage = 0, u = 0;
    uint32_t phase = 0, uphase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      bool ok = true;
      for (int g = 0; g < G; ++g) {
        if (!mbar_wait(&full_bar[stage], phase, abort_flag)) { ok = false; break; }
        if (!mbar_wait(&uempty_bar[u], uphase ^ 1u, abort_flag)) { ok = false; break; }
        const uint4* src = reinterpret_cast<const uint4*>(sBp(stage));
        uint8_t* dst = sBu(u);
#pragma unroll 2
        for (int c = ct; c < L::BP_BYTES / 16; c += 32 * W4_CONV_WARPS) {   // 16-byte chunk c of the packed tile
          const int r = c >> 2, part = c & 3;          // row, quarter of the row's 64 packed bytes
          uint4 lo, hi;
          unpack_int4x32(src[c], lo, hi);
          // row r's 128 int8 bytes: 16-byte chunk ch lives at chunk (ch ^ (r & 7)) of the row
          *reinterpret_cast<uint4*>(dst + r * 128 + (((2 * part) ^ (r & 7)) << 4)) = lo;
          *reinterpret_cast<uint4*>(dst + r * 128 + (((2 * part + 1) ^ (r & 7)) << 4)) = hi;
        }
        fence_proxy_async_smem();   // generic writes -> read by the tensor core (async proxy)
        __syncwarp();
        if (lane == 0) mbar_arrive(&ufull_bar[u]);
        if (++stage == W4_STAGES) { stage = 0; phase ^= 1u; }
        if (++u == W4_URING) { u = 0; uphase ^= 1u; }
      }
      if (!ok) break;
    }
  }
  } else {
    setmaxnreg_inc<W4_REGS_HIGH>();
    // ---------------- promotion + epilogue ----------------
    const int pw = warp - 4;                     // 0..15
    const int q = warp & 3;                      // TMEM lane quarter: output columns 32q..32q+31 of the tile
    const int c0 = (pw >> 2) * W4_PT;            // this warp's first token (TMEM column) of the tile
    const int pt = threadIdx.x - 128;            // 0..511
    const int jl = q * 32 + lane;                // this thread's output column within the tile
    int buf = 0;
    uint32_t buf_phase = 0, bar_phase = 0;
    bool ok = true;
    // TMEM address of this warp's lane quarter, tokens c0 + 8k of accumulator buffer b
    const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(c0);
    auto taddr = [&](int b, int k) { return tq + static_cast<uint32_t>(b * W4_BM + 8 * k); };
    constexpr int NCH = W4_PT / 8;   // 8-token chunks per warp and group
    uint32_t ra[8], rb[8];           // chunks of the warp's share of one group, alternating
    // hand accumulator b to the MMA: this warp's reads of it have completed
    auto release = [&](int b) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&gempty_bar[b]);
    };
    for (int b = 0; b < W4_ACC; ++b) release(b);
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      const int mb = tile % num_m, nb = tile / num_m;
      const int64_t m_base = static_cast<int64_t>(mb) * W4_BM;
      const int64_t n = static_cast<int64_t>(nb) * W4_BN + jl;   // this thread's output column
      const bool n_ok = n < N;
      unsigned long long acc[W4_PT / 2];   // 64 fp32 sums (tokens c0..c0+63) as pairs
#pragma unroll
      for (int j = 0; j < W4_PT / 2; ++j) acc[j] = 0ull;
      // acc[4k..4k+3] += s * C_g for the warp's 8-token chunk k, s = s_w[n, g];
      // r holds the int32 words 16 C_g
      auto promote = [&](int g, int k, const uint32_t (&r)[8], unsigned long long s2) {
        const unsigned long long sixteenth = f32x2_of(0x3D800000u, 0x3D800000u);   // 2^-4
        const unsigned long long neg_base = f32x2_of(0xC9400000u, 0xC9400000u);    // -1.5 * 2^19
#pragma unroll
        for (int j = 0; j < 4; ++j)
          acc[4 * k + j] =
              fma_f32x2(s2, fma2_pk(r[2 * j] + W4_SEED, r[2 * j + 1] + W4_SEED, sixteenth, neg_base), acc[4 * k + j]);
        if constexpr (DBG) {
          if (g == p.dbg_group && n_ok) {
            for (int j = 0; j < 8; ++j) {
              const int64_t i = m_base + c0 + 8 * k + j;
              if (i < M) p.dbg[i * N + n] = static_cast<int32_t>(r[j]) >> 4;
            }
          }
        }
      };
      // wait until the MMA has finished accumulator `buf`, then start reading chunk 0 of it
      auto fetch = [&](uint32_t (&r)[8]) -> bool {
        if (!mbar_wait(&gfull_bar[buf], buf_phase, abort_flag)) return false;
        tc_fence_after();
        __syncwarp();
        tmem_ld8(taddr(buf, 0), r);
        return true;
      };
      // One TMEM load is always in flight while the previous chunk is promoted
      // (tcgen05.wait::ld waits for all of a thread's loads); the last chunk
      // of group g overlaps the first load of group g+1. An accumulator goes
      // back to the MMA once its last chunk is in registers.
      if (!fetch(ra)) { ok = false; break; }
      for (int g = 0; g < G; ++g) {
        if (g % W4_SWIN == 0) {
          // stage the weight scales of groups [g, g + W4_SWIN) for the tile's
          // columns (and, with the first window, the tile's token scales)
          if (!epi_bar(promo_bar, bar_phase, abort_flag)) { ok = false; break; }
          for (int idx = pt; idx < W4_SWIN * W4_BN; idx += 32 * W4_PROMO_WARPS) {
            const int gg = idx / W4_BN, j = idx - gg * W4_BN;
            const int64_t nn = static_cast<int64_t>(nb) * W4_BN + j;
            s_win[idx] = (p.s_w != nullptr && nn < N && g + gg < G) ? __ldg(p.s_w + nn * G + g + gg) : 0.0f;
          }
          if (g == 0 && pt < W4_BM)
            s_xt[pt] = (p.s_x != nullptr && m_base + pt < M) ? __ldg(p.s_x + m_base + pt) : 0.0f;
          if (!epi_bar(promo_bar, bar_phase, abort_flag)) { ok = false; break; }
        }
        const float sw = s_win[(g % W4_SWIN) * W4_BN + jl];
        const unsigned long long s2 = f32x2_of(__float_as_uint(sw), __float_as_uint(sw));
#pragma unroll
        for (int k = 0; k < NCH - 2; k += 2) {
          tmem_wait8(ra);
          tmem_ld8(taddr(buf, k + 1), rb);
          promote(g, k, ra, s2);
          tmem_wait8(rb);
          tmem_ld8(taddr(buf, k + 2), ra);
          promote(g, k + 1, rb, s2);
        }
        tmem_wait8(ra);
        tmem_ld8(taddr(buf, NCH - 1), rb);
        promote(g, NCH - 2, ra, s2);
        tmem_wait8(rb);
        release(buf);
        if (++buf == W4_ACC) { buf = 0; buf_phase ^= 1u; }
        if (g + 1 < G && !fetch(ra)) { ok = false; break; }
        promote(g, NCH - 1, rb, s2);
      }
      if (!ok) {
        // no TMEM load of this warp is left in flight when the CTA winds down
        tmem_ld_wait();
        break;
      }
      if (!DBG && n_ok) {
        const float bn = p.bias != nullptr ? to_f<TOut>(__ldg(p.bias + n)) : 0.0f;
        uint16_t* yp = reinterpret_cast<uint16_t*>(p.Y) + n;
#pragma unroll
        for (int k = 0; k < W4_PT / 16; ++k) {
          const float4* sx4 = reinterpret_cast<const float4*>(s_xt + c0 + 16 * k);
#pragma unroll
          for (int j4 = 0; j4 < 4; ++j4) {
            const float4 sx = sx4[j4];
            const float xs[4] = {sx.x, sx.y, sx.z, sx.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int jj = 4 * j4 + e;   // token c0 + 16k + jj is pair (16k + jj) / 2 of acc
              const int64_t i = m_base + c0 + 16 * k + jj;
              float alo, ahi;
              split2(acc[8 * k + jj / 2], alo, ahi);
              const float a = (jj & 1) ? ahi : alo;
              if (i < M) yp[i * N] = from_f<TOut>(xs[e] * a + bn);
            }
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
