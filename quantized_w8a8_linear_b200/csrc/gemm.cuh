// gemm.cuh -- persistent, warp-specialised tcgen05 GEMM for sm_100a.
//
//   C[M,N] = A[M,K] B[N,K]^T, A and B 8-bit (int8 -> int32 with kind::i8, or
//   E4M3 -> fp32 with kind::f8f6f4) or 16-bit (bf16 or fp16 -> fp32 with
//   kind::f16), both K-major in global memory. Tiles are addressed in bytes:
//   a stage holds 128 bytes of K (128 8-bit or 64 16-bit elements), and every
//   MMA takes 32 bytes of K, so the pipeline is the same for all three kinds.
//
// Roles (one CTA per SM, 20 warps = 5 warpgroups; the last gives most of its
// registers to the first four with setmaxnreg):
//   warp 16     TMA producer: 128x128-byte A tiles and BNx128-byte B tiles,
//               128B-swizzled, into a STAGES-deep shared-memory ring;
//   warp 17     MMA issuer: allocates all 512 TMEM columns (two BN-column
//               accumulators), issues 4 UMMAs (K = 32 each) per stage and
//               commits stage release / accumulator-ready to mbarriers;
//   warps 18-19 idle;
//   warps 0-15  epilogue, four groups of four warps; group g takes columns
//               [g*BN/4, (g+1)*BN/4) of every tile, so four warps share each
//               TMEM lane quarter and hide each other's latencies (the
//               epilogue is latency-bound: shared-memory broadcasts, packed
//               fp32 chains, tcgen05.ld and the Y stores). Each warp
//               reads its 32-lane quarter with tcgen05.ld (the next chunk in
//               flight while the current one is processed) and does the fused
//               dequant (row x column scales), for LLM.int8 the exact
//               removal of the outlier columns' int8 products and the
//               floating-point outlier part as a rank-|O| update, the bias,
//               rounding and the store of Y. With two accumulators the
//               epilogue of tile t overlaps the main loop of tile t+1.
// Tiles are handed out round-robin (tile = blockIdx.x + i * gridDim.x) in
// bands of group_m m-blocks, M fastest within a band, so that the CTAs running
// together share few A and B tiles in L2 (or under stream-K, below).
// Out-of-range rows and K columns are zero-filled by TMA; stores are
// predicated on M and N.
#pragma once
#include <type_traits>

#include "common.cuh"

namespace qlin {

// EPI_INT8_OUTLIER_I32: the int32 accumulator of the LLM.int8 path after the
// outlier-column correction, written out (parity export of the same kernel).
// EPI_F16: Y = dtype(acc + bias), the unquantised 16-bit linear (kind::f16).
enum EpiKind { EPI_I32 = 0, EPI_INT8_OUTLIER = 1, EPI_FP8_TENSOR = 2, EPI_FP8_ROWCOL = 3, EPI_INT8_OUTLIER_I32 = 4,
               EPI_F16 = 5 };

constexpr int GEMM_BM = 128;
constexpr int GEMM_BK = 128;                 // bytes (= elements) per stage along K
constexpr int GEMM_EPI_WARPS = 4;            // per group: one per TMEM lane quarter
constexpr int GEMM_EPI_GROUPS = 4;           // column quarters of every accumulator tile
constexpr int GEMM_EPI_THREADS = 32 * GEMM_EPI_WARPS;
constexpr int GEMM_EPI_ALL = GEMM_EPI_WARPS * GEMM_EPI_GROUPS;   // warps 0..15
constexpr int GEMM_WARP_TMA = GEMM_EPI_ALL;
constexpr int GEMM_WARP_MMA = GEMM_EPI_ALL + 1;
constexpr int GEMM_THREADS = 32 * (GEMM_EPI_ALL + 4);
// Register split (setmaxnreg): the launch gives every thread the kernel's
// register count R (96 for 640 threads); the producer warpgroup drops to
// GEMM_REGS_LOW and the four epilogue warpgroups rise to GEMM_REGS_HIGH. That
// fits the block's pool when 128 (R - LOW) >= 512 (HIGH - R), i.e.
// R >= GEMM_REGS_MIN_LAUNCH; the launch checks R against it.
constexpr int GEMM_REGS_LOW = 56;
constexpr int GEMM_REGS_HIGH = 104;
constexpr int GEMM_REGS_MIN_LAUNCH = 95;
static_assert(128 * (GEMM_REGS_MIN_LAUNCH - GEMM_REGS_LOW) >=
                  32 * GEMM_EPI_ALL * (GEMM_REGS_HIGH - GEMM_REGS_MIN_LAUNCH),
              "register split must fit the launch pool");
constexpr int GEMM_CW = 16;                  // accumulator columns per tcgen05.ld in the epilogue
constexpr int GEMM_OUTL_STAGED = 16;         // outlier counts up to this take the staged fp part in the epilogue
constexpr int GEMM_CORR_K = 32;              // outlier counts up to this take their int8 products out with one MMA
// Stream-K (kind::i8 and kind::f8f6f4, 128 x 256 tiles): at most this many CTAs (partial slots
// in the workspace: two per CTA), each with at least GEMM_SK_MIN_ITERS k-blocks
// unless forced. A cut tile costs its parties about GEMM_SK_COST_KB k-blocks of
// main loop (measured: 4 us to write a partial and fence it, 3 us to add one),
// and the CTAs' k offsets drift apart, so fewer A and B tiles are shared in
// L2; the automatic choice takes stream-K only for a gain of 5% or more.
constexpr int GEMM_SK_MAX_CTAS = 160;
constexpr int GEMM_SK_BN = 256;
constexpr int GEMM_SK_MIN_ITERS = 8;
constexpr int GEMM_SK_COST_KB = 24;
// The LLM.int8 epilogue of a 128 x 256 tile takes about as long as this many
// k-blocks of its main loop (measured: 18K cycles against 0.7K per k-block).
constexpr int GEMM_EPI_KB = 26;
// Tile bands (tile_mn): 16 m-blocks, so 148 tiles in flight share 16 A tiles
// and about 9 B tiles.
constexpr int GEMM_GROUP_M = 16;

struct EpiParams {
  int64_t M, N, K;            // K: bytes of a row of A and of B (elements for 8-bit operands)
  void* Y;                    // [M,N]: int32 (EPI_I32, EPI_INT8_OUTLIER_I32) or 16-bit output dtype
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
  // LLM.int8: the A operand may hold non-zero codes in outlier columns, whose
  // exact int32 contribution sum_o Xq[m,O[o]] * Wq[n,O[o]] leaves the
  // accumulator: for counts up to GEMM_CORR_K by one more MMA per tile over
  // the compact copies -Xq[:,O] and Wq[:,O] (the kernel's tmXc / tmWc tensor
  // maps, [M,32] and [N,32], zero-padded); for larger counts in the epilogue,
  // gathered from Xq / Wq through O.
  const int8_t* Xq;           // [M,K]
  const int8_t* Wq;           // [N,K]
  const int32_t* O;           // [K] ascending outlier columns, first *count valid
  const int8_t* XqO;          // [M,32] -Xq[:,O] (host side: source of tmXc)
  const int8_t* WqO;          // [N,32] Wq[:,O] (host side: source of tmWc)
  // 16-bit Y written through the kernel's Y tensor map (TMA stores of 32-row x
  // 16-column boxes from shared memory) instead of per-thread stores
  int tma_y;
  // Stream-K schedule (kind::i8 only): the T = tiles x k-blocks iterations are
  // cut into gridDim.x equal contiguous ranges, one per CTA, so that no SM
  // idles through a partial last wave. A tile cut between CTAs is finished by
  // exactly one of them from the others' int32 partial accumulators (exact).
  int sk;
  int sk_dp_tiles;     // tiles [0, sk_dp_tiles) go whole and round-robin; stream-K covers the rest
  int32_t* sk_count;   // [tiles][GEMM_EPI_GROUPS] arrival counters: zero on entry, left zero
  int32_t* sk_part;    // [2 * gridDim.x][BN/4][128][4] int32 partial accumulators
  // Tile order: tile t lies in band t / (group_m * num_n) of group_m m-blocks
  // (the last band may be narrower), m fastest within the band; so the tiles
  // in flight together share few A and B tiles. 0: one band of all m-blocks.
  int group_m;
};

__device__ __forceinline__ void tile_mn(int t, int num_m, int num_n, int group_m, int& mb, int& nb) {
  const int gm = group_m > 0 && group_m < num_m ? group_m : num_m;
  const int band = t / (gm * num_n);
  const int m0 = band * gm;
  const int h = num_m - m0 < gm ? num_m - m0 : gm;   // m-blocks in this band
  const int r = t - band * gm * num_n;
  mb = m0 + r % h;
  nb = r / h;
}

// One CTA's share of the work as segments (tile, k-blocks [kb0, kb1)): whole
// tiles round-robin; under stream-K only the tiles below sk_dp_tiles (whole
// waves), then, of the T = (tiles - sk_dp_tiles) x KB iterations of the
// remaining tiles, [b T / G, (b+1) T / G) (b = blockIdx.x, G = gridDim.x) cut
// at tile boundaries. Such a range may start with the tail of a tile that an
// earlier CTA began (a contributor segment) and end with the head of a tile
// (kb0 = 0, the owner segment); tiles in between are whole.
struct Seg {
  int tile, kb0, kb1;
};
__device__ __forceinline__ int64_t sk_begin(int b, int G, int64_t T) { return static_cast<int64_t>(b) * T / G; }
struct SegIter {
  int64_t pos, end;
  int tile, dp_end, KB;
  int head_kb1;   // > 0: the range's cut last tile, taken first (k-blocks [0, head_kb1))
  bool sk;
  __device__ __forceinline__ SegIter(bool sk_, int num_tiles, int dp_tiles, int KB_)
      : tile(static_cast<int>(blockIdx.x)), dp_end(sk_ ? dp_tiles : num_tiles), KB(KB_), head_kb1(0), sk(sk_) {
    const int64_t base = static_cast<int64_t>(dp_end) * KB_;
    const int64_t T = static_cast<int64_t>(num_tiles) * KB_ - base;
    pos = sk_ ? base + sk_begin(blockIdx.x, gridDim.x, T) : 0;
    end = sk_ ? base + sk_begin(blockIdx.x + 1, gridDim.x, T) : 0;
    if (sk_) {
      // A cut head goes before the rest of the range, so that the epilogues
      // of both cut tiles overlap the main loop of whole ones (a short head
      // last would queue its epilogue behind the previous tile's).
      const int64_t last0 = (end - 1) / KB_ * KB_;   // first iteration of the range's last tile
      if (end - last0 < KB_ && last0 > pos) {
        head_kb1 = static_cast<int>(end - last0);
        end = last0;
      }
    }
  }
  __device__ __forceinline__ bool next(Seg& s) {
    if (tile < dp_end) {
      s.tile = tile;
      s.kb0 = 0;
      s.kb1 = KB;
      tile += gridDim.x;
      return true;
    }
    if (!sk) return false;
    if (head_kb1 > 0) {
      s.tile = static_cast<int>(end / KB);
      s.kb0 = 0;
      s.kb1 = head_kb1;
      head_kb1 = 0;
      return true;
    }
    if (pos >= end) return false;
    s.tile = static_cast<int>(pos / KB);
    s.kb0 = static_cast<int>(pos - static_cast<int64_t>(s.tile) * KB);
    const int64_t left = end - pos;
    s.kb1 = left < KB - s.kb0 ? s.kb0 + static_cast<int>(left) : KB;
    pos += s.kb1 - s.kb0;
    return true;
  }
};
// The CTAs that hold parts of a cut tile: the owner ob (its range holds the
// tile's first iteration) and the contributors ob+1 .. ob+nc (their ranges
// start inside the tile). Their partial slots: 2c for contributor c, 2ob+1
// for the owner.
__device__ __forceinline__ void sk_parties(int tile, int KB, int num_tiles, int dp_tiles, int& ob, int& nc) {
  const int G = gridDim.x;
  const int64_t T = static_cast<int64_t>(num_tiles - dp_tiles) * KB;
  const int64_t x0 = static_cast<int64_t>(tile - dp_tiles) * KB, x1 = x0 + KB;
  int b = static_cast<int>(x0 * G / T);
  if (b > G - 1) b = G - 1;
  while (b > 0 && sk_begin(b, G, T) > x0) --b;
  while (b + 1 < G && sk_begin(b + 1, G, T) <= x0) ++b;
  ob = b;
  int c = b + 1;
  while (c < G && sk_begin(c, G, T) < x1) ++c;
  nc = c - b - 1;
}

// Partial-slot traffic of an epilogue group: its BNG columns of one TMEM
// accumulator, 64 columns (4 tcgen05.ld of 16) at a time. Slot layout
// [BN/4 column quads][128 rows] of int4: thread `row` moves its row's quads
// and every warp-wide 16-byte access covers 512 contiguous bytes.
template <int BN, int BNG>
__device__ __forceinline__ void sk_store_partial(int32_t* slot, uint32_t t_row, int g, int row_in_tile) {
  constexpr int NCH = BNG / GEMM_CW;
  static_assert(NCH % 4 == 0, "partials move in groups of four chunks");
  int4* dst = reinterpret_cast<int4*>(slot) + static_cast<int64_t>(g * NCH) * 4 * GEMM_BM + row_in_tile;
#pragma unroll 1
  for (int c0 = 0; c0 < NCH; c0 += 4) {
    uint32_t r[4][GEMM_CW];
#pragma unroll
    for (int i = 0; i < 4; ++i) tmem_ld16(t_row + static_cast<uint32_t>((c0 + i) * GEMM_CW), r[i]);
#pragma unroll
    for (int i = 0; i < 4; ++i) tmem_wait16(r[i]);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int v = 0; v < 4; ++v)
        __stcg(dst + static_cast<int64_t>((c0 + i) * 4 + v) * GEMM_BM,
               make_int4(r[i][4 * v], r[i][4 * v + 1], r[i][4 * v + 2], r[i][4 * v + 3]));
  }
}
// Adds the other parties' partial slots to the group's columns of the TMEM
// accumulator. Parties q = 0..nc: the owner ob (q = 0, slot 2ob+1) and the
// contributors ob+q (slot 2(ob+q)); self_q is this CTA's own party, whose
// part is already in TMEM. int32 (FP false) is exact in any order. fp32 (FP
// true) is summed in party order, p_0 + p_1 + ... + p_nc with this CTA's own
// part taken from TMEM at its place, so the result does not depend on which
// party finishes the tile.
template <int BN, int BNG, bool FP>
__device__ __forceinline__ void sk_add_partials(const int32_t* part, int ob, int nc, int self_q, uint32_t t_row,
                                                int g, int row_in_tile) {
  constexpr int NCH = BNG / GEMM_CW;
  constexpr int64_t SLOT_V4 = static_cast<int64_t>(GEMM_BM) * BN / 4;
  const int4* src0 = reinterpret_cast<const int4*>(part) + static_cast<int64_t>(g * NCH) * 4 * GEMM_BM + row_in_tile;
  if constexpr (FP) {
#pragma unroll 1
    for (int c = 0; c < NCH; ++c) {   // one 16-column chunk at a time
      uint32_t own[GEMM_CW];
      float sum[GEMM_CW];
      tmem_ld16(t_row + static_cast<uint32_t>(c * GEMM_CW), own);
      tmem_wait16(own);
#pragma unroll 1
      for (int q = 0; q <= nc; ++q) {
        float v[GEMM_CW];
        if (q == self_q) {
#pragma unroll
          for (int e = 0; e < GEMM_CW; ++e) v[e] = __uint_as_float(own[e]);
        } else {
          const int slot = q == 0 ? 2 * ob + 1 : 2 * (ob + q);
          const int4* src = src0 + slot * SLOT_V4 + static_cast<int64_t>(c) * 4 * GEMM_BM;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int4 w = __ldcg(src + static_cast<int64_t>(j) * GEMM_BM);
            v[4 * j] = __int_as_float(w.x);
            v[4 * j + 1] = __int_as_float(w.y);
            v[4 * j + 2] = __int_as_float(w.z);
            v[4 * j + 3] = __int_as_float(w.w);
          }
        }
#pragma unroll
        for (int e = 0; e < GEMM_CW; ++e) sum[e] = q == 0 ? v[e] : __fadd_rn(sum[e], v[e]);
      }
      uint32_t out[GEMM_CW];
#pragma unroll
      for (int e = 0; e < GEMM_CW; ++e) out[e] = __float_as_uint(sum[e]);
      tmem_st16(t_row + static_cast<uint32_t>(c * GEMM_CW), out);
    }
    tmem_st_wait();
    return;
  }
#pragma unroll 1
  for (int c0 = 0; c0 < NCH; c0 += 4) {
    uint32_t r[4][GEMM_CW];
#pragma unroll
    for (int i = 0; i < 4; ++i) tmem_ld16(t_row + static_cast<uint32_t>((c0 + i) * GEMM_CW), r[i]);
    bool waited = false;
#pragma unroll 1
    for (int q = 0; q <= nc; ++q) {
      if (q == self_q) continue;
      const int slot = q == 0 ? 2 * ob + 1 : 2 * (ob + q);
      const int4* src = src0 + slot * SLOT_V4 + static_cast<int64_t>(c0) * 4 * GEMM_BM;
      int4 v[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) v[i][j] = __ldcg(src + static_cast<int64_t>(i * 4 + j) * GEMM_BM);
      if (!waited) {
#pragma unroll
        for (int i = 0; i < 4; ++i) tmem_wait16(r[i]);
        waited = true;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          r[i][4 * j] += static_cast<uint32_t>(v[i][j].x);
          r[i][4 * j + 1] += static_cast<uint32_t>(v[i][j].y);
          r[i][4 * j + 2] += static_cast<uint32_t>(v[i][j].z);
          r[i][4 * j + 3] += static_cast<uint32_t>(v[i][j].w);
        }
    }
    if (!waited)
#pragma unroll
      for (int i = 0; i < 4; ++i) tmem_wait16(r[i]);
#pragma unroll
    for (int i = 0; i < 4; ++i) tmem_st16(t_row + static_cast<uint32_t>((c0 + i) * GEMM_CW), r[i]);
  }
  tmem_st_wait();
}

constexpr int GEMM_YBOX_BYTES = 32 * GEMM_CW * 2;   // one warp's 32 rows x 16 columns of 16-bit Y

// Per-tile column data staged in shared memory by an epilogue group, read
// with 16-byte broadcasts (all lanes of a warp read the same address, so no
// bank conflicts and few wavefronts; the tensor core reads its operands from
// the same shared memory):
//   sb[i] = {scale(2i), scale(2i+1), bias(2i), bias(2i+1)} (fp32), a column pair
//   wo[n] = {W_O[n, 0..7], W_O[n, 8..15]} (16-bit)
// Only sb is read without outliers, wo[n][0] for up to 8 outlier columns.
template <int BN>
struct EpiStage {
  float4 sb[BN / 2];
  uint4 wo[BN][2];
};


template <int BN, int STAGES>
struct GemmSmem {
  static constexpr int A_BYTES = GEMM_BM * GEMM_BK;
  static constexpr int B_BYTES = BN * GEMM_BK;
  static constexpr int TILE_BYTES = STAGES * (A_BYTES + B_BYTES);
  static constexpr int EPI_BYTES = static_cast<int>(sizeof(EpiStage<BN / GEMM_EPI_GROUPS>)) * GEMM_EPI_GROUPS;
  // Y staging for the TMA stores: one box per epilogue warp
  static constexpr int Y_BYTES = GEMM_EPI_ALL * GEMM_YBOX_BYTES;
  // full[STAGES], empty[STAGES], tfull[2], tempty[2], drain, epi[GROUPS]; tmem slot, abort flag, sk flags
  static constexpr int BAR_BYTES = 8 * (2 * STAGES + 4 + 1 + GEMM_EPI_GROUPS) + 32;
  static constexpr int TOTAL = 1024 + TILE_BYTES + EPI_BYTES + Y_BYTES + BAR_BYTES;   // 1024: alignment slack
  static_assert(TILE_BYTES % 1024 == 0 && EPI_BYTES % 1024 == 0, "the Y staging boxes stay 1024-byte aligned");
};

template <typename TOut, int EPI, int BN>
__device__ __forceinline__ void epi_stage(const EpiParams& p, EpiStage<BN>& es, int64_t n_base, int et, int cn) {
  constexpr int PER = BN >= GEMM_EPI_THREADS ? BN / GEMM_EPI_THREADS : 1;   // columns per thread
  constexpr bool OUTL = EPI == EPI_INT8_OUTLIER || EPI == EPI_INT8_OUTLIER_I32;
  float sw[PER], b[PER];
  uint4 wo0[PER], wo1[PER];
  // every load first, then every store: one memory round trip per tile
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int64_t n = n_base + et + i * GEMM_EPI_THREADS;
    const bool mine = et + i * GEMM_EPI_THREADS < BN;
    sw[i] = 0.0f;
    b[i] = 0.0f;
    wo0[i] = wo1[i] = make_uint4(0u, 0u, 0u, 0u);
    if (mine && n < p.N) {
      if constexpr (EPI == EPI_INT8_OUTLIER) sw[i] = __ldg(p.s_w + n);
      if constexpr (EPI == EPI_FP8_ROWCOL) sw[i] = to_f<__nv_bfloat16>(__ldg(p.s_w_bf16 + n));
      if constexpr (EPI == EPI_INT8_OUTLIER || EPI == EPI_FP8_TENSOR || EPI == EPI_FP8_ROWCOL || EPI == EPI_F16)
        if (p.bias != nullptr) b[i] = to_f<TOut>(__ldg(p.bias + n));
      if constexpr (OUTL) {
        if (cn > 0) {
          if constexpr (EPI == EPI_INT8_OUTLIER) {
            const uint4* w = reinterpret_cast<const uint4*>(p.W_O + n * p.ostride);
            wo0[i] = __ldg(w);
            if (cn > 8) wo1[i] = __ldg(w + 1);
          }
        }
      }
    }
  }
  float* sbf = reinterpret_cast<float*>(es.sb);
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int j = et + i * GEMM_EPI_THREADS;
    if (j >= BN) continue;
    sbf[(j >> 1) * 4 + (j & 1)] = sw[i];
    sbf[(j >> 1) * 4 + 2 + (j & 1)] = b[i];
    if constexpr (OUTL) {
      es.wo[j][0] = wo0[i];
      es.wo[j][1] = wo1[i];
    }
  }
}

// CW outputs (16-bit pairs, the lower column in the low half) to Y[row, n0..].
// v8: Y is 32-byte aligned and N a multiple of 16, so every 16-column chunk is
// one aligned 32-byte sector, written with one 256-bit store.
template <int CW>
__device__ __forceinline__ void store_chunk(const EpiParams& p, const uint32_t (&out)[CW / 2], int64_t row,
                                            int64_t n0, bool v8) {
  const int64_t N = p.N;
  uint16_t* y = reinterpret_cast<uint16_t*>(p.Y) + row * N + n0;
  if (v8 && n0 + CW <= N) {
    static_assert(CW % 16 == 0, "256-bit stores take 16 columns");
#pragma unroll
    for (int i = 0; i < CW / 16; ++i)
      asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(y + 16 * i), "r"(out[8 * i]),
                   "r"(out[8 * i + 1]), "r"(out[8 * i + 2]), "r"(out[8 * i + 3]), "r"(out[8 * i + 4]),
                   "r"(out[8 * i + 5]), "r"(out[8 * i + 6]), "r"(out[8 * i + 7])
                   : "memory");
  } else if (n0 + CW <= N && (N & 7) == 0) {
#pragma unroll
    for (int i = 0; i < CW / 8; ++i)
      reinterpret_cast<uint4*>(y)[i] = make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
  } else {
#pragma unroll
    for (int j = 0; j < CW; ++j)
      if (n0 + j < N) y[j] = static_cast<uint16_t>(out[j >> 1] >> (16 * (j & 1)));
  }
}

// CW int32 outputs to Y[row, n0..].
template <int CW>
__device__ __forceinline__ void store_chunk_i32(const EpiParams& p, const uint32_t (&r)[CW], int64_t row,
                                                int64_t n0) {
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
}

// One chunk of GEMM_CW accumulator columns of one row: r -> Y[row, n0..).
// CN: outlier columns (0, 2, 4, 8 or 16: a bucket >= the count, the staged
// operands zero-padded) or -1 (more than 16: gathered from global memory,
// correct for any count, not fast).
// 16-bit outputs are returned in `out` (the caller stores them); int32
// outputs are stored here.
template <typename TOut, int EPI, int BN, int CN, int XR, bool FTM>
__device__ __forceinline__ void epi_chunk(const EpiParams& p, const EpiStage<BN>& es, uint32_t (&r)[GEMM_CW],
                                          const uint32_t (&f)[GEMM_CW], int c, int64_t row, int64_t n_base, float sx,
                                          float alpha, int cnt, const uint32_t (&xr)[XR],
                                          uint32_t (&out)[GEMM_CW / 2]) {
  constexpr bool OUTL = EPI == EPI_INT8_OUTLIER || EPI == EPI_INT8_OUTLIER_I32;
  constexpr bool BF = std::is_same<TOut, __nv_bfloat16>::value;
  const int64_t n0 = n_base + c * GEMM_CW;
  // column pairs (j, j+1): one staged record, packed dequant arithmetic
#pragma unroll
  for (int j = 0; j < GEMM_CW; j += 2) {
    int32_t acc[2] = {static_cast<int32_t>(r[j]), static_cast<int32_t>(r[j + 1])};
    if constexpr (OUTL && CN < 0) {
      // more outlier columns than the correction MMA takes: their products
      // leave the accumulator here, exact in int32
#pragma unroll
      for (int e = 0; e < 2; ++e)
        if (cnt > GEMM_CORR_K && n0 + j + e < p.N)
          for (int o = 0; o < cnt; ++o) {
            const int k = __ldg(p.O + o);
            acc[e] -= static_cast<int32_t>(__ldg(p.Xq + row * p.K + k)) *
                      static_cast<int32_t>(__ldg(p.Wq + (n0 + j + e) * p.K + k));
          }
    }
    if constexpr (EPI == EPI_I32 || EPI == EPI_INT8_OUTLIER_I32) {
      r[j] = static_cast<uint32_t>(acc[0]);
      r[j + 1] = static_cast<uint32_t>(acc[1]);
    } else {
      const float4 sbv = es.sb[(c * GEMM_CW + j) >> 1];   // {scale j, scale j+1, bias j, bias j+1}
      const unsigned long long b2 = f32x2_of(__float_as_uint(sbv.z), __float_as_uint(sbv.w));
      unsigned long long v;
      if constexpr (EPI == EPI_FP8_TENSOR || EPI == EPI_F16) {   // alpha = 1 for EPI_F16: fma(acc, 1, b) = acc + b
        v = fma_f32x2(f32x2_of(r[j], r[j + 1]), f32x2_of(__float_as_uint(alpha), __float_as_uint(alpha)), b2);
      } else {
        // acc * (s_x * s_w) + bias, as fmaf(acc, s_x * s_w, bias) per column
        const unsigned long long s2 = mul_f32x2(f32x2_of(__float_as_uint(sx), __float_as_uint(sx)),
                                                f32x2_of(__float_as_uint(sbv.x), __float_as_uint(sbv.y)));
        const unsigned long long a2 =
            EPI == EPI_INT8_OUTLIER
                ? f32x2_of(__float_as_uint(static_cast<float>(acc[0])), __float_as_uint(static_cast<float>(acc[1])))
                : f32x2_of(r[j], r[j + 1]);
        v = fma_f32x2(a2, s2, b2);
      }
      float a0 = lo_f(v), a1 = hi_f(v);
      if constexpr (FTM) {   // the fp outlier part, from its TMEM accumulator
        a0 += __uint_as_float(f[j]);
        a1 += __uint_as_float(f[j + 1]);
      }
      if constexpr (EPI == EPI_INT8_OUTLIER && CN > 0) {
        // floating-point outlier part: sum_o X_O[row,o] W_O[n,o], one
        // mixed-precision fma per outlier column on the 16-bit values
        const uint4 w0 = es.wo[c * GEMM_CW + j][0], w1 = es.wo[c * GEMM_CW + j + 1][0];
        a0 = fma2_mixed<BF>(xr[0], w0.x, a0);
        a1 = fma2_mixed<BF>(xr[0], w1.x, a1);
        if constexpr (CN > 2) {
          a0 = fma2_mixed<BF>(xr[1], w0.y, a0);
          a1 = fma2_mixed<BF>(xr[1], w1.y, a1);
        }
        if constexpr (CN > 4) {
          a0 = fma2_mixed<BF>(xr[2], w0.z, a0);
          a1 = fma2_mixed<BF>(xr[2], w1.z, a1);
          a0 = fma2_mixed<BF>(xr[3], w0.w, a0);
          a1 = fma2_mixed<BF>(xr[3], w1.w, a1);
        }
        if constexpr (CN > 8) {
          const uint4 u0 = es.wo[c * GEMM_CW + j][1], u1 = es.wo[c * GEMM_CW + j + 1][1];
          a0 = fma2_mixed<BF>(xr[4], u0.x, a0);
          a1 = fma2_mixed<BF>(xr[4], u1.x, a1);
          a0 = fma2_mixed<BF>(xr[5], u0.y, a0);
          a1 = fma2_mixed<BF>(xr[5], u1.y, a1);
          a0 = fma2_mixed<BF>(xr[6], u0.z, a0);
          a1 = fma2_mixed<BF>(xr[6], u1.z, a1);
          a0 = fma2_mixed<BF>(xr[7], u0.w, a0);
          a1 = fma2_mixed<BF>(xr[7], u1.w, a1);
        }
      }
      if constexpr (EPI == EPI_INT8_OUTLIER && CN < 0) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float a = e ? a1 : a0;
          if (n0 + j + e < p.N)
            for (int o0 = 0; o0 < cnt; o0 += 8) {
              uint16_t xh[8], wh[8];
              unpack8(__ldg(reinterpret_cast<const uint4*>(p.X_O + row * p.ostride + o0)), xh);
              unpack8(__ldg(reinterpret_cast<const uint4*>(p.W_O + (n0 + j + e) * p.ostride + o0)), wh);
#pragma unroll
              for (int k = 0; k < 8; ++k) a = fmaf(to_f<TOut>(xh[k]), to_f<TOut>(wh[k]), a);
            }
          if (e) a1 = a;
          else a0 = a;
        }
      }
      out[j >> 1] = pack2<TOut>(a0, a1);
    }
  }
  if constexpr (EPI == EPI_I32 || EPI == EPI_INT8_OUTLIER_I32) store_chunk_i32<GEMM_CW>(p, r, row, n0);
}

// One accumulator tile, one thread per row (its TMEM lane): the row's
// operands first, then the accumulator in chunks of GEMM_CW columns with the
// next chunk's tcgen05.ld in flight while the current one is processed.
// FTM: the fp outlier part was computed by the tensor core into a second
// accumulator at t_row_f; the epilogue adds it instead of computing it.
template <typename TOut, int EPI, int BN, int CN, bool FTM = false>
__device__ __forceinline__ void epi_tile(const EpiParams& p, const EpiStage<BN>& es, uint32_t t_row, int64_t row,
                                         bool row_ok, int64_t n_base, float alpha, int cnt, const CUtensorMap* tmY,
                                         uint8_t* ybox, int64_t row0, uint32_t t_row_f = 0) {
  constexpr int XR = CN > 0 ? CN / 2 : 1;
  uint32_t xr[XR];   // the row's outlier values X_O[row, 0..CN), 16-bit pairs
#pragma unroll
  for (int i = 0; i < XR; ++i) xr[i] = 0u;
  float sx = 0.0f;
  if (row_ok) {
    if constexpr (EPI == EPI_INT8_OUTLIER || EPI == EPI_FP8_ROWCOL) sx = __ldg(p.s_x + row);
    if constexpr (CN > 0) {
      if constexpr (EPI == EPI_INT8_OUTLIER) {
#pragma unroll
        for (int qd = 0; qd < (CN + 7) / 8; ++qd) {
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(p.X_O + row * p.ostride + qd * 8));
          const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (qd * 4 + e < XR) xr[qd * 4 + e] = uw[e];
        }
      }
    }
  }
  const bool v8 = (reinterpret_cast<uintptr_t>(p.Y) & 31u) == 0 && (p.N & 15) == 0;
  constexpr int NCH = BN / GEMM_CW;
  static_assert(NCH % 2 == 0, "chunks are processed in pairs");
  const int lane = threadIdx.x & 31;
  // one chunk: compute, then store (TMA box from shared memory, or per-thread stores)
  auto chunk = [&](uint32_t (&r)[GEMM_CW], const uint32_t (&f)[GEMM_CW], int c) {
    const int64_t n0 = n_base + c * GEMM_CW;
    if (n0 >= p.N) return;   // warp-uniform
    uint32_t out[GEMM_CW / 2];
#pragma unroll
    for (int i = 0; i < GEMM_CW / 2; ++i) out[i] = 0u;
    if (row_ok) epi_chunk<TOut, EPI, BN, CN, XR, FTM>(p, es, r, f, c, row, n_base, sx, alpha, cnt, xr, out);
    if constexpr (EPI != EPI_I32 && EPI != EPI_INT8_OUTLIER_I32) {
      if (p.tma_y) {
        uint8_t* box = ybox;
        if (lane == 0) bulk_wait_read<0>();   // the box's previous store has read it
        __syncwarp();
        // row `lane` of the box, 128B-pattern swizzle of the 32-byte rows (SWIZZLE_32B:
        // 16-byte half h sits at h ^ bit 2 of the row): conflict-free quarter-warp writes
        const uint32_t base = smem_u32(box) + static_cast<uint32_t>(lane) * 32u;
        const uint32_t x = ((static_cast<uint32_t>(lane) >> 2) & 1u) << 4;
        st_shared_v4(base + x, out[0], out[1], out[2], out[3]);
        st_shared_v4(base + (16u ^ x), out[4], out[5], out[6], out[7]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(tmY, box, static_cast<int32_t>(n0), static_cast<int32_t>(row0));
          bulk_commit();
        }
      } else if (row_ok) {
        store_chunk<GEMM_CW>(p, out, row, n0, v8);
      }
    }
  };
  uint32_t ra[GEMM_CW], rb[GEMM_CW];
  uint32_t fa[GEMM_CW], fb[GEMM_CW];   // the fp outlier part (FTM); unused otherwise
  __syncwarp();
  tmem_ld16(t_row, ra);
  if constexpr (FTM) tmem_ld16(t_row_f, fa);
#pragma unroll 1
  for (int c = 0; c < NCH; c += 2) {
    __syncwarp();
    tmem_wait16(ra);
    if constexpr (FTM) tmem_wait16(fa);
    tmem_ld16(t_row + static_cast<uint32_t>((c + 1) * GEMM_CW), rb);
    if constexpr (FTM) tmem_ld16(t_row_f + static_cast<uint32_t>((c + 1) * GEMM_CW), fb);
    chunk(ra, fa, c);
    __syncwarp();
    tmem_wait16(rb);
    if constexpr (FTM) tmem_wait16(fb);
    if (c + 2 < NCH) {
      tmem_ld16(t_row + static_cast<uint32_t>((c + 2) * GEMM_CW), ra);
      if constexpr (FTM) tmem_ld16(t_row_f + static_cast<uint32_t>((c + 2) * GEMM_CW), fa);
    }
    chunk(rb, fb, c + 1);
  }
}

template <int KIND, int EPI, typename TOut, int BN, int STAGES>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmXc,
           const __grid_constant__ CUtensorMap tmWc, const __grid_constant__ CUtensorMap tmXo,
           const __grid_constant__ CUtensorMap tmWo, const EpiParams p) {
  using L = GemmSmem<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * L::A_BYTES;
  constexpr int BNG = BN / GEMM_EPI_GROUPS;   // columns per epilogue group
  EpiStage<BNG>* estage = reinterpret_cast<EpiStage<BNG>*>(smem + L::TILE_BYTES);   // [GEMM_EPI_GROUPS]
  uint8_t* ystage = smem + L::TILE_BYTES + L::EPI_BYTES;   // [epilogue warp] boxes
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + L::TILE_BYTES + L::EPI_BYTES + L::Y_BYTES);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* tfull_bar = empty_bar + STAGES;     // [2]
  uint64_t* tempty_bar = tfull_bar + 2;         // [2]
  uint64_t* drain_bar = tempty_bar + 2;         // [1]
  uint64_t* epi_mbar = drain_bar + 1;           // [GEMM_EPI_GROUPS]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epi_mbar + GEMM_EPI_GROUPS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* sk_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);   // [GEMM_EPI_GROUPS]
  static_assert(GEMM_EPI_GROUPS <= 6, "the barrier area's 32 tail bytes hold the TMEM slot, abort and sk flags");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t M = p.M, N = p.N, K = p.K;
  const int num_m = static_cast<int>((M + GEMM_BM - 1) / GEMM_BM);
  const int num_n = static_cast<int>((N + BN - 1) / BN);
  const int num_tiles = num_m * num_n;
  const int num_kb = static_cast<int>((K + GEMM_BK - 1) / GEMM_BK);
  // LLM.int8 with 1..GEMM_CORR_K outlier columns: each tile ends with one more
  // stage, (-Xq[:,O]) x Wq[:,O]^T with K = 32, added to the accumulator
  // FT (LLM.int8, 128-wide tiles): TMEM also holds two fp32 accumulators for
  // the fp outlier part. With 1..16 outlier columns the extra stage carries
  // X_O and W_O (16 columns each, zero-padded) as well, and one kind::f16 MMA
  // (K = 16) computes X_O W_O^T there, so the epilogue only adds it.
  constexpr bool FT = EPI == EPI_INT8_OUTLIER && BN == 128;
  constexpr int TMEM_COLS = FT ? 4 * BN : 2 * BN;
  // stream-K: int32 partials (exact) for kind::i8, fp32 ones summed in party
  // order for kind::f8f6f4; 128 x 256 tiles only, so never with the FT
  // accumulators, which only the tile's owner segment would compute
  constexpr bool SK_OK = (KIND == 0 || KIND == 1) && BN == GEMM_SK_BN;
  const bool sk = SK_OK && p.sk != 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], GEMM_EPI_WARPS * GEMM_EPI_GROUPS);
    }
    mbar_init(drain_bar, 1);
    for (int g = 0; g < GEMM_EPI_GROUPS; ++g) mbar_init(&epi_mbar[g], GEMM_EPI_THREADS);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == GEMM_WARP_TMA && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == GEMM_WARP_MMA) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Launched as a programmatic dependent of the kernel before it (the
  // activation prep): everything above overlapped that kernel's tail; from
  // here on its outputs are read, so wait until it has completed.
  griddep_wait();
  bool corr = false;
  if constexpr (EPI == EPI_INT8_OUTLIER || EPI == EPI_INT8_OUTLIER_I32) {
    const int c = *p.count;
    corr = c > 0 && c <= GEMM_CORR_K;
  }
  bool fmma = false;
  if constexpr (FT) {
    const int c = *p.count;
    fmma = c > 0 && c <= GEMM_OUTL_STAGED;
  }
  // each role's register budget is set inside its branch: code after a merge
  // would be held to the lower of the two
  if (warp >= GEMM_EPI_ALL) {
  setmaxnreg_dec<GEMM_REGS_LOW>();
  if (warp == GEMM_WARP_TMA) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;   // bit s: stage s has a load in flight that nobody consumed yet
      bool ok = true;
      SegIter its(sk, num_tiles, p.sk_dp_tiles, num_kb);
      Seg sg;
      while (ok && its.next(sg)) {
        int mb, nb;
        tile_mn(sg.tile, num_m, num_n, p.group_m, mb, nb);
        for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_bar[stage], L::A_BYTES + L::B_BYTES);
          tma_load_2d(sA + stage * L::A_BYTES, &tmA, &full_bar[stage], kb * GEMM_BK, mb * GEMM_BM);
          tma_load_2d(sB + stage * L::B_BYTES, &tmB, &full_bar[stage], kb * GEMM_BK, nb * BN);
          issued |= 1u << stage;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (ok && corr && sg.kb0 == 0) {   // the tile's owner segment
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_bar[stage], (GEMM_BM + BN) * GEMM_CORR_K * (fmma ? 2 : 1));
          tma_load_2d(sA + stage * L::A_BYTES, &tmXc, &full_bar[stage], 0, mb * GEMM_BM);
          tma_load_2d(sB + stage * L::B_BYTES, &tmWc, &full_bar[stage], 0, nb * BN);
          if (fmma) {
            // X_O and W_O, 16 two-byte columns = 32-byte rows, after the codes
            tma_load_2d(sA + stage * L::A_BYTES + GEMM_BM * GEMM_CORR_K, &tmXo, &full_bar[stage], 0, mb * GEMM_BM);
            tma_load_2d(sB + stage * L::B_BYTES + BN * GEMM_CORR_K, &tmWo, &full_bar[stage], 0, nb * BN);
          }
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
            while (!mbar_try_wait(a, phase) && globaltimer() - t0 < drain_limit_ns()) {}
          }
        }
      }
    }
  } else if (warp == GEMM_WARP_MMA) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = KIND == 0   ? idesc_i8(GEMM_BM, BN)
                                 : KIND == 1 ? idesc_e4m3(GEMM_BM, BN)
                                             : idesc_f16(GEMM_BM, BN, std::is_same<TOut, __nv_bfloat16>::value);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      // test of the abort path (qlin_debug_inject_wait_timeout): nothing has
      // committed to the drain barrier yet, so this bounded wait runs out
      if (g_inject_wait_timeout != 0) ok = mbar_wait(drain_bar, 0u, abort_flag);
      SegIter its(sk, num_tiles, p.sk_dp_tiles, num_kb);
      Seg sg;
      while (ok && its.next(sg)) {
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = sdesc_k128(smem_u32(sA + stage * L::A_BYTES));
          const uint64_t bdesc = sdesc_k128(smem_u32(sB + stage * L::B_BYTES));
#pragma unroll
          for (int k = 0; k < GEMM_BK / 32; ++k)
            umma<KIND>(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc, (kb != sg.kb0 || k != 0) ? 1u : 0u);
          umma_commit(&empty_bar[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (ok && corr && sg.kb0 == 0) {
          if (!mbar_wait(&full_bar[stage], phase, abort_flag)) {
            ok = false;
          } else {
            tc_fence_after();
            umma<KIND>(d_tmem, sdesc_k32(smem_u32(sA + stage * L::A_BYTES)), sdesc_k32(smem_u32(sB + stage * L::B_BYTES)),
                       idesc, 1u);
            if (fmma) {
              constexpr uint32_t idesc_f = idesc_f16(GEMM_BM, BN, std::is_same<TOut, __nv_bfloat16>::value);
              umma<2>(tmem_base + static_cast<uint32_t>(2 * BN + acc * BN),
                      sdesc_k32(smem_u32(sA + stage * L::A_BYTES + GEMM_BM * GEMM_CORR_K)),
                      sdesc_k32(smem_u32(sB + stage * L::B_BYTES + BN * GEMM_CORR_K)), idesc_f, 0u);
            }
            umma_commit(&empty_bar[stage]);
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          }
        }
        if (!ok) break;
        umma_commit(&tfull_bar[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      // every MMA this thread issued has completed before TMEM is released
      umma_commit(drain_bar);
      const uint32_t a = smem_u32(drain_bar);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(a, 0) && globaltimer() - t0 < drain_limit_ns()) {}
    }
  }
  } else {
    setmaxnreg_inc<GEMM_REGS_HIGH>();
    // ---------------- epilogue: group g takes columns [g*BNG, (g+1)*BNG) of every tile ----------------
    const int g = warp / GEMM_EPI_WARPS;
    const int q = warp & 3;   // TMEM lane quarter this warp may access
    const int et = threadIdx.x - g * GEMM_EPI_THREADS;
    EpiStage<BNG>& es = estage[g];
    uint8_t* ybox = ystage + warp * GEMM_YBOX_BYTES;
    int cnt = 0;
    float alpha = 0.0f;
    if constexpr (EPI == EPI_INT8_OUTLIER || EPI == EPI_INT8_OUTLIER_I32) cnt = *p.count;
    if constexpr (EPI == EPI_FP8_TENSOR) alpha = __ldg(p.x_scale) * __ldg(p.w_scale);
    if constexpr (EPI == EPI_F16) alpha = 1.0f;
    const int cn = cnt == 0 ? 0 : cnt <= 2 ? 2 : cnt <= 4 ? 4 : cnt <= 8 ? 8 : cnt <= GEMM_OUTL_STAGED ? 16 : -1;
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t bar_phase = 0;
    SegIter its(sk, num_tiles, p.sk_dp_tiles, num_kb);
    Seg sg;
    while (its.next(sg)) {
      int mb, nb;
      tile_mn(sg.tile, num_m, num_n, p.group_m, mb, nb);
      const int64_t n_base = static_cast<int64_t>(nb) * BN + g * BNG;
      const int64_t row = static_cast<int64_t>(mb) * GEMM_BM + q * 32 + lane;
      const bool row_ok = row < M;
      const uint32_t t_row =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN + g * BNG);
      bool doer = true;   // this group writes the tile's Y
      bool split = false;
      if constexpr (SK_OK) split = sk && (sg.kb0 != 0 || sg.kb1 != num_kb);
      if (!split) {
        if constexpr (EPI != EPI_I32) {
          // the group's readers of the previous tile are done with its staging area
          if (!epi_bar(&epi_mbar[g], bar_phase, abort_flag)) break;
          epi_stage<TOut, EPI, BNG>(p, es, n_base, et, FT && cn > 0 && cnt <= GEMM_OUTL_STAGED ? 0 : cn);
          if (!epi_bar(&epi_mbar[g], bar_phase, abort_flag)) break;
        }
        if (!mbar_wait(&tfull_bar[acc], acc_phase, abort_flag)) break;
        tc_fence_after();
      } else if constexpr (SK_OK) {
        // A cut tile (stream-K). Every party but one leaves its partial (int32,
        // or fp32 for kind::f8f6f4) in its slot and counts itself in; the one that finishes the tile is
        // the owner if all contributors have arrived when its own part is
        // done (then it writes no partial), else the last to arrive. Nobody
        // waits for another CTA.
        if (!mbar_wait(&tfull_bar[acc], acc_phase, abort_flag)) break;
        tc_fence_after();
        int ob, nc;
        sk_parties(sg.tile, num_kb, num_tiles, p.sk_dp_tiles, ob, nc);
        const int self_q = static_cast<int>(blockIdx.x) - ob;   // 0: the owner
        int* ctr = p.sk_count + static_cast<int64_t>(sg.tile) * GEMM_EPI_GROUPS + g;
        const int row_in_tile = q * 32 + lane;
        bool fast = false;
        if (self_q == 0) {
          if (et == 0) sk_flag[g] = ld_acquire_gpu(ctr) == nc ? 1 : 0;
          if (!epi_bar(&epi_mbar[g], bar_phase, abort_flag)) break;
          fast = sk_flag[g] != 0;
        }
        if (!fast) {
          const int64_t slot = 2 * static_cast<int64_t>(blockIdx.x) + (self_q == 0 ? 1 : 0);
          sk_store_partial<BN, BNG>(p.sk_part + slot * (GEMM_BM * BN), t_row, g, row_in_tile);
          __threadfence();
          if (!epi_bar(&epi_mbar[g], bar_phase, abort_flag)) break;
          if (et == 0) sk_flag[g] = atom_add_acq_rel_gpu(ctr, 1) == nc ? 1 : 0;   // the (nc+1)-th arrival
          if (!epi_bar(&epi_mbar[g], bar_phase, abort_flag)) break;
          doer = sk_flag[g] != 0;
        }
        if (doer) {
          __threadfence();
          if (et == 0) *ctr = 0;   // every other party has counted itself in: ready for the next launch
          sk_add_partials<BN, BNG, KIND == 1>(p.sk_part, ob, nc, self_q, t_row, g, row_in_tile);
          if constexpr (EPI != EPI_I32) {
            if (!epi_bar(&epi_mbar[g], bar_phase, abort_flag)) break;
            epi_stage<TOut, EPI, BNG>(p, es, n_base, et, cn);
            if (!epi_bar(&epi_mbar[g], bar_phase, abort_flag)) break;
          }
        }
      }
      if (doer) {
        if constexpr (FT) {
          const uint32_t t_row_f = t_row + static_cast<uint32_t>(2 * BN);
          if (cn == 0) epi_tile<TOut, EPI, BNG, 0>(p, es, t_row, row, row_ok, n_base, alpha, cnt, &tmY, ybox, row - lane);
          else if (cnt <= GEMM_OUTL_STAGED)
            epi_tile<TOut, EPI, BNG, 0, true>(p, es, t_row, row, row_ok, n_base, alpha, cnt, &tmY, ybox, row - lane,
                                              t_row_f);
          else epi_tile<TOut, EPI, BNG, -1>(p, es, t_row, row, row_ok, n_base, alpha, cnt, &tmY, ybox, row - lane);
        } else if constexpr (EPI == EPI_INT8_OUTLIER || EPI == EPI_INT8_OUTLIER_I32) {
          if (cn == 0) epi_tile<TOut, EPI, BNG, 0>(p, es, t_row, row, row_ok, n_base, alpha, cnt, &tmY, ybox,
                                                             row - lane);
          else if (cn == 2) epi_tile<TOut, EPI, BNG, 2>(p, es, t_row, row, row_ok, n_base, alpha, cnt, &tmY, ybox,
                                                             row - lane);
          else if (cn == 4) epi_tile<TOut, EPI, BNG, 4>(p, es, t_row, row, row_ok, n_base, alpha, cnt, &tmY, ybox,
                                                             row - lane);
          else if (cn == 8) epi_tile<TOut, EPI, BNG, 8>(p, es, t_row, row, row_ok, n_base, alpha, cnt, &tmY, ybox,
                                                             row - lane);
          else if (cn == 16) epi_tile<TOut, EPI, BNG, 16>(p, es, t_row, row, row_ok, n_base, alpha, cnt, &tmY, ybox,
                                                             row - lane);
          else epi_tile<TOut, EPI, BNG, -1>(p, es, t_row, row, row_ok, n_base, alpha, cnt, &tmY, ybox,
                                                             row - lane);
        } else {
          epi_tile<TOut, EPI, BNG, 0>(p, es, t_row, row, row_ok, n_base, alpha, cnt, &tmY, ybox,
                                                             row - lane);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) bulk_wait<0>();   // this warp's Y stores are complete before the CTA exits
  }

  __syncthreads();
  if (warp == GEMM_WARP_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace qlin
