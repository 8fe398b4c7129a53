// gemm_cvt.cuh -- GEMMs whose 8-bit weights are dequantised to 16 bits in
// shared memory, tile by tile, and contracted with tcgen05 kind::f16 (fp32
// accumulation); the dequantised weight never reaches global memory.
//
// FMT 0, weight-only FP8 (Qwen-Image-2.1-Text-Encoder-FP8 page, "Format": E4M3
// weights with one bf16 scale per output channel, consumed as
// weight.to(bf16) * weight_scale; the activations stay in bf16):
//   W_deq[j,k] = bf16( decode(Wq[j,k]) * s_w[j] )   (one rounding: the e4m3 value
//                has 4 significant bits and s_w 8, so the fp32 product is exact)
//   Y[i,j]     = bf16( sum_k X[i,k] * W_deq[j,k] + bias[j] )
// FMT 1, block-scaled int8 weights (Qwen-Image-2.1-Text-Encoder-FP8 page, "How
// it was tested": GGUF Q8_0, int8 codes with one scale per 32 weights of a
// row) with per-token int8 activations, whose codes arrive as exact fp16:
//   W_deq[j,k] = fp16( float(Wq[j,k]) * s_w[j, k/32] )   (11 significant bits)
//   Y[i,j]     = dtype( s_x[i] * sum_k Xq[i,k] * W_deq[j,k] + bias[j] )
//   i.e. s_x[i] * sum_b s_w[j,b] * C_b[i,j] with the weight's scale applied
//   per element before the sum instead of per block after it (relative error
//   at most 2^-11 per weight, against the exact int32 block sums).
// FMT 2, NVFP4 weights (a reading of the release format the Darkstar
// ModelOpt-FP8 page names: E2M1 codes, one E4M3 scale per 16 weights of a
// row, one fp32 scale per tensor) with bf16 activations:
//   W_deq[j,k] = bf16( e2m1(code[j,k]) * e4m3(s_b[j,k/16]) )   (exact: at most
//                6 significant bits)
//   Y[i,j]     = bf16( s_t * sum_k X[i,k] * W_deq[j,k] + bias[j] )
//   The raw tile is 256 rows x 32 bytes (64 codes) per stage.
//
// Roles (one CTA per SM, 16 warps, persistent over 128x256 output tiles, two
// 256-column TMEM accumulators so the epilogue of one tile overlaps the main
// loop of the next):
//   warp 0       TMA producer: the 16-bit A tile (128 rows x 64 elements,
//                128B swizzle) and the raw 8-bit B tile (256 rows x 64 bytes)
//                of one stage of K;
//   warp 1       MMA issuer: 4 x kind::f16 (K = 16) per stage;
//   warps 4-11   converters: one 16-byte chunk of raw codes at a time (16
//                weights of one row) -> 16 16-bit values into two 16-byte
//                chunks of the swizzled row, then hand the stage to the MMA;
//   warps 12-15  epilogue, one per TMEM lane quarter: Y = acc + bias (FMT 0)
//                or s_x * acc + bias (FMT 1);
//   warps 2-3    idle.
// All waits are bounded (common.cuh).
#pragma once
#include <type_traits>

#include "common.cuh"

namespace qlin {

constexpr int WO8_BM = 128, WO8_BN = 256;
constexpr int WO8_BK = 64;                 // K elements per stage (128 bytes of a bf16 row)
constexpr int WO8_STAGES = 3;
constexpr int WO8_CONV_WARPS = 8, WO8_EPI_WARPS = 4;
constexpr int WO8_THREADS = 512;
constexpr int WO8_WARP_CONV0 = 4, WO8_WARP_EPI0 = 12;

struct Wo8Params {
  int64_t M, N, K;
  void* Y;                    // [M,N] 16-bit (bf16 for FMT 0)
  const uint16_t* s_w;        // FMT 0: [N] bf16 per-channel weight scale
  const float* s_wb;          // FMT 1: [N, K/32] fp32 block weight scales
  const float* s_x;           // FMT 1: [M] fp32 per-token activation scale
  const uint8_t* s_b4;        // FMT 2: [N, K/16] e4m3 block scales
  const float* s_t;           // FMT 2: [1] fp32 tensor scale
  const uint16_t* bias;       // [N] output dtype, nullable
};

struct Wo8Smem {
  static constexpr int A_BYTES = WO8_BM * WO8_BK * 2;      // 16 KB 16-bit, swizzled
  static constexpr int B_BYTES = WO8_BN * WO8_BK * 2;      // 32 KB 16-bit, swizzled (converted)
  static constexpr int R_BYTES = WO8_BN * WO8_BK;          // 16 KB 8-bit codes (raw)
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + R_BYTES;
  static constexpr int BIAS_BYTES = 2 * WO8_BN * 4;        // two tiles' biases (fp32)
  static constexpr int BAR_BYTES = 8 * (3 * WO8_STAGES + 4 + 2) + 16;
  static constexpr int TOTAL = 1024 + WO8_STAGES * STAGE_BYTES + BIAS_BYTES + BAR_BYTES;
};

// 16 e4m3 codes (one 16-byte chunk, element e in byte e) times the scale s,
// each product rounded once to bf16: 16 bf16 values as two 16-byte chunks.
__device__ __forceinline__ void e4m3x16_to_bf16(const uint4& raw, float s, uint4& lo8, uint4& hi8) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t out[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint16_t pair = static_cast<uint16_t>(w[i] >> (16 * h));   // codes of elements 4i+2h, 4i+2h+1
      uint32_t f16x2;
      asm("{\n\t.reg .b16 t;\n\tmov.b16 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(f16x2) : "h"(pair));
      const float a = __half2float(__ushort_as_half(static_cast<uint16_t>(f16x2 & 0xFFFFu)));
      const float b = __half2float(__ushort_as_half(static_cast<uint16_t>(f16x2 >> 16)));
      uint32_t bf;
      // cvt.rn.bf16x2.f32 d, x, y puts x in the upper half
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(bf) : "f"(__fmul_rn(b, s)), "f"(__fmul_rn(a, s)));
      out[2 * i + h] = bf;
    }
  }
  lo8 = make_uint4(out[0], out[1], out[2], out[3]);
  hi8 = make_uint4(out[4], out[5], out[6], out[7]);
}

// 32 NVFP4 codes (16 packed bytes, byte b holding element b in its low nibble
// and element b + 16 in its high nibble) -> 32 bf16 values code * scale, exact
// (an E2M1 value times an E4M3 scale has at most 6 significant bits).
// sp0 / sp1: the block scales of elements 0..15 / 16..31 as bf16 pairs.
// out[0], out[1]: elements 0-7, 8-15; out[2], out[3]: elements 16-23, 24-31.
// A nibble's magnitude (its low 3 bits) selects the two bytes of its bf16
// value from byte tables (__byte_perm); its bit 3 becomes bit 15 (the sign).
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ void nvfp4x32_to_bf16(const uint4& raw, uint32_t sp0, uint32_t sp1, uint4 (&out)[4]) {
  // bf16 of the magnitudes 0, 0.5, 1, 1.5 | 2, 3, 4, 6: high bytes, low bytes
  constexpr uint32_t HI_A = 0x3F3F3F00u, HI_B = 0x40404040u;
  constexpr uint32_t LO_A = 0xC0800000u, LO_B = 0xC0804000u;
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t lo[8], hi[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      // h = 0: the low nibbles (elements 4i..4i+3), h = 1: the high ones (16+4i..)
      const uint32_t v = h ? (w[i] >> 4) : w[i];
      const uint32_t m = v & 0x07070707u;             // magnitudes m0..m3, one per byte
      const uint32_t sel = m | (m >> 12);              // selector nibbles m0, m2, m1, m3
      const uint32_t hb = __byte_perm(HI_A, HI_B, sel);
      const uint32_t lb = __byte_perm(LO_A, LO_B, sel);   // bytes of elements 0, 2, 1, 3
      uint32_t p01 = __byte_perm(lb, hb, 0x6240);      // bf16 pair (element 0, element 1)
      uint32_t p23 = __byte_perm(lb, hb, 0x7351);      // bf16 pair (element 2, element 3)
      const uint32_t sg = v & 0x08080808u;             // signs at bits 3, 11, 19, 27
      p01 |= ((sg << 12) & 0x00008000u) | ((sg << 20) & 0x80000000u);
      p23 |= ((sg >> 4) & 0x00008000u) | ((sg << 4) & 0x80000000u);
      uint32_t* d = h ? hi : lo;
      const uint32_t sp = h ? sp1 : sp0;
      d[2 * i] = bf16x2_mul(p01, sp);
      d[2 * i + 1] = bf16x2_mul(p23, sp);
    }
  }
  out[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  out[1] = make_uint4(lo[4], lo[5], lo[6], lo[7]);
  out[2] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
  out[3] = make_uint4(hi[4], hi[5], hi[6], hi[7]);
}

// Two e4m3 block scales (low byte first) -> bf16 pairs (s0, s0) and (s1, s1), exact.
__device__ __forceinline__ void e4m3x2_scale_pairs(uint16_t two, uint32_t& sp0, uint32_t& sp1) {
  uint32_t f16x2;
  asm("{\n\t.reg .b16 t;\n\tmov.b16 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(f16x2) : "h"(two));
  const float a = __half2float(__ushort_as_half(static_cast<uint16_t>(f16x2 & 0xFFFFu)));
  const float b = __half2float(__ushort_as_half(static_cast<uint16_t>(f16x2 >> 16)));
  asm("cvt.rn.bf16x2.f32 %0, %1, %1;" : "=r"(sp0) : "f"(a));
  asm("cvt.rn.bf16x2.f32 %0, %1, %1;" : "=r"(sp1) : "f"(b));
}

// 16 int8 codes (element e in byte e) times the scale s, each product
// rounded to fp16 (the fp32 product rounds first when s has more than 16
// significant bits): 16 fp16 values as two 16-byte chunks. A code q reads as
// float from the bits 0x4B000000 | (q ^ 0x80), i.e. 2^23 + 128 + q.
__device__ __forceinline__ void int8x16_to_f16(const uint4& raw, float s, uint4& lo8, uint4& hi8) {
  const uint32_t w[4] = {raw.x ^ 0x80808080u, raw.y ^ 0x80808080u, raw.z ^ 0x80808080u, raw.w ^ 0x80808080u};
  const unsigned long long off2 = f32x2_of(__float_as_uint(-8388736.0f), __float_as_uint(-8388736.0f));
  const unsigned long long s2 = f32x2_of(__float_as_uint(s), __float_as_uint(s));
  uint32_t out[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t a = __byte_perm(w[i], 0x4B000000u, 0x7650u + 2 * h);       // code 4i+2h
      const uint32_t b = __byte_perm(w[i], 0x4B000000u, 0x7650u + 2 * h + 1);   // code 4i+2h+1
      const unsigned long long v = mul_f32x2(add_f32x2(f32x2_of(a, b), off2), s2);
      uint32_t hv;
      // cvt.rn.f16x2.f32 d, x, y puts x in the upper half
      asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(hv) : "f"(hi_f(v)), "f"(lo_f(v)));
      out[2 * i + h] = hv;
    }
  }
  lo8 = make_uint4(out[0], out[1], out[2], out[3]);
  hi8 = make_uint4(out[4], out[5], out[6], out[7]);
}

template <int FMT, typename TOut>
__global__ void __launch_bounds__(WO8_THREADS, 1)
    k_gemm_cvt(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const Wo8Params p) {
  static_assert(FMT == 1 || std::is_same<TOut, __nv_bfloat16>::value, "weight-only FP8 and NVFP4 write bf16");
  // raw weight bytes per row and stage: 64 8-bit codes (FMT 0, 1) or 64 packed 4-bit codes (FMT 2)
  constexpr int RAW_ROW = FMT == 2 ? WO8_BK / 2 : WO8_BK;
  using L = Wo8Smem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // per stage: [A 16 KB | B (converted) 32 KB | raw B 16 KB]
  auto sA = [&](int s) { return smem + s * L::STAGE_BYTES; };
  auto sB = [&](int s) { return smem + s * L::STAGE_BYTES + L::A_BYTES; };
  auto sR = [&](int s) { return smem + s * L::STAGE_BYTES + L::A_BYTES + L::B_BYTES; };
  float* sbias = reinterpret_cast<float*>(smem + WO8_STAGES * L::STAGE_BYTES);   // [2][WO8_BN]
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + WO8_STAGES * L::STAGE_BYTES + L::BIAS_BYTES);
  uint64_t* conv_bar = full_bar + WO8_STAGES;
  uint64_t* empty_bar = conv_bar + WO8_STAGES;
  uint64_t* tfull_bar = empty_bar + WO8_STAGES;   // [2]
  uint64_t* tempty_bar = tfull_bar + 2;           // [2]
  uint64_t* drain_bar = tempty_bar + 2;
  uint64_t* epi_mbar = drain_bar + 1;             // the epilogue warps' barrier (bounded waits)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epi_mbar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t M = p.M, N = p.N, K = p.K;
  const int num_m = static_cast<int>((M + WO8_BM - 1) / WO8_BM);
  const int num_n = static_cast<int>((N + WO8_BN - 1) / WO8_BN);
  const int num_tiles = num_m * num_n;
  const int num_kb = static_cast<int>((K + WO8_BK - 1) / WO8_BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < WO8_STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&conv_bar[s], WO8_CONV_WARPS);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], WO8_EPI_WARPS);
    }
    mbar_init(drain_bar, 1);
    mbar_init(epi_mbar, 32 * WO8_EPI_WARPS);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * WO8_BN);
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
      uint32_t phase = 0, issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        const int mb = tile % num_m, nb = tile / num_m;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_bar[stage], L::A_BYTES + WO8_BN * RAW_ROW);
          tma_load_2d(sA(stage), &tmA, &full_bar[stage], kb * WO8_BK * 2, mb * WO8_BM);
          tma_load_2d(sR(stage), &tmB, &full_bar[stage], kb * RAW_ROW, nb * WO8_BN);
          issued |= 1u << stage;
          if (++stage == WO8_STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // aborted: wait (bounded) for the copies still in flight before the CTA exits
        for (int i = 0; i < WO8_STAGES; ++i) {
          if (--stage < 0) { stage = WO8_STAGES - 1; phase ^= 1u; }
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
      constexpr uint32_t idesc = idesc_f16(WO8_BM, WO8_BN, FMT != 1);   // bf16 (FMT 0, 2) or fp16 operands
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * WO8_BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          // the converters waited for the stage's TMA (A and raw B) before converting
          if (!mbar_wait(&conv_bar[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = sdesc_k128(smem_u32(sA(stage)));
          const uint64_t bdesc = sdesc_k128(smem_u32(sB(stage)));
#pragma unroll
          for (int k = 0; k < WO8_BK / 16; ++k)
            umma<2>(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc, (kb != 0 || k != 0) ? 1u : 0u);
          umma_commit(&empty_bar[stage]);
          if (++stage == WO8_STAGES) { stage = 0; phase ^= 1u; }
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
  } else if (warp >= WO8_WARP_CONV0 && warp < WO8_WARP_CONV0 + WO8_CONV_WARPS) {
    // ---------------- converters: codes * scale -> 16 bits, swizzled ----------------
    const int ct = threadIdx.x - 32 * WO8_WARP_CONV0;   // 0..255
    if constexpr (FMT == 2) {
      // two 16-byte raw chunks per thread and stage: rows ct/2 and ct/2 + 128,
      // chunk ct%2 (codes 32c..32c+31 of the stage, block scales 2c and 2c+1)
      const int c = ct & 1;
      const int64_t nsb = K / 16;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        const int nb = tile / num_m;
        uint16_t sc[2], sn[2];   // the two rows' scale pairs for stage kb, and kb + 1
        auto scale_pairs = [&](int kb, uint16_t (&d)[2]) {
#pragma unroll
          for (int qd = 0; qd < 2; ++qd) {
            const int64_t n = static_cast<int64_t>(nb) * WO8_BN + (ct >> 1) + 128 * qd;
            const int64_t b = 4 * static_cast<int64_t>(kb) + 2 * c;
            d[qd] = (n < N && kb < num_kb)   // K % 64 == 0: b + 1 < K/16
                        ? __ldg(reinterpret_cast<const unsigned short*>(p.s_b4 + n * nsb + b))
                        : static_cast<uint16_t>(0);
          }
        };
        scale_pairs(0, sc);
        for (int kb = 0; kb < num_kb; ++kb) {
          scale_pairs(kb + 1, sn);
          if (!mbar_wait(&full_bar[stage], phase, abort_flag)) { ok = false; break; }
          const uint8_t* raw = sR(stage);
          uint8_t* dst = sB(stage);
#pragma unroll
          for (int qd = 0; qd < 2; ++qd) {
            const int r = (ct >> 1) + 128 * qd;
            const uint4 v = *reinterpret_cast<const uint4*>(raw + r * RAW_ROW + c * 16);
            uint32_t sp0, sp1;
            e4m3x2_scale_pairs(sc[qd], sp0, sp1);
            uint4 o[4];
            nvfp4x32_to_bf16(v, sp0, sp1, o);
            // row r's 128 bf16 bytes: 16-byte chunk ch sits at chunk (ch ^ (r & 7))
#pragma unroll
            for (int x = 0; x < 4; ++x)
              *reinterpret_cast<uint4*>(dst + r * 128 + (((4 * c + x) ^ (r & 7)) << 4)) = o[x];
          }
          fence_proxy_async_smem();   // generic writes -> read by the tensor core (async proxy)
          __syncwarp();
          if (lane == 0) mbar_arrive(&conv_bar[stage]);
          if (++stage == WO8_STAGES) { stage = 0; phase ^= 1u; }
          sc[0] = sn[0];
          sc[1] = sn[1];
        }
      }
    } else {
    const int64_t nblk = K / 32;                        // FMT 1: weight-scale blocks per row
    const int cb = (ct & 3) >> 1;                       // FMT 1: this thread's block within a stage
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      const int nb = tile / num_m;
      // this thread's rows of the tile: ct/4 + 64q, q = 0..3
      float sc[4];       // FMT 0: the rows' scales; FMT 1: their block scales for stage kb
      float sn[4];       // FMT 1: the same for stage kb + 1 (loaded one stage ahead)
      auto block_scales = [&](int kb, float (&d)[4]) {
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
          const int64_t n = static_cast<int64_t>(nb) * WO8_BN + (ct >> 2) + 64 * qd;
          const int64_t b = 2 * static_cast<int64_t>(kb) + cb;
          d[qd] = (n < N && b < nblk) ? __ldg(p.s_wb + n * nblk + b) : 0.0f;
        }
      };
      if constexpr (FMT == 0) {
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
          const int64_t n = static_cast<int64_t>(nb) * WO8_BN + (ct >> 2) + 64 * qd;
          sc[qd] = n < N ? to_f<__nv_bfloat16>(__ldg(p.s_w + n)) : 0.0f;
        }
      } else {
        block_scales(0, sc);
      }
      for (int kb = 0; kb < num_kb; ++kb) {
        if constexpr (FMT == 1) block_scales(kb + 1, sn);
        if (!mbar_wait(&full_bar[stage], phase, abort_flag)) { ok = false; break; }
        const uint8_t* raw = sR(stage);
        uint8_t* dst = sB(stage);
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
          const int id = ct + 256 * qd;          // 16-byte raw chunk: row id/4, chunk id%4
          const int r = id >> 2, c = id & 3;
          const uint4 v = *reinterpret_cast<const uint4*>(raw + r * WO8_BK + c * 16);
          uint4 lo, hi;
          if constexpr (FMT == 0) e4m3x16_to_bf16(v, sc[qd], lo, hi);
          else int8x16_to_f16(v, sc[qd], lo, hi);
          // row r's 128 bf16 bytes: 16-byte chunk ch sits at chunk (ch ^ (r & 7))
          *reinterpret_cast<uint4*>(dst + r * 128 + (((2 * c) ^ (r & 7)) << 4)) = lo;
          *reinterpret_cast<uint4*>(dst + r * 128 + (((2 * c + 1) ^ (r & 7)) << 4)) = hi;
        }
        fence_proxy_async_smem();   // generic writes -> read by the tensor core (async proxy)
        __syncwarp();
        if (lane == 0) mbar_arrive(&conv_bar[stage]);
        if (++stage == WO8_STAGES) { stage = 0; phase ^= 1u; }
        if constexpr (FMT == 1) {
#pragma unroll
          for (int qd = 0; qd < 4; ++qd) sc[qd] = sn[qd];
        }
      }
    }
    }
  } else if (warp >= WO8_WARP_EPI0) {
    // ---------------- epilogue: Y = acc + bias (FMT 0), s_x * acc + bias (FMT 1), s_t * acc + bias (FMT 2) ----------------
    const int q = warp & 3;                      // TMEM lane quarter
    const int et = threadIdx.x - 32 * WO8_WARP_EPI0;   // 0..127
    int acc = 0;
    uint32_t acc_phase = 0, bar_phase = 0;
    const bool vec = (N & 7) == 0 && (reinterpret_cast<uintptr_t>(p.Y) & 15u) == 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int mb = tile % num_m, nb = tile / num_m;
      const int64_t n_base = static_cast<int64_t>(nb) * WO8_BN;
      const int64_t row = static_cast<int64_t>(mb) * WO8_BM + q * 32 + lane;
      // this tile's biases, staged in the slot of its accumulator (the slot's
      // previous readers finished that accumulator's tile two tiles ago)
      float* bt = sbias + acc * WO8_BN;
      for (int j = et; j < WO8_BN; j += 32 * WO8_EPI_WARPS) {
        const int64_t n = n_base + j;
        bt[j] = (p.bias != nullptr && n < N) ? to_f<TOut>(__ldg(p.bias + n)) : 0.0f;
      }
      if (!epi_bar(epi_mbar, bar_phase, abort_flag)) break;
      if (!mbar_wait(&tfull_bar[acc], acc_phase, abort_flag)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * WO8_BN);
      uint32_t r[32];
      float sx = 1.0f;
      if constexpr (FMT == 1) sx = row < M ? __ldg(p.s_x + row) : 0.0f;
      if constexpr (FMT == 2) sx = __ldg(p.s_t);
      for (int c = 0; c < WO8_BN; c += 32) {
        __syncwarp();
        tmem_ld32(t_row + static_cast<uint32_t>(c), r);
        tmem_wait_regs32(r);
        const int64_t n0 = n_base + c;
        if (row < M && n0 < N) {
          uint32_t out[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float2 b2 = *reinterpret_cast<const float2*>(bt + c + 2 * j);
            if constexpr (FMT == 0)
              out[j] = pack2<TOut>(__uint_as_float(r[2 * j]) + b2.x, __uint_as_float(r[2 * j + 1]) + b2.y);
            else
              out[j] = pack2<TOut>(fmaf(__uint_as_float(r[2 * j]), sx, b2.x), fmaf(__uint_as_float(r[2 * j + 1]), sx, b2.y));
          }
          uint16_t* y = reinterpret_cast<uint16_t*>(p.Y) + row * N + n0;
          if (vec && n0 + 32 <= N) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              reinterpret_cast<uint4*>(y)[i] = make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
          } else {
            for (int j = 0; j < 32 && n0 + j < N; ++j) y[j] = static_cast<uint16_t>(out[j >> 1] >> (16 * (j & 1)));
          }
        }
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
    tmem_dealloc(tmem_base, 2 * WO8_BN);
  }
}

}  // namespace qlin
