// prep.cuh -- HBM-bound kernels around the GEMM:
//   * k_prep_rows: per-row absmax, scale and int8 or E4M3 codes (activations
//     and weights); for LLM.int8 activations it also flags the outlier columns
//     (any |x| > threshold in the column, over every token of the call) and
//     leaves entries above the threshold out of the row absmax;
//   * k_ws_reset / k_outlier_finish: the rest of the LLM.int8 prepare stage
//     around that pass (zeroed header before it; after it the outlier list,
//     exact copies X_O of the outlier columns, the rows whose absmax sat in
//     an outlier column requantised, and the outlier weight columns W_O);
//   * k_gather_wo: dequantised outlier weight columns (standalone)
//   * k_zero_outlier_cols: zero codes of the outlier columns (standalone)
//     W_O[j,o] = dtype(fp32(Wq[j,O[o]]) * s_w[j]) (the weight.to(dtype) *
//     weight_scale rule of the Text-Encoder-FP8 page, "Format");
//   * k_fp8_static: per-tensor static E4M3 activation codes;
//   * k_absmax / k_fp8_tensor_quant / k_scale_from_absmax: max calibration and
//     per-tensor FP8 weights;
//   * k_int4_group_quant: int4 per-group weight codes and scales.
// Rows are read as 16-byte vectors of 8 elements (K % 8 == 0), coalesced
// across the threads of a CTA.
#pragma once
#include <type_traits>

#include "common.cuh"

namespace qlin {

constexpr int PREP_THREADS = 128;

// Running per-column maximum of |x| on raw 16-bit patterns: for finite fp16
// or bf16 values, clearing the sign bit gives a pattern whose unsigned order
// is the order of |x|, so two columns are handled per 32-bit max.
__device__ __forceinline__ uint32_t umax16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Running max of |x| over packed 16-bit pairs: the magnitude of the result is
// the larger magnitude (its sign bit is meaningless and cleared at the end).
template <typename T>
__device__ __forceinline__ uint32_t absmax2(uint32_t m, uint32_t x);
template <>
__device__ __forceinline__ uint32_t absmax2<__nv_bfloat16>(uint32_t m, uint32_t x) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(m), "r"(x));
  return d;
}
template <>
__device__ __forceinline__ uint32_t absmax2<__half>(uint32_t m, uint32_t x) {
  uint32_t d;
  asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(d) : "r"(m), "r"(x));
  return d;
}

__device__ __forceinline__ unsigned long long pair_f32(uint32_t lo, uint32_t hi) {
  return static_cast<unsigned long long>(lo) | (static_cast<unsigned long long>(hi) << 32);
}

__device__ __forceinline__ void colmax_accum(uint4& m, const uint4& u) {
  m.x = umax16x2(m.x, u.x & 0x7FFF7FFFu);
  m.y = umax16x2(m.y, u.y & 0x7FFF7FFFu);
  m.z = umax16x2(m.z, u.z & 0x7FFF7FFFu);
  m.w = umax16x2(m.w, u.w & 0x7FFF7FFFu);
}

// Outlier weight column value W_O[j,o] = dtype(fp32(Wq[j,O[o]]) * s_w[j]) for
// o < count, 0 for count <= o < pad (the weight.to(dtype) * weight_scale rule).
template <typename T>
__device__ __forceinline__ void gather_wo_elem(const int8_t* __restrict__ Wq, const float* __restrict__ s_w,
                                               int64_t K, const int32_t* __restrict__ O, int cnt, int pad,
                                               uint16_t* __restrict__ W_O, int64_t ostride, int64_t t) {
  const int64_t j = t / pad;
  const int o = static_cast<int>(t - j * pad);
  float val = 0.0f;
  if (o < cnt) val = __fmul_rn(static_cast<float>(Wq[j * K + __ldg(O + o)]), __ldg(s_w + j));
  W_O[j * ostride + o] = from_f<T>(val);
}

// Optional work folded into the row quantiser's launch: the outlier weight
// columns W_O (N rows), grid-stride over N * pad.
struct WoGather {
  const int8_t* Wq;
  const float* s_w;
  int64_t N;
  const int32_t* O;
  uint16_t* W_O;
  int8_t* WqO;   // [N, OUTL_CODES] weight codes of the outlier columns (count <= OUTL_CODES), or nullptr
};

// Outlier counts up to OUTL_CODES also get compact int8 copies of the codes in
// their columns, zero-padded to OUTL_CODES per row: -Xq[:,O] and Wq[:,O]. The
// GEMM adds their product to its accumulator with one more MMA (K = 32),
// which takes those columns' products back out of the full-K contraction.
constexpr int OUTL_CODES = 32;
constexpr int OUTL_FP_MMA_K = 16;
constexpr int OUTL_LIST = 64;   // outlier counts up to this keep the column list in shared memory
constexpr int OUTL_MAX_K = 32768; // the largest K the library takes

// Round-half-even of an fp32 value in (-2^22, 2^22) to an integer, read from
// the low byte of t + 1.5 * 2^23: the add rounds to nearest even, and within
// [2^23, 2^24) the float spacing is 1, so the low byte is the two's-complement
// low byte of rne(t).
__device__ __forceinline__ uint32_t rne_low_byte(float t) { return __float_as_uint(__fadd_rn(t, 12582912.0f)); }

// 8 int8 codes of one vector, no outlier in it, normal scale (so |t| < 127.5
// and no clamp is needed): code = rne(x * inv), one fp32 multiply (two
// elements per instruction) and one fp32 add. The add is a scalar __fadd_rn on
// purpose: a packed multiply followed by a packed add was measured to be
// contracted into one fused multiply-add, which rounds ties differently.
template <typename T>
__device__ __forceinline__ uint2 quant8_int8_fast(const uint4& u, float inv) {
  const unsigned long long inv2 = pair_f32(__float_as_uint(inv), __float_as_uint(inv));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  uint32_t f[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t lo, hi;
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
      lo = w[i] << 16;
      hi = w[i] & 0xFFFF0000u;
    } else {
      lo = __float_as_uint(to_f<T>(static_cast<uint16_t>(w[i] & 0xFFFFu)));
      hi = __float_as_uint(to_f<T>(static_cast<uint16_t>(w[i] >> 16)));
    }
    const unsigned long long t = mul_f32x2(pair_f32(lo, hi), inv2);
    f[2 * i] = rne_low_byte(__uint_as_float(static_cast<uint32_t>(t)));
    f[2 * i + 1] = rne_low_byte(__uint_as_float(static_cast<uint32_t>(t >> 32)));
  }
  const uint32_t lo = __byte_perm(__byte_perm(f[0], f[1], 0x0040), __byte_perm(f[2], f[3], 0x0040), 0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(f[4], f[5], 0x0040), __byte_perm(f[6], f[7], 0x0040), 0x5410);
  return make_uint2(lo, hi);
}

// Mask that keeps the non-outlier 16-bit lanes of word i (elements 2i, 2i+1)
// of a vector whose outlier flags are the 8 bits of om.
__device__ __forceinline__ uint32_t keep_mask(uint32_t om, int i) {
  return (((om >> (2 * i)) & 1u) ? 0u : 0x0000FFFFu) | (((om >> (2 * i + 1)) & 1u) ? 0u : 0xFFFF0000u);
}

// ---------------------------------------------------------------------------
// Row quantiser (persistent; a "row unit" of RW warps handles one row at a
// time; each thread copies its own V 16-byte vectors of the unit's next
// PF_DEPTH - 1 rows into private shared-memory slots with cp.async, so those
// rows are in flight while the current one is quantised).
//
// CODE 0: int8 (QMAX 127), CODE 1: E4M3 (QMAX 448), CODE 2: the int8 codes
// stored as fp16 values (exact; the A operand of a kind::f16 contraction, 2
// bytes per code: Q is then [rows, K] fp16). SCALE_BF16: the stored
// scale is bf16(absmax / QMAX) and the codes use that rounded value (the
// [out,1] bf16 weight scales of the Text-Encoder-FP8 page).
//
// OUTL (LLM.int8 activations): the streaming pass of the prepare stage. Every
// row is quantised with the absmax over its entries with |x| <= thr; entries
// above the threshold get code 0 and set their column's bit in the outlier
// bitmap. Because a column outside the outlier set O holds no entry above the
// threshold, this absmax equals the exact one (over k not in O) unless the
// maximum sits in a column of O; the raw absmax pattern is kept per row so
// that k_outlier_finish can tell. The bitmap is zeroed by k_ws_reset, the
// kernel launched just before this one: this kernel is its programmatic
// dependent, so it runs while k_ws_reset finishes, and waits for it
// (griddepcontrol.wait) only before OR-ing its columns into the bitmap.
// ---------------------------------------------------------------------------
constexpr int RQ_THREADS = 256;
constexpr int RQ_WARPS = RQ_THREADS / 32;
constexpr int PF_DEPTH = 2;   // row slots per thread (current row + 1 in flight)

struct PrepArgs {
  int64_t M, K;
  float thr;
  uint32_t thr_bits;   // largest 16-bit |x| pattern with value <= thr
  int rw;              // warps per row unit (1, 2, 4 or 8)
  uint8_t* Q;
  float* s_f32;
  uint16_t* s_bf16;
  uint16_t* amax_bits; // [M] pass-1 absmax pattern (OUTL)
  uint32_t* flags;     // [NW] outlier bitmap (zero on entry for OUTL)
};

template <typename T, int CODE>
__device__ __forceinline__ uint2 quant_vec(const uint4& v, uint32_t om, float inv, bool fast, bool zero) {
  if constexpr (CODE == 0) {
    if (fast && om == 0u) return quant8_int8_fast<T>(v, inv);
    uint16_t h[8];
    unpack8(v, h);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int q = (zero || ((om >> e) & 1u)) ? 0 : q_int(to_f<T>(h[e]), inv, 127);
      const uint32_t b = static_cast<uint32_t>(q) & 0xFFu;
      if (e < 4) lo |= b << (8 * e);
      else hi |= b << (8 * (e - 4));
    }
    return make_uint2(lo, hi);
  } else {
    uint16_t h[8];
    unpack8(v, h);
    float t[8];
    if (fast) {
#pragma unroll
      for (int e = 0; e < 8; ++e) t[e] = __fmul_rn(to_f<T>(h[e]), inv);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) t[e] = q_e4m3_in(to_f<T>(h[e]), inv);
    }
    uint2 out;
    out.x = e4m3x2(t[0], t[1]) | (e4m3x2(t[2], t[3]) << 16);
    out.y = e4m3x2(t[4], t[5]) | (e4m3x2(t[6], t[7]) << 16);
    if (zero) out = make_uint2(0u, 0u);
    return out;
  }
}

// 8 int8 codes (element e in byte e) as 8 fp16 values (exact: |code| <= 127).
__device__ __forceinline__ uint4 codes_as_f16x8(const uint2& c) {
  const uint32_t w[2] = {c.x, c.y};
  uint32_t h[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int lo = static_cast<int8_t>((w[i >> 1] >> (16 * (i & 1))) & 0xFFu);
    const int hi = static_cast<int8_t>((w[i >> 1] >> (16 * (i & 1) + 8)) & 0xFFu);
    h[i] = static_cast<uint32_t>(__half_as_ushort(__int2half_rn(lo))) |
           (static_cast<uint32_t>(__half_as_ushort(__int2half_rn(hi))) << 16);
  }
  return make_uint4(h[0], h[1], h[2], h[3]);
}

// Lanes of a packed 16-bit pair whose |x| pattern exceeds tb: with a = |x|
// (<= 0x7FFF) and c = 0x7FFF - tb, a > tb exactly when a + c >= 0x8000, and
// a + c <= 0xFFFE never carries into the other lane, so bit 15 of each lane
// of (a + c) flags it. c2 = c * 0x10001 (both lanes).
__device__ __forceinline__ uint32_t above2(uint32_t w, uint32_t c2) { return ((w & 0x7FFF7FFFu) + c2) & 0x80008000u; }
// All-ones in the flagged lanes of above2's result.
__device__ __forceinline__ uint32_t lanes_of(uint32_t flagged) { return (flagged >> 15) * 0xFFFFu; }
// The 8 flags of a vector (bit e: element e; element 2i is the low lane of word i).
__device__ __forceinline__ uint32_t flag_byte(uint32_t f0, uint32_t f1, uint32_t f2, uint32_t f3) {
  return ((f0 >> 15) & 1u) | ((f0 >> 30) & 2u) | ((f1 >> 13) & 4u) | ((f1 >> 28) & 8u) | ((f2 >> 11) & 16u) |
         ((f2 >> 26) & 32u) | ((f3 >> 9) & 64u) | ((f3 >> 24) & 128u);
}

// Running packed |x| max of one vector into m2 (16-bit pairs).
template <typename T>
__device__ __forceinline__ uint32_t vec_absmax2(uint32_t m2, const uint4& x) {
  return absmax2<T>(absmax2<T>(m2, x.x), absmax2<T>(absmax2<T>(x.y, x.z), x.w));
}

// Largest |x| pattern held in a packed pair accumulator.
__device__ __forceinline__ uint32_t pair_max_bits(uint32_t m2) {
  return max(m2 & 0x7FFFu, (m2 >> 16) & 0x7FFFu);
}

template <typename T, int V, int CODE, bool SCALE_BF16, bool OUTL>
__global__ void __launch_bounds__(RQ_THREADS, 3) k_prep_rows(const T* __restrict__ X, const PrepArgs a) {
  // the kernel that follows may be scheduled now (it waits for this grid's
  // completion before it reads anything this kernel writes)
  griddep_launch_dependents();
  extern __shared__ uint4 stage[];   // [PF_DEPTH][V][RQ_THREADS] 16-byte vectors
  __shared__ uint32_t red[2][RQ_WARPS];
  // OUTL: the CTA's outlier columns, OR-ed into the global bitmap once at the
  // end (per-row global atomics on the few words of the outlier columns
  // contend with every other CTA's and were measured to stall the rows)
  __shared__ uint32_t sbits[OUTL ? (OUTL_MAX_K / 32) : 1];
  const int64_t M = a.M, K = a.K;
  const int KV = static_cast<int>(K / 8);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rw = a.rw;
  const int units = RQ_WARPS / rw;
  const int unit = warp / rw;
  const int ut = tid - unit * rw * 32;   // thread index inside the unit
  const int UT = rw * 32;
  constexpr float QMAX = CODE == 1 ? 448.0f : 127.0f;

  // max over the unit (warp redux, then the unit's warps through shared
  // memory, double-buffered so one named barrier per reduction suffices)
  int rpar = 0;
  auto unit_max = [&](uint32_t v) -> uint32_t {
    v = __reduce_max_sync(0xffffffffu, v);
    if (rw == 1) return v;
    if (lane == 0) red[rpar][warp] = v;
    asm volatile("bar.sync %0, %1;" ::"r"(1 + unit), "r"(UT) : "memory");
    uint32_t m = 0;
    for (int i = 0; i < rw; ++i) m = max(m, red[rpar][unit * rw + i]);
    rpar ^= 1;
    return m;
  };

  // staging: each thread only touches its own column of `stage`, so
  // cp.async.wait_group alone orders it.
  // Rows: unit u of CTA b takes rows (d * G + b) * units + u, d = 0, 1, ...
  // (a static split: a global row counter was measured to cost 2-3 us in
  // contended atomics). The unit's leader keeps a ring of the unit's next row
  // indices in shared memory.
  const int64_t first = static_cast<int64_t>(blockIdx.x) * units + unit;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * units;
  __shared__ long long rowq[RQ_WARPS][8];
  long long* myq = rowq[unit];
  auto grab = [&](int k) -> long long { return static_cast<long long>(first + static_cast<int64_t>(k) * stride); };
  if constexpr (OUTL) {
    for (int i = tid; i < (K + 31) / 32; i += RQ_THREADS) sbits[i] = 0u;
    __syncthreads();
  }
  auto issue = [&](int64_t r, int slot) {
    const uint4* xr = reinterpret_cast<const uint4*>(X + (r < M ? r : 0) * K);
#pragma unroll
    for (int u = 0; u < V; ++u) {
      const int idx = ut + u * UT;
      cp_async16(&stage[(slot * V + u) * RQ_THREADS + tid], xr + idx, r < M && idx < KV);
    }
    cp_async_commit();
  };
  static_assert(PF_DEPTH >= 2 && PF_DEPTH <= 7, "the row ring holds the rows in flight and the next");
  if (ut == 0)
    for (int d = 0; d < PF_DEPTH; ++d) myq[d] = grab(d);
  if (rw == 1) __syncwarp();
  else asm volatile("bar.sync %0, %1;" ::"r"(1 + unit), "r"(UT) : "memory");
#pragma unroll
  for (int d = 0; d < PF_DEPTH - 1; ++d) issue(myq[d], d);
  int slot = 0;
  for (int t = 0;; ++t) {
    const int64_t row = myq[t & 7];
    if (row >= M) break;
    issue(myq[(t + PF_DEPTH - 1) & 7], (slot + PF_DEPTH - 1) % PF_DEPTH);
    // ring entry (t+D)&7 last held row t+D-8, read at iteration t+D-8 < t
    // before that iteration's barrier (unit_max); its new row is first read
    // at iteration t+1 (prefetch), after this iteration's barrier
    if (ut == 0) myq[(t + PF_DEPTH) & 7] = grab(t + PF_DEPTH);
    if (rw == 1) __syncwarp();
    cp_async_wait<PF_DEPTH - 1>();   // this thread's copies of `row` have landed
    uint4 cur[V];
#pragma unroll
    for (int u = 0; u < V; ++u) {
      const int idx = ut + u * UT;
      cur[u] = idx < KV ? stage[(slot * V + u) * RQ_THREADS + tid] : make_uint4(0u, 0u, 0u, 0u);
    }
    slot = (slot + 1) % PF_DEPTH;
    uint32_t m2 = 0;
#pragma unroll
    for (int u = 0; u < V; ++u) m2 = vec_absmax2<T>(m2, cur[u]);
    uint32_t mb = unit_max(pair_max_bits(m2));
    if (OUTL && mb > a.thr_bits) {
      // some entry of this row exceeds the threshold: flag its column, and
      // zero it, which leaves it out of the absmax and gives it code 0
      const uint32_t c2 = (0x7FFFu - a.thr_bits) * 0x10001u;
      uint32_t mm = 0;
#pragma unroll
      for (int u = 0; u < V; ++u) {
        const int idx = ut + u * UT;   // vectors past the row are zero: never flagged
        uint4 x = cur[u];
        const uint32_t f0 = above2(x.x, c2), f1 = above2(x.y, c2), f2 = above2(x.z, c2), f3 = above2(x.w, c2);
        if ((f0 | f1 | f2 | f3) != 0u) {
          atomicOr(&sbits[idx >> 2], flag_byte(f0, f1, f2, f3) << ((idx & 3) * 8));
          x.x &= ~lanes_of(f0);
          x.y &= ~lanes_of(f1);
          x.z &= ~lanes_of(f2);
          x.w &= ~lanes_of(f3);
          cur[u] = x;
        }
        mm = vec_absmax2<T>(mm, x);
      }
      mb = unit_max(pair_max_bits(mm));
    }
    float s = to_f<T>(static_cast<uint16_t>(mb)) / QMAX;
    if constexpr (SCALE_BF16) {
      const uint16_t sb = __bfloat16_as_ushort(__float2bfloat16_rn(s));
      s = __uint_as_float(static_cast<uint32_t>(sb) << 16);
      if (ut == 0) a.s_bf16[row] = sb;
    } else {
      if (ut == 0) a.s_f32[row] = s;
    }
    if constexpr (OUTL) {
      if (ut == 0) a.amax_bits[row] = static_cast<uint16_t>(mb);
    }
    const float inv = 1.0f / s;
    const bool zero = (s == 0.0f);
    // a normal scale keeps |x * inv| below QMAX + 1/2 for every entry in the absmax
    const bool fast = s >= 1.17549435e-38f;
    if constexpr (CODE == 2) {
      uint4* qr = reinterpret_cast<uint4*>(a.Q + row * K * 2);
#pragma unroll
      for (int u = 0; u < V; ++u) {
        const int idx = ut + u * UT;
        if (idx < KV) qr[idx] = codes_as_f16x8(quant_vec<T, 0>(cur[u], 0u, inv, fast, zero));
      }
    } else {
      uint2* qr = reinterpret_cast<uint2*>(a.Q + row * K);
#pragma unroll
      for (int u = 0; u < V; ++u) {
        const int idx = ut + u * UT;
        if (idx < KV) qr[idx] = quant_vec<T, CODE>(cur[u], 0u, inv, fast, zero);
      }
    }
  }
  cp_async_wait<0>();
  if constexpr (OUTL) {
    // the global bitmap was zeroed by the kernel before this one (this grid is
    // its programmatic dependent; a no-op without a programmatic launch)
    griddep_wait();
    __syncthreads();
    for (int i = tid; i < (K + 31) / 32; i += RQ_THREADS)
      if (sbits[i] != 0u) atomicOr(a.flags + i, sbits[i]);
  }
}

// Zeroes the per-call header of the LLM.int8 workspace (row counter, outlier
// count and bitmap, stream-K arrival counters) at the start of a prepare
// stage. The streaming pass is launched as its programmatic dependent.
__global__ void __launch_bounds__(256) k_ws_reset(uint32_t* __restrict__ hdr, int64_t words) {
  griddep_launch_dependents();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < words;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    hdr[i] = 0u;
}

// ---------------------------------------------------------------------------
// The rest of the LLM.int8 prepare stage, once the streaming pass has seen
// every row (a programmatic dependent of it: scheduled as its CTAs leave,
// then griddepcontrol.wait until it has completed):
//   compact  every CTA scans the bitmap into shared memory (per-word prefix
//            counts; the ascending list itself for up to OUTL_LIST columns);
//            CTA 0 writes the list O and the count;
//   W_O      one thread per weight row: its codes in the O columns, then
//            W_O[j, 0..pad) = dtype(fp32(code) * s_w[j]) and, for up to
//            OUTL_CODES columns, WqO[j, 0..32) = the codes (zero-padded), as
//            16-byte stores;
//   fix-up   one lane segment (8, 16 or 32 lanes) per activation row: the
//            row's values in the O columns go to X_O (zero-padded to `pad`)
//            and, for up to OUTL_CODES columns, minus the codes the streaming
//            pass left there to XqO (the GEMM takes those codes' products back
//            out, so Xq keeps them); if the largest of those values that is
//            <= thr reaches the pass-1 absmax, the absmax may sit in an
//            outlier column: the row is requantised with the exact absmax by
//            the whole CTA (its outlier codes then 0, its XqO row 0).
// ---------------------------------------------------------------------------
// The (o+1)-th outlier column, from the shared bitmap and its word prefixes.
__device__ __forceinline__ int outlier_col(const uint32_t* sflags, const int32_t* swpre, int NW, int o) {
  int lo = 0, hi = NW - 1;   // largest w with swpre[w] <= o
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (swpre[mid] <= o) lo = mid;
    else hi = mid - 1;
  }
  return lo * 32 + static_cast<int>(__fns(sflags[lo], 0, o - swpre[lo] + 1));
}

constexpr int FIN_THREADS = 256;
constexpr int FIN_WARPS = FIN_THREADS / 32;
constexpr int FIN_RQ_LIST = 64;   // rows a CTA queues for requantisation by the whole CTA

struct FinishArgs {
  int64_t M, K;
  uint32_t thr_bits;
  const uint32_t* flags;     // [NW]
  int32_t* O;                // [K]
  int32_t* count;            // [1]
  const uint16_t* amax_bits; // [M]
  float* s_x;                // [M]
  uint8_t* Q;                // [M,K]
  uint16_t* X_O;             // [M, ostride]
  int64_t ostride;
  int8_t* XqO;               // [M, OUTL_CODES] or nullptr
  WoGather wo;
};

template <typename T>
__global__ void __launch_bounds__(FIN_THREADS) k_outlier_finish(const T* __restrict__ X, const FinishArgs a) {
  griddep_launch_dependents();   // the GEMM may be scheduled now; it waits for this grid to complete
  griddep_wait();                // the streaming pass has completed and its writes are visible
  extern __shared__ uint32_t fsm[];   // sflags[NW], swpre[NW]
  __shared__ int warp_tot[FIN_WARPS];
  __shared__ int o_list[OUTL_LIST];
  __shared__ long long rq_rows[FIN_RQ_LIST];
  __shared__ int rq_n;
  __shared__ uint32_t red[FIN_WARPS];
  const int64_t M = a.M, K = a.K;
  const int KV = static_cast<int>(K / 8);
  const int NW = static_cast<int>((K + 31) / 32);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t* sflags = fsm;
  int32_t* swpre = reinterpret_cast<int32_t*>(fsm + NW);
  constexpr float QMAX = 127.0f;

  // ---------------- compaction of the bitmap into shared memory ----------------
  const int per = (NW + FIN_THREADS - 1) / FIN_THREADS;   // <= 4 (K <= 32768)
  int local = 0;
  for (int u = 0; u < per; ++u) {
    const int w = tid * per + u;
    if (w < NW) {
      const uint32_t word = __ldcg(a.flags + w);
      sflags[w] = word;
      local += __popc(word);
    }
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_tot[warp] = incl;
  if (tid == 0) rq_n = 0;
  __syncthreads();
  int base = 0, cnt = 0;
  for (int i = 0; i < FIN_WARPS; ++i) {
    if (i < warp) base += warp_tot[i];
    cnt += warp_tot[i];
  }
  int run = base + incl - local;
  for (int u = 0; u < per; ++u) {
    const int w = tid * per + u;
    if (w < NW) {
      swpre[w] = run;
      uint32_t bits = sflags[w];
      int o = run;
      while (bits) {
        const int col = w * 32 + (__ffs(bits) - 1);
        if (blockIdx.x == 0) a.O[o] = col;
        if (o < OUTL_LIST) o_list[o] = col;
        ++o;
        bits &= bits - 1;
      }
      run += __popc(sflags[w]);
    }
  }
  if (blockIdx.x == 0 && tid == 0) *a.count = cnt;
  __syncthreads();
  if (cnt == 0) return;
  auto ocol = [&](int o) -> int { return cnt <= OUTL_LIST ? o_list[o] : outlier_col(sflags, swpre, NW, o); };
  // X_O and W_O are zero-padded to a multiple of 8 columns, and to 16 for up
  // to 16 outlier columns (one K = 16 tensor-core step of the fp part)
  const int pad = cnt <= OUTL_FP_MMA_K ? OUTL_FP_MMA_K : (cnt + 7) & ~7;
  const bool codes = a.XqO != nullptr && cnt <= OUTL_CODES;

  // a vector of row xr with its outlier columns' entries zeroed
  auto masked_vec = [&](const T* xr, int64_t idx) -> uint4 {
    uint4 x = ld_nc_v4(reinterpret_cast<const uint4*>(xr) + idx);
    const uint32_t omv = (sflags[idx >> 2] >> ((idx & 3) * 8)) & 0xFFu;
    x.x &= keep_mask(omv, 0);
    x.y &= keep_mask(omv, 1);
    x.z &= keep_mask(omv, 2);
    x.w &= keep_mask(omv, 3);
    return x;
  };
  // the CTA requantises a row below (or this thread alone, if its list is full)
  auto queue_requant = [&](int64_t row) {
    const int slot = atomicAdd(&rq_n, 1);
    if (slot < FIN_RQ_LIST) {
      rq_rows[slot] = row;
      return;
    }
    const T* xr = X + row * K;
    uint32_t m = 0;
    for (int64_t idx = 0; idx < KV; ++idx) m = vec_absmax2<T>(m, masked_vec(xr, idx));
    const float sc = to_f<T>(static_cast<uint16_t>(pair_max_bits(m))) / QMAX;
    a.s_x[row] = sc;
    const float inv = 1.0f / sc;
    const bool zero = (sc == 0.0f), fast = sc >= 1.17549435e-38f;
    for (int64_t idx = 0; idx < KV; ++idx) {
      const uint4 x = ld_nc_v4(reinterpret_cast<const uint4*>(xr) + idx);
      const uint32_t omv = (sflags[idx >> 2] >> ((idx & 3) * 8)) & 0xFFu;
      *reinterpret_cast<uint2*>(a.Q + row * K + idx * 8) = quant_vec<T, 0>(x, omv, inv, fast, zero);
    }
  };

  // Work of this thread: (1) at most one weight row j of the compact gather
  // (counts up to OUTL_CODES; rows go to warp w of every CTA before warp w+1
  // of any, so that the gather spreads over all CTAs); (2) per pass, one
  // outlier column o of one activation row in a segment of L lanes (counts up
  // to 32; larger counts loop over the columns). Every independent load is
  // issued before any of them is used: the kernel is latency-bound.
  const int64_t wg = static_cast<int64_t>(warp) * gridDim.x + blockIdx.x;
  const int64_t wstride = static_cast<int64_t>(gridDim.x) * FIN_WARPS;
  const bool wcompact = a.wo.N > 0 && a.wo.WqO != nullptr && cnt <= OUTL_CODES;
  const int64_t j = wg * 32 + lane;
  const bool has_j = wcompact && j < a.wo.N;
  int8_t wc[OUTL_CODES];   // the weight row's codes in the O columns
  float sw = 0.0f;
  if (has_j) {
    const int8_t* wr = a.wo.Wq + j * K;
    sw = __ldg(a.wo.s_w + j);
#pragma unroll
    for (int o = 0; o < OUTL_CODES; ++o) wc[o] = o < cnt ? __ldg(wr + o_list[o]) : int8_t{0};
  }
  // the weight row's stores: WqO[j, 0..32) and W_O[j, 0..pad), 16 bytes at a time
  auto store_w = [&]() {
    if (!has_j) return;
    uint32_t cw[OUTL_CODES / 4];
#pragma unroll
    for (int i = 0; i < OUTL_CODES / 4; ++i)
      cw[i] = static_cast<uint32_t>(static_cast<uint8_t>(wc[4 * i])) |
              (static_cast<uint32_t>(static_cast<uint8_t>(wc[4 * i + 1])) << 8) |
              (static_cast<uint32_t>(static_cast<uint8_t>(wc[4 * i + 2])) << 16) |
              (static_cast<uint32_t>(static_cast<uint8_t>(wc[4 * i + 3])) << 24);
    uint4* q4 = reinterpret_cast<uint4*>(a.wo.WqO + j * OUTL_CODES);
    q4[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    q4[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
    uint4* w4 = reinterpret_cast<uint4*>(a.wo.W_O + j * a.ostride);
#pragma unroll
    for (int v = 0; v < OUTL_CODES / 8; ++v) {
      if (v * 8 >= pad) break;
      uint32_t hw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int oo = v * 8 + 2 * e;
        hw[e] = static_cast<uint32_t>(from_f<T>(__fmul_rn(static_cast<float>(wc[oo]), sw))) |
                (static_cast<uint32_t>(from_f<T>(__fmul_rn(static_cast<float>(wc[oo + 1]), sw))) << 16);
      }
      w4[v] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    }
  };

  if (a.wo.N > 0 && !wcompact) {   // the element-wise gather (counts above OUTL_CODES)
    const int64_t total = a.wo.N * pad;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * FIN_THREADS + tid; t < total;
         t += static_cast<int64_t>(gridDim.x) * FIN_THREADS) {
      const int64_t jj = t / pad;
      const int oo = static_cast<int>(t - jj * pad);
      float val = 0.0f;
      if (oo < cnt) val = __fmul_rn(static_cast<float>(a.wo.Wq[jj * K + ocol(oo)]), __ldg(a.wo.s_w + jj));
      a.wo.W_O[jj * a.ostride + oo] = from_f<T>(val);
    }
  }

  const int L = pad <= 8 ? 8 : pad <= 16 ? 16 : 32;
  const int rpw = 32 / L;                 // rows per warp and pass
  const int seg = lane / L, sl = lane - seg * L;
  if (pad <= 32) {
    // one column per lane: o = sl (pad <= L)
    const int o = sl;
    const int k = o < cnt ? o_list[o] : 0;   // cnt <= 32 <= OUTL_LIST
    bool first = true;
    for (int64_t rb = wg * rpw; rb < M; rb += wstride * rpw) {   // warp-uniform
      const int64_t row = rb + seg;
      const bool ok = row < M;
      // loads: the value and the pass-1 code in column O[o], the pass-1 absmax
      uint16_t h = 0;
      int8_t c = 0;
      uint32_t mb = 0xFFFFu;
      if (ok) {
        mb = __ldcg(a.amax_bits + row);
        if (o < cnt) {
          h = __ldg(reinterpret_cast<const uint16_t*>(X + row * K) + k);
          if (codes) c = static_cast<int8_t>(__ldcg(a.Q + row * K + k));
        }
      }
      if (first) {   // the weight row's stores, once these loads are in flight
        first = false;
        store_w();
      }
      const uint32_t ah = h & 0x7FFFu;
      uint32_t mo = (o < cnt && ah <= a.thr_bits) ? ah : 0u;   // largest |x| <= thr among the O columns
#pragma unroll
      for (int off = 1; off < 32; off <<= 1)
        if (off < L) mo = max(mo, __shfl_xor_sync(0xffffffffu, mo, off));
      const bool requant = ok && mo >= mb;
      if (ok) {
        if (o < pad) a.X_O[row * a.ostride + o] = h;
        if (codes)   // minus the pass-1 codes of the O columns (a requantised row has 0 there)
          for (int oo = o; oo < OUTL_CODES; oo += L)
            a.XqO[row * OUTL_CODES + oo] = static_cast<int8_t>(oo == o && !requant ? -c : 0);
      }
      if (requant && sl == 0) queue_requant(row);
    }
    if (first) store_w();   // this warp had no activation row
  } else {
    // more than 32 columns: each lane loops over its columns
    for (int64_t rb = wg; rb < M; rb += wstride) {   // one row per warp
      const int64_t row = rb;
      const T* xr = X + row * K;
      uint32_t mo = 0;
      for (int o = lane; o < pad; o += 32) {
        uint16_t h = 0;
        if (o < cnt) {
          h = reinterpret_cast<const uint16_t*>(xr)[ocol(o)];
          const uint32_t ah = h & 0x7FFFu;
          if (ah <= a.thr_bits) mo = max(mo, ah);
        }
        a.X_O[row * a.ostride + o] = h;
      }
      mo = __reduce_max_sync(0xffffffffu, mo);
      const uint32_t mb = __ldcg(a.amax_bits + row);
      if (mo >= mb && lane == 0) queue_requant(row);
    }
  }
  __syncthreads();
  // the CTA's listed rows: absmax over the non-outlier columns, then the codes;
  // rows of up to FIN_THREADS * 8 vectors (K <= 16384) are held in registers
  // (one read), longer ones are read twice (the second read hits L2)
  const int nrq = min(rq_n, FIN_RQ_LIST);
  constexpr int RV = 8;
  auto block_max = [&](uint32_t m) -> uint32_t {
    m = __reduce_max_sync(0xffffffffu, pair_max_bits(m));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = 0;
#pragma unroll
    for (int w = 0; w < FIN_WARPS; ++w) m = max(m, red[w]);
    return m;
  };
  auto vec_mask = [&](int idx) -> uint32_t { return (sflags[idx >> 2] >> ((idx & 3) * 8)) & 0xFFu; };
  for (int i = 0; i < nrq; ++i) {
    const int64_t row = rq_rows[i];
    const uint4* xr = reinterpret_cast<const uint4*>(X + row * K);
    uint2* qr = reinterpret_cast<uint2*>(a.Q + row * K);
    if (KV <= FIN_THREADS * RV) {
      uint4 v[RV];
      uint32_t m = 0;
#pragma unroll
      for (int r = 0; r < RV; ++r) {
        const int idx = tid + r * FIN_THREADS;
        v[r] = idx < KV ? ld_nc_v4(xr + idx) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int r = 0; r < RV; ++r) {
        const int idx = tid + r * FIN_THREADS;
        if (idx < KV) {
          const uint32_t omv = vec_mask(idx);
          uint4 x = v[r];
          x.x &= keep_mask(omv, 0);
          x.y &= keep_mask(omv, 1);
          x.z &= keep_mask(omv, 2);
          x.w &= keep_mask(omv, 3);
          m = vec_absmax2<T>(m, x);
        }
      }
      m = block_max(m);
      const float sc = to_f<T>(static_cast<uint16_t>(m)) / QMAX;
      if (tid == 0) a.s_x[row] = sc;
      const float inv = 1.0f / sc;
      const bool zero = (sc == 0.0f), fast = sc >= 1.17549435e-38f;
#pragma unroll
      for (int r = 0; r < RV; ++r) {
        const int idx = tid + r * FIN_THREADS;
        if (idx < KV) qr[idx] = quant_vec<T, 0>(v[r], vec_mask(idx), inv, fast, zero);
      }
    } else {
      uint32_t m = 0;
      for (int idx = tid; idx < KV; idx += FIN_THREADS) m = vec_absmax2<T>(m, masked_vec(X + row * K, idx));
      m = block_max(m);
      const float sc = to_f<T>(static_cast<uint16_t>(m)) / QMAX;
      if (tid == 0) a.s_x[row] = sc;
      const float inv = 1.0f / sc;
      const bool zero = (sc == 0.0f), fast = sc >= 1.17549435e-38f;
      for (int idx = tid; idx < KV; idx += FIN_THREADS) qr[idx] = quant_vec<T, 0>(ld_nc_v4(xr + idx), vec_mask(idx), inv, fast, zero);
    }
    __syncthreads();   // red is reused by the next row
  }
}

// Standalone outlier weight gather (grid-stride over N * pad).
template <typename T>
__global__ void __launch_bounds__(256) k_gather_wo(const int8_t* __restrict__ Wq, const float* __restrict__ s_w,
                                                 int64_t N, int64_t K, const int32_t* __restrict__ O,
                                                 const int32_t* __restrict__ count_ptr, uint16_t* __restrict__ W_O,
                                                 int64_t ostride) {
  const int cnt = *count_ptr;
  if (cnt == 0) return;
  const int pad = (cnt + 7) & ~7;
  const int64_t total = N * pad;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x)
    gather_wo_elem<T>(Wq, s_w, K, O, cnt, pad, W_O, ostride, t);
}

// Static per-tensor E4M3 codes: Xq = e4m3(x * (1 / *x_scale)); all-zero
// codes if the scale is 0. Grid-stride over 8-element vectors.
// E4M3 codes of n fp32 values (grid-stride, two per conversion).
__global__ void __launch_bounds__(256) k_e4m3_encode(const float* __restrict__ t, uint8_t* __restrict__ codes,
                                                   int64_t n) {
  for (int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x); i < n;
       i += 2 * static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float a = t[i], b = i + 1 < n ? t[i + 1] : 0.0f;
    const uint32_t c = e4m3x2(a, b);
    codes[i] = static_cast<uint8_t>(c & 0xFFu);
    if (i + 1 < n) codes[i + 1] = static_cast<uint8_t>(c >> 8);
  }
}

// The codes of the outlier columns set to 0 in Q [M,K] (a warp per row). The
// fused forward never needs this: its GEMM takes those codes as 0 on its own.
__global__ void __launch_bounds__(256) k_zero_outlier_cols(int8_t* __restrict__ Q, int64_t M, int64_t K,
                                                         const int32_t* __restrict__ O,
                                                         const int32_t* __restrict__ count_ptr) {
  const int cnt = *count_ptr;
  const int lane = threadIdx.x & 31;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5); row < M;
       row += static_cast<int64_t>(gridDim.x) * 8)
    for (int o = lane; o < cnt; o += 32) Q[row * K + __ldg(O + o)] = 0;
}

template <typename T>
__global__ void __launch_bounds__(256) k_fp8_static(const T* __restrict__ X, int64_t nvec,
                                                  const float* __restrict__ x_scale, uint8_t* __restrict__ Q) {
  griddep_launch_dependents();   // the GEMM may be scheduled now (it waits for this grid to complete)
  const float s = __ldg(x_scale);
  const float inv = 1.0f / s;
  const bool zero = (s == 0.0f);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nvec;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 u = ld_nc_v4(reinterpret_cast<const uint4*>(X) + i);
    uint16_t h[8];
    unpack8(u, h);
    float t[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) t[e] = q_e4m3_in(to_f<T>(h[e]), inv);
    uint32_t lo = e4m3x2(t[0], t[1]) | (e4m3x2(t[2], t[3]) << 16);
    uint32_t hi = e4m3x2(t[4], t[5]) | (e4m3x2(t[6], t[7]) << 16);
    if (zero) lo = hi = 0u;
    reinterpret_cast<uint2*>(Q)[i] = make_uint2(lo, hi);
  }
}

// absmax over a whole tensor into *out (a non-negative float's bits order
// like the float, so an unsigned atomicMax works). *out must be 0 on entry.
template <typename T>
__global__ void __launch_bounds__(256) k_absmax(const T* __restrict__ X, int64_t nvec, uint32_t* out) {
  __shared__ float red[8];
  float m = 0.0f;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nvec;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    uint16_t h[8];
    unpack8(ld_nc_v4(reinterpret_cast<const uint4*>(X) + i), h);
#pragma unroll
    for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(to_f<T>(h[e])));
  }
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < static_cast<int>(blockDim.x / 32); ++w) m = fmaxf(m, red[w]);
    m = fmaxf(m, red[0]);
    atomicMax(out, __float_as_uint(m));
  }
}

// *scale = absmax / qmax (IEEE fp32).
__global__ void k_scale_from_absmax(const uint32_t* absmax_bits, float qmax, float* scale) {
  *scale = __uint_as_float(*absmax_bits) / qmax;
}

// Per-tensor E4M3 weight codes with s = absmax / 448, written to *s_out.
template <typename T>
__global__ void __launch_bounds__(256) k_fp8_tensor_quant(const T* __restrict__ W, int64_t nvec,
                                                        const uint32_t* __restrict__ absmax_bits,
                                                        uint8_t* __restrict__ Q, float* s_out) {
  const float s = __uint_as_float(*absmax_bits) / 448.0f;
  const float inv = 1.0f / s;
  const bool zero = (s == 0.0f);
  if (blockIdx.x == 0 && threadIdx.x == 0) *s_out = s;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nvec;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    uint16_t h[8];
    unpack8(ld_nc_v4(reinterpret_cast<const uint4*>(W) + i), h);
    float t[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) t[e] = q_e4m3_in(to_f<T>(h[e]), inv);
    uint32_t lo = e4m3x2(t[0], t[1]) | (e4m3x2(t[2], t[3]) << 16);
    uint32_t hi = e4m3x2(t[4], t[5]) | (e4m3x2(t[6], t[7]) << 16);
    if (zero) lo = hi = 0u;
    reinterpret_cast<uint2*>(Q)[i] = make_uint2(lo, hi);
  }
}

// int4 per-group weights: one warp per (row, group of 128). Lane l holds
// columns [4l, 4l+4) of the group; s = absmax / 7; codes in [-7, 7]. Each
// block of 32 columns is stored in 16 bytes, byte b holding column b of the
// block in its low nibble and column b + 16 in its high nibble: lanes
// 8m..8m+3 own the low nibbles of block m and take the high nibbles from
// lanes 8m+4..8m+7.
template <typename T>
__global__ void __launch_bounds__(256) k_int4_group_quant(const T* __restrict__ W, int64_t N, int64_t K,
                                                        uint8_t* __restrict__ Q4, float* __restrict__ s_w) {
  const int64_t G = 128, ng = K / G;
  const int64_t gw = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= N * ng) return;
  const int64_t j = gw / ng, g = gw - j * ng;
  const T* src = W + j * K + g * G + lane * 4;
  const uint2 u = *reinterpret_cast<const uint2*>(src);
  uint16_t h[4] = {static_cast<uint16_t>(u.x & 0xFFFF), static_cast<uint16_t>(u.x >> 16),
                   static_cast<uint16_t>(u.y & 0xFFFF), static_cast<uint16_t>(u.y >> 16)};
  float m = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e) m = fmaxf(m, fabsf(to_f<T>(h[e])));
  m = warp_max(m);
  const float s = m / 7.0f;
  const float inv = 1.0f / s;
  uint32_t nib = 0;   // code e in the low nibble of byte e
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int q = (s == 0.0f) ? 0 : q_int(to_f<T>(h[e]), inv, 7);
    nib |= (static_cast<uint32_t>(q) & 0xFu) << (8 * e);
  }
  const uint32_t upper = __shfl_down_sync(0xFFFFFFFFu, nib, 4);
  if ((lane & 4) == 0)
    *reinterpret_cast<uint32_t*>(Q4 + j * (K / 2) + g * (G / 2) + (lane >> 3) * 16 + (lane & 3) * 4) =
        nib | (upper << 4);
  if (lane == 0) s_w[j * ng + g] = s;
}

// NVFP4 weights (a reading of the release format the Darkstar ModelOpt-FP8
// page names): one thread per (row j, block of 32 columns), each step one
// IEEE fp32 operation:
//   s_t  = absmax(W) / 2688                 (2688 = 6 * 448)
//   s_b  = e4m3(absmax(16 weights) / (6 * s_t))   (rne, saturating; 0 if s_t == 0)
//   code = e2m1(w / (decode(s_b) * s_t))    (0 where that divisor is 0)
// packed like the int4 format: byte b of the block's 16 holds element b in
// its low nibble and element b + 16 in its high nibble.
// E2M1 rounding: the magnitude's code is the number of rounding boundaries
// below it (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5 between 0, 0.5, 1, 1.5, 2, 3,
// 4, 6); at a boundary it goes to the even mantissa (> or >=), and anything
// above 5 saturates to 6.
__device__ __forceinline__ uint32_t e2m1_rne(float t) {
  const float a = fabsf(t);
  const uint32_t c = static_cast<uint32_t>(a > 0.25f) + static_cast<uint32_t>(a >= 0.75f) +
                     static_cast<uint32_t>(a > 1.25f) + static_cast<uint32_t>(a >= 1.75f) +
                     static_cast<uint32_t>(a > 2.5f) + static_cast<uint32_t>(a >= 3.5f) + static_cast<uint32_t>(a > 5.0f);
  return c | (signbit(t) ? 8u : 0u);
}
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  uint32_t f16x2;
  const uint16_t pair = static_cast<uint16_t>(code & 0xFFu);
  asm("{\n\t.reg .b16 t;\n\tmov.b16 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(f16x2) : "h"(pair));
  return __half2float(__ushort_as_half(static_cast<uint16_t>(f16x2 & 0xFFFFu)));
}
template <typename T>
__global__ void __launch_bounds__(256) k_nvfp4_quant(const T* __restrict__ W, int64_t N, int64_t K,
                                                     const uint32_t* __restrict__ amax_bits, uint8_t* __restrict__ Q,
                                                     uint8_t* __restrict__ s_b, float* __restrict__ s_t) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nb = K / 32;
  if (t >= N * nb) return;
  const int64_t j = t / nb, m = t - j * nb;
  const float st = __fdiv_rn(__uint_as_float(*amax_bits), 2688.0f);
  const float six_st = __fmul_rn(6.0f, st);
  if (t == 0) *s_t = st;
  float w[32];
  const uint4* src = reinterpret_cast<const uint4*>(W + j * K + m * 32);
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    uint16_t h[8];
    unpack8(__ldg(src + v), h);
#pragma unroll
    for (int e = 0; e < 8; ++e) w[8 * v + e] = to_f<T>(h[e]);
  }
  uint32_t sc[2];
  float d[2];
#pragma unroll
  for (int hb = 0; hb < 2; ++hb) {
    float bm = 0.0f;
#pragma unroll
    for (int e = 0; e < 16; ++e) bm = fmaxf(bm, fabsf(w[16 * hb + e]));
    sc[hb] = six_st == 0.0f ? 0u : (e4m3x2(__fdiv_rn(bm, six_st), 0.0f) & 0xFFu);
    d[hb] = __fmul_rn(e4m3_value(sc[hb]), st);
  }
  uint32_t out[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int b = 4 * i + e;
      const uint32_t lo = d[0] == 0.0f ? 0u : e2m1_rne(__fdiv_rn(w[b], d[0]));
      const uint32_t hi = d[1] == 0.0f ? 0u : e2m1_rne(__fdiv_rn(w[16 + b], d[1]));
      word |= (lo | (hi << 4)) << (8 * e);
    }
    out[i] = word;
  }
  *reinterpret_cast<uint4*>(Q + j * (K / 2) + m * 16) = make_uint4(out[0], out[1], out[2], out[3]);
  *reinterpret_cast<uint16_t*>(s_b + j * (K / 16) + 2 * m) = static_cast<uint16_t>(sc[0] | (sc[1] << 8));
}

// Block-scaled int8 weights: one thread per (row j, block b of 32 weights
// along K): s_w[j,b] = absmax / 127, codes rne(w * (1/s)) clamped to +-127
// (the row format's quantiser on each block), 0 for an all-zero block.
template <typename T>
__global__ void __launch_bounds__(256) k_int8_block_quant(const T* __restrict__ W, int64_t N, int64_t K,
                                                        int8_t* __restrict__ Q, float* __restrict__ s_w) {
  const int64_t nb = K / 32;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < N * nb;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t j = t / nb, b = t - j * nb;
    const uint4* src = reinterpret_cast<const uint4*>(W + j * K + b * 32);
    uint16_t h[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint16_t e[8];
      unpack8(ld_nc_v4(src + i), e);
#pragma unroll
      for (int k = 0; k < 8; ++k) h[8 * i + k] = e[k];
    }
    float m = 0.0f;
#pragma unroll
    for (int k = 0; k < 32; ++k) m = fmaxf(m, fabsf(to_f<T>(h[k])));
    const float s = m / 127.0f;
    const float inv = 1.0f / s;
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t v = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int q = s == 0.0f ? 0 : q_int(to_f<T>(h[4 * i + k]), inv, 127);
        v |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * k);
      }
      w[i] = v;
    }
    uint4* dst = reinterpret_cast<uint4*>(Q + j * K + b * 32);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    s_w[t] = s;
  }
}

}  // namespace qlin
