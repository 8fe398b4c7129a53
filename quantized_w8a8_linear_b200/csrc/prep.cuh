// prep.cuh -- HBM-bound kernels around the GEMM:
//   * k_outlier_flags: LLM.int8 outlier-column detection (any |x| > threshold
//     in the column, over every token of the call) into a bitmap, with the
//     last CTA compacting the bitmap into the ascending outlier list O, the
//     outlier count and per-word prefix counts;
//   * k_rowquant: per-row absmax (optionally excluding outlier columns),
//     scale, and int8 or E4M3 codes, plus the exact copy of the outlier
//     columns into X_O; it also quantises weights row by row;
//   * k_gather_wo: dequantised outlier weight columns
//     W_O[j,o] = dtype(fp32(Wq[j,O[o]]) * s_w[j]) (the weight.to(dtype) *
//     weight_scale rule of the Text-Encoder-FP8 page, "Format");
//   * k_fp8_static: per-tensor static E4M3 activation codes;
//   * k_absmax / k_fp8_tensor_quant / k_scale_from_absmax: max calibration and
//     per-tensor FP8 weights;
//   * k_int4_group_quant: int4 per-group weight codes and scales.
// Rows are read as 16-byte vectors of 8 elements (K % 8 == 0), coalesced
// across the threads of a CTA.
#pragma once
#include "common.cuh"

namespace qlin {

constexpr int PREP_THREADS = 128;

// 8 flags (bit e set iff |x_e| > thr) for one 16-byte vector of 8 elements.
template <typename T>
__device__ __forceinline__ uint32_t outlier_bits8(const uint4& u, float thr) {
  uint16_t h[8];
  unpack8(u, h);
  uint32_t m = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) m |= (fabsf(to_f<T>(h[e])) > thr ? 1u : 0u) << e;
  return m;
}

// Compaction of the outlier bitmap by one CTA of PREP_THREADS threads:
// wpre[w] = number of set bits in words [0, w); O lists the set columns in
// ascending order; *count = total. NW <= 8 * PREP_THREADS.
__device__ void compact_flags(const uint32_t* flags, int NW, int32_t* wpre, int32_t* O, int32_t* count) {
  __shared__ int warp_tot[PREP_THREADS / 32];
  const int tid = threadIdx.x;
  const int per = (NW + PREP_THREADS - 1) / PREP_THREADS;   // <= 8
  const int w0 = tid * per;
  uint32_t words[8];
  int local = 0;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int w = w0 + u;
    words[u] = (u < per && w < NW) ? __ldcg(flags + w) : 0u;
    local += __popc(words[u]);
  }
  // exclusive scan of `local` over the CTA
  const int lane = tid & 31, warp = tid >> 5;
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int base = 0;
  for (int i = 0; i < warp; ++i) base += warp_tot[i];
  int run = base + incl - local;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int w = w0 + u;
    if (u < per && w < NW) {
      wpre[w] = run;
      uint32_t bits = words[u];
      while (bits) {
        const int b = __ffs(bits) - 1;
        O[run++] = w * 32 + b;
        bits &= bits - 1;
      }
    }
  }
  if (tid == PREP_THREADS - 1) *count = run;
}

// grid: (ceil(KV / PREP_THREADS), ceil(M / rows_per_block)); KV = K / 8.
// flags and *done must be zero on entry.
template <typename T>
__global__ void __launch_bounds__(PREP_THREADS) k_outlier_flags(const T* __restrict__ X, int64_t M, int64_t K,
                                                              float thr, int rows_per_block, uint32_t* flags,
                                                              int32_t* wpre, int32_t* O, int32_t* count,
                                                              uint32_t* done) {
  const int64_t KV = K / 8;
  const int64_t v = static_cast<int64_t>(blockIdx.x) * PREP_THREADS + threadIdx.x;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_block;
  const int64_t r1 = min(M, r0 + rows_per_block);
  uint32_t mask = 0;
  if (v < KV) {
    const uint4* p = reinterpret_cast<const uint4*>(X + r0 * K) + v;
    int64_t r = r0;
    for (; r + 4 <= r1; r += 4) {
      const uint4 a = ld_nc_v4(p), b = ld_nc_v4(p + KV), c = ld_nc_v4(p + 2 * KV), d = ld_nc_v4(p + 3 * KV);
      mask |= outlier_bits8<T>(a, thr) | outlier_bits8<T>(b, thr) | outlier_bits8<T>(c, thr) |
              outlier_bits8<T>(d, thr);
      p += 4 * KV;
    }
    for (; r < r1; ++r, p += KV) mask |= outlier_bits8<T>(ld_nc_v4(p), thr);
  }
  // four consecutive threads hold the 32 columns of one bitmap word
  uint32_t w = mask << ((v & 3) * 8);
  w |= __shfl_xor_sync(0xffffffffu, w, 1);
  w |= __shfl_xor_sync(0xffffffffu, w, 2);
  if ((v & 3) == 0 && v < KV && w != 0u) atomicOr(flags + (v >> 2), w);

  // the last CTA to finish compacts the bitmap
  __shared__ int is_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(done, 1u) == gridDim.x * gridDim.y - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  compact_flags(flags, static_cast<int>((K + 31) / 32), wpre, O, count);
}

// One CTA per row. CODE 0: int8 (QMAX 127), CODE 1: E4M3 (QMAX 448).
// SCALE_BF16: the stored scale is bf16(absmax / QMAX) and the codes use that
// rounded value (the [out,1] bf16 weight scales of the Text-Encoder-FP8 page).
// OUTL: columns flagged in `flags` are excluded from the absmax, get code 0,
// and are copied exactly into X_O[row, o] (o = rank of the column in O), the
// row zero-padded to a multiple of 8 outlier columns.
template <typename T, int V, int CODE, bool SCALE_BF16, bool OUTL>
__global__ void __launch_bounds__(PREP_THREADS) k_rowquant(const T* __restrict__ X, int64_t K, uint8_t* __restrict__ Q,
                                                         float* __restrict__ s_f32, uint16_t* __restrict__ s_bf16,
                                                         const uint32_t* __restrict__ flags,
                                                         const int32_t* __restrict__ wpre,
                                                         const int32_t* __restrict__ count_ptr,
                                                         uint16_t* __restrict__ X_O, int64_t ostride) {
  __shared__ float red[PREP_THREADS / 32];
  const int64_t row = blockIdx.x;
  const int64_t KV = K / 8;
  const uint4* xr = reinterpret_cast<const uint4*>(X + row * K);
  uint4 vals[V];
  uint32_t om[V];
  float amax = 0.0f;
#pragma unroll
  for (int u = 0; u < V; ++u) {
    const int64_t idx = threadIdx.x + static_cast<int64_t>(u) * PREP_THREADS;
    om[u] = 0u;
    if (idx < KV) {
      vals[u] = ld_nc_v4(xr + idx);
      if constexpr (OUTL) om[u] = (__ldg(flags + (idx >> 2)) >> ((idx & 3) * 8)) & 0xFFu;
      uint16_t h[8];
      unpack8(vals[u], h);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (!((om[u] >> e) & 1u)) amax = fmaxf(amax, fabsf(to_f<T>(h[e])));
    } else {
      vals[u] = make_uint4(0, 0, 0, 0);
    }
  }
  amax = warp_max(amax);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < PREP_THREADS / 32; ++w) amax = fmaxf(amax, red[w]);

  constexpr float QMAX = CODE == 0 ? 127.0f : 448.0f;
  float s = amax / QMAX;
  if constexpr (SCALE_BF16) {
    const uint16_t sb = __bfloat16_as_ushort(__float2bfloat16_rn(s));
    s = __uint_as_float(static_cast<uint32_t>(sb) << 16);
    if (threadIdx.x == 0) s_bf16[row] = sb;
  } else {
    if (threadIdx.x == 0) s_f32[row] = s;
  }
  const float inv = 1.0f / s;
  const bool zero = (s == 0.0f);

#pragma unroll
  for (int u = 0; u < V; ++u) {
    const int64_t idx = threadIdx.x + static_cast<int64_t>(u) * PREP_THREADS;
    if (idx < KV) {
      uint16_t h[8];
      unpack8(vals[u], h);
      uint32_t lo = 0, hi = 0;
      if constexpr (CODE == 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int q = (zero || ((om[u] >> e) & 1u)) ? 0 : q_int(to_f<T>(h[e]), inv, 127);
          const uint32_t b = static_cast<uint32_t>(q) & 0xFFu;
          if (e < 4) lo |= b << (8 * e);
          else hi |= b << (8 * (e - 4));
        }
      } else {
        float t[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) t[e] = q_e4m3_in(to_f<T>(h[e]), inv);
        lo = e4m3x2(t[0], t[1]) | (e4m3x2(t[2], t[3]) << 16);
        hi = e4m3x2(t[4], t[5]) | (e4m3x2(t[6], t[7]) << 16);
        if (zero) lo = hi = 0u;
      }
      *reinterpret_cast<uint2*>(Q + row * K + idx * 8) = make_uint2(lo, hi);
      if constexpr (OUTL) {
        if (om[u]) {
          const uint32_t word = __ldg(flags + (idx >> 2));
          const int base = __ldg(wpre + (idx >> 2));
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if ((om[u] >> e) & 1u) {
              const int bit = static_cast<int>((idx & 3) * 8) + e;
              const int o = base + __popc(word & ((1u << bit) - 1u));
              X_O[row * ostride + o] = h[e];
            }
          }
        }
      }
    }
  }
  if constexpr (OUTL) {
    const int cnt = __ldg(count_ptr);
    const int pad = (cnt + 7) & ~7;
    for (int o = cnt + threadIdx.x; o < pad; o += PREP_THREADS) X_O[row * ostride + o] = 0;
  }
}

// W_O[j,o] = dtype(fp32(Wq[j,O[o]]) * s_w[j]) for o < count, 0 up to the
// next multiple of 8. Grid-stride over N * pad.
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
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t j = t / pad;
    const int o = static_cast<int>(t - j * pad);
    float val = 0.0f;
    if (o < cnt) val = __fmul_rn(static_cast<float>(Wq[j * K + __ldg(O + o)]), __ldg(s_w + j));
    W_O[j * ostride + o] = from_f<T>(val);
  }
}

// Static per-tensor E4M3 codes: Xq = e4m3(x * (1 / *x_scale)); all-zero
// codes if the scale is 0. Grid-stride over 8-element vectors.
template <typename T>
__global__ void __launch_bounds__(256) k_fp8_static(const T* __restrict__ X, int64_t nvec,
                                                  const float* __restrict__ x_scale, uint8_t* __restrict__ Q) {
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
// columns [4l, 4l+4) of the group; s = absmax / 7; codes in [-7, 7]; byte
// k/2 holds column k even in the low nibble, k odd in the high nibble.
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
  uint32_t packed = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int q = (s == 0.0f) ? 0 : q_int(to_f<T>(h[e]), inv, 7);
    packed |= (static_cast<uint32_t>(q) & 0xFu) << (4 * e);
  }
  *reinterpret_cast<uint16_t*>(Q4 + j * (K / 2) + g * (G / 2) + lane * 2) = static_cast<uint16_t>(packed);
  if (lane == 0) s_w[j * ng + g] = s;
}

}  // namespace qlin
