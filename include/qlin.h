/*
 * qlin.h -- C ABI of libqlin.so: one quantized linear layer, Y = X W^T, on
 * NVIDIA B200 (sm_100a), in the four weight/activation formats the
 * Qwen-Image-2.1 model-card pages use:
 *
 *   - LLM.int8 mixed-precision decomposition (ixim/Image21-INT8, section
 *     "Quantization": bitsandbytes LLM.int8, outlier threshold 6.0, outlier
 *     handling in floating point) with vector-wise int8: per-token absmax/127
 *     activation scales, per-output-channel absmax/127 weight scales, int32
 *     accumulation, dequant by the outer product of the two scale vectors;
 *   - FP8 E4M3 W8A8 with static per-tensor fp32 weight_scale and input_scale
 *     (Darkstar-Qwen-Image-2.1-Base-ModelOpt-FP8, section "Precision map");
 *   - FP8 E4M3 weights with one bf16 scale per output channel, shape [out,1],
 *     and dynamic per-token FP8 activations (Qwen-Image-2.1-Text-Encoder-FP8,
 *     section "Format"; dequant rule weight.to(bf16) * weight_scale);
 *   - int4 per-group weights with int8 activations and fp32 scales
 *     (Qwen-Image-fni8, section "Format"), group 128 along K.
 *
 * Conventions shared by every entry point:
 *   - Shapes: X is [M,K] row-major, W is [N,K] row-major (K contiguous), Y is
 *     [M,N] row-major. M = tokens, K = in-features, N = out-features.
 *   - Every data pointer is a DEVICE pointer unless its comment says "host".
 *     The caller owns all memory. The library allocates and frees no device
 *     memory and never synchronises the stream inside a forward: all work is
 *     enqueued on `stream` (a cudaStream_t passed as void*; NULL = the legacy
 *     default stream).
 *   - Alignment: every device pointer must be 16-byte aligned; K must be a
 *     positive multiple of 16 (of 128 for the int4 format) and at most 32768.
 *     M and N are arbitrary (M = 0 or N = 0 is a no-op that returns QLIN_OK).
 *   - Scratch: entry points that need scratch take `workspace` (device) and
 *     `ws_bytes`; qlin_workspace_bytes() gives the size. A workspace may be
 *     reused by calls that are ordered on one stream, not by calls that may
 *     overlap.
 *   - dtype of X, bias and Y: QLIN_F16 or QLIN_BF16 (all three the same).
 *     bias is nullable ([N]).
 *   - Errors: every call returns a qlin_status; nothing crosses the ABI as an
 *     exception. Argument errors are detected on the host before anything is
 *     enqueued. A device-side wait that runs out of time (QLIN_ERR_TIMEOUT)
 *     is recorded in a device status word that qlin_get_device_status()
 *     reads. qlin_last_error_string() describes the last error of the
 *     calling thread.
 *   - Thread safety: calls from several host threads are safe; the error
 *     string is thread-local.
 */
#ifndef QLIN_H
#define QLIN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QLIN_API __attribute__((visibility("default")))
#else
#define QLIN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum qlin_status {
    QLIN_OK = 0,
    QLIN_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad enum            */
    QLIN_ERR_UNSUPPORTED = 2,   /* shape / device outside what the kernels support  */
    QLIN_ERR_ALIGNMENT = 3,     /* pointer not 16-byte aligned, K not a multiple    */
    QLIN_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required       */
    QLIN_ERR_CUDA = 5,          /* a CUDA runtime call or a launch failed           */
    QLIN_ERR_TIMEOUT = 6        /* a bounded device-side wait ran out of time       */
} qlin_status;

typedef enum qlin_dtype { QLIN_F16 = 0, QLIN_BF16 = 1 } qlin_dtype;

/* Weight formats (offline quantisation, qlin_quantize_weight). */
typedef enum qlin_wmode {
    QLIN_W_INT8_ROW = 0,     /* Wq int8 [N,K];  w_scale fp32 [N]   = absmax_k|W[j,k]| / 127          */
    QLIN_W_FP8_TENSOR = 1,   /* Wq e4m3 [N,K];  w_scale fp32 [1]   = absmax|W| / 448                 */
    QLIN_W_FP8_CHANNEL = 2,  /* Wq e4m3 [N,K];  w_scale bf16 [N,1] = bf16(absmax_k|W[j,k]| / 448)    */
    QLIN_W_INT4_G128 = 3,    /* Wq uint8 [N,K/2]: each block of 32 consecutive k in 16 bytes, byte b
                                holding element b (low nibble) and element b+16 (high nibble), two's
                                complement, codes in [-7,7]; w_scale fp32 [N,K/128] = absmax/7      */
    QLIN_W_INT8_BLOCK32 = 4, /* Wq int8 [N,K]; w_scale fp32 [N,K/32] = absmax of each run of 32
                                weights of a row / 127 (K % 32 == 0)                               */
    QLIN_W_NVFP4 = 5         /* Wq uint8 [N,K/2]: E2M1 codes packed like QLIN_W_INT4_G128 (blocks
                                of 32 k in 16 bytes, byte b: element b low nibble, b+16 high);
                                w_scale: E4M3 block scales uint8 [N,K/16] (one per 16 weights of
                                a row), then at byte offset round_up(N*K/16, 16) the fp32 tensor
                                scale s_t: 16-byte aligned, round_up(N*K/16,16) + 4 bytes.
                                s_t = absmax(W)/2688, s_b = e4m3(absmax(block)/(6 s_t)),
                                code = e2m1_rne(w/(s_b s_t)), saturating at 6. K % 64 == 0.
                                Workspace: QLIN_OP_QUANTIZE_WEIGHT.                               */
} qlin_wmode;

/* Operations whose scratch size qlin_workspace_bytes() reports. */
typedef enum qlin_op {
    QLIN_OP_INT8_OUTLIER = 0,   /* qlin_int8_outlier_forward                        */
    QLIN_OP_FP8 = 1,            /* qlin_fp8_forward                                 */
    QLIN_OP_W4A8 = 2,           /* qlin_w4a8_forward                                */
    QLIN_OP_QUANTIZE_WEIGHT = 3,/* qlin_quantize_weight and qlin_calibrate_input_scale */
    QLIN_OP_INT8_PREP = 4,      /* qlin_int8_prep                                   */
    QLIN_OP_INT8_BLOCK = 5,     /* qlin_int8_block_forward                          */
    QLIN_OP_FP8_GEMM = 6        /* qlin_fp8_gemm's optional scratch                 */
} qlin_op;

/* Bytes of device scratch `op` needs for an [M,K] x [N,K]^T problem (0 when
 * none is needed). Host-only, never fails; returns 0 for invalid sizes. */
QLIN_API size_t qlin_workspace_bytes(qlin_op op, int64_t M, int64_t N, int64_t K);

/* Offline weight quantisation (not part of the timed forward).
 * W: [N,K] in `wdt`. Wq / w_scale: layouts listed with qlin_wmode. Codes are
 * round-half-even (int8/int4, clamped to +-127 / +-7) or round-to-nearest-even
 * saturating E4M3 (max 448), computed as code(w * (1/s)) with every step in
 * IEEE fp32. workspace: qlin_workspace_bytes(QLIN_OP_QUANTIZE_WEIGHT, 0, N, K)
 * bytes (only QLIN_W_FP8_TENSOR uses it). */
QLIN_API qlin_status qlin_quantize_weight(const void *W, qlin_dtype wdt, int64_t N, int64_t K,
                                 qlin_wmode mode, void *Wq, void *w_scale,
                                 void *workspace, size_t ws_bytes, void *stream);

/* Max calibration of a static FP8 input scale (Darkstar ModelOpt-FP8 page,
 * "Provenance": calibration with the max algorithm):
 * *x_scale (device fp32) = absmax(X) / 448 over a calibration batch X [M,K].
 * workspace: qlin_workspace_bytes(QLIN_OP_QUANTIZE_WEIGHT, M, 0, K) bytes. */
QLIN_API qlin_status qlin_calibrate_input_scale(const void *X, qlin_dtype xdt, int64_t M, int64_t K,
                                       float *x_scale, void *workspace, size_t ws_bytes,
                                       void *stream);

/* LLM.int8 forward (ixim/Image21-INT8, "Quantization"):
 *   O       = { k : |X[i,k]| > threshold for some token i of this call }
 *   s_x[i]  = max_{k not in O} |X[i,k]| / 127;  Xq = rne(X / s_x), 0 on O
 *   C       = Xq Wq^T (int8 x int8 -> int32, tcgen05 kind::i8)
 *   F       = X[:,O] W_O^T, W_O = dtype(fp32(Wq[:,O]) * w_scale)  (the
 *             floating-point outlier part, dequant rule weight.to(dtype)*scale)
 *   Y       = dtype(C * s_x[i] * w_scale[j] + F + bias[j]).
 * threshold <= 0 or +inf turns the decomposition off (pure vector-wise int8).
 * Wq int8 [N,K], w_scale fp32 [N] from qlin_quantize_weight(QLIN_W_INT8_ROW).
 * Y [M,N] in xdt. workspace: qlin_workspace_bytes(QLIN_OP_INT8_OUTLIER, M, N, K).
 * The number of outlier columns stays on the device (no host sync). */
QLIN_API qlin_status qlin_int8_outlier_forward(const void *X, qlin_dtype xdt, int64_t M, int64_t K,
                                      const int8_t *Wq, const float *w_scale, int64_t N,
                                      float threshold, const void *bias, void *Y,
                                      void *workspace, size_t ws_bytes, void *stream);

/* The two stages of qlin_int8_outlier_forward, for callers that schedule
 * (or time) them separately; the forward is exactly prepare then gemm on the
 * same stream and workspace.
 *   prepare: outlier detection, activation codes/scales, X_O and W_O
 *            (HBM-bound kernels), all written into `workspace`;
 *   gemm:    the tcgen05 int8 GEMM with the fused dequant + outlier + bias
 *            epilogue, reading what prepare left in `workspace`. */
QLIN_API qlin_status qlin_int8_outlier_prepare(const void *X, qlin_dtype xdt, int64_t M, int64_t K,
                                      const int8_t *Wq, const float *w_scale, int64_t N,
                                      float threshold, void *workspace, size_t ws_bytes,
                                      void *stream);
QLIN_API qlin_status qlin_int8_outlier_gemm(qlin_dtype xdt, int64_t M, int64_t K, const int8_t *Wq,
                                   const float *w_scale, int64_t N, const void *bias, void *Y,
                                   void *workspace, size_t ws_bytes, void *stream);

/* FP8 E4M3 W8A8 forward.
 *   wmode QLIN_W_FP8_TENSOR: w_scale -> fp32 scalar (ModelOpt-FP8 page,
 *     "Precision map"); wmode QLIN_W_FP8_CHANNEL: w_scale -> bf16 [N]
 *     (Text-Encoder-FP8 page, "Format").
 *   x_scale -> fp32 scalar: static per-tensor input scale, Xq = e4m3(X / x_scale)
 *     (required with QLIN_W_FP8_TENSOR);
 *   x_scale == NULL: dynamic per-token scales s_x[i] = absmax_i / 448
 *     (required with QLIN_W_FP8_CHANNEL). Other pairings return
 *     QLIN_ERR_UNSUPPORTED: the pages pair the scales this way.
 *   acc = sum_k dec(Xq) dec(Wq) (fp32 accumulate, tcgen05 kind::f8f6f4),
 *   Y = dtype(acc * s_x * s_w + bias).
 * workspace: qlin_workspace_bytes(QLIN_OP_FP8, M, N, K). */
QLIN_API qlin_status qlin_fp8_forward(const void *X, qlin_dtype xdt, int64_t M, int64_t K,
                             const uint8_t *Wq, const void *w_scale, qlin_wmode wmode,
                             int64_t N, const float *x_scale, const void *bias, void *Y,
                             void *workspace, size_t ws_bytes, void *stream);

/* The GEMM stage of qlin_fp8_forward: Xq e4m3 [M,K] and (dynamic mode) s_x
 * fp32 [M] as qlin_fp8_prep wrote them. Same wmode / x_scale rules.
 * workspace: NULL (whole output tiles per CTA), or a 16-byte aligned buffer of
 * qlin_workspace_bytes(QLIN_OP_FP8_GEMM, M, N, K) bytes, owned by the caller
 * and not shared with a concurrent call: the GEMM may then split tiles along K
 * across CTAs (stream-K), with fp32 partial sums added in a fixed order, so
 * the output does not depend on timing. When it cuts tiles, the call clears
 * the buffer's arrival counters itself (a memset on `stream`); no other
 * initialisation. */
QLIN_API qlin_status qlin_fp8_gemm(qlin_dtype xdt, int64_t M, int64_t K, const uint8_t *Xq,
                          const float *s_x, const uint8_t *Wq, const void *w_scale,
                          qlin_wmode wmode, int64_t N, const float *x_scale, const void *bias,
                          void *Y, void *workspace, size_t ws_bytes, void *stream);

/* NVFP4 weight-only linear (a reading of the release format the Darkstar
 * ModelOpt-FP8 page names; the page gives no layout): weights from
 * qlin_quantize_weight(QLIN_W_NVFP4), bf16 activations as they are:
 *   W_deq[j,k] = e2m1(code[j,k]) * e4m3(s_b[j,k/16])   (exact in bf16)
 *   Y = bf16( s_t * sum_k X[i,k] * W_deq[j,k] + bias[j] ), fp32 accumulation.
 * The weight is dequantised tile by tile in shared memory and contracted with
 * tcgen05 kind::f16 (bf16). X bf16 [M,K], K % 64 == 0; Y bf16 [M,N]. */
QLIN_API qlin_status qlin_nvfp4_weight_only_forward(const void *X, qlin_dtype xdt, int64_t M, int64_t K,
                                           const uint8_t *Wq, const void *w_scale, int64_t N,
                                           const void *bias, void *Y, void *stream);

/* W4A8 forward (Qwen-Image-fni8 page, "Format": int4 per-group weights,
 * int8 activations, fp32 scales; group 128 along K):
 *   activations: per-token int8, s_x[i] = absmax_i / 127 (no outlier split);
 *   C_g = sum over the 128 columns of group g of Xq * Wq4 (int32, exact; the
 *         int4 weights are unpacked to int8 (as 16 * code) in shared memory
 *         and contracted with tcgen05 kind::i8, one TMEM accumulator per
 *         group);
 *   Y   = dtype(s_x[i] * sum_g w_scale[j,g] * C_g + bias[j]), the group sum in
 *         fp32 in ascending g.
 * Wq4 uint8 [N, K/2] and w_scale fp32 [N, K/128] from
 * qlin_quantize_weight(QLIN_W_INT4_G128). K must be a multiple of 128.
 * workspace: qlin_workspace_bytes(QLIN_OP_W4A8, M, N, K). */
QLIN_API qlin_status qlin_w4a8_forward(const void *X, qlin_dtype xdt, int64_t M, int64_t K,
                              const uint8_t *Wq4, const float *w_scale, int64_t N,
                              const void *bias, void *Y, void *workspace, size_t ws_bytes,
                              void *stream);

/* The activation stage of qlin_w4a8_forward: per-token int8 codes Xq [M,K]
 * (round-half-even of X * (1/s_x), IEEE fp32) and fp32 scales s_x [M] =
 * absmax_i / 127, written to caller memory; one HBM-bound kernel. */
QLIN_API qlin_status qlin_w4a8_prep(const void *X, qlin_dtype xdt, int64_t M, int64_t K, int8_t *Xq,
                           float *s_x, void *stream);

/* The GEMM stage of qlin_w4a8_forward, on int8 codes Xq [M,K] and fp32 s_x [M]
 * (qlin_w4a8_prep, or qlin_int8_prep with the threshold off, writes them). */
QLIN_API qlin_status qlin_w4a8_gemm(qlin_dtype xdt, int64_t M, int64_t K, const int8_t *Xq,
                           const float *s_x, const uint8_t *Wq4, const float *w_scale,
                           int64_t N, const void *bias, void *Y, void *stream);

/* Unquantised 16-bit linear, for the layers a model keeps in floating point
 * (Image21-Turbo-OrbitQuant-W4A4 page, "What 4-bit breaks here and what stays
 * in fp16": the projections that write or cancel the massive activations stay
 * in fp16 while the rest are quantised):
 *   Y = dtype(X W^T + bias), X [M,K], W [N,K], bias [N] and Y [M,N] all in
 *   xdt (QLIN_F16 or QLIN_BF16); products exact, fp32 accumulation in the
 *   tensor cores (tcgen05 kind::f16), one rounding to xdt at the end.
 * No workspace. Same shape and alignment rules as the other forwards. */
QLIN_API qlin_status qlin_fp_linear_forward(const void *X, qlin_dtype xdt, int64_t M, int64_t K, const void *W,
                                   int64_t N, const void *bias, void *Y, void *stream);

/* Weight-only FP8 linear (Qwen-Image-2.1-Text-Encoder-FP8 page, "Format": the
 * E4M3 weights and their bf16 [out,1] scales are consumed as
 * weight.to(bf16) * weight_scale, the activations are not quantised):
 *   W_deq[j,k] = bf16(decode(Wq[j,k]) * w_scale[j])  (one rounding: the fp32
 *                product of the 4-bit and 8-bit significands is exact)
 *   Y = bf16(X W_deq^T + bias), fp32 accumulation (tcgen05 kind::f16).
 * W_deq is formed tile by tile in shared memory and never written out.
 * X, bias and Y are bf16 (xdt must be QLIN_BF16: the tensor core multiplies
 * operands of one type, and the rule dequantises to bf16; QLIN_ERR_UNSUPPORTED
 * otherwise). Wq e4m3 [N,K] and w_scale bf16 [N] as qlin_quantize_weight
 * (QLIN_W_FP8_CHANNEL) writes them. No workspace. */
QLIN_API qlin_status qlin_fp8_weight_only_forward(const void *X, qlin_dtype xdt, int64_t M, int64_t K,
                                         const uint8_t *Wq, const void *w_scale, int64_t N,
                                         const void *bias, void *Y, void *stream);

/* Block-scaled int8 linear (Qwen-Image-2.1-Text-Encoder-FP8 page, "How it was
 * tested": GGUF Q8_0 stores int8 weight codes with one scale per run of 32
 * weights of a row and was measured closest to bf16):
 *   activations: per-token int8, s_x[i] = absmax_i / 127, as in W4A8 mode;
 *   weights: Wq int8 [N,K], w_scale fp32 [N,K/32] from
 *            qlin_quantize_weight(QLIN_W_INT8_BLOCK32);
 *   Y = dtype(s_x[i] * sum_b w_scale[j,b] * C_b[i,j] + bias[j]),
 *   C_b = sum over the 32 columns of block b of Xq * Wq.
 * The kernel applies each weight's block scale before the sum: the weight
 * tile is dequantised on chip to fp16 (q * s rounded to 11 significant bits),
 * the activation codes enter as exact fp16 values, and tcgen05 kind::f16
 * accumulates in fp32, so the result is within 2^-11 relative per weight of
 * the exact int32 block sums (the per-block int32 partials are not formed).
 * K % 32 == 0. workspace: qlin_workspace_bytes(QLIN_OP_INT8_BLOCK, M, N, K). */
QLIN_API qlin_status qlin_int8_block_forward(const void *X, qlin_dtype xdt, int64_t M, int64_t K,
                                    const int8_t *Wq, const float *w_scale, int64_t N, const void *bias,
                                    void *Y, void *workspace, size_t ws_bytes, void *stream);

/* ---------------- parity exports: the same kernels, intermediates written out ------ */

/* The activation stage of qlin_int8_block_forward: per-token int8 codes
 * (round-half-even of X * (1/s_x), IEEE fp32) written as fp16 values Xq16
 * [M,K] (exact), and s_x fp32 [M] = absmax_i / 127. */
QLIN_API qlin_status qlin_int8_block_prep(const void *X, qlin_dtype xdt, int64_t M, int64_t K, void *Xq16,
                                 float *s_x, void *stream);

/* LLM.int8 activation prep alone. Outputs: Xq int8 [M,K]; s_x fp32 [M];
 * flags uint32 [ceil(K/32)] (bit k%32 of word k/32 set iff column k is an
 * outlier); O int32 [K] (ascending outlier columns, first *count valid);
 * count int32 [1]; X_O [M, ostride] in xdt (X[:,O], zero-padded to a multiple
 * of 8 columns, and to 16 columns when 1 <= count <= 16; ostride >=
 * round_up(K,8), a multiple of 8).
 * workspace: qlin_workspace_bytes(QLIN_OP_INT8_PREP, M, 0, K). */
QLIN_API qlin_status qlin_int8_prep(const void *X, qlin_dtype xdt, int64_t M, int64_t K, float threshold,
                           int8_t *Xq, float *s_x, uint32_t *flags, int32_t *O, int32_t *count,
                           void *X_O, int64_t ostride, void *workspace, size_t ws_bytes,
                           void *stream);

/* Outlier weight columns: W_O[j,o] = dtype(fp32(Wq[j,O[o]]) * w_scale[j]) for
 * o < *count, zero up to the next multiple of 8; W_O is [N, ostride] in dt. */
QLIN_API qlin_status qlin_outlier_weights(const int8_t *Wq, const float *w_scale, int64_t N, int64_t K,
                                 const int32_t *O, const int32_t *count, qlin_dtype dt,
                                 void *W_O, int64_t ostride, void *stream);

/* The int32 accumulator of qlin_int8_outlier_gemm, written out instead of Y:
 * C[M,N] = sum over non-outlier columns k of Xq[m,k] * Wq[n,k], exact, from
 * the workspace a qlin_int8_outlier_prepare call on the same stream filled
 * (ixim/Image21-INT8, "Quantization": the int8 part of the decomposition).
 * The same kernel as the fused forward with its output stage replaced: the
 * MMA sums all K columns and the epilogue subtracts the outlier columns'
 * products in int32. */
QLIN_API qlin_status qlin_int8_outlier_gemm_i32(int64_t M, int64_t K, const int8_t *Wq, int64_t N,
                                       int32_t *C, void *workspace, size_t ws_bytes, void *stream);

/* Raw int8 GEMM: C[M,N] int32 = Xq[M,K] Wq[N,K]^T, exact (|C| <= K*127^2). */
QLIN_API qlin_status qlin_int8_gemm_i32(const int8_t *Xq, const int8_t *Wq, int64_t M, int64_t N,
                               int64_t K, int32_t *C, void *stream);

/* The int32 group partials C_g [M,N] of one group (0 <= group < K/128) as the
 * W4A8 GEMM computes them (parity export; the same kernel, its output stage
 * replaced by the export). */
QLIN_API qlin_status qlin_w4a8_group_i32(const int8_t *Xq, const uint8_t *Wq4, int64_t M, int64_t N,
                                int64_t K, int group, int32_t *C, void *stream);

/* FP8 activation prep alone: Xq e4m3 [M,K]; s_x fp32 [M] (dynamic mode,
 * x_scale == NULL; ignored and may be NULL in static mode). */
QLIN_API qlin_status qlin_fp8_prep(const void *X, qlin_dtype xdt, int64_t M, int64_t K,
                          const float *x_scale, uint8_t *Xq, float *s_x, void *stream);

/* The E4M3 conversion every FP8 kernel uses (cvt.rn.satfinite.e4m3x2.f32),
 * applied to n fp32 values t: codes[i] = round-to-nearest-even E4M3 of t[i],
 * saturating to +-448 (Text-Encoder-FP8 page, "How it was tested": 3-bit
 * mantissa). Parity export; n >= 0, no alignment requirement. */
QLIN_API qlin_status qlin_e4m3_encode_f32(const float *t, uint8_t *codes, int64_t n, void *stream);

/* ---------------- LLM.int8 forward with built-in scratch ------------------------------ */

/* Size of the library's built-in scratch array (64 MiB per device). */
#define QLIN_NOALLOC_SCRATCH_BYTES (64LL * 1024 * 1024)

/* The same LLM.int8 forward as qlin_int8_outlier_forward, for callers that
 * cannot allocate device memory where they run the layer (for example a
 * plugin whose host framework owns all device allocations, or a
 * latency-critical path that must not call cudaMalloc, which can synchronise
 * the device). It takes no workspace: its scratch is a file-scope device
 * array of QLIN_NOALLOC_SCRATCH_BYTES inside the library, which every GPU
 * that loads the library holds until the process exits. The model-card pages
 * have no counterpart of this entry point.
 *   - Its scratch holds the workspace layout of qlin_int8_outlier_forward
 *     without the stream-K partial slots (the GEMM then takes whole tiles;
 *     the results are the same). That is about M*K bytes of codes plus
 *     2*(M+N)*round_up(K,8) bytes for the worst-case outlier columns X_O and
 *     W_O: M = 2048, K = N = 4096 needs 56.3 MiB and fits; the 1024^2 DiT
 *     linears (M = 4352, K or N = 12288) do not. Larger shapes are rejected
 *     with QLIN_ERR_UNSUPPORTED and a message; nothing is enqueued. Arguments
 *     are otherwise validated as in qlin_int8_outlier_forward.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - Every call uses the same array and finds the previous call's contents
 *     in it; the parts that must start at zero are cleared on the call's
 *     stream. Calls ordered on one stream are safe; calls that may overlap on
 *     the GPU (different streams or host threads) race on the array. */
QLIN_API qlin_status qlin_int8_outlier_forward_noalloc(const void *X, qlin_dtype xdt, int64_t M, int64_t K,
                                              const int8_t *Wq, const float *w_scale, int64_t N,
                                              float threshold, const void *bias, void *Y,
                                              void *stream);

/* ---------------- status ------------------------------------------------------------ */

/* Reads (and with reset != 0 clears) the device status word of the current
 * device into *status (host pointer): QLIN_OK, or QLIN_ERR_TIMEOUT if a
 * kernel gave up on a bounded wait. Synchronises the device. */
QLIN_API qlin_status qlin_get_device_status(int32_t *status, int reset);

/* Sets the limit of every bounded device-side wait, in nanoseconds (default
 * 2e9). Synchronous; call it outside stream capture. */
QLIN_API qlin_status qlin_set_wait_timeout_ns(uint64_t ns);

/* Test switch of the failure path (the model-card pages have no counterpart):
 * with on != 0, every later launch of the int8 / FP8 / 16-bit GEMM first waits
 * on a barrier that nothing arrives on, so that its bounded wait runs out
 * after the wait limit (qlin_set_wait_timeout_ns). The kernel then records
 * QLIN_ERR_TIMEOUT in the device status word, stops its other roles, waits
 * (up to max(limit, 1 s)) for its own copies and MMAs in flight, frees its
 * TMEM and returns, leaving Y unwritten; later launches work normally once the
 * switch is off again. Off by default. Synchronous; call it outside stream
 * capture. */
QLIN_API qlin_status qlin_debug_inject_wait_timeout(int on);

/* Work schedule of the LLM.int8 GEMMs (qlin_int8_outlier_forward / _gemm /
 * _gemm_i32), process-wide, read at each launch:
 *   0  automatic (default): whole output tiles handed out round-robin, or
 *      stream-K when a cost model predicts a gain of 5% or more (few tiles
 *      over a long K: the split-K case);
 *   1  whole tiles only;
 *   2  stream-K whenever the shape has more than one k-block iteration in
 *      total, down to one iteration per CTA (exercises cut tiles; slow).
 * Under stream-K each CTA takes an equal contiguous range of the
 * tiles x k-blocks iterations; a tile cut between CTAs is summed from int32
 * partial accumulators in the workspace, so the int32 accumulator (and Y, for
 * the same tile width) is the same bit for bit under every schedule. No CTA
 * waits for another. QLIN_ERR_INVALID_ARG for another mode. */
QLIN_API qlin_status qlin_set_gemm_schedule(int mode);

/* Message for the last error returned on the calling thread ("" if none). */
QLIN_API const char *qlin_last_error_string(void);

/* ABI version of this header (major * 100 + minor). */
QLIN_API int qlin_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QLIN_H */
