/*
 * razer.h -- C ABI of the B200 (sm_100a) RaZeR hot path.
 *
 * RaZeR ("RaZeR: Pushing the Limits of NVFP4 Quantization with Redundant Zero
 * Remapping") keeps the NVFP4 layout -- 16-element blocks of FP4-E2M1 codes,
 * one FP8 block scale per block and one FP32 tensor scale -- and reuses two
 * redundancies: the FP4 code 0b1000 (-0) decodes to a per-block special value
 * v, and spare bits of the block-scale byte select v.
 *
 * Formats (razer_format):
 *   RAZER_FMT_WEIGHT  scale byte = meta[7:6] | E3M3[5:0] (bias 3, subnormals,
 *                     max 30); meta 0..3 selects v in {+5, -5, +8, -8}.
 *                     (RaZeR notes, 关键设计 1: weight scales narrowed to
 *                     E3M3 free 2 bits; 训练策略: V_w = {+-5, +-8}.)
 *   RAZER_FMT_ACT     scale byte = meta[7] | E4M3[6:0] (OCP E4M3, max 448);
 *                     meta 0..1 selects v in {+5, -5}.  (关键设计 1: the
 *                     activation scale keeps E4M3 and frees its sign bit.)
 *   RAZER_FMT_NVFP4   scale byte = E4M3[6:0], no remap: 0b1000 means 0.
 *                     Plain NVFP4, kept as an ablation of the remap.
 *
 * Layout (all row-major, blocks along K; K must be a multiple of 16):
 *   codes  [R, K/2]  uint8, element 2i in the low nibble of byte i
 *   scales [R, K/16] uint8
 *   ts     one float in DEVICE memory (the FP32 tensor scale)
 *   A weight matrix is W [N, K] (output features x input features); the
 *   products are y = W x per vector, Y = X W^T for matrices.
 *
 * Quantizer semantics (关键设计 2; gist.science summary 2.2): with
 *   ts   = amax(|X|) / (6 * S_max)            (S_max = 30 or 448; fp32)
 *   s    = nearest scale code to amax_b / (6*ts) (ties to the even code,
 *          saturating), decoded exactly
 *   xs   = x / (s * ts)                         (IEEE fp32, nearest-even)
 * each block picks v* = argmin_{v in V} || round(xs, Q_FP4 u {v}) - xs ||^2
 * (rounding to the nearest point, ties to the smaller magnitude; the squared
 * errors are compared exactly; ties go to the lowest meta index) and stores
 * the codes of round(xs, Q_FP4 u {v*}); every element that rounds to 0 is
 * coded 0b0000.  A block with scale code 0 (or ts <= 0) is all zeros.
 * Codes, scale bytes and meta bits are bit-exact against this definition.
 *
 * Conventions for every call:
 *   - All array pointers are DEVICE pointers owned by the caller; the library
 *     keeps none of them after the call returns and allocates nothing.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream) and
 *     never synchronise; they keep no global state and are thread-safe.
 *   - Argument errors are reported synchronously through the return value
 *     and nothing is launched.  A failed launch returns RAZER_ERR_CUDA.
 *   - Input, code, output and workspace pointers must be 16-byte aligned;
 *     scale pointers 4-byte aligned; a null pointer where one is required
 *     gives RAZER_ERR_INVALID_ARG; sizes that are negative, K % 16 != 0, or
 *     beyond a call's stated range give RAZER_ERR_SHAPE.
 */
#ifndef RAZER_H
#define RAZER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *razer_stream_t; /* same type as cudaStream_t */

typedef enum {
    RAZER_OK = 0,
    RAZER_ERR_INVALID_ARG = 1, /* null pointer, unknown enum value            */
    RAZER_ERR_SHAPE = 2,       /* negative size, K % 16 != 0, out of range      */
    RAZER_ERR_ALIGN = 3,       /* pointer alignment below the stated minimum    */
    RAZER_ERR_DTYPE = 4,       /* unsupported element type for this call        */
    RAZER_ERR_WORKSPACE = 5,   /* workspace smaller than razer_workspace_size() */
    RAZER_ERR_UNSUPPORTED = 6, /* valid request this build does not implement   */
    RAZER_ERR_TIMEOUT = 7,     /* a bounded device-side wait gave up            */
    RAZER_ERR_CUDA = 8         /* CUDA launch / runtime error                   */
} razer_status;

typedef enum { RAZER_F16 = 0, RAZER_BF16 = 1, RAZER_F32 = 2 } razer_dtype;

typedef enum {
    RAZER_FMT_WEIGHT = 0,
    RAZER_FMT_ACT = 1,
    RAZER_FMT_NVFP4 = 2,
    /* razer_quantize_weights only (accuracy ablation): FourOverSix -- NVFP4
     * encoding (decode it as RAZER_FMT_NVFP4), but each block is scaled so
     * that its amax maps to 6 or to 4, whichever leaves the smaller squared
     * error sum_j (x_j - q_j*d)^2 (double, element order; ties take 6).
     * Four Over Six summary page, 方法详解. */
    RAZER_FMT_FOUR_OVER_SIX = 3,
    /* razer_quantize_variant / razer_quant_error_variant only: the FP16 block
     * scale of the pages' kernel format (RaZeR notes, 关键设计 3) -- a 16-bit
     * scale word per block, s = RN_fp16(amax_b / 6) in bits 13..0 (saturating
     * at 0x3FFF), the meta in bits 15..14, no tensor scale (ts = 1). */
    RAZER_SCALE_F16 = 4
} razer_format;

typedef enum { RAZER_OP_GEMV = 0, RAZER_OP_GEMM = 1, RAZER_OP_GEMM_W4A4 = 2, RAZER_OP_GEMM_VARIANT = 3 } razer_op;

/*
 * razer_quantize_weights -- offline weight quantizer (RaZeR notes, 关键设计
 * 1-2: E3M3 block scale, 2 meta bits, per-block argmin over V_w).
 *   W             [N, K] input, in_dt = RAZER_F16 or RAZER_BF16
 *   codes         [N, K/2] output
 *   scales        [N, K/16] output
 *   tensor_scale  device float, output: ts = amax(|W|) / (6 * S_max); it is
 *                 also used as scratch for the amax during the call
 *   fmt           RAZER_FMT_WEIGHT, or RAZER_FMT_NVFP4 for the ablation
 * N >= 0, K >= 0 (an empty tensor writes ts = 0 and nothing else).
 */
razer_status razer_quantize_weights(const void *W, razer_dtype in_dt, int64_t N, int64_t K,
                                    uint8_t *codes, uint8_t *scales, float *tensor_scale,
                                    razer_format fmt, razer_stream_t stream);

/*
 * razer_quantize_weights_batch -- razer_quantize_weights on count matrices in
 * one call; matrix i gets exactly the codes, scales and ts a separate
 * razer_quantize_weights call would give it.  The amax pass of matrix i + 1
 * (bandwidth-bound) runs in the same kernel as the quantization of matrix i
 * (arithmetic-bound), so a batch streams closer to the HBM rate than the
 * separate calls.
 *   count          number of matrices (0: nothing is done)
 *   W, N, K        HOST arrays of count entries: device pointer of matrix i
 *                  ([N[i], K[i]], in_dt = RAZER_F16 or RAZER_BF16) and sizes
 *   codes, scales  HOST arrays of count device pointers ([N[i], K[i]/2] and
 *                  [N[i], K[i]/16] outputs)
 *   tensor_scales  DEVICE array of count floats, output: ts of each matrix
 *                  (also the amax scratch during the call)
 *   fmt            RAZER_FMT_WEIGHT or RAZER_FMT_NVFP4 (one format for all)
 * The host arrays are read before the call returns.  Each matrix is checked
 * like razer_quantize_weights' arguments; the first failure is returned and
 * nothing is launched.
 */
razer_status razer_quantize_weights_batch(int count, const void *const *W, razer_dtype in_dt,
                                          const int64_t *N, const int64_t *K, uint8_t *const *codes,
                                          uint8_t *const *scales, float *tensor_scales,
                                          razer_format fmt, razer_stream_t stream);

/*
 * razer_quantize_acts -- online activation quantizer (关键设计 1-2; the
 * "double quantization" of 训练策略 / gist.science 2.2: each block is
 * quantized once per candidate in V_a = {+5, -5} and the smaller error wins).
 *   X          [M, K] input, in_dt = RAZER_F16 or RAZER_BF16
 *   ts_in      device float or NULL.  Given: the tensor scale to use (static
 *              scaling).  NULL: ts is computed from amax(|X|) (dynamic).
 *   codes      [M, K/2] output;  scales [M, K/16] output
 *   ts_out     device float, output: the tensor scale used (may equal ts_in)
 *   meta_hist  device unsigned long long[4] or NULL.  Overwritten with
 *              [blocks choosing meta 0, blocks choosing meta 1, blocks where
 *              meta 0 strictly lowered the squared error, same for meta 1].
 *   fmt        RAZER_FMT_ACT, or RAZER_FMT_NVFP4 for the ablation
 */
razer_status razer_quantize_acts(const void *X, razer_dtype in_dt, int64_t M, int64_t K,
                                 const float *ts_in, uint8_t *codes, uint8_t *scales, float *ts_out,
                                 unsigned long long *meta_hist, razer_format fmt,
                                 razer_stream_t stream);

/*
 * razer_dequant -- decoder (关键设计 3: the special value replaces -0):
 *   out[r, k] = round_out( (q * s) * ts ),
 * q*s exact, one fp32 multiply by *ts, one rounding to out_dt (f16 / bf16 /
 * f32).  Bit-exact.  out is [R, K].
 */
razer_status razer_dequant(const uint8_t *codes, const uint8_t *scales, const float *ts,
                           razer_format fmt, int64_t R, int64_t K, void *out, razer_dtype out_dt,
                           razer_stream_t stream);

/*
 * razer_gemv -- W4A16 small-batch product (关键设计 3: weight-only kernels
 * that decode the remapped codes on the fly):
 *   y[b, n] = ts * sum_k x[b, k] * (q*s)[n, k],   1 <= B <= 32,
 * with fp32 accumulation.
 *   x          [B, K] activations, act_dt = RAZER_F16 or RAZER_BF16
 *   codes/scales/ts  a weight tensor [N, K] in format wfmt
 *   y          [B, N] output, out_dt = RAZER_F16, RAZER_BF16 or RAZER_F32
 *   workspace  device scratch of at least
 *              razer_workspace_size(RAZER_OP_GEMV, B, N, K) bytes (16-byte
 *              aligned), or NULL when that size is 0.  Contents on entry are
 *              ignored (it holds split-K partials while a call runs).
 * Any K % 16 == 0.  K % 256 == 0 with a 16-byte aligned scale pointer takes
 * the bulk-tensor (TMA) kernel -- one persistent CTA per SM plus a small
 * split-K reduction kernel launched as its programmatic dependent; other
 * K % 128 == 0 calls take a per-warp cp.async kernel and a reduction kernel;
 * K % 128 != 0 takes a row-per-thread kernel that decodes each block exactly
 * in fp32 (no workspace: razer_workspace_size returns 0).
 */
razer_status razer_gemv(const void *x, razer_dtype act_dt, int64_t B, const uint8_t *codes,
                        const uint8_t *scales, const float *ts, razer_format wfmt, int64_t N,
                        int64_t K, void *y, razer_dtype out_dt, void *workspace, size_t ws_bytes,
                        razer_stream_t stream);

/*
 * razer_gemm -- W4A16 large-M product on the tcgen05 tensor cores:
 *   Y[m, n] = ts * sum_k X[m, k] * (q*s)[n, k],   fp32 accumulation.
 *   X   [M, K] activations, act_dt = RAZER_BF16 or RAZER_F16; the decoded
 *       weights use the same 16-bit type (q*s is exact in both).
 *   Y   [M, N] output, out_dt = RAZER_BF16, RAZER_F16 or RAZER_F32
 *   workspace  device scratch of razer_workspace_size(RAZER_OP_GEMM, M, N, K)
 *              bytes (16-byte aligned; contents on entry ignored).  For
 *              M >= 1024 that is N * K * 2 bytes: the packed weights are
 *              decoded once into a 16-bit copy (exact q*s, the same type as
 *              X) and the tensor-core pipeline loads both operands by TMA.
 *              For smaller M it is 0 and the weights are decoded per CTA tile
 *              into shared memory (each weight once per 256 rows of X).
 *              When K is split, a further S * M * N * 4 bytes follow.  S =
 *              the number of 16384-long chunks K needs (one tensor-memory
 *              accumulator chain over a longer K loses precision), raised
 *              to min(SMs / tiles, K / 512) when the ceil(M/256) *
 *              ceil(N/256) output tiles cannot occupy the SMs.  The S splits
 *              run in parallel, each writes its scaled fp32 sum to its own
 *              [M, N] slice, and a reduction kernel adds the slices in split
 *              order (deterministic) and converts to out_dt.
 * Any K % 16 == 0 and any N, M.  K % 64 != 0 or N % 16 != 0 take the
 * decode-once path whatever M (workspace N * K * 2 bytes first): the
 * bulk-tensor copies zero-fill the last, partial k-step of both operands.
 */
razer_status razer_gemm(const void *X, razer_dtype act_dt, int64_t M, const uint8_t *codes,
                        const uint8_t *scales, const float *ts, razer_format wfmt, int64_t N,
                        int64_t K, void *Y, razer_dtype out_dt, void *workspace, size_t ws_bytes,
                        razer_stream_t stream);

/*
 * razer_gemv_batch -- several independent razer_gemv products in one call
 * (for example the projections of one layer that read the same activations):
 *   y_i[b, n] = ts_i * sum_k x_i[b, k] * (q*s)_i[n, k]   for i < count.
 * One activation type, weight format and output type for all problems.
 * Problems that razer_gemv would run on its bulk-tensor kernel (K % 256 == 0,
 * 16-byte aligned scales) share launches: their tiles are concatenated into
 * one stream-K pass per group of up to 8 problems with the same n-tile class
 * (B <= 8, B <= 16, B <= 32), so the pipeline fill, drain and split-K
 * reduction are paid once per group instead of once per product.  The other
 * problems run one by one after them.  Each y_i equals razer_gemv's result up
 * to the order of the fp32 partial sums.
 *   problems   HOST array of count razer_gemv_problem (device pointers in
 *              it, each argument as for razer_gemv), read during the call
 *   workspace  device scratch of razer_gemv_batch_workspace_size(count,
 *              problems) bytes (16-byte aligned; contents on entry ignored),
 *              or NULL when that size is 0
 * Errors: those of razer_gemv for the first problem that fails a check
 * (nothing is launched then); count < 0 or a NULL array -> INVALID_ARG.
 */
typedef struct {
    const void *x;         /* [B, K] activations */
    int64_t B;             /* 1 .. 32 */
    const uint8_t *codes;  /* [N, K/2] */
    const uint8_t *scales; /* [N, K/16] */
    const float *ts;       /* device */
    int64_t N, K;
    void *y;               /* [B, N] */
} razer_gemv_problem;

razer_status razer_gemv_batch(int count, const razer_gemv_problem *problems, razer_dtype act_dt,
                              razer_format wfmt, razer_dtype out_dt, void *workspace,
                              size_t ws_bytes, razer_stream_t stream);
size_t razer_gemv_batch_workspace_size(int count, const razer_gemv_problem *problems);

/*
 * razer_gemm_w4a4 -- W4A4 product of two RaZeR-packed operands (the
 * weight-activation kernels of the gist.science summary 2.3; the RaZeR notes,
 * 局限与展望, note that current Blackwell tensor cores run it only emulated):
 *   Y[m, n] = ts_a * ts_w * sum_k (q*s)_a[m, k] * (q*s)_w[n, k],  fp32 accumulation.
 *   codes_a, scales_a, ts_a, afmt   A [M, K] as razer_quantize_acts writes it
 *                                   (any format; RAZER_FMT_ACT or NVFP4 for activations)
 *   codes_w, scales_w, ts_w, wfmt   W [N, K] as razer_quantize_weights writes it
 *   Y          [M, N], out_dt = RAZER_F32, RAZER_F16 or RAZER_BF16
 *   workspace  razer_workspace_size(RAZER_OP_GEMM_W4A4, M, N, K) bytes
 *              (16-byte aligned, contents on entry ignored): both operands
 *              are decoded exactly to fp16 there (q*s*2^-bias is exact in
 *              fp16 for every code and scale of the three formats), the
 *              tcgen05 pipeline of razer_gemm multiplies them, and the
 *              epilogue applies ts_a * ts_w (one fp32 rounding) and the
 *              bias; K > 16384 runs in chunks as for razer_gemm.
 * Any K % 16 == 0 and any N (a partial last k-step is zero-filled as for
 * razer_gemm).  ts_a and ts_w are device floats.
 */
razer_status razer_gemm_w4a4(const uint8_t *codes_a, const uint8_t *scales_a, const float *ts_a,
                             razer_format afmt, int64_t M, const uint8_t *codes_w,
                             const uint8_t *scales_w, const float *ts_w, razer_format wfmt,
                             int64_t N, int64_t K, void *Y, razer_dtype out_dt, void *workspace,
                             size_t ws_bytes, razer_stream_t stream);

/*
 * razer_gemm_w4a4_online -- the online W4A4 path in one call: quantize the
 * activations X [M, K] (fp16/bf16) as razer_quantize_acts does (ts_in = NULL:
 * dynamic tensor scale; otherwise the given device scale) and multiply them
 * with the packed weights as razer_gemm_w4a4 does.  The activation quantizer
 * writes the decoded operand of the product directly (one pass over X; the
 * codes are not read back), so
 *   Y == razer_gemm_w4a4(razer_quantize_acts(X), W)   bit for bit.
 *   afmt            RAZER_FMT_ACT or RAZER_FMT_NVFP4
 *   codes_a, scales_a  optional outputs ([M, K/2], [M, K/16]); both NULL or
 *                   both set
 *   ts_a_out        device float, output: the activations' tensor scale
 *   meta_hist       optional, as for razer_quantize_acts
 *   W, Y, workspace as razer_gemm_w4a4 (razer_workspace_size(RAZER_OP_GEMM_W4A4, M, N, K))
 */
razer_status razer_gemm_w4a4_online(const void *X, razer_dtype x_dt, int64_t M, const float *ts_in,
                                    razer_format afmt, uint8_t *codes_a, uint8_t *scales_a,
                                    float *ts_a_out, unsigned long long *meta_hist,
                                    const uint8_t *codes_w, const uint8_t *scales_w,
                                    const float *ts_w, razer_format wfmt, int64_t N, int64_t K,
                                    void *Y, razer_dtype out_dt, void *workspace, size_t ws_bytes,
                                    razer_stream_t stream);

/*
 * razer_quant_error -- quantization error of a packed tensor (accuracy
 * ablations): *sse = sum over [R, K] of (X - q*s*ts)^2 in double (q*s*ts is
 * exact in double).  X is the tensor that was quantized (RAZER_F16 or
 * RAZER_BF16), codes/scales/ts its packed form in format fmt (a tensor
 * quantized with RAZER_FMT_FOUR_OVER_SIX is decoded as RAZER_FMT_NVFP4).  sse
 * is a device double, overwritten; partial sums meet in atomic adds, so its
 * last bits depend on the order the thread blocks finish in.
 */
razer_status razer_quant_error(const void *X, razer_dtype in_dt, int64_t R, int64_t K,
                               const uint8_t *codes, const uint8_t *scales, const float *ts,
                               razer_format fmt, double *sse, razer_stream_t stream);

/*
 * razer_quantize_variant / razer_quant_error_variant -- format variants for
 * accuracy studies (the block-size study of the RaZeR notes, 主实验, and the
 * per-model special-value choice of 训练策略): the RaZeR quantizer with a
 * block of `block` elements (16, 32, 64 or 128) and the special values
 * special_values[0..n_special) (host array; each a multiple of 0.5 with
 * magnitude in [2.5, 9.5] and not an E2M1 magnitude 3, 4 or 6; the
 * gist.science summary 2.2 gives the constraint).  scale_fmt RAZER_FMT_WEIGHT:
 * E3M3 scale, meta in bits 7..6 (n_special <= 4); RAZER_FMT_ACT or NVFP4:
 * E4M3 scale, meta in bit 7 (n_special <= 2); RAZER_SCALE_F16: the pages'
 * kernel format, 16-bit scale words (n_special <= 4, ts = 1); n_special = 0
 * is plain rounding.  Dynamic ts = amax / (6 * S_max).  codes [R, K/2]
 * (16-byte aligned), scales [R, K/block] bytes ([R, K/block] 16-bit words,
 * 2-byte aligned, for RAZER_SCALE_F16).  The decision per block is exact (the
 * candidates' squared-error differences are summed exactly).  The error
 * variant writes sum (X - q*s*ts)^2 (double) to the device double *sse.
 * razer_dequant_variant and razer_gemv_variant (below) decode these
 * tensors; the hot-path GEMV / GEMM calls read the 16-element formats only.
 */
razer_status razer_quantize_variant(const void *X, razer_dtype in_dt, int64_t R, int64_t K, int block,
                                    razer_format scale_fmt, const float *special_values,
                                    int n_special, uint8_t *codes, uint8_t *scales, float *ts_out,
                                    razer_stream_t stream);
razer_status razer_quant_error_variant(const void *X, razer_dtype in_dt, int64_t R, int64_t K,
                                       int block, razer_format scale_fmt,
                                       const float *special_values, int n_special,
                                       const uint8_t *codes, const uint8_t *scales, const float *ts,
                                       double *sse, razer_stream_t stream);

/*
 * razer_dequant_variant -- decoder of a razer_quantize_variant tensor (the
 * same block, scale_fmt and special values; RaZeR notes, 关键设计 3: the FP4
 * -0 code decodes to the special value the block's meta selects):
 *   out[r, k] = round_out( (q * s) * ts ),
 * q*s exact in binary32, one binary32 multiply by *ts, one rounding to out_dt
 * (f16 / bf16 / f32).  Bit-exact.  codes [R, K/2] (8-byte aligned); scales
 * as razer_quantize_variant writes them; out [R, K] (16-byte aligned).  A
 * meta value at or past n_special decodes the 0b1000 code to 0.
 */
razer_status razer_dequant_variant(const uint8_t *codes, const uint8_t *scales, const float *ts, int64_t R, int64_t K,
                                   int block, razer_format scale_fmt, const float *special_values, int n_special,
                                   void *out, razer_dtype out_dt, razer_stream_t stream);

/*
 * razer_gemv_variant -- W4A16 small-batch product on a format-variant weight
 * tensor (the per-model special values of the RaZeR notes, 训练策略, and the
 * pages' own kernel format of 关键设计 3: blocks of 128, FP16 scale words):
 *   y[b, n] = ts * sum_k x[b, k] * (q*s)[n, k],   1 <= B <= 32,
 * fp32 accumulation.  Arguments as razer_gemv, plus block / scale_fmt /
 * special_values / n_special as razer_quantize_variant.  workspace: at least
 * razer_workspace_size(RAZER_OP_GEMV, B, N, K) bytes (16-byte aligned; NULL
 * when that is 0), contents ignored.  K % 128 == 0; codes 16-byte aligned.
 * Byte scales (RAZER_FMT_WEIGHT / ACT / NVFP4): any block; the decoded
 * weights q*s enter the tensor-core MMA exactly, so bf16 activations with
 * +-9.5 in the set give RAZER_ERR_UNSUPPORTED (9.5 times a scale of
 * significand 1.875 needs 9 significant bits; every other allowed value
 * fits the 8 of bf16).
 * RAZER_SCALE_F16: block 128 only (others RAZER_ERR_UNSUPPORTED); the MMA
 * sums q * x and each block's fp32 sum is multiplied by its scale.
 */
razer_status razer_gemv_variant(const void *x, razer_dtype act_dt, int64_t B, const uint8_t *codes,
                                const uint8_t *scales, const float *ts, int block, razer_format scale_fmt,
                                const float *special_values, int n_special, int64_t N, int64_t K, void *y,
                                razer_dtype out_dt, void *workspace, size_t ws_bytes, razer_stream_t stream);

/*
 * razer_gemm_variant -- prefill GEMM on a format-variant weight tensor (RaZeR
 * notes, 关键设计 3: the pages' W4A16 kernels on group-128 FP16-scale
 * weights; 训练策略: per-model special values):
 *   Y[m, n] = ts * sum_k X[m, k] * (q*s)[n, k],   fp32 accumulation,
 * on the tcgen05 tensor cores.  Arguments as razer_gemm, plus block /
 * scale_fmt / special_values / n_special as razer_quantize_variant.  codes
 * 8-byte aligned; FP16 scale words 2-byte aligned.
 *   workspace  at least razer_workspace_size(RAZER_OP_GEMM_VARIANT, M, N, K)
 *              bytes, 16-byte aligned (a decoded [N, K] 16-bit copy of q*s,
 *              the partial sums of long or split K, one float); contents
 *              ignored.  M = 0, N = 0 or K = 0 need none.
 * The weights are decoded once to the activations' 16-bit type.  Byte-scale
 * formats: q*s is exact in fp16, and in bf16 unless +-9.5 is in the set
 * (bf16 activations with +-9.5 give RAZER_ERR_UNSUPPORTED).  FP16 scale
 * words: q*s has up to 16 significant bits, so the copy holds two 16-bit
 * terms hi + lo of q*s*2^11 (exact in bf16; in fp16 to within 2^-25 where lo
 * is subnormal) and the product runs over 2 K (twice the tensor-core work);
 * K % 64 == 0 (else RAZER_ERR_UNSUPPORTED).  Any M >= 0, N, and K a multiple
 * of block.
 */
razer_status razer_gemm_variant(const void *X, razer_dtype act_dt, int64_t M, const uint8_t *codes,
                                const uint8_t *scales, const float *ts, int block, razer_format scale_fmt,
                                const float *special_values, int n_special, int64_t N, int64_t K, void *Y,
                                razer_dtype out_dt, void *workspace, size_t ws_bytes, razer_stream_t stream);

/*
 * razer_gemv_noalloc -- razer_gemv for callers that cannot allocate device
 * memory (the paper has no counterpart: this is a deployment convenience).
 * Some callers cannot call cudaMalloc at all, e.g. a runtime that gives every
 * byte of the GPU to its own pool up front or code under a fixed static
 * memory budget, so they cannot hand razer_gemv a workspace.  This entry point
 * takes the same arguments minus the workspace and uses a fixed scratch array
 * inside the library instead (razer_gemv_noalloc_max_scratch() bytes, held on
 * every GPU that loads the library until the process exits).
 *   - It allocates nothing.  Its first call on a device looks up the device
 *     address of the array (with that device current), and so does its first
 *     call after the device's context is re-created (e.g. by cudaDeviceReset);
 *     make that first call before any stream capture.
 *   - Arguments are checked as razer_gemv checks them; K = 0 writes y = 0 and
 *     N = 0 writes nothing (null x / y are then allowed).
 *   - Sizes whose scratch need (razer_workspace_size(RAZER_OP_GEMV, B, N, K))
 *     exceeds the maximum are rejected with RAZER_ERR_WORKSPACE.
 *   - All calls on a device share the array and it keeps the last call's
 *     contents (nothing in it needs to start at zero).  Calls whose kernels can
 *     overlap on the GPU -- e.g. on two unordered streams -- race on it; order
 *     them on one stream.
 * Results equal razer_gemv's for the same inputs.
 */
razer_status razer_gemv_noalloc(const void *x, razer_dtype act_dt, int64_t B, const uint8_t *codes,
                                const uint8_t *scales, const float *ts, razer_format wfmt, int64_t N,
                                int64_t K, void *y, razer_dtype out_dt, razer_stream_t stream);

/* Size in bytes of the fixed scratch array used by razer_gemv_noalloc. */
size_t razer_gemv_noalloc_max_scratch(void);

/* Bytes of workspace razer_gemv (RAZER_OP_GEMV; M_or_B = B), razer_gemm
 * (RAZER_OP_GEMM), razer_gemm_w4a4 / razer_gemm_w4a4_online
 * (RAZER_OP_GEMM_W4A4) and razer_gemm_variant (RAZER_OP_GEMM_VARIANT) need
 * for these sizes (M_or_B = M for the GEMMs); 0 when none. */
size_t razer_workspace_size(razer_op op, int64_t M_or_B, int64_t N, int64_t K);

/*
 * razer_get_device_status -- the device-side error word of the current
 * device: RAZER_OK, or RAZER_ERR_TIMEOUT when a bounded wait inside a kernel
 * (pipeline barrier of razer_gemm or of the TMA razer_gemv) gave up.  Synchronises `stream`, then
 * reads and clears the word.
 */
razer_status razer_get_device_status(razer_stream_t stream);

/* Static description of a status code. */
const char *razer_status_string(razer_status status);

/* Library version, as major*10000 + minor*100 + patch. */
int razer_version(void);

/*
 * razer_set_quantize_path -- how razer_quantize_weights and
 * razer_quantize_acts compute a DYNAMIC tensor scale (ts_in == NULL);
 * process-wide, default RAZER_QPATH_TWO_PASS.  Both paths write identical
 * codes, scales, ts and histogram.
 *   RAZER_QPATH_TWO_PASS     an amax kernel, then the block quantizer reads X
 *                            again (from L2 when X fits there).
 *   RAZER_QPATH_SINGLE_PASS  one cooperative kernel, one CTA per SM: each CTA
 *                            copies its contiguous slice of blocks into shared
 *                            memory, the CTAs merge their amax and meet at a
 *                            grid barrier (bounded wait: on expiry the outputs
 *                            are void and razer_get_device_status reports
 *                            RAZER_ERR_TIMEOUT), then each quantizes its slice
 *                            from shared memory: X is read from HBM once.
 *                            Taken when at least one block per SM exists and
 *                            each slice fits in 224 KB (X of at most
 *                            SMs x 224 KB); other sizes and partitioned GPUs
 *                            that cannot hold every CTA at once use the
 *                            two-pass path.  The batched weight quantizer is
 *                            not affected.
 * Returns the previous setting, or -1 (and changes nothing) for an unknown
 * value.  Not meant to be changed while other threads launch quantizers.
 */
typedef enum { RAZER_QPATH_TWO_PASS = 0, RAZER_QPATH_SINGLE_PASS = 1 } razer_qpath;
int razer_set_quantize_path(int path);

/*
 * razer_debug_set_fault_injection -- for tests of the failure path only (the
 * paper has no counterpart).  While on (on != 0), each launch of the
 * bulk-tensor razer_gemv kernel leaves one pipeline stage of one CTA unfilled,
 * each razer_gemm launch withholds one decoder warp's arrivals and one CTA of
 * the single-pass quantizer never arrives at its grid barrier, so their
 * bounded waits expire: the call still returns RAZER_OK and
 * razer_get_device_status then reports RAZER_ERR_TIMEOUT; outputs of such a
 * call are void.  No GPU fault, trap or hang results.  Returns the previous
 * setting.  The initial setting is 1 when the environment variable
 * RAZER_FAULT_INJECT_STALL is "1" when the library is loaded, else 0.
 * Process-wide; not meant to be toggled while other threads launch.
 */
int razer_debug_set_fault_injection(int on);

#ifdef __cplusplus
}
#endif

#endif /* RAZER_H */
