/*
 * RaZeR CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded C implementation of what the RaZeR hot path
 * computes.  Only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark may load it; the product path (the CUDA library) never does, and
 * the two share no code, header, table or constant generator.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared
 * (no FMA contraction: every float operation below is one IEEE binary32
 * operation rounded to nearest-even, as written).
 *
 * Sources (the RaZeR pages):
 *  - "RaZeR: Pushing the Limits of NVFP4 Quantization with Redundant Zero
 *    Remapping" notes (papernotes.org), sections 研究背景与动机 (NVFP4 = E2M1
 *    elements + 16-element FP8-E4M3 block scale + FP32 tensor scale),
 *    关键设计 1 (weights: block scale narrowed to E3M3 -> 2 free bits, 4 special
 *    values; activations: E4M3 kept, 1 free sign bit, 2 special values),
 *    关键设计 2 (the FP4 -0 code is remapped to a special value; the block
 *    objective v_i = argmin_{v in V} || round(X_i^scaled, Q^FP4 u {v}) - X_i^scaled ||^2),
 *    关键设计 3 (decoder: special value rebuilt from a base value and an
 *    offset, joined with a sign bit), 一个完整示例 (worked example: a block
 *    with values near 5.2 and -4.8 selects +5), 训练策略 (V_w = {+-5, +-8}
 *    for Llama, V_a = {+-5}).
 *  - gist.science technical summary, sections 1 (FP4 set {+-0, +-0.5, +-1,
 *    +-1.5, +-2, +-3, +-4, +-6}), 2.1 (E3M3 weights / E4M3 activations) and
 *    2.2 (per-block special value chosen to minimise the squared error).
 *
 * Readings where the pages leave a step open (each is also listed with its
 * reason in the design notes of the repository):
 *  R1  E3M3 = 3 exponent bits, bias 3, 3 mantissa bits, subnormals, no
 *      inf/NaN: normal (1+m/8)*2^(e-3), subnormal m/32, max 30 (0x3F).
 *  R2  E4M3 = OCP E4M3 magnitude (bias 7, subnormal m*2^-9, max 448 = 0x7E;
 *      0x7F is never produced).
 *  R3  Special-value order: weights meta 0..3 -> {+5, -5, +8, -8}; activations
 *      meta 0..1 -> {+5, -5}.  Weight scale byte = meta<<6 | E3M3; activation
 *      scale byte = meta<<7 | E4M3.  Plain NVFP4 (ablation) = E4M3, no meta.
 *  R4  Tensor scale ts = amax(|X|) / (6 * S_max) (fp32 divide), S_max = 30
 *      (E3M3) or 448 (E4M3).
 *  R5  Block scale code = nearest E3M3/E4M3 value to s_f = amax_b / (6*ts)
 *      (both fp32 ops: 6*ts rounded first), ties to the even code, saturating
 *      at the largest code.
 *  R6  X^scaled = x / (s*ts): one fp32 multiply s*ts per block, one fp32
 *      IEEE divide per element.
 *  R7  Rounding to Q^FP4 u {v}: nearest point, ties to the smaller magnitude.
 *  R8  The argmin compares squared errors exactly (as real numbers); exact
 *      ties go to the lowest meta index.
 *  R9  Every element that rounds to 0 is coded 0b0000; 0b1000 means only v.
 *  R10 A block whose scale code is 0, or with ts <= 0, or whose s*ts
 *      underflows to 0, is all-zero codes with meta 0.
 *  R11 Packing: codes [R, K/2], element 2i in the low nibble of byte i;
 *      scales [R, K/16]; blocks run along K.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

/* format ids (the oracle's own numbering; the Python wrapper maps them) */
#define RO_FMT_WEIGHT 0 /* E3M3 scale, 2-bit meta, V_w = {+5,-5,+8,-8} */
#define RO_FMT_ACT 1    /* E4M3 scale, 1-bit meta, V_a = {+5,-5}       */
#define RO_FMT_NVFP4 2  /* E4M3 scale, no remap (plain NVFP4)          */
#define RO_SCALE_F16 4  /* format variants only: FP16 block scale, meta in bits 15..14 (R17) */

/* input / output element types */
#define RO_F16 0
#define RO_BF16 1
#define RO_F32 2

/* ---------------------------------------------------------------------- */
/* 16-bit float <-> double, written from the IEEE 754 / bfloat16 layouts.  */
/* ---------------------------------------------------------------------- */

double ro_f16_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24); /* subnormal: m * 2^-14 / 1024 */
    else if (e == 31)
        v = (m == 0) ? INFINITY : NAN;
    else
        v = ldexp(1.0 + (double)m / 1024.0, e - 15);
    return sign ? -v : v;
}

double ro_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16; /* bfloat16 is the top half of binary32 */
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static float load_elem(const void *x, int dtype, int64_t i)
{
    if (dtype == RO_F16)
        return (float)ro_f16_to_double(((const uint16_t *)x)[i]);
    if (dtype == RO_BF16)
        return (float)ro_bf16_to_double(((const uint16_t *)x)[i]);
    return ((const float *)x)[i];
}

/* Round a binary32 value to binary16 / bfloat16, nearest-even, by scanning
 * the two neighbouring representable values (slow and plain). */
uint16_t ro_float_to_f16(float f)
{
    if (isnan(f))
        return 0x7e00;
    uint16_t sign = signbit(f) ? 0x8000 : 0;
    double a = fabs((double)f);
    if (a >= 65520.0) /* half-way between 65504 and 2^16 rounds to inf */
        return sign | 0x7c00;
    /* find the largest non-negative finite half <= a */
    uint16_t lo = 0;
    for (int step = 1 << 14; step > 0; step >>= 1)
        if (lo + step <= 0x7bff && ro_f16_to_double((uint16_t)(lo + step)) <= a)
            lo = (uint16_t)(lo + step);
    double vlo = ro_f16_to_double(lo);
    if (vlo == a)
        return sign | lo;
    uint16_t hi = (uint16_t)(lo + 1);
    double vhi = ro_f16_to_double(hi);
    double dlo = a - vlo, dhi = vhi - a;
    uint16_t r;
    if (dlo < dhi)
        r = lo;
    else if (dhi < dlo)
        r = hi;
    else
        r = (lo & 1) ? hi : lo;
    return sign | r;
}

uint16_t ro_float_to_bf16(float f)
{
    if (isnan(f))
        return 0x7fc0;
    uint16_t sign = signbit(f) ? 0x8000 : 0;
    double a = fabs((double)f);
    uint16_t lo = 0;
    for (int step = 1 << 14; step > 0; step >>= 1)
        if (lo + step <= 0x7f80 && ro_bf16_to_double((uint16_t)(lo + step)) <= a)
            lo = (uint16_t)(lo + step);
    double vlo = ro_bf16_to_double(lo);
    if (vlo == a || lo == 0x7f80)
        return sign | lo;
    uint16_t hi = (uint16_t)(lo + 1);
    double vhi = ro_bf16_to_double(hi);
    double dlo = a - vlo, dhi = vhi - a;
    uint16_t r;
    if (dlo < dhi)
        r = lo;
    else if (dhi < dlo)
        r = hi;
    else
        r = (lo & 1) ? hi : lo;
    return sign | r;
}

/* ---------------------------------------------------------------------- */
/* Block-scale formats (readings R1, R2).                                  */
/* ---------------------------------------------------------------------- */

/* number of scale codes a format may produce */
static int scale_code_count(int fmt) { return fmt == RO_FMT_WEIGHT ? 64 : 127; }

/* value of a scale code (magnitude bits only, meta stripped) */
double ro_scale_value(int fmt, int code)
{
    if (fmt == RO_FMT_WEIGHT) { /* E3M3, bias 3 */
        int e = (code >> 3) & 7, m = code & 7;
        if (e == 0)
            return (double)m / 32.0;
        return ldexp(1.0 + m / 8.0, e - 3);
    } else { /* E4M3, bias 7 */
        int e = (code >> 3) & 15, m = code & 7;
        if (e == 0)
            return ldexp((double)m, -9);
        return ldexp(1.0 + m / 8.0, e - 7);
    }
}

double ro_scale_max(int fmt) { return ro_scale_value(fmt, scale_code_count(fmt) - 1); }

/* R5: nearest scale value by brute-force search, ties to the even code;
 * values above the largest code land on it (it is the nearest). */
int ro_scale_encode(int fmt, float s_f)
{
    int n = scale_code_count(fmt);
    int best = 0;
    double bestd = INFINITY;
    if (!(s_f < ro_scale_value(fmt, n - 1))) /* saturate (also +inf) */
        return n - 1;
    for (int c = 0; c < n; c++) {
        double d = fabs((double)s_f - ro_scale_value(fmt, c));
        if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            bestd = d;
        }
    }
    return best;
}

/* ---------------------------------------------------------------------- */
/* Special values (reading R3) and the FP4 grid.                           */
/* ---------------------------------------------------------------------- */

int ro_num_specials(int fmt) { return fmt == RO_FMT_WEIGHT ? 4 : (fmt == RO_FMT_ACT ? 2 : 0); }

double ro_special_value(int fmt, int meta)
{
    static const double vw[4] = {5.0, -5.0, 8.0, -8.0};
    static const double va[2] = {5.0, -5.0};
    if (fmt == RO_FMT_WEIGHT)
        return vw[meta & 3];
    if (fmt == RO_FMT_ACT)
        return va[meta & 1];
    return 0.0;
}

/* E2M1 magnitudes in code order 0..7 (gist.science summary, section 1) */
static const double Q_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* Decode one 4-bit code under special value v (has_v = 0: plain NVFP4). */
double ro_fp4_value(int code, int has_v, double v)
{
    code &= 15;
    if (code == 8)
        return has_v ? v : 0.0; /* the redundant -0 */
    double mag = Q_MAG[code & 7];
    return (code & 8) ? -mag : mag;
}

/* R7 + R9: nearest point of Q^FP4 u {v} to xs, ties to the smaller
 * magnitude.  Returns the 4-bit code and stores the point in *pt.
 * The candidate list is scanned in full; |xs| above 16 is treated as 16,
 * which leaves the nearest point unchanged (every point is within 9.5). */
static int round_to_grid(double xs, int has_v, double v, double *pt)
{
    double x = xs;
    if (x > 16.0)
        x = 16.0;
    if (x < -16.0)
        x = -16.0;
    int best_code = 0;
    double best_pt = 0.0;
    double best_d = fabs(x);
    for (int code = 1; code < 16; code++) {
        double p;
        if (code == 8) {
            if (!has_v)
                continue;
            p = v;
        } else {
            p = ro_fp4_value(code, 0, 0.0);
        }
        double d = fabs(x - p);
        if (d < best_d || (d == best_d && fabs(p) < fabs(best_pt))) {
            best_d = d;
            best_pt = p;
            best_code = code;
        }
    }
    *pt = best_pt;
    return best_code;
}

/* ---------------------------------------------------------------------- */
/* Tensor scale (reading R4).                                              */
/* ---------------------------------------------------------------------- */

float ro_tensor_scale(const void *x, int dtype, int64_t n, int fmt)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < n; i++) {
        float a = fabsf(load_elem(x, dtype, i));
        if (a > amax)
            amax = a;
    }
    float c = (float)(6.0 * ro_scale_max(fmt)); /* 180 or 2688, exact */
    return amax / c;
}

/* ---------------------------------------------------------------------- */
/* One 16-element block (关键设计 2).                                       */
/* ---------------------------------------------------------------------- */

/*
 * Quantize one block x[0..15] (binary32 values of the 16-bit inputs) under
 * tensor scale ts.  Outputs: codes[16] (4-bit each), the scale byte, and,
 * when the pointers are non-NULL, xs[16] = X^scaled and the exact SSE
 * difference of each candidate against plain rounding (sse_delta[meta]).
 */
void ro_quantize_block(const float *x, float ts, int fmt, uint8_t *codes, uint8_t *scale_byte,
                       float *xs_out, double *sse_delta)
{
    int nv = ro_num_specials(fmt);
    float xs[16];
    memset(codes, 0, 16);
    *scale_byte = 0;
    for (int j = 0; j < 16; j++)
        xs[j] = 0.0f;
    if (sse_delta)
        for (int m = 0; m < 4; m++)
            sse_delta[m] = 0.0;

    /* block amax */
    float amax_b = 0.0f;
    for (int j = 0; j < 16; j++) {
        float a = fabsf(x[j]);
        if (a > amax_b)
            amax_b = a;
    }
    if (!(ts > 0.0f)) { /* R10 */
        if (xs_out)
            memcpy(xs_out, xs, sizeof xs);
        return;
    }

    /* block scale: s_f = amax_b / (6 * ts), then the nearest scale code */
    float six_ts = 6.0f * ts;
    float s_f = amax_b / six_ts;
    int sc = ro_scale_encode(fmt, s_f);
    float s = (float)ro_scale_value(fmt, sc); /* exact in binary32 */
    float d = s * ts;
    if (sc == 0 || d == 0.0f) { /* R10 */
        if (xs_out)
            memcpy(xs_out, xs, sizeof xs);
        return;
    }

    /* X^scaled */
    for (int j = 0; j < 16; j++)
        xs[j] = x[j] / d;

    /* v_i = argmin over V of the squared error; compare candidates exactly.
     * For two candidates v, w: SSE_v - SSE_w = sum_j (e_vj^2 - e_wj^2) with
     * e = xs - r(xs).  Elements that round to the same point under v and w
     * contribute exactly 0; at the others |xs| > 4.5, so the factored term
     * (r_w - r_v) * (2 xs - r_v - r_w) is exact in double and so is the sum
     * (all terms are multiples of 2^-22 well below 2^30 in magnitude). */
    int meta = 0;
    double delta[4] = {0.0, 0.0, 0.0, 0.0}; /* SSE_v - SSE_plain, exact */
    if (nv > 0) {
        double rp[16]; /* plain rounding (the +-0 grid only) */
        for (int j = 0; j < 16; j++)
            round_to_grid(xs[j], 0, 0.0, &rp[j]);
        for (int m = 0; m < nv; m++) {
            double v = ro_special_value(fmt, m);
            for (int j = 0; j < 16; j++) {
                double rv;
                round_to_grid(xs[j], 1, v, &rv);
                if (rv != rp[j]) {
                    if (!(fabs((double)xs[j]) < 1073741824.0)) {
                        fprintf(stderr, "razer oracle: |X^scaled| out of the exact range\n");
                        abort();
                    }
                    delta[m] += (rp[j] - rv) * (2.0 * (double)xs[j] - rv - rp[j]);
                }
            }
        }
        for (int m = 1; m < nv; m++) /* strict '<': ties keep the lower index */
            if (delta[m] < delta[meta])
                meta = m;
        if (sse_delta)
            for (int m = 0; m < nv; m++)
                sse_delta[m] = delta[m];
    }

    /* final encode with the chosen special value */
    int has_v = nv > 0;
    double v = has_v ? ro_special_value(fmt, meta) : 0.0;
    for (int j = 0; j < 16; j++) {
        double pt;
        int code = round_to_grid(xs[j], has_v, v, &pt);
        if (pt == 0.0)
            code = 0; /* R9 */
        codes[j] = (uint8_t)code;
    }
    if (fmt == RO_FMT_WEIGHT)
        *scale_byte = (uint8_t)(sc | (meta << 6));
    else if (fmt == RO_FMT_ACT)
        *scale_byte = (uint8_t)(sc | (meta << 7));
    else
        *scale_byte = (uint8_t)sc;
    if (xs_out)
        memcpy(xs_out, xs, sizeof xs);
}

/* ---------------------------------------------------------------------- */
/* Whole-tensor quantizer.                                                 */
/* ---------------------------------------------------------------------- */

/*
 * x: [R, K] elements of dtype; ts: tensor scale; codes: [R, K/2];
 * scales: [R, K/16]; hist (may be NULL): hist[m] = blocks that chose meta m
 * (m < 4), hist[4 + m] = of those, blocks where the choice strictly lowered
 * the squared error (exact SSE difference < 0).
 */
int ro_quantize(const void *x, int dtype, int64_t R, int64_t K, int fmt, float ts, uint8_t *codes,
                uint8_t *scales, uint64_t *hist)
{
    if (K % 16 != 0)
        return 1;
    float blk[16];
    uint8_t c[16];
    double dl[4];
    for (int64_t r = 0; r < R; r++) {
        for (int64_t b = 0; b < K / 16; b++) {
            for (int j = 0; j < 16; j++)
                blk[j] = load_elem(x, dtype, r * K + b * 16 + j);
            uint8_t sb;
            ro_quantize_block(blk, ts, fmt, c, &sb, NULL, dl);
            for (int j = 0; j < 8; j++)
                codes[r * (K / 2) + b * 8 + j] = (uint8_t)(c[2 * j] | (c[2 * j + 1] << 4));
            scales[r * (K / 16) + b] = sb;
            if (hist && ro_num_specials(fmt) > 0) {
                int meta = fmt == RO_FMT_WEIGHT ? (sb >> 6) : (sb >> 7);
                hist[meta]++;
                if (dl[meta] < 0.0)
                    hist[4 + meta]++;
            }
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------- */
/* Dequantization (decoder of 关键设计 3) and the GEMM reference.          */
/* ---------------------------------------------------------------------- */

/* Value of element (r, k) as q * s (exact) in double. */
static double elem_qs(const uint8_t *codes, const uint8_t *scales, int fmt, int64_t K, int64_t r,
                      int64_t k)
{
    uint8_t byte = codes[r * (K / 2) + k / 2];
    int code = (k & 1) ? (byte >> 4) : (byte & 15);
    uint8_t sb = scales[r * (K / 16) + k / 16];
    int sc, meta;
    if (fmt == RO_FMT_WEIGHT) {
        sc = sb & 0x3f;
        meta = sb >> 6;
    } else if (fmt == RO_FMT_ACT) {
        sc = sb & 0x7f;
        meta = sb >> 7;
    } else {
        sc = sb & 0x7f;
        meta = 0;
    }
    int has_v = ro_num_specials(fmt) > 0;
    double q = ro_fp4_value(code, has_v, ro_special_value(fmt, meta));
    return q * ro_scale_value(fmt, sc);
}

/*
 * out[r, k] = round_out( fp32( (q*s) * ts ) ): q*s is exact in binary32,
 * one binary32 multiply by ts, then one rounding to the output type.
 */
int ro_dequant(const uint8_t *codes, const uint8_t *scales, float ts, int fmt, int64_t R, int64_t K,
               int out_dtype, void *out)
{
    if (K % 16 != 0)
        return 1;
    for (int64_t r = 0; r < R; r++)
        for (int64_t k = 0; k < K; k++) {
            float qs = (float)elem_qs(codes, scales, fmt, K, r, k);
            float v = qs * ts;
            int64_t i = r * K + k;
            if (out_dtype == RO_F16)
                ((uint16_t *)out)[i] = ro_float_to_f16(v);
            else if (out_dtype == RO_BF16)
                ((uint16_t *)out)[i] = ro_float_to_bf16(v);
            else
                ((float *)out)[i] = v;
        }
    return 0;
}

/*
 * Reference product r[m, n] = ts * sum_k x[m, k] * (q*s)[n, k], accumulated
 * in double (x: [M, K] of x_dtype; weights: codes [N, K/2], scales [N, K/16]).
 * rows: optional list of n_rows row indices of x to evaluate (NULL = all M);
 * out is [n_rows or M, N].
 */
int ro_gemm_ref(const void *x, int x_dtype, int64_t M, const uint8_t *codes, const uint8_t *scales,
                float ts, int fmt, int64_t N, int64_t K, const int64_t *rows, int64_t n_rows, double *out)
{
    if (K % 16 != 0)
        return 1;
    int64_t nm = rows ? n_rows : M;
    double *wrow = (double *)malloc(sizeof(double) * (size_t)K);
    if (!wrow)
        return 2;
    for (int64_t n = 0; n < N; n++) {
        for (int64_t k = 0; k < K; k++)
            wrow[k] = elem_qs(codes, scales, fmt, K, n, k);
        for (int64_t i = 0; i < nm; i++) {
            int64_t m = rows ? rows[i] : i;
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += (double)load_elem(x, x_dtype, m * K + k) * wrow[k];
            out[i * N + n] = acc * (double)ts;
        }
    }
    free(wrow);
    return 0;
}

/*
 * W4A4 product (RaZeR notes, 局限与展望: on current Blackwell tensor cores the
 * W4A4 multiply-add is emulated -- here by decoding both operands; gist.science
 * summary 2.3: weight-activation kernels): both operands are RaZeR-packed,
 *   r[m, n] = ts_a * ts_w * sum_k (q*s)_a[m, k] * (q*s)_w[n, k],
 * every q*s exact, the sum accumulated in double, then one multiply by each
 * tensor scale (in double).  rows: optional list of n_rows rows of A (NULL =
 * all M); out is [n_rows or M, N].
 */
int ro_gemm_w4a4_ref(const uint8_t *codes_a, const uint8_t *scales_a, float ts_a, int afmt, int64_t M,
                     const uint8_t *codes_w, const uint8_t *scales_w, float ts_w, int wfmt, int64_t N, int64_t K,
                     const int64_t *rows, int64_t n_rows, double *out)
{
    if (K % 16 != 0)
        return 1;
    int64_t nm = rows ? n_rows : M;
    double *arow = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
    double *wrows = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1) * (size_t)(N > 0 ? N : 1));
    if (!arow || !wrows) {
        free(arow);
        free(wrows);
        return 2;
    }
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++)
            wrows[n * K + k] = elem_qs(codes_w, scales_w, wfmt, K, n, k);
    for (int64_t i = 0; i < nm; i++) {
        int64_t m = rows ? rows[i] : i;
        for (int64_t k = 0; k < K; k++)
            arow[k] = elem_qs(codes_a, scales_a, afmt, K, m, k);
        for (int64_t n = 0; n < N; n++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += arow[k] * wrows[n * K + k];
            out[i * N + n] = acc * (double)ts_a * (double)ts_w;
        }
    }
    free(arow);
    free(wrows);
    return 0;
}

/* ---------------------------------------------------------------------- */
/* Accuracy ablations: FourOverSix and the quantization error.            */
/* ---------------------------------------------------------------------- */

/*
 * FourOverSix (Four Over Six summary page, 方法详解: 技术框架 and 关键创新):
 * plain NVFP4 blocks, but each block may be scaled so that its amax maps to
 * 4 instead of 6, whichever leaves the smaller error.  Reading R15: for
 * c in {6, 4}: s_f = amax_b / fp32(c * ts), sc = nearest E4M3 code (R5),
 * d = fp32(s * ts), codes by plain rounding of x / d (R6, R7, R9); the
 * block's squared error is sum_j (x_j - q_j * d)^2 in double, each term and
 * the running sum rounded in element order (q_j * d and x_j - q_j * d are
 * exact in double).  The 4-candidate wins only with a strictly smaller error.
 * A block whose scale code is 0 (or d = 0) is all zeros with error sum x^2.
 * Output: NVFP4 encoding (scale byte = E4M3 code); n_four (may be NULL)
 * counts the blocks that took 4.
 */
static double block_46(const float *x, float ts, float c, uint8_t *codes, int *sc_out)
{
    float amax_b = 0.0f;
    for (int j = 0; j < 16; j++) {
        float a = fabsf(x[j]);
        if (a > amax_b)
            amax_b = a;
    }
    float c_ts = c * ts;
    float s_f = amax_b / c_ts;
    int sc = ro_scale_encode(RO_FMT_NVFP4, s_f);
    float d = (float)ro_scale_value(RO_FMT_NVFP4, sc) * ts;
    double sse = 0.0;
    *sc_out = sc;
    if (sc == 0 || d == 0.0f) {
        memset(codes, 0, 16);
        *sc_out = 0;
        for (int j = 0; j < 16; j++)
            sse += (double)x[j] * (double)x[j];
        return sse;
    }
    for (int j = 0; j < 16; j++) {
        float xs = x[j] / d;
        double pt;
        int code = round_to_grid(xs, 0, 0.0, &pt);
        if (pt == 0.0)
            code = 0;
        codes[j] = (uint8_t)code;
        double t = (double)x[j] - pt * (double)d;
        sse += t * t;
    }
    return sse;
}

int ro_quantize_46(const void *x, int dtype, int64_t R, int64_t K, float ts, uint8_t *codes, uint8_t *scales,
                   uint64_t *n_four)
{
    if (K % 16 != 0)
        return 1;
    float blk[16];
    uint8_t c6[16], c4[16];
    if (n_four)
        *n_four = 0;
    for (int64_t r = 0; r < R; r++)
        for (int64_t b = 0; b < K / 16; b++) {
            for (int j = 0; j < 16; j++)
                blk[j] = load_elem(x, dtype, r * K + b * 16 + j);
            int sc6 = 0, sc4 = 0;
            const uint8_t *c = c6;
            int sc = 0;
            if (ts > 0.0f) { /* R10: ts <= 0 leaves the block zero */
                double e6 = block_46(blk, ts, 6.0f, c6, &sc6);
                double e4 = block_46(blk, ts, 4.0f, c4, &sc4);
                sc = sc6;
                if (e4 < e6) {
                    c = c4;
                    sc = sc4;
                    if (n_four)
                        (*n_four)++;
                }
            } else {
                memset(c6, 0, 16);
            }
            for (int j = 0; j < 8; j++)
                codes[r * (K / 2) + b * 8 + j] = (uint8_t)(c[2 * j] | (c[2 * j + 1] << 4));
            scales[r * (K / 16) + b] = (uint8_t)sc;
        }
    return 0;
}

/*
 * Quantization error of a packed tensor against its input:
 * sum over [R, K] (row-major order) of (x - q*s*ts)^2 in double (q*s*ts is
 * exact in double; each difference, square and running sum rounded).
 */
double ro_quant_sse(const void *x, int dtype, int64_t R, int64_t K, const uint8_t *codes, const uint8_t *scales, float ts,
                    int fmt)
{
    double sse = 0.0;
    for (int64_t r = 0; r < R; r++)
        for (int64_t k = 0; k < K; k++) {
            double v = elem_qs(codes, scales, fmt, K, r, k) * (double)ts;
            double t = (double)load_elem(x, dtype, r * K + k) - v;
            sse += t * t;
        }
    return sse;
}

/* ---------------------------------------------------------------------- */
/* Format variants (block size, special-value set) for accuracy studies.  */
/* ---------------------------------------------------------------------- */

/*
 * The RaZeR quantizer with a block of bs elements (16, 32, 64 or 128; the
 * RaZeR notes, 主实验, report the block-size study) and a special-value set
 * V[0..nv) given by the caller (multiples of 0.5 in [2.5, 9.5], the
 * constraint of the gist.science summary 2.2).  Scale format sfmt:
 * RO_FMT_WEIGHT (E3M3, meta in bits 7..6, nv <= 4) or RO_FMT_ACT /
 * RO_FMT_NVFP4 (E4M3, meta in bit 7, nv <= 2; nv = 0 is plain NVFP4).  The
 * steps are those of ro_quantize_block over bs elements: s_f = amax_b /
 * fp32(6 ts), nearest scale code, d = fp32(s ts), xs = x / d, the candidate
 * whose exact squared-error difference against plain rounding is smallest
 * (ties: lowest index), the final encode against Q u {v*}.  scales is
 * [R, K/bs].
 */
/*
 * Reading R17 (RaZeR notes, 关键设计 3: the authors' Blackwell kernels use
 * blocks of 128 with an FP16 block scale whose sign bit and top exponent bit
 * carry the meta): the scale is s = RN_fp16(amax_b / 6) with bits 15..14
 * clear, saturating at 0x3FFF (the largest such value, 2 - 2^-10); no tensor
 * scale (ts = 1); meta in bits 15..14 of the 16-bit scale word.
 */
static int f16_scale_code(float amax_b)
{
    uint16_t h = ro_float_to_f16(amax_b / 6.0f);
    return h > 0x3FFF ? 0x3FFF : h;
}

static void block_generic(const float *x, int bs, float ts, int sfmt, const double *V, int nv, uint8_t *codes, uint16_t *scale_word)
{
    memset(codes, 0, (size_t)bs);
    *scale_word = 0;
    float amax_b = 0.0f;
    for (int j = 0; j < bs; j++) {
        float a = fabsf(x[j]);
        if (a > amax_b)
            amax_b = a;
    }
    int sc;
    float d;
    if (sfmt == RO_SCALE_F16) {
        sc = f16_scale_code(amax_b);
        d = (float)ro_f16_to_double((uint16_t)sc);
    } else {
        if (!(ts > 0.0f))
            return;
        float six_ts = 6.0f * ts;
        float s_f = amax_b / six_ts;
        sc = ro_scale_encode(sfmt, s_f);
        d = (float)ro_scale_value(sfmt, sc) * ts;
    }
    if (sc == 0 || d == 0.0f)
        return;
    int meta = 0;
    double best = 0.0;
    for (int m = 0; m < nv; m++) {
        double delta = 0.0;
        for (int j = 0; j < bs; j++) {
            float xs = x[j] / d;
            double rp, rv;
            round_to_grid(xs, 0, 0.0, &rp);
            round_to_grid(xs, 1, V[m], &rv);
            if (rv != rp)
                delta += (rp - rv) * (2.0 * (double)xs - rv - rp);
        }
        if (m == 0 || delta < best) {
            best = delta;
            meta = m;
        }
    }
    for (int j = 0; j < bs; j++) {
        double pt;
        int code = round_to_grid(x[j] / d, nv > 0, nv > 0 ? V[meta] : 0.0, &pt);
        codes[j] = (uint8_t)(pt == 0.0 ? 0 : code);
    }
    if (sfmt == RO_SCALE_F16)
        *scale_word = (uint16_t)(sc | (nv > 0 ? meta << 14 : 0));
    else
        *scale_word = (uint16_t)(sc | (nv > 0 ? meta << (sfmt == RO_FMT_WEIGHT ? 6 : 7) : 0));
}

int ro_quantize_generic(const void *x, int dtype, int64_t R, int64_t K, int bs, int sfmt, const double *V, int nv, float ts,
                        uint8_t *codes, uint8_t *scales)
{
    if (bs <= 0 || bs > 128 || K % bs != 0 || (bs & 15) != 0)
        return 1;
    float blk[128];
    uint8_t c[128];
    for (int64_t r = 0; r < R; r++)
        for (int64_t b = 0; b < K / bs; b++) {
            for (int j = 0; j < bs; j++)
                blk[j] = load_elem(x, dtype, r * K + b * bs + j);
            uint16_t sw;
            block_generic(blk, bs, ts, sfmt, V, nv, c, &sw);
            for (int j = 0; j < bs / 2; j++)
                codes[r * (K / 2) + b * (bs / 2) + j] = (uint8_t)(c[2 * j] | (c[2 * j + 1] << 4));
            if (sfmt == RO_SCALE_F16) { /* 16-bit scale words, little-endian */
                scales[2 * (r * (K / bs) + b)] = (uint8_t)(sw & 0xFF);
                scales[2 * (r * (K / bs) + b) + 1] = (uint8_t)(sw >> 8);
            } else {
                scales[r * (K / bs) + b] = (uint8_t)sw;
            }
        }
    return 0;
}

/* q*s of element (r, k) of a tensor of ro_quantize_generic (exact in double) */
static double generic_qs(const uint8_t *codes, const uint8_t *scales, int64_t K, int bs, int sfmt, const double *V, int nv,
                         int64_t r, int64_t k)
{
    uint8_t byte = codes[r * (K / 2) + k / 2];
    int code = (k & 1) ? (byte >> 4) : (byte & 15);
    double sv;
    int meta;
    if (sfmt == RO_SCALE_F16) {
        int64_t bi = r * (K / bs) + k / bs;
        uint16_t sw = (uint16_t)(scales[2 * bi] | (scales[2 * bi + 1] << 8));
        sv = ro_f16_to_double((uint16_t)(sw & 0x3FFF));
        meta = nv > 0 ? sw >> 14 : 0;
    } else {
        uint8_t sb = scales[r * (K / bs) + k / bs];
        sv = ro_scale_value(sfmt, sb & (sfmt == RO_FMT_WEIGHT ? 0x3f : 0x7f));
        meta = nv > 0 ? (sfmt == RO_FMT_WEIGHT ? sb >> 6 : sb >> 7) : 0;
    }
    /* a meta value at or past nv (never written by the quantizer) selects 0 */
    double q = ro_fp4_value(code, nv > 0, (nv > 0 && meta < nv) ? V[meta] : 0.0);
    return q * sv;
}

/* sum (x - q*s*ts)^2 for a tensor of ro_quantize_generic (row-major order, double) */
double ro_quant_sse_generic(const void *x, int dtype, int64_t R, int64_t K, int bs, int sfmt, const double *V, int nv,
                            const uint8_t *codes, const uint8_t *scales, float ts)
{
    double sse = 0.0;
    for (int64_t r = 0; r < R; r++)
        for (int64_t k = 0; k < K; k++) {
            double v = generic_qs(codes, scales, K, bs, sfmt, V, nv, r, k) * (double)ts;
            double t = (double)load_elem(x, dtype, r * K + k) - v;
            sse += t * t;
        }
    return sse;
}

/*
 * Decoder of the format variants, defined like ro_dequant: out[r, k] =
 * round_out( fp32( (q*s) * ts ) ) -- q*s is exact in binary32 for every
 * variant (at most 5 significant bits of q times at most 11 of s), one
 * binary32 multiply by ts, one rounding to the output type.
 */
int ro_dequant_generic(const uint8_t *codes, const uint8_t *scales, float ts, int64_t R, int64_t K, int bs, int sfmt,
                       const double *V, int nv, int out_dtype, void *out)
{
    if (bs <= 0 || bs > 128 || (bs & 15) != 0 || K % bs != 0)
        return 1;
    for (int64_t r = 0; r < R; r++)
        for (int64_t k = 0; k < K; k++) {
            float qs = (float)generic_qs(codes, scales, K, bs, sfmt, V, nv, r, k);
            float v = qs * ts;
            int64_t i = r * K + k;
            if (out_dtype == RO_F16)
                ((uint16_t *)out)[i] = ro_float_to_f16(v);
            else if (out_dtype == RO_BF16)
                ((uint16_t *)out)[i] = ro_float_to_bf16(v);
            else
                ((float *)out)[i] = v;
        }
    return 0;
}

/*
 * Reference W4A16 product on a variant weight tensor [N, K]:
 * r[b, n] = ts * sum_k x[b, k] * (q*s)[n, k], accumulated in double (x is
 * [B, K] of x_dtype); out is [B, N].
 */
int ro_gemv_generic(const void *x, int x_dtype, int64_t B, const uint8_t *codes, const uint8_t *scales, float ts, int bs,
                    int sfmt, const double *V, int nv, int64_t N, int64_t K, double *out)
{
    if (bs <= 0 || bs > 128 || (bs & 15) != 0 || K % bs != 0)
        return 1;
    double *wrow = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
    if (!wrow)
        return 2;
    for (int64_t n = 0; n < N; n++) {
        for (int64_t k = 0; k < K; k++)
            wrow[k] = generic_qs(codes, scales, K, bs, sfmt, V, nv, n, k);
        for (int64_t b = 0; b < B; b++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += (double)load_elem(x, x_dtype, b * K + k) * wrow[k];
            out[b * N + n] = acc * (double)ts;
        }
    }
    free(wrow);
    return 0;
}

