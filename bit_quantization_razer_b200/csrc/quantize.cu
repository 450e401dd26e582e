// RaZeR block quantizer for sm_100a.
//
// Follows RaZeR notes 关键设计 1-2 (two-level scaling; E3M3 weight scale with a
// 2-bit meta, E4M3 activation scale with a 1-bit meta; per-block argmin of the
// squared error over Q_FP4 u {v}) and the gist.science summary, section 2.2
// (activations: one quantization per candidate, keep the smaller error).
//
// One thread owns one 16-element block: it streams 32 bytes of fp16/bf16 in
// (two 128-bit loads), and writes 8 bytes of codes and one scale byte.  The
// path is HBM-bound only if the per-element ALU work stays small, so:
//   * X^scaled = RN(x / d) uses one correctly rounded reciprocal per block and
//     Markstein's correction per element (q = x*y, r = fma(-q,d,x),
//     q' = fma(r,y,q)); tests/markstein_check.c proves q' == RN(x/d) for every
//     16-bit input significand and every binary32 divisor significand, so the
//     result is the IEEE quotient (blocks with d outside [2^-90, 2^90] take
//     the plain IEEE divide);
//   * the plain E2M1 codes (ties to the smaller magnitude) come from two
//     hardware conversions and a 3-operation select per 8 codes (fix_codes);
//   * the squared-error comparison of the candidates is exact: only elements
//     whose nearest point changes contribute, each term (q - v)(2 xs - q - v)
//     is a multiple of 2^-20 computed exactly in binary32, and the partial
//     sums stay exact (see the notes on each accumulator below).
#include <atomic>

#include "razer_internal.cuh"
#include "sm100_async.cuh"

namespace razer {

// Packed binary32 pair arithmetic (two lanes per instruction on sm_100a).
__device__ __forceinline__ float2 mul2(float2 a, float2 b)
{
    float2 d;
    asm("{ .reg .b64 A, B, D; mov.b64 A, {%2, %3}; mov.b64 B, {%4, %5}; mul.rn.f32x2 D, A, B; mov.b64 {%0, %1}, D; }"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c)
{
    float2 d;
    asm("{ .reg .b64 A, B, C, D; mov.b64 A, {%2, %3}; mov.b64 B, {%4, %5}; mov.b64 C, {%6, %7}; fma.rn.f32x2 D, A, B, C; mov.b64 {%0, %1}, D; }"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// Hardware E2M1 conversion (round to nearest even, saturating) of 8 values
// into one word: nibble j holds the code of v[j].
__device__ __forceinline__ float2 add2(float2 a, float2 b)
{
    float2 d;
    asm("{ .reg .b64 A, B, D; mov.b64 A, {%2, %3}; mov.b64 B, {%4, %5}; add.rn.f32x2 D, A, B; mov.b64 {%0, %1}, D; }"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ unsigned cvt_e2m1x8(const float *v)
{
    unsigned w;
    asm("{ .reg .b8 b0, b1, b2, b3;"
        " cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;"
        " cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;"
        " cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;"
        " cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;"
        " mov.b32 %0, {b0, b1, b2, b3}; }"
        : "=r"(w)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return w;
}

// Plain E2M1 codes with ties to the SMALLER magnitude from two hardware
// conversions (ties to even): c1 of xs and c2 of pred(xs) = xs * (1 - 2^-24)
// (one ulp toward zero).  They differ only when a midpoint lies in
// [pred(xs), xs]; the two codes are then adjacent and the right one is the
// odd one (tests/test_e2m1_tie_identity.py checks this for every binary32 in
// [0, 16]).  Finally the codes of values that rounded to -0 become 0b0000.
__device__ __forceinline__ unsigned fix_codes(unsigned c1, unsigned c2)
{
    const unsigned odd = (c1 & 0x11111111u) * 15u;  // whole nibble set where c1 is odd
    const unsigned w = (c1 & odd) | (c2 & ~odd);
    const unsigned z = w & ~((w & 0x77777777u) + 0x77777777u) & 0x88888888u;  // nibbles == 0b1000
    return w & ~z;
}

// Nearest scale code of s_f >= 0 (ties to even, saturating) from the hardware
// E4M3 convert.  E4M3 (bias 7) codes are the activation scale codes; an E3M3
// (bias 3) value times 2^-4 has the same exponent and mantissa fields in E4M3,
// subnormals included, so the weight code is the E4M3 code of s_f * 2^-4
// clamped to the largest E3M3 code (anything above it saturates there).
template <int FMT> __device__ __forceinline__ unsigned encode_scale_cvt(float sf)
{
    using F = Fmt<FMT>;
    const float v = FMT == RAZER_FMT_WEIGHT ? __fmul_rn(sf, 0.0625f) : sf;
    unsigned short h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(v));
    const unsigned c = (unsigned)h & 0x7Fu;
    return FMT == RAZER_FMT_WEIGHT ? min(c, (unsigned)F::kMagMask) : c;
}

struct BlockOut {
    uint2 packed;    // 16 nibbles
    unsigned sbyte;  // scale byte (meta | magnitude code)
    unsigned meta;
    bool effective;  // the chosen special value strictly lowered the error
};

// Per-launch constants of the block quantizer: ts, 6*ts with its correctly
// rounded reciprocal, and per scale code c the divisor d = dec(c) * ts and
// RN(1/d) (0 where d is outside [2^-90, 2^90], where the IEEE divide is used).
struct ScaleCtx {
    float ts, six_ts, y6;
    const float *tab_d, *tab_y;  // shared memory, one entry per magnitude code
};

// FAST: the launch-wide preconditions of the fast path hold (ts in
// [2^-62, 2^57]): RN(1/(6 ts)) and RN(1/d) of every non-zero scale code are
// valid Markstein reciprocals, so the block needs no divide fallback and no
// early exit (a zero scale code is zeroed by selects at the end).  F16IN: the
// elements are fp16, whose amax is 0 or in [2^-24, 65504].
template <int FMT, bool FAST, bool F16IN>
__device__ __forceinline__ BlockOut quantize_block(const float (&x)[16], const ScaleCtx &k)
{
    const float ts = k.ts;
    using F = Fmt<FMT>;
    BlockOut o;
    o.packed = make_uint2(0u, 0u);
    o.sbyte = 0u;
    o.meta = 0u;
    o.effective = false;

    float m8[8];
#pragma unroll
    for (int j = 0; j < 8; j++) m8[j] = fmaxf(fabsf(x[2 * j]), fabsf(x[2 * j + 1]));
#pragma unroll
    for (int j = 0; j < 4; j++) m8[j] = fmaxf(m8[j], m8[j + 4]);
    const float amax = fmaxf(fmaxf(m8[0], m8[2]), fmaxf(m8[1], m8[3]));
    if (!FAST && !(ts > 0.0f)) return o;

    // block scale: s_f = RN(amax_b / RN(6 ts)), nearest scale code.  amax_b is
    // an fp16/bf16 value, so Markstein's correction of amax_b * RN(1/(6 ts))
    // is the IEEE quotient (the same proof as for X^scaled) while both
    // operands stay well inside the normal range.
    float sf;
    if ((FAST && F16IN) || (k.y6 != 0.0f && ((amax >= 0x1p-60f && amax <= 0x1p60f) || amax == 0.0f))) {
        const float q = __fmul_rn(amax, k.y6);
        sf = __fmaf_rn(__fmaf_rn(-q, k.six_ts, amax), k.y6, q);
    } else {
        sf = __fdiv_rn(amax, k.six_ts);
    }
    const unsigned sc = FAST ? encode_scale_cvt<FMT>(sf) : encode_scale<FMT>(sf);
    const float d = k.tab_d[sc];  // dec(sc) * ts
    if (!FAST && (sc == 0u || d == 0.0f)) return o;

    // X^scaled = RN(x / d).  Markstein's correction needs its intermediates in
    // the normal range: with a caller-given ts a saturated block scale can
    // leave x / d near or past the binary32 maximum (bf16 input only: an fp16
    // amax is at most 65504), so such blocks take the IEEE divide (which
    // overflows to inf like the oracle's quotient).
    float xs[16];
    const float y = k.tab_y[sc];  // RN(1/d), or 0 outside the Markstein range
    if ((FAST || y != 0.0f) && (F16IN || __fmul_rn(amax, y) <= 0x1p126f)) {
        const float2 y2 = make_float2(y, y), nd2 = make_float2(-d, -d);
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
            const float2 xv = make_float2(x[j], x[j + 1]);
            const float2 q = mul2(xv, y2);
            const float2 r = fma2(q, nd2, xv);
            const float2 q2 = fma2(r, y2, q);
            xs[j] = q2.x;
            xs[j + 1] = q2.y;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; j++) xs[j] = __fdiv_rn(x[j], d);
    }

    // plain codes (ties to the smaller magnitude, 0b1000 never produced)
    float pv[16];
    const float2 down = make_float2(1.0f - 0x1p-24f, 1.0f - 0x1p-24f);
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
        const float2 p = mul2(make_float2(xs[j], xs[j + 1]), down);
        pv[j] = p.x;
        pv[j + 1] = p.y;
    }
    unsigned w0 = fix_codes(cvt_e2m1x8(xs), cvt_e2m1x8(pv));
    unsigned w1 = fix_codes(cvt_e2m1x8(xs + 8), cvt_e2m1x8(pv + 8));

    unsigned meta = 0u;
    if constexpr (F::kSpecials > 0) {
        // v = +5 / -5: an element changes only inside (4.5, 5.5] (resp.
        // [-5.5, -4.5)), where the squared-error difference is
        // t = |2|xs| - 10| - 1 in [-1, 0]; outside, the clamped t is exactly 0.
        // In the region 2|xs| - 10 is exact (Sterbenz) and t is a multiple of
        // 2^-20.  A = sum t and B = sum copysign(t, xs) are exact binary32 sums
        // (|A|, |B| <= 16); then the +5 sum is (A - B) / 2 and the -5 sum is
        // (A + B) / 2, both exact.
        float ea[16];  // 2|xs| - 10, reused by the final encode
        // -t = sat(1 - |e|) in one saturating add; copysign(-t, xs) =
        // copysign(t, xs) for t <= 0, so the second sum is B itself
        float2 AB = make_float2(0.0f, 0.0f);  // (-A, B), one packed add per element
#pragma unroll
        for (int j = 0; j < 16; j++) {
            ea[j] = __fmaf_rn(2.0f, fabsf(xs[j]), -10.0f);
            const float nt = __saturatef(__fadd_rn(1.0f, -fabsf(ea[j])));
            AB = add2(AB, make_float2(nt, copysignf(nt, xs[j])));
        }
        const float A = -AB.x, Bs = AB.y;
        const float dp5 = __fmul_rn(__fsub_rn(A, Bs), 0.5f);
        const float dn5 = __fmul_rn(__fadd_rn(A, Bs), 0.5f);
        float best = dp5;
        if (dn5 < best) { best = dn5; meta = 1u; }
        // final encode against Q_FP4 u {v*}: elements nearest to v* take
        // 0b1000.  For v* = +5 the region is xs in (4.5, 5.5], for v* = -5 it
        // is [-5.5, -4.5) (ties go to the smaller magnitude): |xs| in
        // (4.5, 5.5] with the sign of v*.  y = |xs|/2 - (1 + 2^-23) is exact
        // for |xs| in [4, 8) (a multiple of 2^-23 in [1, 2)) and lies in
        // (1.25, 1.75) -- the open interval the E2M1 convert sends to code
        // 0b0011 -- exactly when |xs| is in (4.5, 5.5]; smaller |xs| give
        // y < 1 and larger ones (<= 9) y > 1.75.  Four converts gather the 16
        // tests; the sign of xs is the plain code's sign bit (the plain code is
        // +-4 or +-6 there).
        unsigned o0, o1;
        {
            float yv[16];
#pragma unroll
            for (int j = 0; j < 16; j++) yv[j] = __fmaf_rn(fabsf(xs[j]), 0.5f, -(1.0f + 0x1p-23f));
            const unsigned v0 = cvt_e2m1x8(yv) ^ 0x33333333u, v1 = cvt_e2m1x8(yv + 8) ^ 0x33333333u;
            // bit 3 of every nibble equal to 0b0011
            const unsigned in0 = ~(((v0 & 0x77777777u) + 0x77777777u) | v0) & 0x88888888u;
            const unsigned in1 = ~(((v1 & 0x77777777u) + 0x77777777u) | v1) & 0x88888888u;
            o0 = in0 & (meta ? w0 : ~w0);
            o1 = in1 & (meta ? w1 : ~w1);
        }
        if constexpr (F::kSpecials == 4) {
            // v = +8 / -8 changes an element only when |xs| > 7.  With a
            // normal scale code |xs| <= 6 / (1 - 2^-4) < 7, so only blocks with
            // a subnormal scale code (0 < sc < 8) can use them; there |xs| <= 9
            // and the terms are summed exactly as integers in units of 2^-20.
            if (sc - 1u < 7u) {
                int ip5 = 0, in5 = 0, ip8 = 0, in8 = 0;
#pragma unroll
                for (int j = 0; j < 16; j++) {
                    const float t5p = fminf(__fadd_rn(fabsf(__fmaf_rn(2.0f, xs[j], -10.0f)), -1.0f), 0.0f);
                    const float t5n = fminf(__fadd_rn(fabsf(__fmaf_rn(2.0f, xs[j], 10.0f)), -1.0f), 0.0f);
                    const float t8p = fminf(__fmaf_rn(-4.0f, xs[j], 28.0f), 0.0f);
                    const float t8n = fminf(__fmaf_rn(4.0f, xs[j], 28.0f), 0.0f);
                    ip5 += __float2int_rn(__fmul_rn(t5p, 1048576.0f));
                    in5 += __float2int_rn(__fmul_rn(t5n, 1048576.0f));
                    ip8 += __float2int_rn(__fmul_rn(t8p, 1048576.0f));
                    in8 += __float2int_rn(__fmul_rn(t8n, 1048576.0f));
                }
                int ib = ip5;
                unsigned m8 = 0u;
                if (in5 < ib) { ib = in5; m8 = 1u; }
                if (ip8 < ib) { ib = ip8; m8 = 2u; }
                if (in8 < ib) { ib = in8; m8 = 3u; }
                best = (float)ib;
                if (m8 >= 2u) {
                    // +8 (7, inf] / -8 [-inf, -7): one interval of bit patterns each
                    const unsigned lo = 0x40E00001u | ((m8 & 1u) << 31), span = 0x7F800000u - 0x40E00001u;
                    o0 = o1 = 0u;
#pragma unroll
                    for (int j = 0; j < 8; j++) {
                        o0 |= (__float_as_uint(xs[j]) - lo <= span) ? (8u << (4 * j)) : 0u;
                        o1 |= (__float_as_uint(xs[j + 8]) - lo <= span) ? (8u << (4 * j)) : 0u;
                    }
                }
                // below 2 the integer decision repeats the +-5 one (the same exact sums)
                meta = m8;
            }
        }
        o.effective = best < 0.0f;
        w0 = (w0 & ~((o0 >> 3) * 15u)) | o0;
        w1 = (w1 & ~((o1 >> 3) * 15u)) | o1;
    }

    if (FAST && sc == 0u) {  // amax_b rounds to a zero scale: all-zero block (selects, no branch)
        w0 = w1 = 0u;
        meta = 0u;
        o.effective = false;
    }
    o.packed = make_uint2(w0, w1);
    o.meta = meta;
    o.sbyte = sc | (meta << F::kMetaShift);
    return o;
}

constexpr int kQThreads = 256;

template <int FMT, typename TIn, bool FAST, bool HIST>
__device__ __forceinline__ void quant_one(const uint4 v0, const uint4 v1, int64_t b, const ScaleCtx &k, uint8_t *__restrict__ codes,
                                          uint8_t *__restrict__ scales, unsigned (&cnt)[4])
{
    float xv[16];
    const unsigned wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const float2 f = In16<TIn>::to_f2(wv[i]);
        xv[2 * i] = f.x;
        xv[2 * i + 1] = f.y;
    }
    const BlockOut o = quantize_block<FMT, FAST, std::is_same<TIn, __half>::value>(xv, k);
    reinterpret_cast<uint2 *>(codes)[b] = o.packed;
    scales[b] = (uint8_t)o.sbyte;
    if constexpr (HIST) {
        const unsigned m1 = o.meta & 1u, e = o.effective ? 1u : 0u;
        cnt[0] += 1u - m1;
        cnt[1] += m1;
        cnt[2] += e & (1u - m1);
        cnt[3] += e & m1;
    }
}

// Thread t of T quantizes blocks t, t + T, ...  The next block's 32 bytes are
// loaded before the current block is quantized, so every thread keeps one
// load in flight while it computes.
template <int FMT, typename TIn, bool FAST, bool HIST>
__device__ __forceinline__ void quant_range(const TIn *__restrict__ x, int64_t nblk, const ScaleCtx &k, uint8_t *__restrict__ codes,
                                            uint8_t *__restrict__ scales, int64_t t, int64_t T, unsigned (&cnt)[4])
{
    const uint4 *p = reinterpret_cast<const uint4 *>(x);
    int64_t b = t;
    if (b >= nblk) return;
    uint4 v0 = ldg_stream(p + 2 * b), v1 = ldg_stream(p + 2 * b + 1);
    for (; b < nblk; b += T) {
        const int64_t bn = b + T < nblk ? b + T : b;
        const uint4 n0 = ldg_stream(p + 2 * bn), n1 = ldg_stream(p + 2 * bn + 1);
        quant_one<FMT, TIn, FAST, HIST>(v0, v1, b, k, codes, scales, cnt);
        v0 = n0;
        v1 = n1;
    }
}

template <int FMT, typename TIn, bool FAST, bool HIST>
__device__ __forceinline__ void quant_loop(const TIn *__restrict__ x, int64_t nblk, const ScaleCtx &k, uint8_t *__restrict__ codes,
                                           uint8_t *__restrict__ scales, unsigned (&cnt)[4])
{
    quant_range<FMT, TIn, FAST, HIST>(x, nblk, k, codes, scales, (int64_t)blockIdx.x * blockDim.x + threadIdx.x,
                                      (int64_t)gridDim.x * blockDim.x, cnt);
}

// Fills the per-code tables (shared memory) and the launch constants for ts;
// the caller synchronises the block before using them.
template <int FMT>
__device__ __forceinline__ ScaleCtx make_ctx(float ts, float *tab_d, float *tab_y)
{
    using F = Fmt<FMT>;
    for (int c = threadIdx.x; c <= (int)F::kMagMask; c += blockDim.x) {
        const float d = __fmul_rn(decode_scale<FMT>((unsigned)c), ts);
        tab_d[c] = d;
        tab_y[c] = (d >= 0x1p-90f && d <= 0x1p90f) ? __frcp_rn(d) : 0.0f;
    }
    ScaleCtx k;
    k.ts = ts;
    k.six_ts = __fmul_rn(6.0f, ts);
    k.y6 = (k.six_ts >= 0x1p-60f && k.six_ts <= 0x1p60f) ? __frcp_rn(k.six_ts) : 0.0f;
    k.tab_d = tab_d;
    k.tab_y = tab_y;
    return k;
}

// launch-wide: with ts in [2^-62, 2^57] every reciprocal the blocks need is a
// valid Markstein reciprocal (d of a non-zero scale code lies in
// [2^-71, 2^66]), so the per-block fallbacks and early exits drop out
__device__ __forceinline__ bool fast_ts(float ts) { return ts >= 0x1p-62f && ts <= 0x1p57f; }

// max(m, |x|) over the eight 16-bit values of one 16-byte vector
template <typename TIn> __device__ __forceinline__ float amax_vec(float m, const uint4 v)
{
    const unsigned w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const float2 f = In16<TIn>::to_f2(w[k]);
        m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    return m;
}

// block-wide max of m, merged into *out as binary32 bits (atomicMax is
// order-preserving for non-negative floats)
__device__ __forceinline__ void commit_amax(float m, unsigned *out)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float sm[32];
    if ((threadIdx.x & 31) == 0) sm[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float r = sm[0];
        for (int i = 1; i < (int)(blockDim.x >> 5); i++) r = fmaxf(r, sm[i]);
        if (r > 0.0f) atomicMax(out, __float_as_uint(r));
    }
}

template <int FMT, typename TIn, bool HIST>
__global__ void __launch_bounds__(kQThreads) quantize_kernel(const TIn *__restrict__ x, int64_t nblk,
                                                             const float *__restrict__ ts_src, int ts_is_amax,
                                                             uint8_t *__restrict__ codes, uint8_t *__restrict__ scales,
                                                             unsigned long long *__restrict__ hist)
{
    using F = Fmt<FMT>;
    pdl_wait();  // x, ts and the histogram come from earlier kernels in the stream
    pdl_trigger();
    const float tv = *ts_src;
    const float ts = ts_is_amax ? __fdiv_rn(tv, F::kC) : tv;
    unsigned cnt[4] = {0u, 0u, 0u, 0u};

    __shared__ float tab_d[F::kMagMask + 1], tab_y[F::kMagMask + 1];
    const ScaleCtx k = make_ctx<FMT>(ts, tab_d, tab_y);
    __syncthreads();

    if (fast_ts(ts)) quant_loop<FMT, TIn, true, HIST>(x, nblk, k, codes, scales, cnt);
    else quant_loop<FMT, TIn, false, HIST>(x, nblk, k, codes, scales, cnt);

    if constexpr (HIST) {
        __shared__ unsigned long long sh[4];
        if (threadIdx.x < 4) sh[threadIdx.x] = 0ull;
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 4; i++) {
            unsigned c = cnt[i];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
            if ((threadIdx.x & 31) == 0 && c) atomicAdd(&sh[i], (unsigned long long)c);
        }
        __syncthreads();
        if (threadIdx.x < 4 && sh[threadIdx.x]) atomicAdd(&hist[threadIdx.x], sh[threadIdx.x]);
    }
}

// amax(|x|) over n16 / 8 128-bit vectors; result as binary32 bits via
// atomicMax (order-preserving for non-negative floats) into *out.
template <typename TIn>
__global__ void __launch_bounds__(256) amax_kernel(const TIn *__restrict__ x, int64_t nvec, unsigned *__restrict__ out)
{
    pdl_wait();
    pdl_trigger();
    float m = 0.0f;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const uint4 *p = reinterpret_cast<const uint4 *>(x);
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    // four independent 16-byte loads in flight per thread
    for (; i + 3 * stride < nvec; i += 4 * stride) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; u++) v[u] = ldg_stream(p + i + u * stride);
#pragma unroll
        for (int u = 0; u < 4; u++) m = amax_vec<TIn>(m, v[u]);
    }
    for (; i < nvec; i += stride) m = amax_vec<TIn>(m, ldg_stream(p + i));
    commit_amax(m, out);
}

// Thread t of T reduces max(m, |x|) over the 16-byte vectors t, t + T, ...
// with eight loads in flight.
template <typename TIn>
__device__ __forceinline__ void amax_range(const TIn *__restrict__ x, int64_t nvec, int64_t t, int64_t T, float &m)
{
    const uint4 *p = reinterpret_cast<const uint4 *>(x);
    int64_t i = t;
    for (; i + 7 * T < nvec; i += 8 * T) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; u++) v[u] = ldg_stream(p + i + u * T);
#pragma unroll
        for (int u = 0; u < 8; u++) m = amax_vec<TIn>(m, v[u]);
    }
    for (; i < nvec; i += T) m = amax_vec<TIn>(m, ldg_stream(p + i));
}

// One stage of the batched weight quantizer: quantizes tensor q, whose amax
// an earlier kernel in the stream completed, while reducing amax(|x|) of the
// next tensor a.  Quantization is arithmetic-bound and the amax pass is
// bandwidth-bound, so each CTA splits its warps: the first amax_warps stream
// tensor a (eight 16-byte loads in flight per thread, few instructions), the
// others quantize tensor q with the prefetching loop.  The host picks the
// split from the two parts' expected times so that both finish together.
template <int FMT, typename TIn>
__global__ void __launch_bounds__(kQThreads, 4) quant_amax_kernel(const TIn *__restrict__ xq, int64_t nblk, const float *__restrict__ amax_q,
                                                                  uint8_t *__restrict__ codes, uint8_t *__restrict__ scales,
                                                                  const TIn *__restrict__ xa, int64_t nva, unsigned *__restrict__ amax_a,
                                                                  int amax_warps)
{
    using F = Fmt<FMT>;
    pdl_wait();  // amax_q and the zeroed amax_a come from earlier kernels
    pdl_trigger();
    const float ts = __fdiv_rn(*amax_q, F::kC);
    __shared__ float tab_d[F::kMagMask + 1], tab_y[F::kMagMask + 1];
    const ScaleCtx k = make_ctx<FMT>(ts, tab_d, tab_y);
    __syncthreads();
    float m = 0.0f;
    const int warp = threadIdx.x >> 5;
    if (warp < amax_warps) {
        const int64_t per = 32 * amax_warps;
        amax_range<TIn>(xa, nva, (int64_t)blockIdx.x * per + threadIdx.x, (int64_t)gridDim.x * per, m);
    } else {
        const int64_t per = kQThreads - 32 * amax_warps;
        const int64_t t = (int64_t)blockIdx.x * per + threadIdx.x - 32 * amax_warps, T = (int64_t)gridDim.x * per;
        unsigned cnt[4] = {0u, 0u, 0u, 0u};
        if (fast_ts(ts)) quant_range<FMT, TIn, true, false>(xq, nblk, k, codes, scales, t, T, cnt);
        else quant_range<FMT, TIn, false, false>(xq, nblk, k, codes, scales, t, T, cnt);
    }
    commit_amax(m, amax_a);
}

// zeroes count amax words (one launch for a whole batch)
__global__ void init_many_kernel(unsigned *bits, int count)
{
    pdl_wait();
    pdl_trigger();
    for (int i = threadIdx.x; i < count; i += blockDim.x) bits[i] = 0u;
}

// ts[i] = amax[i] / (6 * S_max) for a whole batch, written over the amax words
__global__ void finalize_many_kernel(float *ts, int count, float c)
{
    pdl_wait();
    for (int i = threadIdx.x; i < count; i += blockDim.x) ts[i] = __fdiv_rn(__uint_as_float(reinterpret_cast<unsigned *>(ts)[i]), c);
}

// ts = amax / (6 * S_max), written over the amax word.
__global__ void finalize_ts_kernel(float *ts, float c)
{
    pdl_wait();
    const float amax = __uint_as_float(*reinterpret_cast<unsigned *>(ts));
    *ts = __fdiv_rn(amax, c);
}

__global__ void copy_ts_kernel(const float *src, float *dst)
{
    pdl_wait();
    *dst = *src;
}

// zeroes the histogram and the amax accumulator of a quantizer call (one
// launch instead of two memsets), and the two barrier words of the
// single-pass kernel when it runs (the first 8 code bytes)
__global__ void quant_init_kernel(unsigned long long *hist, unsigned *amax_bits, unsigned *bar_words)
{
    pdl_wait();
    pdl_trigger();
    if (hist && threadIdx.x < 4) hist[threadIdx.x] = 0ull;
    if (amax_bits && threadIdx.x == 0) *amax_bits = 0u;
    if (bar_words && threadIdx.x < 2) bar_words[threadIdx.x] = 0u;
}

// ---------------------------------------------------------------------------
// Single-pass quantizer with a dynamic tensor scale: X is read from HBM once.
// One CTA per SM, all co-resident (cooperative launch), each holding its
// contiguous slice of blocks in shared memory:
//   1. bulk copies bring the slice in (8 chunks at most, one mbarrier each);
//      the block-wide amax is reduced chunk by chunk as they land and merged
//      into the amax word (*ts_out, zeroed by the init kernel);
//   2. a grid barrier: arrivals count up in bar[0], bounded wait for all G;
//   3. every CTA reads the tensor amax, ts = amax / (6 S_max) (the same fp32
//      divide as the two-pass path), counts itself out in bar[1], and
//      quantizes its slice from shared memory with the same block quantizer;
//   4. CTA 0 waits (bounded) until every CTA has counted out, then writes
//      what the barrier words overlay -- the code bytes of block 0 -- and ts.
// bar[] is the first 8 bytes of this call's code output: no state outlives
// the call, and concurrent calls do not share it.  On a timeout the device
// status word records RAZER_ERR_TIMEOUT and the outputs are void.
// ---------------------------------------------------------------------------
constexpr int kOneThreads = 1024;
constexpr int kOneChunk = 32768;                  // bytes per bulk copy
constexpr int kOneMaxChunks = 7;
constexpr int kOneMaxSlice = kOneChunk * kOneMaxChunks;  // 224 KB of blocks per CTA

__device__ __forceinline__ uint32_t ld_acquire_u32(const unsigned *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

template <int FMT, typename TIn, bool HIST>
__global__ void __launch_bounds__(kOneThreads, 1)
    quantize_onepass_kernel(const TIn *__restrict__ x, int64_t nblk, uint8_t *__restrict__ codes, uint8_t *__restrict__ scales,
                            float *ts_out, unsigned long long *__restrict__ hist, int inject_stall)
{
    using F = Fmt<FMT>;
    extern __shared__ __align__(128) uint8_t slice[];
    __shared__ __align__(8) uint64_t bars[kOneMaxChunks];
    __shared__ int s_abort;
    __shared__ float s_amax;
    __shared__ float tab_d[F::kMagMask + 1], tab_y[F::kMagMask + 1];
    // launched as a programmatic dependent of the init kernel: resident early,
    // it touches no global memory before that kernel (and the stream's earlier
    // work) has completed
    pdl_wait();
    const int G = gridDim.x, c = blockIdx.x;
    const int64_t b0 = (int64_t)c * nblk / G, b1 = (int64_t)(c + 1) * nblk / G;
    const int nb = (int)(b1 - b0), bytes = nb * 32, nch = (bytes + kOneChunk - 1) / kOneChunk;
    unsigned *bar = reinterpret_cast<unsigned *>(codes);  // [0] arrived, [1] departed (zeroed by the init kernel)
    unsigned *amax_bits = reinterpret_cast<unsigned *>(ts_out);
    const uint32_t bar0 = smem_addr(bars), sl = smem_addr(slice);
    if (threadIdx.x == 0) {
        for (int i = 0; i < nch; i++) mbar_init(bar0 + 8 * i, 1);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint8_t *src = reinterpret_cast<const uint8_t *>(x) + b0 * 32;
        for (int i = 0; i < nch; i++) {
            const uint32_t sz = (uint32_t)min(kOneChunk, bytes - i * kOneChunk);
            mbar_expect_tx(bar0 + 8 * i, sz);
            bulk_load(sl + (uint32_t)(i * kOneChunk), src + (size_t)i * kOneChunk, sz, bar0 + 8 * i);
        }
    }
    // 1. amax of the slice, chunk by chunk
    float m = 0.0f;
    for (int i = 0; i < nch; i++) {
        if (!mbar_try_wait(bar0 + 8 * i, 0)) (void)mbar_wait(bar0 + 8 * i, 0, &s_abort);
        const int nv = min(kOneChunk, bytes - i * kOneChunk) / 16;
        const uint4 *v = reinterpret_cast<const uint4 *>(slice + i * kOneChunk);
        for (int j = threadIdx.x; j < nv; j += kOneThreads) m = amax_vec<TIn>(m, v[j]);
    }
    commit_amax(m, amax_bits);  // ends with thread 0's atomicMax (after a block barrier)
    // 2. grid barrier
    if (threadIdx.x == 0) {
        __threadfence();
        if (!(inject_stall && c == 0)) atomicAdd(&bar[0], 1u);  // fault injection (tests only): CTA 0 never arrives
        const uint64_t t0 = globaltimer();
        while (ld_acquire_u32(&bar[0]) < (unsigned)G) {
            if (globaltimer() - t0 > kTimeoutNs) {
                set_device_status(RAZER_ERR_TIMEOUT);
                s_abort = 1;
                break;
            }
            __nanosleep(64);
        }
        // 3. the tensor amax, read once; then this CTA counts itself out (it
        // touches neither the barrier words nor the amax word again)
        s_amax = __uint_as_float(ld_acquire_u32(amax_bits));
        atomicAdd(&bar[1], 1u);
    }
    __syncthreads();
    const float ts = __fdiv_rn(s_amax, F::kC);
    const ScaleCtx k = make_ctx<FMT>(ts, tab_d, tab_y);
    __syncthreads();
    unsigned cnt[4] = {0u, 0u, 0u, 0u};
    uint2 block0 = make_uint2(0u, 0u);  // CTA 0's first block: written last
    const bool fast = fast_ts(ts);
    for (int j = threadIdx.x; j < nb; j += kOneThreads) {
        const uint4 *v = reinterpret_cast<const uint4 *>(slice + j * 32);
        const uint4 v0 = v[0], v1 = v[1];
        float xv[16];
        const unsigned wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const float2 f = In16<TIn>::to_f2(wv[i]);
            xv[2 * i] = f.x;
            xv[2 * i + 1] = f.y;
        }
        const BlockOut o = fast ? quantize_block<FMT, true, std::is_same<TIn, __half>::value>(xv, k)
                                : quantize_block<FMT, false, std::is_same<TIn, __half>::value>(xv, k);
        const int64_t b = b0 + j;
        if (b == 0) block0 = o.packed;
        else reinterpret_cast<uint2 *>(codes)[b] = o.packed;
        scales[b] = (uint8_t)o.sbyte;
        if constexpr (HIST) {
            const unsigned m1 = o.meta & 1u, e = o.effective ? 1u : 0u;
            cnt[0] += 1u - m1;
            cnt[1] += m1;
            cnt[2] += e & (1u - m1);
            cnt[3] += e & m1;
        }
    }
    if constexpr (HIST) {
        __shared__ unsigned long long sh[4];
        if (threadIdx.x < 4) sh[threadIdx.x] = 0ull;
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 4; i++) {
            unsigned cc = cnt[i];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) cc += __shfl_xor_sync(0xffffffffu, cc, o);
            if ((threadIdx.x & 31) == 0 && cc) atomicAdd(&sh[i], (unsigned long long)cc);
        }
        __syncthreads();
        if (threadIdx.x < 4 && sh[threadIdx.x]) atomicAdd(&hist[threadIdx.x], sh[threadIdx.x]);
    }
    // 4. block 0's codes and ts, once no CTA reads the barrier words or the amax word
    if (c == 0 && threadIdx.x == 0) {
        const uint64_t t0 = globaltimer();
        while (ld_acquire_u32(&bar[1]) < (unsigned)G && globaltimer() - t0 < kTimeoutNs) __nanosleep(64);
        if (nb > 0) reinterpret_cast<uint2 *>(codes)[0] = block0;
        *ts_out = ts;
    }
}

// ---------------------------------------------------------------------------
// Host launchers.
// ---------------------------------------------------------------------------
// CTAs of kQThreads threads of kernel f resident per SM (cached per kernel)
template <typename Kern> static int resident_ctas(Kern f)
{
    static int cached = 0;
    if (!cached) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, f, kQThreads, 0) != cudaSuccess || n <= 0) n = 4;
        cached = n;
    }
    return cached;
}

static int quant_grid(int64_t work, int threads, int per_sm)
{
    int64_t g = (work + threads - 1) / threads;
    int64_t cap = (int64_t)sm_count() * per_sm;
    if (g > cap) g = cap;
    return g < 1 ? 1 : (int)g;
}

template <typename TIn>
static void launch_amax(const void *x, int64_t n, unsigned *out, cudaStream_t st)
{
    const int64_t nvec = n / 8;
    launch_pdl(amax_kernel<TIn>, (unsigned)quant_grid(nvec, 256, 8), 256u, 0, st, reinterpret_cast<const TIn *>(x), nvec, out);
}

template <int FMT, typename TIn>
static void launch_quant(const void *x, int64_t nblk, const float *ts_src, int is_amax, uint8_t *codes,
                         uint8_t *scales, unsigned long long *hist, cudaStream_t st)
{
    // one wave of resident CTAs: a second, partial wave costs more than the
    // grid-stride loop's extra iterations
    static int per_sm[2] = {0, 0};
    const bool h = hist && Fmt<FMT>::kSpecials > 0;
    if (!per_sm[h]) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, h ? quantize_kernel<FMT, TIn, true> : quantize_kernel<FMT, TIn, false>,
                                                          kQThreads, 0) != cudaSuccess ||
            n <= 0)
            n = 4;
        per_sm[h] = n;
    }
    const unsigned grid = (unsigned)quant_grid(nblk, kQThreads, per_sm[h]);
    if (h)
        launch_pdl(quantize_kernel<FMT, TIn, true>, grid, (unsigned)kQThreads, 0, st, reinterpret_cast<const TIn *>(x), nblk, ts_src,
                   is_amax, codes, scales, hist);
    else
        launch_pdl(quantize_kernel<FMT, TIn, false>, grid, (unsigned)kQThreads, 0, st, reinterpret_cast<const TIn *>(x), nblk, ts_src,
                   is_amax, codes, scales, hist);
}

template <int FMT>
static void launch_quant_dt(razer_dtype dt, const void *x, int64_t nblk, const float *ts_src, int is_amax,
                            uint8_t *codes, uint8_t *scales, unsigned long long *hist, cudaStream_t st)
{
    if (dt == RAZER_F16) launch_quant<FMT, __half>(x, nblk, ts_src, is_amax, codes, scales, hist, st);
    else launch_quant<FMT, __nv_bfloat16>(x, nblk, ts_src, is_amax, codes, scales, hist, st);
}

// the single-pass kernel takes a dynamic-scale call when it is selected and
// each SM's slice fits in shared memory.  It is not the default: on a B200 the
// two-pass form measured faster (2048 x 4096 bf16 activations: 14.9 us against
// 17.1 us), because its quantize phase cannot start before the slowest slice
// has landed and the grid has met, while the two-pass form's amax kernel hands
// over to the quantizer through a programmatic dependent launch and the
// quantizer's second read of X comes from L2.
static std::atomic<bool> g_single_pass{false};
bool set_single_pass_quantizer(bool on) { return g_single_pass.exchange(on, std::memory_order_relaxed); }

static bool onepass_eligible(int64_t nblk)
{
    if (!g_single_pass.load(std::memory_order_relaxed)) return false;
    const int64_t G = sm_count();
    return nblk >= G && (nblk + G - 1) / G * 32 <= kOneMaxSlice;
}

template <int FMT, typename TIn>
static razer_status launch_onepass(const void *x, int64_t nblk, uint8_t *codes, uint8_t *scales, float *ts_out, unsigned long long *hist,
                                   cudaStream_t st)
{
    const int G = sm_count();
    const int64_t slice = (nblk + G - 1) / G * 32;
    static bool attr_done[2][64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    const bool h = hist && Fmt<FMT>::kSpecials > 0;
    auto kern = h ? quantize_onepass_kernel<FMT, TIn, true> : quantize_onepass_kernel<FMT, TIn, false>;
    if (dev >= 0 && dev < 64 && !attr_done[h][dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kOneMaxSlice) != cudaSuccess) return RAZER_ERR_CUDA;
        attr_done[h][dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)G);
    cfg.blockDim = dim3((unsigned)kOneThreads);
    cfg.dynamicSmemBytes = (size_t)slice;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident at once: the grid barrier cannot wait on an unscheduled CTA
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const int inject = fault_injection_enabled() ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, reinterpret_cast<const TIn *>(x), nblk, codes, scales, ts_out, hist, inject);
    if (e == cudaErrorCooperativeLaunchTooLarge) {
        (void)cudaGetLastError();
        return RAZER_ERR_UNSUPPORTED;  // fewer SMs than the device reports (a partitioned GPU): the caller takes the two-pass path
    }
    return e == cudaSuccess ? RAZER_OK : RAZER_ERR_CUDA;
}

// Runs the whole quantizer on one stream.  ts_in == nullptr: dynamic scale
// (the single-pass kernel when each SM's slice fits in shared memory, else
// memset + amax + quantize + finalize into ts_out); otherwise static.
razer_status run_quantize(const void *x, razer_dtype dt, int64_t R, int64_t K, const float *ts_in, uint8_t *codes,
                          uint8_t *scales, float *ts_out, unsigned long long *hist, razer_format fmt, cudaStream_t st)
{
    const int64_t n = R * K;
    const int64_t nblk = n / 16;
    const float C = fmt == RAZER_FMT_WEIGHT ? Fmt<RAZER_FMT_WEIGHT>::kC : Fmt<RAZER_FMT_ACT>::kC;
    if (!ts_in && onepass_eligible(nblk)) {
        if (launch_pdl(quant_init_kernel, 1u, 32u, 0, st, hist, reinterpret_cast<unsigned *>(ts_out), reinterpret_cast<unsigned *>(codes)) !=
            cudaSuccess)
            return RAZER_ERR_CUDA;
        const bool h = dt == RAZER_F16;
        razer_status r;
        if (fmt == RAZER_FMT_WEIGHT)
            r = h ? launch_onepass<RAZER_FMT_WEIGHT, __half>(x, nblk, codes, scales, ts_out, nullptr, st)
                  : launch_onepass<RAZER_FMT_WEIGHT, __nv_bfloat16>(x, nblk, codes, scales, ts_out, nullptr, st);
        else if (fmt == RAZER_FMT_ACT)
            r = h ? launch_onepass<RAZER_FMT_ACT, __half>(x, nblk, codes, scales, ts_out, hist, st)
                  : launch_onepass<RAZER_FMT_ACT, __nv_bfloat16>(x, nblk, codes, scales, ts_out, hist, st);
        else
            r = h ? launch_onepass<RAZER_FMT_NVFP4, __half>(x, nblk, codes, scales, ts_out, nullptr, st)
                  : launch_onepass<RAZER_FMT_NVFP4, __nv_bfloat16>(x, nblk, codes, scales, ts_out, nullptr, st);
        if (r != RAZER_ERR_UNSUPPORTED) return r;
    }
    // every kernel of the chain is a programmatic dependent of the previous one
    // (it is scheduled early and waits before touching memory)
    if (hist || !ts_in) {
        if (launch_pdl(quant_init_kernel, 1u, 32u, 0, st, hist, ts_in ? (unsigned *)nullptr : reinterpret_cast<unsigned *>(ts_out),
                   (unsigned *)nullptr) !=
            cudaSuccess)
            return RAZER_ERR_CUDA;
    }
    const float *ts_src = ts_in;
    int is_amax = 0;
    if (!ts_in) {
        if (n > 0) {
            if (dt == RAZER_F16) launch_amax<__half>(x, n, reinterpret_cast<unsigned *>(ts_out), st);
            else launch_amax<__nv_bfloat16>(x, n, reinterpret_cast<unsigned *>(ts_out), st);
        }
        ts_src = ts_out;
        is_amax = 1;
    }
    if (nblk > 0) {
        if (fmt == RAZER_FMT_WEIGHT) launch_quant_dt<RAZER_FMT_WEIGHT>(dt, x, nblk, ts_src, is_amax, codes, scales, nullptr, st);
        else if (fmt == RAZER_FMT_ACT) launch_quant_dt<RAZER_FMT_ACT>(dt, x, nblk, ts_src, is_amax, codes, scales, hist, st);
        else launch_quant_dt<RAZER_FMT_NVFP4>(dt, x, nblk, ts_src, is_amax, codes, scales, nullptr, st);
    }
    if (!ts_in) {
        if (launch_pdl(finalize_ts_kernel, 1u, 1u, 0, st, ts_out, C) != cudaSuccess) return RAZER_ERR_CUDA;
    } else if (ts_out != ts_in) {
        if (launch_pdl(copy_ts_kernel, 1u, 1u, 0, st, ts_in, ts_out) != cudaSuccess) return RAZER_ERR_CUDA;
    }
    return last_launch_status();
}

// Warps (of the 8 in a CTA) that stream the amax of the next tensor in a
// batch stage: proportional to that part's expected share of the stage time,
// at rates measured on this GPU (the amax warps ~8 TB/s of 16-byte vectors,
// tuned so that the stage time is lowest; the quantizer ~92 G blocks/s).
#ifndef RAZER_QSTAGE_AMAX_RATE
#define RAZER_QSTAGE_AMAX_RATE 5.0e11  // 16-byte vectors per second
#endif
#ifndef RAZER_QSTAGE_QUANT_RATE
#define RAZER_QSTAGE_QUANT_RATE 9.2e10  // 16-element blocks per second
#endif
static int stage_amax_warps(int64_t nblk, int64_t nva)
{
    if (nva == 0) return 0;
    if (nblk == 0) return kQThreads / 32;
    const double ta = (double)nva / RAZER_QSTAGE_AMAX_RATE, tq = (double)nblk / RAZER_QSTAGE_QUANT_RATE;
    int aw = (int)(8.0 * ta / (ta + tq) + 0.5);
    return aw < 1 ? 1 : (aw > 6 ? 6 : aw);
}

// Batched weight quantizer: tensors 0..count-1 with their amax words in
// ts[0..count).  Stage 0 reduces amax of tensor 0; stage i (1 <= i < count)
// quantizes tensor i-1 and reduces amax of tensor i in one kernel; the last
// stage quantizes tensor count-1.  Each tensor's codes, scales and ts are
// those of a separate run_quantize call.
template <int FMT, typename TIn>
static razer_status run_batch_t(int count, const void *const *W, const int64_t *R, const int64_t *K, uint8_t *const *codes,
                                uint8_t *const *scales, float *ts, cudaStream_t st)
{
    const float C = Fmt<FMT>::kC;
    unsigned *bits = reinterpret_cast<unsigned *>(ts);
    if (launch_pdl(init_many_kernel, 1u, 256u, 0, st, bits, count) != cudaSuccess) return RAZER_ERR_CUDA;
    if (R[0] * K[0] > 0) launch_amax<TIn>(W[0], R[0] * K[0], bits, st);
    for (int i = 1; i < count; i++) {
        const int64_t nblk = R[i - 1] * K[i - 1] / 16, nva = R[i] * K[i] / 8;
        if (nblk + nva == 0) continue;
        const int aw = stage_amax_warps(nblk, nva);
        // one CTA per resident slot, fewer when a thread would otherwise get no work
        const int qw = kQThreads / 32 - aw;
        const int64_t need_q = qw ? (nblk + 32 * qw - 1) / (32 * qw) : 0, need_a = aw ? (nva + 32 * aw - 1) / (32 * aw) : 0;
        const int64_t cap = (int64_t)sm_count() * resident_ctas(quant_amax_kernel<FMT, TIn>);
        const int64_t need = need_q > need_a ? need_q : need_a;
        const unsigned grid = (unsigned)(need < 1 ? 1 : (need > cap ? cap : need));
        if (launch_pdl(quant_amax_kernel<FMT, TIn>, grid, (unsigned)kQThreads, 0, st, reinterpret_cast<const TIn *>(W[i - 1]), nblk,
                       const_cast<const float *>(ts + i - 1), codes[i - 1], scales[i - 1], reinterpret_cast<const TIn *>(W[i]), nva,
                       bits + i, aw) != cudaSuccess)
            return RAZER_ERR_CUDA;
    }
    const int l = count - 1;
    if (R[l] * K[l] > 0) launch_quant<FMT, TIn>(W[l], R[l] * K[l] / 16, ts + l, 1, codes[l], scales[l], nullptr, st);
    if (launch_pdl(finalize_many_kernel, 1u, 256u, 0, st, ts, count, C) != cudaSuccess) return RAZER_ERR_CUDA;
    return last_launch_status();
}

razer_status run_quantize_batch(int count, const void *const *W, razer_dtype dt, const int64_t *R, const int64_t *K,
                                uint8_t *const *codes, uint8_t *const *scales, float *ts, razer_format fmt, cudaStream_t st)
{
    if (count == 0) return RAZER_OK;
    const bool h = dt == RAZER_F16;
    if (fmt == RAZER_FMT_WEIGHT)
        return h ? run_batch_t<RAZER_FMT_WEIGHT, __half>(count, W, R, K, codes, scales, ts, st)
                 : run_batch_t<RAZER_FMT_WEIGHT, __nv_bfloat16>(count, W, R, K, codes, scales, ts, st);
    return h ? run_batch_t<RAZER_FMT_NVFP4, __half>(count, W, R, K, codes, scales, ts, st)
             : run_batch_t<RAZER_FMT_NVFP4, __nv_bfloat16>(count, W, R, K, codes, scales, ts, st);
}

}  // namespace razer
