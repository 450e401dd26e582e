// Accuracy ablations on sm_100a: the FourOverSix block quantizer and the
// quantization error of a packed tensor.
//
// FourOverSix (Four Over Six summary page, 方法详解: 技术框架, 关键创新)
// keeps the NVFP4 encoding but lets each block scale its amax to 4 instead of
// 6 when that leaves the smaller error.  One thread per 16-element block
// quantizes the block under both scales -- IEEE divides throughout, the plain
// E2M1 codes with ties to the smaller magnitude -- and compares the squared
// errors sum_j (x_j - q_j * d)^2 accumulated in double in element order with
// explicitly rounded operations (no contraction), so the choice is the one
// the CPU reference makes.  The 4-candidate wins only with a strictly
// smaller error.  This is an accuracy tool, not a hot path: it spends two
// divides per element and a few double operations.
//
// The error kernel sums (x - q*s*ts)^2 over a packed tensor in double (q*s*ts
// is exact in double); the partial sums meet in an atomic add, so the last
// bits depend on the order the blocks finish in.
#include "razer_internal.cuh"
#include "variant.cuh"

namespace razer {

// signed value of a plain E2M1 code (no remap)
__device__ __forceinline__ float e2m1_value(unsigned c)
{
    const float m = fp4_mag(c & 7u);
    return (c & 8u) ? -m : m;
}

// Plain E2M1 code of xs, ties to the smaller magnitude, -0 -> 0b0000: the odd
// one of the hardware RNE conversions of xs and of xs * (1 - 2^-24) (the
// identity the quantizer uses, checked on the CPU for every binary32 in
// [0, 16]).
__device__ __forceinline__ unsigned e2m1_code_down(float xs)
{
    unsigned short a, b;
    asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u16.u8 %0, t; }" : "=h"(a) : "f"(0.0f), "f"(xs));
    asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u16.u8 %0, t; }"
        : "=h"(b)
        : "f"(0.0f), "f"(__fmul_rn(xs, 1.0f - 0x1p-24f)));
    const unsigned c1 = a & 15u, c2 = b & 15u;
    const unsigned c = (c1 & 1u) ? c1 : c2;
    return (c & 7u) ? c : 0u;
}

// One candidate of a block: scale amax_b -> cmax (6 or 4).  Returns the
// squared error; codes (4 bits each, element j at nibble j of the 64-bit
// word) and the E4M3 scale code through the references.
__device__ __forceinline__ double block_candidate(const float (&x)[16], float amax, float ts, float cmax, unsigned long long &codes,
                                                  unsigned &sc_out)
{
    const float s_f = __fdiv_rn(amax, __fmul_rn(cmax, ts));
    unsigned short h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(s_f));
    const unsigned sc = (unsigned)h & 0x7Fu;
    const float d = __fmul_rn(decode_scale<RAZER_FMT_NVFP4>(sc), ts);
    double sse = 0.0;
    codes = 0ull;
    sc_out = sc;
    if (sc == 0u || d == 0.0f) {
        sc_out = 0u;
#pragma unroll
        for (int j = 0; j < 16; j++) sse = __dadd_rn(sse, __dmul_rn((double)x[j], (double)x[j]));
        return sse;
    }
#pragma unroll
    for (int j = 0; j < 16; j++) {
        const unsigned c = e2m1_code_down(__fdiv_rn(x[j], d));
        codes |= (unsigned long long)c << (4 * j);
        const double t = __dsub_rn((double)x[j], __dmul_rn((double)e2m1_value(c), (double)d));
        sse = __dadd_rn(sse, __dmul_rn(t, t));
    }
    return sse;
}

template <typename TIn>
__global__ void __launch_bounds__(256) quantize46_kernel(const TIn *__restrict__ x, int64_t nblk, const float *__restrict__ ts_src,
                                                         int ts_is_amax, uint8_t *__restrict__ codes, uint8_t *__restrict__ scales,
                                                         unsigned long long *__restrict__ n_four)
{
    pdl_wait();
    pdl_trigger();
    const float tv = *ts_src;
    const float ts = ts_is_amax ? __fdiv_rn(tv, Fmt<RAZER_FMT_NVFP4>::kC) : tv;
    unsigned fours = 0u;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk; b += stride) {
        const uint4 *p = reinterpret_cast<const uint4 *>(x) + 2 * b;
        const uint4 v0 = ldg_stream(p), v1 = ldg_stream(p + 1);
        const unsigned wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        float xv[16];
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const float2 f = In16<TIn>::to_f2(wv[i]);
            xv[2 * i] = f.x;
            xv[2 * i + 1] = f.y;
        }
        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < 16; j++) amax = fmaxf(amax, fabsf(xv[j]));
        unsigned long long c = 0ull;
        unsigned sc = 0u;
        if (ts > 0.0f) {  // ts <= 0 leaves the block zero
            unsigned long long c6, c4;
            unsigned sc6, sc4;
            const double e6 = block_candidate(xv, amax, ts, 6.0f, c6, sc6);
            const double e4 = block_candidate(xv, amax, ts, 4.0f, c4, sc4);
            const bool four = e4 < e6;
            c = four ? c4 : c6;
            sc = four ? sc4 : sc6;
            fours += four ? 1u : 0u;
        }
        // element 2i in the low nibble of byte i: the nibble order of c
        reinterpret_cast<uint2 *>(codes)[b] = make_uint2((unsigned)c, (unsigned)(c >> 32));
        scales[b] = (uint8_t)sc;
    }
    if (n_four) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) fours += __shfl_xor_sync(0xffffffffu, fours, o);
        if ((threadIdx.x & 31) == 0 && fours) atomicAdd(n_four, (unsigned long long)fours);
    }
}

// q * s of element (code nibble, scale byte) of a format, exact in binary32
template <int FMT> __device__ __forceinline__ float elem_qs(unsigned code, unsigned sb)
{
    using F = Fmt<FMT>;
    const float s = decode_scale<FMT>(sb & F::kMagMask);
    if (F::kSpecials > 0 && code == 8u) return __fmul_rn(special_value((int)(sb >> F::kMetaShift)), s);
    return __fmul_rn(e2m1_value(code), s);
}

template <int FMT, typename TIn>
__global__ void __launch_bounds__(256) quant_sse_kernel(const TIn *__restrict__ x, int64_t nblk, const uint8_t *__restrict__ codes,
                                                        const uint8_t *__restrict__ scales, const float *__restrict__ ts_p,
                                                        double *__restrict__ out)
{
    pdl_wait();
    pdl_trigger();
    const double ts = (double)*ts_p;
    double acc = 0.0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk; b += stride) {
        const uint4 *p = reinterpret_cast<const uint4 *>(x) + 2 * b;
        const uint4 v0 = ldg_stream(p), v1 = ldg_stream(p + 1);
        const unsigned wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        const uint2 cw = reinterpret_cast<const uint2 *>(codes)[b];
        const unsigned long long c = (unsigned long long)cw.x | ((unsigned long long)cw.y << 32);
        const unsigned sb = scales[b];
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const float2 f = In16<TIn>::to_f2(wv[i]);
            const double v0d = __dmul_rn((double)elem_qs<FMT>((unsigned)(c >> (8 * i)) & 15u, sb), ts);
            const double v1d = __dmul_rn((double)elem_qs<FMT>((unsigned)(c >> (8 * i + 4)) & 15u, sb), ts);
            const double t0 = __dsub_rn((double)f.x, v0d), t1 = __dsub_rn((double)f.y, v1d);
            acc = __dadd_rn(acc, __dadd_rn(__dmul_rn(t0, t0), __dmul_rn(t1, t1)));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    __shared__ double sm[8];
    if ((threadIdx.x & 31) == 0) sm[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double r = 0.0;
        for (int i = 0; i < (int)(blockDim.x >> 5); i++) r += sm[i];
        atomicAdd(out, r);
    }
}

// ---------------------------------------------------------------------------
// Format variants: any block size (16..128) and special-value set.
// ---------------------------------------------------------------------------
// nearest of the grid u {v} to xs, given the plain rounding rp: v wins when
// strictly nearer, or equally near with the smaller magnitude (the grid tie
// rule); distances are exact in binary32 (xs and the points are multiples of
// xs's ulp, |xs| <= 16)
__device__ __forceinline__ bool takes_v(float xs, float rp, float v)
{
    const float dv = fabsf(__fsub_rn(xs, v)), dp = fabsf(__fsub_rn(xs, rp));
    return dv < dp || (dv == dp && fabsf(v) < fabsf(rp));
}

// Scale formats of the variants: E3M3 / E4M3 codes (with the tensor scale),
// or the FP16 word of the pages' kernel format (R17: s = RN_fp16(amax / 6)
// with bits 15..14 clear, saturating at 0x3FFF; no tensor scale; meta in bits
// 15..14).
constexpr int kScaleF16 = RAZER_SCALE_F16;
template <int SFMT> struct VarScale {
    static constexpr float kC = Fmt<SFMT>::kC;
    static constexpr int kMetaShift = Fmt<SFMT>::kMetaShift;
    static constexpr unsigned kMagMask = Fmt<SFMT>::kMagMask;
    static constexpr int kBytes = 1;
    static __device__ __forceinline__ unsigned encode(float amax, float ts)
    {
        return ts > 0.0f ? encode_scale<SFMT>(__fdiv_rn(amax, __fmul_rn(6.0f, ts))) : 0u;
    }
    static __device__ __forceinline__ float value(unsigned code) { return decode_scale<SFMT>(code); }
    static __device__ __forceinline__ float d(unsigned code, float ts) { return __fmul_rn(decode_scale<SFMT>(code), ts); }
};
template <> struct VarScale<kScaleF16> {
    static constexpr float kC = 1.0f;
    static constexpr int kMetaShift = 14;
    static constexpr unsigned kMagMask = 0x3FFFu;
    static constexpr int kBytes = 2;
    static __device__ __forceinline__ unsigned encode(float amax, float)
    {
        const unsigned h = __half_as_ushort(__float2half_rn(__fdiv_rn(amax, 6.0f)));
        return h > 0x3FFFu ? 0x3FFFu : h;
    }
    static __device__ __forceinline__ float value(unsigned code) { return __half2float(__ushort_as_half((unsigned short)code)); }
    static __device__ __forceinline__ float d(unsigned code, float) { return value(code); }
};

// One thread per 16 elements; the bs / 16 lanes of a block (consecutive,
// inside one warp) reduce its amax and the candidates' exact error
// differences with shuffles.  Decisions as the oracle's ro_quantize_generic.
template <int SFMT, typename TIn>
__global__ void __launch_bounds__(256) quantize_variant_kernel(const TIn *__restrict__ x, int64_t nsub, int group,
                                                               const float *__restrict__ ts_src, int ts_is_amax, VariantV V,
                                                               uint8_t *__restrict__ codes, uint8_t *__restrict__ scales)
{
    using F = VarScale<SFMT>;
    pdl_wait();
    pdl_trigger();
    const float tv = SFMT == kScaleF16 ? 1.0f : *ts_src;
    const float ts = (ts_is_amax && SFMT != kScaleF16) ? __fdiv_rn(tv, F::kC) : tv;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;  // a multiple of 32: groups never straddle warps
    const int64_t nsub_pad = (nsub + 31) / 32 * 32;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < nsub_pad; t += stride) {
        const bool live = t < nsub;
        float xv[16];
        if (live) {
            const uint4 *p = reinterpret_cast<const uint4 *>(x) + 2 * t;
            const uint4 v0 = ldg_stream(p), v1 = ldg_stream(p + 1);
            const unsigned wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const float2 f = In16<TIn>::to_f2(wv[i]);
                xv[2 * i] = f.x;
                xv[2 * i + 1] = f.y;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 16; j++) xv[j] = 0.0f;
        }
        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < 16; j++) amax = fmaxf(amax, fabsf(xv[j]));
        for (int o = 1; o < group; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        // every lane of the warp runs the same shuffle sequence below; a
        // block with a zero scale (or ts <= 0) contributes nothing and stays 0
        const unsigned sc = F::encode(amax, ts);
        const float d = F::d(sc, ts);
        const bool active = ts > 0.0f && sc != 0u && d != 0.0f;
        const float dd = active ? d : 1.0f;
        float xs[16], rp[16];
        unsigned pc[16];
#pragma unroll
        for (int j = 0; j < 16; j++) {
            xs[j] = active ? fminf(fmaxf(__fdiv_rn(xv[j], dd), -16.0f), 16.0f) : 0.0f;
            pc[j] = e2m1_code_down(xs[j]);
            rp[j] = e2m1_value(pc[j]);
        }
        int meta = 0;
        double best = 0.0;
        for (int m = 0; m < V.nv; m++) {
            double delta = 0.0;
#pragma unroll
            for (int j = 0; j < 16; j++) {
                if (takes_v(xs[j], rp[j], V.v[m])) {
                    const double r0 = rp[j], r1 = V.v[m];
                    delta = __dadd_rn(delta, __dmul_rn(__dsub_rn(r0, r1), __dsub_rn(__dsub_rn(2.0 * (double)xs[j], r1), r0)));
                }
            }
            for (int o = 1; o < group; o <<= 1) delta += __shfl_xor_sync(0xffffffffu, delta, o);
            if (m == 0 || delta < best) {
                best = delta;
                meta = m;
            }
        }
        unsigned long long c = 0ull;
        unsigned sb = 0u;
        if (active) {
#pragma unroll
            for (int j = 0; j < 16; j++) {
                const unsigned code = (V.nv > 0 && takes_v(xs[j], rp[j], V.v[meta])) ? 8u : pc[j];
                c |= (unsigned long long)code << (4 * j);
            }
            sb = sc | (V.nv > 0 ? (unsigned)meta << F::kMetaShift : 0u);
        }
        if (live) {
            reinterpret_cast<uint2 *>(codes)[t] = make_uint2((unsigned)c, (unsigned)(c >> 32));
            if (t % group == 0) {
                if (F::kBytes == 2) reinterpret_cast<uint16_t *>(scales)[t / group] = (uint16_t)sb;
                else scales[t / group] = (uint8_t)sb;
            }
        }
    }
}

template <int SFMT, typename TIn>
__global__ void __launch_bounds__(256) quant_sse_variant_kernel(const TIn *__restrict__ x, int64_t nsub, int group,
                                                                const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scales,
                                                                const float *__restrict__ ts_p, VariantV V, double *__restrict__ out)
{
    using F = VarScale<SFMT>;
    pdl_wait();
    pdl_trigger();
    const double ts = (double)*ts_p;
    double acc = 0.0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < nsub; t += stride) {
        const uint4 *p = reinterpret_cast<const uint4 *>(x) + 2 * t;
        const uint4 v0 = ldg_stream(p), v1 = ldg_stream(p + 1);
        const unsigned wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        const uint2 cw = reinterpret_cast<const uint2 *>(codes)[t];
        const unsigned long long c = (unsigned long long)cw.x | ((unsigned long long)cw.y << 32);
        const unsigned sb = F::kBytes == 2 ? (unsigned)reinterpret_cast<const uint16_t *>(scales)[t / group] : (unsigned)scales[t / group];
        const double s = (double)F::value(sb & F::kMagMask);
        const float vm = V.nv > 0 ? V.v[sb >> F::kMetaShift] : 0.0f;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const float2 f = In16<TIn>::to_f2(wv[i]);
            const unsigned c0 = (unsigned)(c >> (8 * i)) & 15u, c1 = (unsigned)(c >> (8 * i + 4)) & 15u;
            const double q0 = (V.nv > 0 && c0 == 8u) ? vm : e2m1_value(c0), q1 = (V.nv > 0 && c1 == 8u) ? vm : e2m1_value(c1);
            const double t0 = __dsub_rn((double)f.x, __dmul_rn(__dmul_rn(q0, s), ts));
            const double t1 = __dsub_rn((double)f.y, __dmul_rn(__dmul_rn(q1, s), ts));
            acc = __dadd_rn(acc, __dadd_rn(__dmul_rn(t0, t0), __dmul_rn(t1, t1)));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    __shared__ double sm[8];
    if ((threadIdx.x & 31) == 0) sm[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double r = 0.0;
        for (int i = 0; i < (int)(blockDim.x >> 5); i++) r += sm[i];
        atomicAdd(out, r);
    }
}

__global__ void set_one_kernel(float *p)
{
    pdl_wait();
    *p = 1.0f;
}

__global__ void zero_u64_kernel(unsigned long long *a, unsigned long long *b)
{
    pdl_wait();
    pdl_trigger();
    if (threadIdx.x == 0) {
        if (a) *a = 0ull;
        if (b) *b = 0ull;
    }
}

// FourOverSix quantizer: dynamic ts = amax / (6 * 448) as for NVFP4 (init,
// amax, quantize, finalize on one stream); n_four (device, may be NULL)
// receives the number of blocks that took the amax -> 4 scale.
razer_status run_quantize_46(const void *x, razer_dtype dt, int64_t R, int64_t K, uint8_t *codes, uint8_t *scales, float *ts_out,
                             unsigned long long *n_four, cudaStream_t st)
{
    const int64_t n = R * K, nblk = n / 16;
    if (launch_pdl(zero_u64_kernel, 1u, 32u, 0, st, n_four, (unsigned long long *)nullptr) != cudaSuccess) return RAZER_ERR_CUDA;
    if (launch_pdl(quant_init_kernel, 1u, 32u, 0, st, (unsigned long long *)nullptr, reinterpret_cast<unsigned *>(ts_out), (unsigned *)nullptr) !=
        cudaSuccess)
        return RAZER_ERR_CUDA;
    if (n > 0) {
        if (dt == RAZER_F16) launch_amax<__half>(x, n, reinterpret_cast<unsigned *>(ts_out), st);
        else launch_amax<__nv_bfloat16>(x, n, reinterpret_cast<unsigned *>(ts_out), st);
    }
    if (nblk > 0) {
        const unsigned grid = (unsigned)quant_grid(nblk, 256, 8);
        const cudaError_t e =
            dt == RAZER_F16
                ? launch_pdl(quantize46_kernel<__half>, grid, 256u, 0, st, reinterpret_cast<const __half *>(x), nblk, (const float *)ts_out, 1,
                             codes, scales, n_four)
                : launch_pdl(quantize46_kernel<__nv_bfloat16>, grid, 256u, 0, st, reinterpret_cast<const __nv_bfloat16 *>(x), nblk,
                             (const float *)ts_out, 1, codes, scales, n_four);
        if (e != cudaSuccess) return RAZER_ERR_CUDA;
    }
    if (launch_pdl(finalize_ts_kernel, 1u, 1u, 0, st, ts_out, Fmt<RAZER_FMT_NVFP4>::kC) != cudaSuccess) return RAZER_ERR_CUDA;
    return last_launch_status();
}

template <int FMT>
static cudaError_t launch_sse(razer_dtype dt, const void *x, int64_t nblk, const uint8_t *codes, const uint8_t *scales, const float *ts,
                              double *out, cudaStream_t st)
{
    const unsigned grid = (unsigned)quant_grid(nblk, 256, 8);
    if (dt == RAZER_F16)
        return launch_pdl(quant_sse_kernel<FMT, __half>, grid, 256u, 0, st, reinterpret_cast<const __half *>(x), nblk, codes, scales, ts, out);
    return launch_pdl(quant_sse_kernel<FMT, __nv_bfloat16>, grid, 256u, 0, st, reinterpret_cast<const __nv_bfloat16 *>(x), nblk, codes,
                      scales, ts, out);
}

razer_status run_quant_sse(const void *x, razer_dtype dt, int64_t R, int64_t K, const uint8_t *codes, const uint8_t *scales,
                           const float *ts, razer_format fmt, double *out, cudaStream_t st)
{
    const int64_t nblk = R * K / 16;
    if (launch_pdl(zero_u64_kernel, 1u, 32u, 0, st, reinterpret_cast<unsigned long long *>(out), (unsigned long long *)nullptr) !=
        cudaSuccess)
        return RAZER_ERR_CUDA;
    if (nblk == 0) return last_launch_status();
    cudaError_t e;
    if (fmt == RAZER_FMT_WEIGHT) e = launch_sse<RAZER_FMT_WEIGHT>(dt, x, nblk, codes, scales, ts, out, st);
    else if (fmt == RAZER_FMT_ACT) e = launch_sse<RAZER_FMT_ACT>(dt, x, nblk, codes, scales, ts, out, st);
    else e = launch_sse<RAZER_FMT_NVFP4>(dt, x, nblk, codes, scales, ts, out, st);
    return e == cudaSuccess ? RAZER_OK : RAZER_ERR_CUDA;
}

// Format-variant quantizer (block bs, special values V, scale format sfmt):
// dynamic ts = amax / (6 * S_max(sfmt)).
razer_status run_quantize_variant(const void *x, razer_dtype dt, int64_t R, int64_t K, int bs, razer_format sfmt, const VariantV &V,
                                  uint8_t *codes, uint8_t *scales, float *ts_out, cudaStream_t st)
{
    const int64_t n = R * K, nsub = n / 16;
    const float C = sfmt == RAZER_FMT_WEIGHT ? Fmt<RAZER_FMT_WEIGHT>::kC : Fmt<RAZER_FMT_ACT>::kC;
    if (launch_pdl(quant_init_kernel, 1u, 32u, 0, st, (unsigned long long *)nullptr, reinterpret_cast<unsigned *>(ts_out), (unsigned *)nullptr) !=
        cudaSuccess)
        return RAZER_ERR_CUDA;
    if (n > 0) {
        if (dt == RAZER_F16) launch_amax<__half>(x, n, reinterpret_cast<unsigned *>(ts_out), st);
        else launch_amax<__nv_bfloat16>(x, n, reinterpret_cast<unsigned *>(ts_out), st);
    }
    if (nsub > 0) {
        const unsigned grid = (unsigned)quant_grid((nsub + 31) / 32 * 32, 256, 8);
        const int group = bs / 16;
        const float *tsrc = ts_out;
        cudaError_t e;
        const bool h = dt == RAZER_F16;
        if (sfmt == RAZER_SCALE_F16)
            e = h ? launch_pdl(quantize_variant_kernel<kScaleF16, __half>, grid, 256u, 0, st, reinterpret_cast<const __half *>(x), nsub,
                               group, tsrc, 1, V, codes, scales)
                  : launch_pdl(quantize_variant_kernel<kScaleF16, __nv_bfloat16>, grid, 256u, 0, st, reinterpret_cast<const __nv_bfloat16 *>(x),
                               nsub, group, tsrc, 1, V, codes, scales);
        else if (sfmt == RAZER_FMT_WEIGHT)
            e = h ? launch_pdl(quantize_variant_kernel<RAZER_FMT_WEIGHT, __half>, grid, 256u, 0, st, reinterpret_cast<const __half *>(x), nsub,
                               group, tsrc, 1, V, codes, scales)
                  : launch_pdl(quantize_variant_kernel<RAZER_FMT_WEIGHT, __nv_bfloat16>, grid, 256u, 0, st,
                               reinterpret_cast<const __nv_bfloat16 *>(x), nsub, group, tsrc, 1, V, codes, scales);
        else
            e = h ? launch_pdl(quantize_variant_kernel<RAZER_FMT_ACT, __half>, grid, 256u, 0, st, reinterpret_cast<const __half *>(x), nsub,
                               group, tsrc, 1, V, codes, scales)
                  : launch_pdl(quantize_variant_kernel<RAZER_FMT_ACT, __nv_bfloat16>, grid, 256u, 0, st,
                               reinterpret_cast<const __nv_bfloat16 *>(x), nsub, group, tsrc, 1, V, codes, scales);
        if (e != cudaSuccess) return RAZER_ERR_CUDA;
    }
    if (sfmt == RAZER_SCALE_F16) {  // no tensor scale: ts = 1
        if (launch_pdl(set_one_kernel, 1u, 1u, 0, st, ts_out) != cudaSuccess) return RAZER_ERR_CUDA;
    } else if (launch_pdl(finalize_ts_kernel, 1u, 1u, 0, st, ts_out, C) != cudaSuccess) {
        return RAZER_ERR_CUDA;
    }
    return last_launch_status();
}

razer_status run_quant_sse_variant(const void *x, razer_dtype dt, int64_t R, int64_t K, int bs, razer_format sfmt, const VariantV &V,
                                   const uint8_t *codes, const uint8_t *scales, const float *ts, double *out, cudaStream_t st)
{
    const int64_t nsub = R * K / 16;
    if (launch_pdl(zero_u64_kernel, 1u, 32u, 0, st, reinterpret_cast<unsigned long long *>(out), (unsigned long long *)nullptr) !=
        cudaSuccess)
        return RAZER_ERR_CUDA;
    if (nsub == 0) return last_launch_status();
    const unsigned grid = (unsigned)quant_grid(nsub, 256, 8);
    const int group = bs / 16;
    const bool h = dt == RAZER_F16;
    cudaError_t e;
    if (sfmt == RAZER_SCALE_F16)
        e = h ? launch_pdl(quant_sse_variant_kernel<kScaleF16, __half>, grid, 256u, 0, st, reinterpret_cast<const __half *>(x), nsub, group,
                           codes, scales, ts, V, out)
              : launch_pdl(quant_sse_variant_kernel<kScaleF16, __nv_bfloat16>, grid, 256u, 0, st, reinterpret_cast<const __nv_bfloat16 *>(x),
                           nsub, group, codes, scales, ts, V, out);
    else if (sfmt == RAZER_FMT_WEIGHT)
        e = h ? launch_pdl(quant_sse_variant_kernel<RAZER_FMT_WEIGHT, __half>, grid, 256u, 0, st, reinterpret_cast<const __half *>(x), nsub,
                           group, codes, scales, ts, V, out)
              : launch_pdl(quant_sse_variant_kernel<RAZER_FMT_WEIGHT, __nv_bfloat16>, grid, 256u, 0, st,
                           reinterpret_cast<const __nv_bfloat16 *>(x), nsub, group, codes, scales, ts, V, out);
    else
        e = h ? launch_pdl(quant_sse_variant_kernel<RAZER_FMT_ACT, __half>, grid, 256u, 0, st, reinterpret_cast<const __half *>(x), nsub,
                           group, codes, scales, ts, V, out)
              : launch_pdl(quant_sse_variant_kernel<RAZER_FMT_ACT, __nv_bfloat16>, grid, 256u, 0, st,
                           reinterpret_cast<const __nv_bfloat16 *>(x), nsub, group, codes, scales, ts, V, out);
    return e == cudaSuccess ? RAZER_OK : RAZER_ERR_CUDA;
}

}  // namespace razer
