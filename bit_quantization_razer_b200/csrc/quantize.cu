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
//   * the squared-error comparison of the candidates is exact: only elements
//     whose nearest point changes contribute, each term (q - v)(2 xs - q - v)
//     is a multiple of 2^-20 computed exactly in binary32, and the partial
//     sums stay exact (see the notes on each accumulator below).
#include "razer_internal.cuh"

namespace razer {

// Plain E2M1 magnitude code of a = |xs|, nearest with ties to the smaller
// magnitude.  For a >= 1 the code is a half-down rounding of the binary32
// bit pattern to one mantissa bit (adding 2^21 - 1 then truncating rounds
// ties down); below 1 the two thresholds are compared directly.
__device__ __forceinline__ unsigned e2m1_mag_code(float a)
{
    unsigned u = __float_as_uint(a);
    unsigned hi = min(((u + 0x1FFFFFu) >> 22) - 252u, 7u);
    unsigned lo = (unsigned)(a > 0.25f) + (unsigned)(a > 0.75f);
    return a >= 1.0f ? hi : lo;
}

struct BlockOut {
    uint2 packed;    // 16 nibbles
    unsigned sbyte;  // scale byte (meta | magnitude code)
    unsigned meta;
    bool effective;  // the chosen special value strictly lowered the error
};

template <int FMT>
__device__ __forceinline__ BlockOut quantize_block(const float (&x)[16], float ts)
{
    using F = Fmt<FMT>;
    BlockOut o;
    o.packed = make_uint2(0u, 0u);
    o.sbyte = 0u;
    o.meta = 0u;
    o.effective = false;

    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; j++) amax = fmaxf(amax, fabsf(x[j]));
    if (!(ts > 0.0f)) return o;

    // block scale: s_f = amax_b / (6 ts), nearest scale code, exact decode
    const float sf = __fdiv_rn(amax, __fmul_rn(6.0f, ts));
    const unsigned sc = encode_scale<FMT>(sf);
    const float s = decode_scale<FMT>(sc);
    const float d = __fmul_rn(s, ts);
    if (sc == 0u || d == 0.0f) return o;

    // X^scaled = RN(x / d)
    float xs[16];
    if (d >= 0x1p-90f && d <= 0x1p90f) {
        const float y = __frcp_rn(d);
#pragma unroll
        for (int j = 0; j < 16; j++) {
            const float q = __fmul_rn(x[j], y);
            const float r = __fmaf_rn(-q, d, x[j]);
            xs[j] = __fmaf_rn(r, y, q);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; j++) xs[j] = __fdiv_rn(x[j], d);
    }

    unsigned meta = 0u;
    if constexpr (F::kSpecials > 0) {
        // v = +5 / -5: an element changes only inside (4.5, 5.5] (resp.
        // [-5.5, -4.5)), where the error difference is |2 xs -+ 10| - 1 in
        // [-1, 0].  2 xs -+ 10 is exact there (Sterbenz), and outside the
        // region the clamped term is exactly 0.  Terms are multiples of
        // 2^-20 and |sum| <= 16, so the binary32 sums are exact.
        float dp5 = 0.0f, dn5 = 0.0f;
#pragma unroll
        for (int j = 0; j < 16; j++) {
            dp5 = __fadd_rn(dp5, fminf(__fadd_rn(fabsf(__fmaf_rn(2.0f, xs[j], -10.0f)), -1.0f), 0.0f));
            dn5 = __fadd_rn(dn5, fminf(__fadd_rn(fabsf(__fmaf_rn(2.0f, xs[j], 10.0f)), -1.0f), 0.0f));
        }
        float best = dp5;
        if (dn5 < best) { best = dn5; meta = 1u; }
        if constexpr (F::kSpecials == 4) {
            // v = +8 / -8 changes an element only when |xs| > 7.  With a
            // normal scale code |xs| <= 6 / (1 - 2^-4) < 7, so only blocks with
            // a subnormal scale code (sc < 8) can use them; there |xs| <= 9
            // and the terms 2*(7 - |xs|)*2 = 28 - 4|xs| are summed exactly as
            // integers in units of 2^-20 together with the +-5 terms.
            if (sc < 8u) {
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
                meta = 0u;
                if (in5 < ib) { ib = in5; meta = 1u; }
                if (ip8 < ib) { ib = ip8; meta = 2u; }
                if (in8 < ib) { ib = in8; meta = 3u; }
                best = (float)ib;
            }
        }
        o.effective = best < 0.0f;
    }

    // final encode against Q_FP4 u {v*}
    const float v = special_value((int)meta);
    const float vsign = v < 0.0f ? -1.0f : 1.0f;
    const float rlo = fabsf(v) == 5.0f ? 4.5f : 7.0f;
    const float rhi = fabsf(v) == 5.0f ? 5.5f : 3.0e38f;
    unsigned w0 = 0u, w1 = 0u;
#pragma unroll
    for (int j = 0; j < 16; j++) {
        const float a = fabsf(xs[j]);
        const unsigned c = e2m1_mag_code(a);
        unsigned code = (c != 0u && xs[j] < 0.0f) ? (c | 8u) : c;
        if constexpr (F::kSpecials > 0) {
            const float sx = xs[j] * vsign;  // exact (multiplication by +-1)
            if (sx > rlo && sx <= rhi) code = 8u;
        }
        if (j < 8) w0 |= code << (4 * j);
        else w1 |= code << (4 * (j - 8));
    }
    o.packed = make_uint2(w0, w1);
    o.meta = meta;
    o.sbyte = sc | (meta << F::kMetaShift);
    return o;
}

constexpr int kQThreads = 256;

template <int FMT, typename TIn>
__global__ void __launch_bounds__(kQThreads) quantize_kernel(const TIn *__restrict__ x, int64_t nblk,
                                                             const float *__restrict__ ts_src, int ts_is_amax,
                                                             uint8_t *__restrict__ codes, uint8_t *__restrict__ scales,
                                                             unsigned long long *__restrict__ hist)
{
    using F = Fmt<FMT>;
    const float tv = *ts_src;
    const float ts = ts_is_amax ? __fdiv_rn(tv, F::kC) : tv;
    unsigned cnt[4] = {0u, 0u, 0u, 0u};

    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk; b += stride) {
        const uint4 *p = reinterpret_cast<const uint4 *>(x) + 2 * b;
        const uint4 v0 = ldg_stream(p);
        const uint4 v1 = ldg_stream(p + 1);
        float xv[16];
        const unsigned wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const float2 f = In16<TIn>::to_f2(wv[i]);
            xv[2 * i] = f.x;
            xv[2 * i + 1] = f.y;
        }
        const BlockOut o = quantize_block<FMT>(xv, ts);
        reinterpret_cast<uint2 *>(codes)[b] = o.packed;
        scales[b] = (uint8_t)o.sbyte;
        if constexpr (F::kSpecials > 0) {
            if (hist) {
                const unsigned m1 = o.meta & 1u, e = o.effective ? 1u : 0u;
                cnt[0] += 1u - m1;
                cnt[1] += m1;
                cnt[2] += e & (1u - m1);
                cnt[3] += e & m1;
            }
        }
    }
    if constexpr (F::kSpecials > 0) {
        if (hist) {
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
}

// amax(|x|) over n16 / 8 128-bit vectors; result as binary32 bits via
// atomicMax (order-preserving for non-negative floats) into *out.
template <typename TIn>
__global__ void __launch_bounds__(256) amax_kernel(const TIn *__restrict__ x, int64_t nvec, unsigned *__restrict__ out)
{
    float m = 0.0f;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const uint4 *p = reinterpret_cast<const uint4 *>(x);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += stride) {
        const uint4 v = ldg_stream(p + i);
        const unsigned w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const float2 f = In16<TIn>::to_f2(w[k]);
            m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float sm[8];
    if ((threadIdx.x & 31) == 0) sm[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float r = sm[0];
        for (int i = 1; i < (int)(blockDim.x >> 5); i++) r = fmaxf(r, sm[i]);
        if (r > 0.0f) atomicMax(out, __float_as_uint(r));
    }
}

// ts = amax / (6 * S_max), written over the amax word.
__global__ void finalize_ts_kernel(float *ts, float c)
{
    const float amax = __uint_as_float(*reinterpret_cast<unsigned *>(ts));
    *ts = __fdiv_rn(amax, c);
}

__global__ void copy_ts_kernel(const float *src, float *dst) { *dst = *src; }

// ---------------------------------------------------------------------------
// Host launchers.
// ---------------------------------------------------------------------------
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
    amax_kernel<TIn><<<quant_grid(nvec, 256, 8), 256, 0, st>>>(reinterpret_cast<const TIn *>(x), nvec, out);
}

template <int FMT, typename TIn>
static void launch_quant(const void *x, int64_t nblk, const float *ts_src, int is_amax, uint8_t *codes,
                         uint8_t *scales, unsigned long long *hist, cudaStream_t st)
{
    quantize_kernel<FMT, TIn><<<quant_grid(nblk, kQThreads, 8), kQThreads, 0, st>>>(
        reinterpret_cast<const TIn *>(x), nblk, ts_src, is_amax, codes, scales, hist);
}

template <int FMT>
static void launch_quant_dt(razer_dtype dt, const void *x, int64_t nblk, const float *ts_src, int is_amax,
                            uint8_t *codes, uint8_t *scales, unsigned long long *hist, cudaStream_t st)
{
    if (dt == RAZER_F16) launch_quant<FMT, __half>(x, nblk, ts_src, is_amax, codes, scales, hist, st);
    else launch_quant<FMT, __nv_bfloat16>(x, nblk, ts_src, is_amax, codes, scales, hist, st);
}

// Runs the whole quantizer on one stream.  ts_in == nullptr: dynamic scale
// (memset + amax + quantize + finalize into ts_out); otherwise static.
razer_status run_quantize(const void *x, razer_dtype dt, int64_t R, int64_t K, const float *ts_in, uint8_t *codes,
                          uint8_t *scales, float *ts_out, unsigned long long *hist, razer_format fmt, cudaStream_t st)
{
    const int64_t n = R * K;
    const int64_t nblk = n / 16;
    const float C = fmt == RAZER_FMT_WEIGHT ? Fmt<RAZER_FMT_WEIGHT>::kC : Fmt<RAZER_FMT_ACT>::kC;
    if (hist && cudaMemsetAsync(hist, 0, 4 * sizeof(unsigned long long), st) != cudaSuccess) return RAZER_ERR_CUDA;
    const float *ts_src = ts_in;
    int is_amax = 0;
    if (!ts_in) {
        if (cudaMemsetAsync(ts_out, 0, sizeof(float), st) != cudaSuccess) return RAZER_ERR_CUDA;
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
    if (!ts_in) finalize_ts_kernel<<<1, 1, 0, st>>>(ts_out, C);
    else if (ts_out != ts_in) copy_ts_kernel<<<1, 1, 0, st>>>(ts_in, ts_out);
    return last_launch_status();
}

}  // namespace razer
