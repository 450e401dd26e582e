// RaZeR decoder (RaZeR notes 关键设计 3: the FP4 -0 code decodes to the
// block's special value, selected by the meta bits of the scale byte).
//   out = round_out( (q * s) * ts ): q*s is exact in binary32, one binary32
//   multiply by ts, one rounding to the output type.
#include "razer_internal.cuh"

namespace razer {

template <typename TOut> struct Out16;
template <> struct Out16<__half> {
    static __device__ __forceinline__ unsigned pack(float a, float b)
    {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<unsigned *>(&h);
    }
};
template <> struct Out16<__nv_bfloat16> {
    static __device__ __forceinline__ unsigned pack(float a, float b)
    {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<unsigned *>(&h);
    }
};

template <int FMT, typename TOut>
__global__ void __launch_bounds__(256) dequant_kernel(const uint2 *__restrict__ codes, const uint8_t *__restrict__ scales,
                                                      const float *__restrict__ ts_p, int64_t nblk, TOut *__restrict__ out)
{
    using F = Fmt<FMT>;
    const float ts = *ts_p;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk; b += stride) {
        const uint2 c = codes[b];
        const unsigned sb = scales[b];
        const float s = decode_scale<FMT>(sb);
        const float v = F::kSpecials > 0 ? special_value((int)(sb >> F::kMetaShift)) : 0.0f;
        float val[16];
#pragma unroll
        for (int j = 0; j < 16; j++) {
            const unsigned code = ((j < 8 ? c.x : c.y) >> (4 * (j & 7))) & 15u;
            float q;
            if (code == 8u) q = v;
            else q = (code & 8u) ? -fp4_mag(code & 7u) : fp4_mag(code & 7u);
            val[j] = __fmul_rn(__fmul_rn(q, s), ts);
        }
        if constexpr (sizeof(TOut) == 4) {
            float4 *o = reinterpret_cast<float4 *>(out) + 4 * b;
#pragma unroll
            for (int i = 0; i < 4; i++) o[i] = make_float4(val[4 * i], val[4 * i + 1], val[4 * i + 2], val[4 * i + 3]);
        } else {
            uint4 *o = reinterpret_cast<uint4 *>(out) + 2 * b;
#pragma unroll
            for (int i = 0; i < 2; i++) {
                o[i] = make_uint4(Out16<TOut>::pack(val[8 * i], val[8 * i + 1]), Out16<TOut>::pack(val[8 * i + 2], val[8 * i + 3]),
                                  Out16<TOut>::pack(val[8 * i + 4], val[8 * i + 5]), Out16<TOut>::pack(val[8 * i + 6], val[8 * i + 7]));
            }
        }
    }
}

template <int FMT>
static void launch_dequant_fmt(const uint8_t *codes, const uint8_t *scales, const float *ts, int64_t nblk, void *out,
                               razer_dtype dt, cudaStream_t st)
{
    int64_t g = (nblk + 255) / 256;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (g > cap) g = cap;
    if (g < 1) g = 1;
    const uint2 *c = reinterpret_cast<const uint2 *>(codes);
    if (dt == RAZER_F32) dequant_kernel<FMT, float><<<(int)g, 256, 0, st>>>(c, scales, ts, nblk, reinterpret_cast<float *>(out));
    else if (dt == RAZER_F16) dequant_kernel<FMT, __half><<<(int)g, 256, 0, st>>>(c, scales, ts, nblk, reinterpret_cast<__half *>(out));
    else dequant_kernel<FMT, __nv_bfloat16><<<(int)g, 256, 0, st>>>(c, scales, ts, nblk, reinterpret_cast<__nv_bfloat16 *>(out));
}

razer_status run_dequant(const uint8_t *codes, const uint8_t *scales, const float *ts, razer_format fmt, int64_t R, int64_t K,
                         void *out, razer_dtype dt, cudaStream_t st)
{
    const int64_t nblk = R * K / 16;
    if (nblk == 0) return RAZER_OK;
    if (fmt == RAZER_FMT_WEIGHT) launch_dequant_fmt<RAZER_FMT_WEIGHT>(codes, scales, ts, nblk, out, dt, st);
    else if (fmt == RAZER_FMT_ACT) launch_dequant_fmt<RAZER_FMT_ACT>(codes, scales, ts, nblk, out, dt, st);
    else launch_dequant_fmt<RAZER_FMT_NVFP4>(codes, scales, ts, nblk, out, dt, st);
    return last_launch_status();
}

}  // namespace razer
