// Internal device helpers of the RaZeR B200 library (not part of the ABI).
//
// Format facts used below (RaZeR notes, 关键设计 1: weight block scale in
// E3M3 with 2 meta bits, activation block scale in E4M3 with 1 meta bit;
// 关键设计 2: the FP4 -0 code carries the special value; 训练策略: V_w =
// {+-5, +-8}, V_a = {+-5}; gist.science summary, section 1: the E2M1 set).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "razer.h"

namespace razer {

// ---------------------------------------------------------------------------
// Device status word (bounded waits record RAZER_ERR_TIMEOUT here).
// ---------------------------------------------------------------------------
// Defined once: the library is built as a single translation unit.
__device__ unsigned int g_device_status = 0u;

__device__ __forceinline__ void set_device_status(unsigned s) { atomicCAS(&g_device_status, 0u, s); }

// ---------------------------------------------------------------------------
// Format traits.
// ---------------------------------------------------------------------------
template <int FMT> struct Fmt;

template <> struct Fmt<RAZER_FMT_WEIGHT> {
    static constexpr int kSpecials = 4;        // meta 0..3 -> +5, -5, +8, -8
    static constexpr unsigned kMagMask = 0x3F; // E3M3
    static constexpr int kMetaShift = 6;
    static constexpr float kSmax = 30.0f;
    static constexpr float kC = 180.0f;        // 6 * S_max
    static constexpr int kBias = 3;
    static constexpr float kSubStep = 0.03125f; // 2^-5
    static constexpr float kMinNormal = 0.25f;  // 2^-2
    static constexpr unsigned kMaxCode = 0x3F;
};

template <> struct Fmt<RAZER_FMT_ACT> {
    static constexpr int kSpecials = 2;        // meta 0..1 -> +5, -5
    static constexpr unsigned kMagMask = 0x7F; // E4M3
    static constexpr int kMetaShift = 7;
    static constexpr float kSmax = 448.0f;
    static constexpr float kC = 2688.0f;
    static constexpr int kBias = 7;
    static constexpr float kSubStep = 0.001953125f; // 2^-9
    static constexpr float kMinNormal = 0.015625f;  // 2^-6
    static constexpr unsigned kMaxCode = 0x7E;
};

template <> struct Fmt<RAZER_FMT_NVFP4> : Fmt<RAZER_FMT_ACT> {
    static constexpr int kSpecials = 0;
};

// Special value of a meta index (weights: +5, -5, +8, -8; activations: +5, -5).
__host__ __device__ __forceinline__ float special_value(int meta)
{
    return ((meta & 2) ? 8.0f : 5.0f) * ((meta & 1) ? -1.0f : 1.0f);
}

// Nearest scale code (ties to the even code), saturating at the largest code.
// Normal range: round the binary32 significand to 3 bits, nearest-even; the
// subnormal range (below the smallest normal) has a uniform step, so the code
// is the nearest-even integer multiple of that step (which may become the
// first normal code).
template <int FMT> __device__ __forceinline__ unsigned encode_scale(float sf)
{
    using F = Fmt<FMT>;
    if (!(sf < F::kSmax)) return F::kMaxCode;
    if (sf < F::kMinNormal) return (unsigned)__float2int_rn(__fmul_rn(sf, 1.0f / F::kSubStep));
    unsigned u = __float_as_uint(sf);
    unsigned r = u + 0x7FFFFu + ((u >> 20) & 1u);
    unsigned e = (r >> 23) - 127u + (unsigned)F::kBias;
    unsigned c = (e << 3) | ((r >> 20) & 7u);
    return c > F::kMaxCode ? F::kMaxCode : c;
}

// Exact binary32 value of a scale code (meta bits stripped).
template <int FMT> __device__ __forceinline__ float decode_scale(unsigned c)
{
    using F = Fmt<FMT>;
    c &= F::kMagMask;
    unsigned e = c >> 3, m = c & 7u;
    if (e == 0) return (float)m * F::kSubStep;
    return __uint_as_float(((e - (unsigned)F::kBias + 127u) << 23) | (m << 20));
}

// binary16 bit pattern of (scale value) * 2^-(12 or 8): placing the scale
// code's exponent/mantissa fields into the binary16 fields is an exact
// multiplication by a power of two, subnormals included.
template <int FMT> __device__ __forceinline__ unsigned scale_f16_bits(unsigned c)
{
    return (c & Fmt<FMT>::kMagMask) << 7;
}
template <int FMT> constexpr float scale_f16_unbias() { return FMT == RAZER_FMT_WEIGHT ? 4096.0f : 256.0f; }

// E2M1 magnitudes of codes 0..7 (binary32).
__device__ __forceinline__ float fp4_mag(unsigned c)
{
    // 0, 0.5, 1, 1.5, 2, 3, 4, 6
    return c < 2 ? 0.5f * (float)c : __uint_as_float(0x3F000000u + (c << 22));
}

// 16-bit loads/stores helpers ------------------------------------------------
template <typename T> struct In16;
template <> struct In16<__half> {
    static __device__ __forceinline__ float2 to_f2(unsigned w) { return __half22float2(*reinterpret_cast<__half2 *>(&w)); }
};
template <> struct In16<__nv_bfloat16> {
    static __device__ __forceinline__ float2 to_f2(unsigned w)
    {
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    }
};

__device__ __forceinline__ uint2 ldg_stream_u2(const uint2 *p)
{
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}
__device__ __forceinline__ uint4 ldg_stream(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

}  // namespace razer

// Launch helpers shared by the host files --------------------------------------
namespace razer {
// launch with the programmatic-stream-serialization attribute: the kernel may
// be scheduled before its predecessor in the stream has finished, and waits
// for it with griddepcontrol.wait before touching memory the predecessor wrote
template <typename... KArgs, typename... Args>
static inline cudaError_t launch_pdl(void (*kern)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t st, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// in a kernel launched that way: wait for the predecessor grid (no-op otherwise)
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// let the dependent grid be scheduled (it still waits for this grid to finish)
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

int sm_count();
razer_status last_launch_status();
// Test-only fault injection (razer_debug_set_fault_injection): a plain load
// on the launch path, no environment lookup per call.
bool fault_injection_enabled();
// dynamic-scale quantizer path (false: two-pass); returns the previous value
bool set_single_pass_quantizer(bool on);
}  // namespace razer
