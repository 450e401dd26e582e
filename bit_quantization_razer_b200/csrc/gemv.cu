// RaZeR W4A16 GEMV / skinny GEMM (1 <= B <= 32) for sm_100a.
//
// y[b, n] = ts * sum_k x[b, k] * (q*s)[n, k]      (RaZeR notes 关键设计 3:
// weight-only kernels that decode the remapped codes in registers; the
// small-batch split-K sizing of the same section is done per launch for the
// 148 SMs of a B200).
//
// Design (HBM-bound: 0.5625 byte of weights per multiply-add at B = 1):
//   * a warp owns 16 weight rows; each step consumes a 16-row x 128-k slice of
//     codes (64 contiguous bytes per row, 4 lanes per row) plus the matching
//     scale bytes, streamed through a 4-stage per-warp shared-memory ring with
//     16-byte cp.async copies, so three slices per warp are in flight without
//     holding registers;
//   * each code byte becomes one f16x2 pair with the hardware E2M1 convert;
//     the redundant-zero codes receive v*s through the convert of an
//     indicator word folded in with one packed FMA, and the block scale is a
//     packed multiply -- q*s*2^-12 (E3M3) or q*s*2^-8 (E4M3) is exact in fp16
//     (the integer / convert work runs on the half-rate ALU pipe, which bounds
//     this kernel, so the decode keeps it to 11 operations per 8 codes);
//   * the decoded pairs are already in the register layout of the A operand of
//     the warp-level m16n8k16 tensor-core MMA, so the products accumulate in
//     fp32 without any shared-memory round trip; the activations form the
//     n8 operand (B <= 8 uses one MMA per k16, B <= 32 four).  The reduction
//     order over k within each 16 columns is permuted identically on both
//     operands, which leaves the sum unchanged;
//   * split-K partials go to a caller-provided fp32 workspace and a second
//     small kernel sums them, applies ts (and the 2^12 / 2^8 unbias) and
//     converts to the output type.
#include <algorithm>

#include "razer_internal.cuh"

namespace razer {

constexpr int kGemvWarps = 4;
constexpr int kGemvThreads = kGemvWarps * 32;

// E2M1 pair -> f16x2 of byte lane L of w (the convert reads the byte lane
// directly, no shift).
template <int L>
__device__ __forceinline__ unsigned cvt_lane(unsigned w)
{
    unsigned r;
    if constexpr (L == 0) asm("{ .reg .b8 b0, b1, b2, b3; mov.b32 {b0, b1, b2, b3}, %1; cvt.rn.f16x2.e2m1x2 %0, b0; }" : "=r"(r) : "r"(w));
    if constexpr (L == 1) asm("{ .reg .b8 b0, b1, b2, b3; mov.b32 {b0, b1, b2, b3}, %1; cvt.rn.f16x2.e2m1x2 %0, b1; }" : "=r"(r) : "r"(w));
    if constexpr (L == 2) asm("{ .reg .b8 b0, b1, b2, b3; mov.b32 {b0, b1, b2, b3}, %1; cvt.rn.f16x2.e2m1x2 %0, b2; }" : "=r"(r) : "r"(w));
    if constexpr (L == 3) asm("{ .reg .b8 b0, b1, b2, b3; mov.b32 {b0, b1, b2, b3}, %1; cvt.rn.f16x2.e2m1x2 %0, b3; }" : "=r"(r) : "r"(w));
    return r;
}

__device__ __forceinline__ unsigned hfma2u(unsigned a, unsigned b, unsigned c)
{
    unsigned r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}

__device__ __forceinline__ unsigned hmul2u(unsigned a, unsigned b)
{
    unsigned r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// f16x2 -> bf16x2 (exact for the decoded values: at most 7 significant bits,
// inside the bf16 range).  Through fp32: the direct 16-bit convert is a slow
// instruction on this GPU, the f16 -> f32 converts and the f32 pair pack are not.
__device__ __forceinline__ unsigned f16x2_to_bf16x2(unsigned h)
{
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h));
    __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
    return *reinterpret_cast<unsigned *>(&b);
}

__device__ __forceinline__ unsigned prmt(unsigned a, unsigned b, unsigned sel)
{
    unsigned r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// Decode 8 codes of one block (a 32-bit word) into 4 packed pairs of
// (q * s * 2^-bias): pair b holds nibbles 2b (low half) and 2b+1.  The
// redundant-zero codes (0b1000, converted to -0) receive v*s through a
// second conversion of an indicator word holding the code of 1.0 (0b0010)
// exactly where the code is 0b1000, folded in with one packed FMA.  Integer
// and conversion work shares the half-rate ALU pipe, so the indicator shift
// is a high multiply (FMA pipe) and the converts read byte lanes directly.
template <int FMT, bool BF16>
__device__ __forceinline__ void decode_word(unsigned w, unsigned s2, unsigned vs2, unsigned (&h)[4])
{
    unsigned q[4] = {cvt_lane<0>(w), cvt_lane<1>(w), cvt_lane<2>(w), cvt_lane<3>(w)};
    if constexpr (Fmt<FMT>::kSpecials > 0) {
        // bit 3 set where the magnitude is non-zero; the add is issued as an
        // integer multiply-add so that it runs on the FMA pipe -- the ALU pipe
        // (converts, logic) bounds this decode (three 8B projections at
        // B = 1: 30.3 -> 29.1 us)
        unsigned t;
        asm("mad.lo.u32 %0, %1, 1, 0x77777777;" : "=r"(t) : "r"(w & 0x77777777u));
        const unsigned is8 = w & ~t & 0x88888888u;                 // bit 3 set where the code is 0b1000
        const unsigned ind = __umulhi(is8, 0x40000000u);          // is8 >> 2: nibble 0b0010 (= 1.0)
        const unsigned i[4] = {cvt_lane<0>(ind), cvt_lane<1>(ind), cvt_lane<2>(ind), cvt_lane<3>(ind)};
#pragma unroll
        for (int b = 0; b < 4; b++) {
            const unsigned r = hfma2u(i[b], vs2, hmul2u(q[b], s2));
            h[b] = BF16 ? f16x2_to_bf16x2(r) : r;
        }
    } else {
#pragma unroll
        for (int b = 0; b < 4; b++) {
            const unsigned r = hmul2u(q[b], s2);
            h[b] = BF16 ? f16x2_to_bf16x2(r) : r;
        }
    }
}

template <bool BF16>
__device__ __forceinline__ void mma16816(float (&d)[4], unsigned a0, unsigned a1, unsigned a2, unsigned a3, unsigned b0, unsigned b1)
{
    if constexpr (BF16) {
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                     : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                     : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    } else {
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                     : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                     : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
}

// fp16 pairs of s * 2^-bias and of v * s * 2^-bias for the two blocks held in
// the low 16 bits of sb (one scale byte per block).
template <int FMT>
__device__ __forceinline__ void scale_pairs2(unsigned sb, unsigned (&s2)[2], unsigned (&v2)[2])
{
    const unsigned x = prmt(sb, 0u, 0x4140u);  // 16-bit lanes: byte 0, byte 1
    const unsigned sx = (x & (Fmt<FMT>::kMagMask * 0x10001u)) << 7;  // fp16 [s0, s1] * 2^-12 (E3M3) / 2^-8 (E4M3)
    s2[0] = prmt(sx, 0u, 0x1010u);
    s2[1] = prmt(sx, 0u, 0x3232u);
    if constexpr (Fmt<FMT>::kSpecials > 0) {
        // fp16 high bytes of +5, -5, +8, -8 indexed by the meta value; one
        // permute builds [v0, v1] for both blocks
        constexpr unsigned kVHigh = 0xC848C545u;
        const unsigned m = (x >> Fmt<FMT>::kMetaShift) & 0x00030003u;  // meta0 | meta1 << 16
        const unsigned sel = 0x0404u | ((m & 3u) << 4) | ((m >> 16) << 12);
        const unsigned vs = hmul2u(prmt(kVHigh, 0u, sel), sx);          // [v0 * s0, v1 * s1]
        v2[0] = prmt(vs, 0u, 0x1010u);
        v2[1] = prmt(vs, 0u, 0x3232u);
    } else {
        v2[0] = v2[1] = 0u;
    }
}

// One 16-row x 128-k slice: ca / cb are this lane's 16 code bytes of MMA
// rows g and g+8 (32 codes = two blocks each), sA / sB their two scale bytes,
// xw the activation fragments of the same 32 k (zero for batch rows past B).
template <int FMT, bool BF16, int NB>
__device__ __forceinline__ void slice_mma(const uint4 &ca, const uint4 &cb, unsigned sA, unsigned sB, const unsigned (&xw)[NB][16],
                                          float (&acc)[NB][4])
{
    unsigned s2A[2], vA[2], s2B[2], vB[2];
    scale_pairs2<FMT>(sA, s2A, vA);
    scale_pairs2<FMT>(sB, s2B, vB);
    const unsigned wa[4] = {ca.x, ca.y, ca.z, ca.w};
    const unsigned wb[4] = {cb.x, cb.y, cb.z, cb.w};
#pragma unroll
    for (int m = 0; m < 4; m++) {
        unsigned hA[4], hB[4];
        decode_word<FMT, BF16>(wa[m], s2A[m >> 1], vA[m >> 1], hA);
        decode_word<FMT, BF16>(wb[m], s2B[m >> 1], vB[m >> 1], hB);
#pragma unroll
        for (int j = 0; j < NB; j++) {
            mma16816<BF16>(acc[j], hA[0], hB[0], hA[1], hB[1], xw[j][4 * m], xw[j][4 * m + 1]);
            mma16816<BF16>(acc[j], hA[2], hB[2], hA[3], hB[3], xw[j][4 * m + 2], xw[j][4 * m + 3]);
        }
    }
}

constexpr int kRing = 4;                          // stages per warp ring
constexpr int kCodeBytes = 16 * 64;               // 16 rows x 64 bytes per chunk
constexpr int kScaleBytes = 16 * 8;               // 16 rows x 8 scale bytes
constexpr int kXRowBytes = 128 * 2;               // one activation row of a chunk
// stage = codes | scales | activations (B <= 8 rows, only when NB == 1)
__host__ __device__ constexpr int gemv_stage_bytes(int xrows) { return kCodeBytes + kScaleBytes + xrows * kXRowBytes; }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int FMT, bool BF16, int NB>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(const uint16_t *__restrict__ x, int B, const uint8_t *__restrict__ codes,
                                                            const uint8_t *__restrict__ scales, int N, int K, int S,
                                                            float *__restrict__ ws)
{
    extern __shared__ __align__(16) uint8_t gemv_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int row0 = (blockIdx.x * kGemvWarps + warp) * 16;
    if (row0 >= N) return;
    const int s = blockIdx.y;
    const int chunks = K >> 7;
    const int c_begin = (int)((int64_t)s * chunks / S), c_end = (int)((int64_t)(s + 1) * chunks / S);
    const int rA = min(row0 + g, N - 1), rB = min(row0 + g + 8, N - 1);
    const uint8_t *pa = codes + (size_t)rA * (K >> 1) + 16 * t;
    const uint8_t *pb = codes + (size_t)rB * (K >> 1) + 16 * t;
    const uint8_t *sa = scales + (size_t)rA * (K >> 4);
    const uint8_t *sbp = scales + (size_t)rB * (K >> 4);

    // this warp's ring: stage = [16 rows x 64 B of codes][16 rows x 8 B of
    // scales][activation rows of the chunk, B <= 8 only]
    const int xrows = NB == 1 ? B : 0;
    const int stage_bytes = gemv_stage_bytes(xrows);
    uint8_t *ring = gemv_smem + warp * (kRing * stage_bytes);
    const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
    auto issue = [&](int c, int slot) {
        if (c < c_end) {
            const uint32_t st = ring_s + slot * stage_bytes;
            cp_async16(st + g * 64 + 16 * t, pa + (size_t)c * 64);
            cp_async16(st + (g + 8) * 64 + 16 * t, pb + (size_t)c * 64);
            if (t < 2) {  // 8 scale bytes per row (scales are only 4-byte aligned)
                cp_async4(st + kCodeBytes + g * 8 + 4 * t, sa + (size_t)c * 8 + 4 * t);
                cp_async4(st + kCodeBytes + (g + 8) * 8 + 4 * t, sbp + (size_t)c * 8 + 4 * t);
            }
            if (NB == 1 && g < B) {  // this lane's 64 activation bytes
                const uint8_t *src = reinterpret_cast<const uint8_t *>(x + (size_t)g * K + (size_t)c * 128 + 32 * t);
                const uint32_t dst = st + kCodeBytes + kScaleBytes + g * kXRowBytes + 64 * t;
#pragma unroll
                for (int q = 0; q < 4; q++) cp_async16(dst + 16 * q, src + 16 * q);
            }
        }
        cp_async_commit();  // one group per chunk (possibly empty) keeps the counting uniform
    };

    float acc[NB][4];
#pragma unroll
    for (int j = 0; j < NB; j++) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;

    unsigned xw[NB][16];
#pragma unroll
    for (int j = 0; j < NB; j++)
#pragma unroll
        for (int q = 0; q < 16; q++) xw[j][q] = 0u;

#pragma unroll
    for (int i = 0; i < kRing - 1; i++) issue(c_begin + i, i);
    for (int c = c_begin; c < c_end; c++) {
        const int i = c - c_begin;
        __syncwarp();  // every lane is done with the slot refilled next
        issue(c + kRing - 1, (i + kRing - 1) % kRing);
        cp_async_wait<kRing - 1>();  // this chunk's group has landed
        __syncwarp();                // scale bytes were copied by lanes t < 2 of each row group
        const uint8_t *st = ring + (i % kRing) * stage_bytes;
        const uint4 ca = *reinterpret_cast<const uint4 *>(st + g * 64 + 16 * t);
        const uint4 cb = *reinterpret_cast<const uint4 *>(st + (g + 8) * 64 + 16 * t);
        const unsigned sA = *reinterpret_cast<const unsigned short *>(st + kCodeBytes + g * 8 + 2 * t);
        const unsigned sB = *reinterpret_cast<const unsigned short *>(st + kCodeBytes + (g + 8) * 8 + 2 * t);
#pragma unroll
        for (int j = 0; j < NB; j++) {
            if (8 * j + g < B) {  // lanes past the batch keep their zero fragments
                const uint4 *px = NB == 1 ? reinterpret_cast<const uint4 *>(st + kCodeBytes + kScaleBytes + g * kXRowBytes + 64 * t)
                                          : reinterpret_cast<const uint4 *>(x + (size_t)(8 * j + g) * K + (size_t)c * 128 + 32 * t);
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    const uint4 v = NB == 1 ? px[q] : __ldg(px + q);
                    xw[j][4 * q] = v.x;
                    xw[j][4 * q + 1] = v.y;
                    xw[j][4 * q + 2] = v.z;
                    xw[j][4 * q + 3] = v.w;
                }
            }
        }
        slice_mma<FMT, BF16, NB>(ca, cb, sA, sB, xw, acc);
    }
    cp_async_wait<0>();

    // partials: D[g][2t..2t+1] -> rows row0+g, D[g+8][..] -> rows row0+g+8
    float *wsb = ws + (size_t)s * B * N;
#pragma unroll
    for (int j = 0; j < NB; j++) {
        const int n0 = 8 * j + 2 * t;
#pragma unroll
        for (int h = 0; h < 2; h++) {
            const int row = row0 + g + 8 * h;
            if (row < N) {
                if (n0 < B) wsb[(size_t)n0 * N + row] = acc[j][2 * h];
                if (n0 + 1 < B) wsb[(size_t)(n0 + 1) * N + row] = acc[j][2 * h + 1];
            }
        }
    }
}

template <typename TOut>
__global__ void __launch_bounds__(256) gemv_reduce_kernel(const float *__restrict__ ws, int S, int64_t BN, const float *__restrict__ ts_p,
                                                          float unbias, TOut *__restrict__ y)
{
    const float scale = __fmul_rn(*ts_p, unbias);
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < BN; i += stride) {
        // independent loads, eight at a time, added in split order
        float a = 0.0f;
        for (int s0 = 0; s0 < S; s0 += 8) {
            float v[8];
#pragma unroll
            for (int k = 0; k < 8; k++) v[k] = s0 + k < S ? ws[(size_t)(s0 + k) * BN + i] : 0.0f;
#pragma unroll
            for (int k = 0; k < 8; k++)
                if (s0 + k < S) a += v[k];
        }
        a = __fmul_rn(a, scale);
        if constexpr (sizeof(TOut) == 4) y[i] = a;
        else if constexpr (std::is_same<TOut, __half>::value) y[i] = __float2half_rn(a);
        else y[i] = __float2bfloat16_rn(a);
    }
}

// ---------------------------------------------------------------------------
// Split-K sizing: enough CTAs for ~8 resident 4-warp CTAs per SM, never more
// splits than 128-wide k chunks (each split keeps at least two chunks when K
// allows, so the reduction stays small against the weight stream).
// ---------------------------------------------------------------------------
int gemv_splits(int64_t B, int64_t N, int64_t K)
{
    (void)B;
    const int64_t ctas_x = ((N + 15) / 16 + kGemvWarps - 1) / kGemvWarps;
    const int64_t chunks = K / 128;
    const int64_t target = (int64_t)sm_count() * 8;
    int64_t S = (target + ctas_x - 1) / ctas_x;
    const int64_t max_s = chunks >= 4 ? chunks / 2 : (chunks > 0 ? chunks : 1);
    if (S > max_s) S = max_s;
    if (S < 1) S = 1;
    return (int)S;
}

// ---------------------------------------------------------------------------
// Any K % 16 == 0 (K % 128 != 0 has no 128-k chunking): one thread per weight
// row, every block decoded exactly in binary32 (q*s, or v*s for the
// redundant-zero code) and multiplied into B fp32 accumulators; y = ts * sum.
// The activations are read through the read-only cache (every thread of a
// warp reads the same element).  No workspace.
// ---------------------------------------------------------------------------
template <int FMT, typename TIn>
__global__ void __launch_bounds__(128) gemv_generic_kernel(const TIn *__restrict__ x, int B, const uint8_t *__restrict__ codes,
                                                           const uint8_t *__restrict__ scales, const float *__restrict__ ts_p, int N, int K,
                                                           void *y, int out_dt)
{
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    float acc[32];
#pragma unroll
    for (int b = 0; b < 32; b++) acc[b] = 0.0f;
    const int nb = K >> 4;
    const uint2 *crow = reinterpret_cast<const uint2 *>(codes + (size_t)n * (K >> 1));  // 8 bytes per block (K/2 % 8 == 0)
    const uint8_t *srow = scales + (size_t)n * nb;
    for (int kb = 0; kb < nb; kb++) {
        const uint2 cw = __ldg(crow + kb);
        const unsigned sb = srow[kb];
        const float s = decode_scale<FMT>(sb);
        float v = 0.0f;
        if constexpr (Fmt<FMT>::kSpecials > 0) v = special_value((int)(sb >> Fmt<FMT>::kMetaShift));
#pragma unroll
        for (int e = 0; e < 16; e++) {
            const unsigned c = ((e < 8 ? cw.x : cw.y) >> (4 * (e & 7))) & 0xFu;
            float q = fp4_mag(c & 7u);
            if (c & 8u) q = (Fmt<FMT>::kSpecials > 0 && c == 8u) ? v : -q;
            const float w = __fmul_rn(q, s);  // exact
            const size_t k = (size_t)kb * 16 + e;
            for (int b = 0; b < B; b++) {
                const TIn xv = x[(size_t)b * K + k];
                float xf;
                if constexpr (std::is_same<TIn, __half>::value) xf = __half2float(xv);
                else xf = __bfloat162float(xv);
                acc[b] = fmaf(xf, w, acc[b]);
            }
        }
    }
    const float ts = *ts_p;
    for (int b = 0; b < B; b++) {
        const float a = __fmul_rn(acc[b], ts);
        const size_t i = (size_t)b * N + n;
        if (out_dt == RAZER_F32) reinterpret_cast<float *>(y)[i] = a;
        else if (out_dt == RAZER_F16) reinterpret_cast<__half *>(y)[i] = __float2half_rn(a);
        else reinterpret_cast<__nv_bfloat16 *>(y)[i] = __float2bfloat16_rn(a);
    }
}

template <int FMT>
static razer_status launch_gemv_generic(const void *x, razer_dtype act_dt, int B, const uint8_t *codes, const uint8_t *scales,
                                        const float *ts, int N, int K, void *y, razer_dtype out_dt, cudaStream_t st)
{
    const unsigned grid = (unsigned)((N + 127) / 128);
    if (act_dt == RAZER_F16)
        gemv_generic_kernel<FMT, __half><<<grid, 128, 0, st>>>(reinterpret_cast<const __half *>(x), B, codes, scales, ts, N, K, y, (int)out_dt);
    else
        gemv_generic_kernel<FMT, __nv_bfloat16><<<grid, 128, 0, st>>>(reinterpret_cast<const __nv_bfloat16 *>(x), B, codes, scales, ts, N, K, y,
                                                                     (int)out_dt);
    return last_launch_status();
}

bool gemv_tma_eligible(int64_t B, int64_t N, int64_t K);
size_t gemv_tma_workspace_bytes(int64_t B, int64_t N, int64_t K);
razer_status run_gemv_tma(const void *x, razer_dtype act_dt, int64_t B, const uint8_t *codes, const uint8_t *scales, const float *ts,
                          razer_format wfmt, int64_t N, int64_t K, void *y, razer_dtype out_dt, void *workspace, cudaStream_t st);

size_t gemv_workspace_bytes(int64_t B, int64_t N, int64_t K)
{
    if (B <= 0 || N <= 0 || K <= 0 || K % 128 != 0) return 0;  // K % 128 != 0: the generic kernel, no workspace
    // the per-warp kernel also serves eligible shapes whose scale pointer is
    // only 4-byte aligned (a tensor map needs 16), so size for both
    const size_t split = (size_t)gemv_splits(B, N, K) * (size_t)B * (size_t)N * sizeof(float);
    return gemv_tma_eligible(B, N, K) ? std::max(split, gemv_tma_workspace_bytes(B, N, K)) : split;
}

template <int FMT, bool BF16>
static void launch_gemv_fmt(const void *x, int B, const uint8_t *codes, const uint8_t *scales, int N, int K, int S, float *ws,
                            cudaStream_t st)
{
    dim3 grid((unsigned)(((N + 15) / 16 + kGemvWarps - 1) / kGemvWarps), (unsigned)S);
    const uint16_t *xp = reinterpret_cast<const uint16_t *>(x);
    const int smem1 = kGemvWarps * kRing * gemv_stage_bytes(B), smem0 = kGemvWarps * kRing * gemv_stage_bytes(0);
    static bool attr_done[64] = {false};  // per device: allow up to 8 activation rows in the ring (> 48 KB)
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        cudaFuncSetAttribute(gemv_kernel<FMT, BF16, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kGemvWarps * kRing * gemv_stage_bytes(8));
        attr_done[dev] = true;
    }
    if (B <= 8) gemv_kernel<FMT, BF16, 1><<<grid, kGemvThreads, smem1, st>>>(xp, B, codes, scales, N, K, S, ws);
    else if (B <= 16) gemv_kernel<FMT, BF16, 2><<<grid, kGemvThreads, smem0, st>>>(xp, B, codes, scales, N, K, S, ws);
    else gemv_kernel<FMT, BF16, 4><<<grid, kGemvThreads, smem0, st>>>(xp, B, codes, scales, N, K, S, ws);
}

razer_status run_gemv(const void *x, razer_dtype act_dt, int64_t B, const uint8_t *codes, const uint8_t *scales, const float *ts,
                      razer_format wfmt, int64_t N, int64_t K, void *y, razer_dtype out_dt, void *workspace, cudaStream_t st)
{
    if (K % 128 != 0) {
        if (wfmt == RAZER_FMT_WEIGHT) return launch_gemv_generic<RAZER_FMT_WEIGHT>(x, act_dt, (int)B, codes, scales, ts, (int)N, (int)K, y, out_dt, st);
        if (wfmt == RAZER_FMT_ACT) return launch_gemv_generic<RAZER_FMT_ACT>(x, act_dt, (int)B, codes, scales, ts, (int)N, (int)K, y, out_dt, st);
        return launch_gemv_generic<RAZER_FMT_NVFP4>(x, act_dt, (int)B, codes, scales, ts, (int)N, (int)K, y, out_dt, st);
    }
    if (gemv_tma_eligible(B, N, K) && (reinterpret_cast<uintptr_t>(scales) & 15) == 0)
        return run_gemv_tma(x, act_dt, B, codes, scales, ts, wfmt, N, K, y, out_dt, workspace, st);
    const int S = gemv_splits(B, N, K);
    float *ws = reinterpret_cast<float *>(workspace);
    const bool bf = act_dt == RAZER_BF16;
    if (wfmt == RAZER_FMT_WEIGHT) {
        if (bf) launch_gemv_fmt<RAZER_FMT_WEIGHT, true>(x, (int)B, codes, scales, (int)N, (int)K, S, ws, st);
        else launch_gemv_fmt<RAZER_FMT_WEIGHT, false>(x, (int)B, codes, scales, (int)N, (int)K, S, ws, st);
    } else if (wfmt == RAZER_FMT_ACT) {
        if (bf) launch_gemv_fmt<RAZER_FMT_ACT, true>(x, (int)B, codes, scales, (int)N, (int)K, S, ws, st);
        else launch_gemv_fmt<RAZER_FMT_ACT, false>(x, (int)B, codes, scales, (int)N, (int)K, S, ws, st);
    } else {
        if (bf) launch_gemv_fmt<RAZER_FMT_NVFP4, true>(x, (int)B, codes, scales, (int)N, (int)K, S, ws, st);
        else launch_gemv_fmt<RAZER_FMT_NVFP4, false>(x, (int)B, codes, scales, (int)N, (int)K, S, ws, st);
    }
    const float unbias = wfmt == RAZER_FMT_WEIGHT ? scale_f16_unbias<RAZER_FMT_WEIGHT>() : scale_f16_unbias<RAZER_FMT_ACT>();
    const int64_t BN = B * N;
    int64_t g = (BN + 255) / 256;
    if (g > (int64_t)sm_count() * 8) g = (int64_t)sm_count() * 8;
    if (g < 1) g = 1;
    if (out_dt == RAZER_F32) gemv_reduce_kernel<float><<<(int)g, 256, 0, st>>>(ws, S, BN, ts, unbias, reinterpret_cast<float *>(y));
    else if (out_dt == RAZER_F16) gemv_reduce_kernel<__half><<<(int)g, 256, 0, st>>>(ws, S, BN, ts, unbias, reinterpret_cast<__half *>(y));
    else gemv_reduce_kernel<__nv_bfloat16><<<(int)g, 256, 0, st>>>(ws, S, BN, ts, unbias, reinterpret_cast<__nv_bfloat16 *>(y));
    return last_launch_status();
}

}  // namespace razer
