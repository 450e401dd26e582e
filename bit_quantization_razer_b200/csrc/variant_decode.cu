// Decoder and W4A16 GEMV of the RaZeR format variants: blocks of 16, 32, 64
// or 128 elements, a caller-chosen special-value set (multiples of 0.5 in
// [2.5, 9.5], gist.science summary 2.2; per-model pairs such as +-5/+-7 in
// the RaZeR notes, 训练策略), and the pages' own kernel format (RaZeR notes,
// 关键设计 3: blocks of 128 with an FP16 scale whose sign bit and top
// exponent bit hold the meta).
//
// GEMV design: the per-warp split-K kernel of the 16-element format (a warp
// owns 16 weight rows, 16-row x 128-k code slices stream through a 4-stage
// cp.async ring, warp-level m16n8k16 MMAs with fp32 accumulation), with two
// ways of applying the block scale:
//   * byte scales (E3M3 / E4M3): each decoded weight is q * s * 2^-bias in
//     fp16 -- exact for every allowed special value (q has at most 5
//     significant bits, s at most 4) -- so the MMA sees exact operands and the
//     scale is applied before it, as in the 16-element kernel.  For bf16
//     activations the operand must be bf16 (8 significant bits), which holds
//     for every allowed value except +-9.5 (19 * 15 = 285 needs 9 bits); sets
//     with it are refused for bf16 activations;
//   * FP16 scale words (11 significant bits): q * s is not an fp16 value, so
//     the MMA multiplies the exact q and the scale multiplies each block's
//     fp32 partial sum afterwards.  A 128-k slice is one block, so every MMA
//     of a slice lies inside one block; blocks shorter than 128 are refused.
// The scale bytes / words of the next slice are fetched into registers one
// slice ahead (they are a few bytes per row; their pointer may have any
// alignment the format allows).
#include "variant.cuh"

namespace razer {

enum { kVarE3M3 = 0, kVarE4M3 = 1, kVarF16 = 2 };

// fp16 bit patterns of the special values, two per word (v0 | v1 << 16,
// v2 | v3 << 16); unused entries are 0.
struct VarTable {
    unsigned lo, hi;
};

static inline VarTable var_table(const VariantV &V)
{
    uint16_t h[4] = {0, 0, 0, 0};
    for (int i = 0; i < V.nv && i < 4; i++) {
        // multiples of 0.5 up to 9.5: exact in fp16 (sign, exponent, 4 fraction bits)
        const __half hv = __float2half_rn(V.v[i]);
        h[i] = *reinterpret_cast<const uint16_t *>(&hv);
    }
    return VarTable{(unsigned)h[0] | ((unsigned)h[1] << 16), (unsigned)h[2] | ((unsigned)h[3] << 16)};
}

// 16-bit lane selector of a prmt over {lo, hi} picking entry m (bytes 2m, 2m+1)
__device__ __forceinline__ unsigned var_sel(unsigned m) { return m * 0x22u + 0x10u; }

// fp16 pairs of s * 2^-bias and of v * s * 2^-bias for the two 16-element
// sub-blocks whose scale bytes sit in the low 16 bits of sb.
template <int SF>
__device__ __forceinline__ void var_scale_pairs(unsigned sb, VarTable T, unsigned (&s2)[2], unsigned (&v2)[2])
{
    constexpr unsigned kMag = SF == kVarE3M3 ? 0x3Fu : 0x7Fu;
    const unsigned x = prmt(sb, 0u, 0x4140u);   // 16-bit lanes: byte 0, byte 1
    const unsigned sx = (x & (kMag * 0x10001u)) << 7;  // fp16 [s0, s1] * 2^-12 (E3M3) / 2^-8 (E4M3)
    s2[0] = prmt(sx, 0u, 0x1010u);
    s2[1] = prmt(sx, 0u, 0x3232u);
    const unsigned m0 = SF == kVarE3M3 ? (sb >> 6) & 3u : (sb >> 7) & 1u;
    const unsigned m1 = SF == kVarE3M3 ? (sb >> 14) & 3u : (sb >> 15) & 1u;
    const unsigned vs = hmul2u(prmt(T.lo, T.hi, var_sel(m0) | (var_sel(m1) << 8)), sx);  // [v0 * s0, v1 * s1]
    v2[0] = prmt(vs, 0u, 0x1010u);
    v2[1] = prmt(vs, 0u, 0x3232u);
}

// One 16-row x 128-k slice, byte scales: the block scale is folded into the
// decoded operands (exact), as in the 16-element kernel.
template <int SF, bool BF16, int NB>
__device__ __forceinline__ void var_slice_prescaled(const uint4 &ca, const uint4 &cb, unsigned sA, unsigned sB, VarTable T,
                                                    const unsigned (&xw)[NB][16], float (&acc)[NB][4])
{
    unsigned s2A[2], vA[2], s2B[2], vB[2];
    var_scale_pairs<SF>(sA, T, s2A, vA);
    var_scale_pairs<SF>(sB, T, s2B, vB);
    const unsigned wa[4] = {ca.x, ca.y, ca.z, ca.w};
    const unsigned wb[4] = {cb.x, cb.y, cb.z, cb.w};
#pragma unroll
    for (int m = 0; m < 4; m++) {
        unsigned hA[4], hB[4];
        decode_word<RAZER_FMT_WEIGHT, BF16>(wa[m], s2A[m >> 1], vA[m >> 1], hA);
        decode_word<RAZER_FMT_WEIGHT, BF16>(wb[m], s2B[m >> 1], vB[m >> 1], hB);
#pragma unroll
        for (int j = 0; j < NB; j++) {
            mma16816<BF16>(acc[j], hA[0], hB[0], hA[1], hB[1], xw[j][4 * m], xw[j][4 * m + 1]);
            mma16816<BF16>(acc[j], hA[2], hB[2], hA[3], hB[3], xw[j][4 * m + 2], xw[j][4 * m + 3]);
        }
    }
}

// Decode 8 codes into 4 pairs of q (no scale): the E2M1 convert, and v at
// the 0b1000 codes through the indicator convert and one packed FMA.
template <bool BF16>
__device__ __forceinline__ void decode_q(unsigned w, unsigned v2, unsigned (&h)[4])
{
    const unsigned t = (w & 0x77777777u) + 0x77777777u;  // bit 3 set where the magnitude is non-zero
    const unsigned is8 = w & ~t & 0x88888888u;            // bit 3 set where the code is 0b1000
    const unsigned ind = __umulhi(is8, 0x40000000u);     // nibble 0b0010 (= 1.0) there
    const unsigned q[4] = {cvt_lane<0>(w), cvt_lane<1>(w), cvt_lane<2>(w), cvt_lane<3>(w)};
    const unsigned i[4] = {cvt_lane<0>(ind), cvt_lane<1>(ind), cvt_lane<2>(ind), cvt_lane<3>(ind)};
#pragma unroll
    for (int b = 0; b < 4; b++) {
        const unsigned r = hfma2u(i[b], v2, q[b]);  // q values are exact in fp16 and bf16
        h[b] = BF16 ? f16x2_to_bf16x2(r) : r;
    }
}

// One 16-row x 128-k slice = one block per row, FP16 scale words: the MMAs
// sum q * x exactly-multiplied in fp32, then each row's block sum is scaled.
template <bool BF16, int NB>
__device__ __forceinline__ void var_slice_postscaled(const uint4 &ca, const uint4 &cb, unsigned swA, unsigned swB, VarTable T,
                                                     const unsigned (&xw)[NB][16], float (&acc)[NB][4])
{
    const unsigned vA = prmt(T.lo, T.hi, var_sel(swA >> 14) * 0x101u);  // [v, v] of row g's meta
    const unsigned vB = prmt(T.lo, T.hi, var_sel(swB >> 14) * 0x101u);
    const float sA = __half2float(__ushort_as_half((unsigned short)(swA & 0x3FFFu)));
    const float sB = __half2float(__ushort_as_half((unsigned short)(swB & 0x3FFFu)));
    float part[NB][4];
#pragma unroll
    for (int j = 0; j < NB; j++) part[j][0] = part[j][1] = part[j][2] = part[j][3] = 0.0f;
    const unsigned wa[4] = {ca.x, ca.y, ca.z, ca.w};
    const unsigned wb[4] = {cb.x, cb.y, cb.z, cb.w};
#pragma unroll
    for (int m = 0; m < 4; m++) {
        unsigned hA[4], hB[4];
        decode_q<BF16>(wa[m], vA, hA);
        decode_q<BF16>(wb[m], vB, hB);
#pragma unroll
        for (int j = 0; j < NB; j++) {
            mma16816<BF16>(part[j], hA[0], hB[0], hA[1], hB[1], xw[j][4 * m], xw[j][4 * m + 1]);
            mma16816<BF16>(part[j], hA[2], hB[2], hA[3], hB[3], xw[j][4 * m + 2], xw[j][4 * m + 3]);
        }
    }
#pragma unroll
    for (int j = 0; j < NB; j++) {  // d[0..1]: row g, d[2..3]: row g + 8
        acc[j][0] = fmaf(sA, part[j][0], acc[j][0]);
        acc[j][1] = fmaf(sA, part[j][1], acc[j][1]);
        acc[j][2] = fmaf(sB, part[j][2], acc[j][2]);
        acc[j][3] = fmaf(sB, part[j][3], acc[j][3]);
    }
}

__host__ __device__ constexpr int var_stage_bytes(int xrows) { return kCodeBytes + xrows * kXRowBytes; }

// bs_shift = log2(block / 16).  Byte scales: [N, K / block] bytes; FP16 scale
// words: [N, K / 128] 16-bit words.  Launch bounds: the B <= 8 kernel fits 64
// registers without spilling (8 CTAs per SM); the B <= 16 and B <= 32 kernels
// keep their natural register counts (about 90 and 150).
template <int SF, bool BF16, int NB>
__global__ void __launch_bounds__(kGemvThreads, NB == 1 ? 8 : (NB == 2 ? 5 : 3)) gemv_variant_kernel(const uint16_t *__restrict__ x, int B, const uint8_t *__restrict__ codes,
                                                                    const uint8_t *__restrict__ scales, int N, int K, int S, int bs_shift,
                                                                    VarTable T, float *__restrict__ ws)
{
    extern __shared__ __align__(16) uint8_t gemv_var_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int row0 = (blockIdx.x * kGemvWarps + warp) * 16;
    if (row0 >= N) return;
    const int s = blockIdx.y;
    const int chunks = K >> 7;
    const int c_begin = (int)((int64_t)s * chunks / S), c_end = (int)((int64_t)(s + 1) * chunks / S);
    const int rA = min(row0 + g, N - 1), rB = min(row0 + g + 8, N - 1);
    const uint8_t *pa = codes + (size_t)rA * (K >> 1) + 16 * t;
    const uint8_t *pb = codes + (size_t)rB * (K >> 1) + 16 * t;
    const int64_t per_row = SF == kVarF16 ? (K >> 7) : (K >> (4 + bs_shift));  // scale entries per row
    const uint8_t *sa_row = scales + (size_t)rA * per_row * (SF == kVarF16 ? 2 : 1);
    const uint8_t *sb_row = scales + (size_t)rB * per_row * (SF == kVarF16 ? 2 : 1);

    const int xrows = NB == 1 ? B : 0;
    const int stage_bytes = var_stage_bytes(xrows);
    uint8_t *ring = gemv_var_smem + warp * (kRing * stage_bytes);
    const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
    auto issue = [&](int c, int slot) {
        if (c < c_end) {
            const uint32_t st = ring_s + slot * stage_bytes;
            cp_async16(st + g * 64 + 16 * t, pa + (size_t)c * 64);
            cp_async16(st + (g + 8) * 64 + 16 * t, pb + (size_t)c * 64);
            if (NB == 1 && g < B) {  // this lane's 64 activation bytes
                const uint8_t *src = reinterpret_cast<const uint8_t *>(x + (size_t)g * K + (size_t)c * 128 + 32 * t);
                const uint32_t dst = st + kCodeBytes + g * kXRowBytes + 64 * t;
#pragma unroll
                for (int q = 0; q < 4; q++) cp_async16(dst + 16 * q, src + 16 * q);
            }
        }
        cp_async_commit();
    };
    // this lane's scale entries of slice c: byte scales -> the bytes of its
    // two 16-element sub-blocks (low 16 bits), FP16 -> the slice's word
    auto load_scales = [&](int c, unsigned &sA, unsigned &sB) {
        if (SF == kVarF16) {
            sA = __ldg(reinterpret_cast<const unsigned short *>(sa_row) + c);
            sB = __ldg(reinterpret_cast<const unsigned short *>(sb_row) + c);
        } else {
            const int u0 = c * 8 + 2 * t;
            const int b0 = u0 >> bs_shift, b1 = (u0 + 1) >> bs_shift;
            sA = (unsigned)__ldg(sa_row + b0) | ((unsigned)__ldg(sa_row + b1) << 8);
            sB = (unsigned)__ldg(sb_row + b0) | ((unsigned)__ldg(sb_row + b1) << 8);
        }
    };

    float acc[NB][4];
#pragma unroll
    for (int j = 0; j < NB; j++) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
    unsigned xw[NB][16];
#pragma unroll
    for (int j = 0; j < NB; j++)
#pragma unroll
        for (int q = 0; q < 16; q++) xw[j][q] = 0u;

    unsigned scA = 0u, scB = 0u;
    if (c_begin < c_end) load_scales(c_begin, scA, scB);
#pragma unroll
    for (int i = 0; i < kRing - 1; i++) issue(c_begin + i, i);
    for (int c = c_begin; c < c_end; c++) {
        const int i = c - c_begin;
        unsigned nA = 0u, nB = 0u;
        if (c + 1 < c_end) load_scales(c + 1, nA, nB);  // one slice ahead
        __syncwarp();  // every lane is done with the slot refilled next
        issue(c + kRing - 1, (i + kRing - 1) % kRing);
        cp_async_wait<kRing - 1>();
        __syncwarp();
        const uint8_t *st = ring + (i % kRing) * stage_bytes;
        const uint4 ca = *reinterpret_cast<const uint4 *>(st + g * 64 + 16 * t);
        const uint4 cb = *reinterpret_cast<const uint4 *>(st + (g + 8) * 64 + 16 * t);
#pragma unroll
        for (int j = 0; j < NB; j++) {
            if (8 * j + g < B) {
                const uint4 *px = NB == 1 ? reinterpret_cast<const uint4 *>(st + kCodeBytes + g * kXRowBytes + 64 * t)
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
        if constexpr (SF == kVarF16) var_slice_postscaled<BF16, NB>(ca, cb, scA, scB, T, xw, acc);
        else var_slice_prescaled<SF, BF16, NB>(ca, cb, scA, scB, T, xw, acc);
        scA = nA;
        scB = nB;
    }
    cp_async_wait<0>();

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

// Split count for a launch: every CTA of the grid resident at once (the
// 4-warp CTAs have equal work, so a second partial wave would leave SMs
// half idle), at most S_max (the count the workspace is sized for).
template <typename Kern>
static int one_wave_splits(Kern kern, int smem, int N, int S_max)
{
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kGemvThreads, (size_t)smem) != cudaSuccess || occ < 1) occ = 1;
    const int64_t ctas_x = ((N + 15) / 16 + kGemvWarps - 1) / kGemvWarps;
    const int64_t s = (int64_t)sm_count() * occ / ctas_x;
    return (int)std::max<int64_t>(1, std::min<int64_t>(s, S_max));
}

// Launches the GEMV kernel; returns the split count it used (<= S_max).
template <int SF, bool BF16>
static int launch_gemv_variant(const void *x, int B, const uint8_t *codes, const uint8_t *scales, int N, int K, int S_max, int bs_shift,
                               VarTable T, float *ws, cudaStream_t st)
{
    const unsigned gx = (unsigned)(((N + 15) / 16 + kGemvWarps - 1) / kGemvWarps);
    const uint16_t *xp = reinterpret_cast<const uint16_t *>(x);
    const int smem1 = kGemvWarps * kRing * var_stage_bytes(B), smem0 = kGemvWarps * kRing * var_stage_bytes(0);
    static bool attr_done[64] = {false};  // per device: up to 8 activation rows in the ring (> 48 KB)
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        cudaFuncSetAttribute(gemv_variant_kernel<SF, BF16, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kGemvWarps * kRing * var_stage_bytes(8));
        attr_done[dev] = true;
    }
    int S;
    if (B <= 8) {
        S = one_wave_splits(gemv_variant_kernel<SF, BF16, 1>, smem1, N, S_max);
        gemv_variant_kernel<SF, BF16, 1><<<dim3(gx, S), kGemvThreads, smem1, st>>>(xp, B, codes, scales, N, K, S, bs_shift, T, ws);
    } else if (B <= 16) {
        S = one_wave_splits(gemv_variant_kernel<SF, BF16, 2>, smem0, N, S_max);
        gemv_variant_kernel<SF, BF16, 2><<<dim3(gx, S), kGemvThreads, smem0, st>>>(xp, B, codes, scales, N, K, S, bs_shift, T, ws);
    } else {
        S = one_wave_splits(gemv_variant_kernel<SF, BF16, 4>, smem0, N, S_max);
        gemv_variant_kernel<SF, BF16, 4><<<dim3(gx, S), kGemvThreads, smem0, st>>>(xp, B, codes, scales, N, K, S, bs_shift, T, ws);
    }
    return S;
}

static int var_sf(razer_format sfmt) { return sfmt == RAZER_SCALE_F16 ? kVarF16 : (sfmt == RAZER_FMT_WEIGHT ? kVarE3M3 : kVarE4M3); }
static int bs_shift_of(int bs) { return bs == 16 ? 0 : (bs == 32 ? 1 : (bs == 64 ? 2 : 3)); }

size_t gemv_variant_workspace_bytes(int64_t B, int64_t N, int64_t K)
{
    if (B <= 0 || N <= 0 || K <= 0) return 0;
    return (size_t)gemv_splits(B, N, K) * (size_t)B * (size_t)N * sizeof(float);
}

razer_status run_gemv_variant(const void *x, razer_dtype act_dt, int64_t B, const uint8_t *codes, const uint8_t *scales, const float *ts,
                              int bs, razer_format sfmt, const VariantV &V, int64_t N, int64_t K, void *y, razer_dtype out_dt,
                              void *workspace, cudaStream_t st)
{
    const int S_max = gemv_splits(B, N, K);  // the workspace holds S_max partial sets
    float *ws = reinterpret_cast<float *>(workspace);
    const VarTable T = var_table(V);
    const int sf = var_sf(sfmt), sh = bs_shift_of(bs);
    const bool bf = act_dt == RAZER_BF16;
    int S;
    if (sf == kVarE3M3)
        S = bf ? launch_gemv_variant<kVarE3M3, true>(x, (int)B, codes, scales, (int)N, (int)K, S_max, sh, T, ws, st)
               : launch_gemv_variant<kVarE3M3, false>(x, (int)B, codes, scales, (int)N, (int)K, S_max, sh, T, ws, st);
    else if (sf == kVarE4M3)
        S = bf ? launch_gemv_variant<kVarE4M3, true>(x, (int)B, codes, scales, (int)N, (int)K, S_max, sh, T, ws, st)
               : launch_gemv_variant<kVarE4M3, false>(x, (int)B, codes, scales, (int)N, (int)K, S_max, sh, T, ws, st);
    else
        S = bf ? launch_gemv_variant<kVarF16, true>(x, (int)B, codes, scales, (int)N, (int)K, S_max, sh, T, ws, st)
               : launch_gemv_variant<kVarF16, false>(x, (int)B, codes, scales, (int)N, (int)K, S_max, sh, T, ws, st);
    const float unbias = sf == kVarE3M3 ? 4096.0f : (sf == kVarE4M3 ? 256.0f : 1.0f);
    const int64_t BN = B * N;
    int64_t g = (BN + 255) / 256;
    if (g > (int64_t)sm_count() * 8) g = (int64_t)sm_count() * 8;
    if (g < 1) g = 1;
    if (out_dt == RAZER_F32) gemv_reduce_kernel<float><<<(int)g, 256, 0, st>>>(ws, S, BN, ts, unbias, reinterpret_cast<float *>(y));
    else if (out_dt == RAZER_F16) gemv_reduce_kernel<__half><<<(int)g, 256, 0, st>>>(ws, S, BN, ts, unbias, reinterpret_cast<__half *>(y));
    else gemv_reduce_kernel<__nv_bfloat16><<<(int)g, 256, 0, st>>>(ws, S, BN, ts, unbias, reinterpret_cast<__nv_bfloat16 *>(y));
    return last_launch_status();
}

// ---------------------------------------------------------------------------
// Decoder: one thread per 16-element sub-block; out = round_out((q*s) * ts)
// with q*s exact in binary32 (at most 5 + 11 significant bits).
// ---------------------------------------------------------------------------
template <int SF, typename TOut>
__global__ void __launch_bounds__(256) dequant_variant_kernel(const uint2 *__restrict__ codes, const uint8_t *__restrict__ scales,
                                                              const float *__restrict__ ts_p, int64_t nsub, int64_t sub_per_row, int bs_shift,
                                                              VariantV V, TOut *__restrict__ out)
{
    const float ts = *ts_p;
    const int64_t per_row = sub_per_row >> bs_shift;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nsub; b += stride) {
        const int64_t r = b / sub_per_row, u = b - r * sub_per_row;
        const int64_t bi = r * per_row + (u >> bs_shift);
        float s;
        unsigned meta;
        if constexpr (SF == kVarF16) {
            const unsigned sw = reinterpret_cast<const unsigned short *>(scales)[bi];
            s = __half2float(__ushort_as_half((unsigned short)(sw & 0x3FFFu)));
            meta = sw >> 14;
        } else if constexpr (SF == kVarE3M3) {
            const unsigned sb = scales[bi];
            s = decode_scale<RAZER_FMT_WEIGHT>(sb);
            meta = sb >> 6;
        } else {
            const unsigned sb = scales[bi];
            s = decode_scale<RAZER_FMT_ACT>(sb);
            meta = sb >> 7;
        }
        // entries past n_special are 0 (the quantizer never writes such a meta)
        const float v = meta == 0 ? V.v[0] : (meta == 1 ? V.v[1] : (meta == 2 ? V.v[2] : V.v[3]));
        const uint2 c = codes[b];
        float val[16];
#pragma unroll
        for (int j = 0; j < 16; j++) {
            const unsigned code = ((j < 8 ? c.x : c.y) >> (4 * (j & 7))) & 15u;
            float q;
            if (code == 8u) q = V.nv > 0 ? v : 0.0f;
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

template <int SF>
static void launch_dequant_variant(const uint8_t *codes, const uint8_t *scales, const float *ts, int64_t nsub, int64_t sub_per_row,
                                   int sh, const VariantV &V, void *out, razer_dtype dt, cudaStream_t st)
{
    int64_t g = (nsub + 255) / 256;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (g > cap) g = cap;
    if (g < 1) g = 1;
    const uint2 *c = reinterpret_cast<const uint2 *>(codes);
    if (dt == RAZER_F32)
        dequant_variant_kernel<SF, float><<<(int)g, 256, 0, st>>>(c, scales, ts, nsub, sub_per_row, sh, V, reinterpret_cast<float *>(out));
    else if (dt == RAZER_F16)
        dequant_variant_kernel<SF, __half><<<(int)g, 256, 0, st>>>(c, scales, ts, nsub, sub_per_row, sh, V, reinterpret_cast<__half *>(out));
    else
        dequant_variant_kernel<SF, __nv_bfloat16>
            <<<(int)g, 256, 0, st>>>(c, scales, ts, nsub, sub_per_row, sh, V, reinterpret_cast<__nv_bfloat16 *>(out));
}

razer_status run_dequant_variant(const uint8_t *codes, const uint8_t *scales, const float *ts, int64_t R, int64_t K, int bs,
                                 razer_format sfmt, const VariantV &V, void *out, razer_dtype dt, cudaStream_t st)
{
    const int64_t nsub = R * K / 16;
    if (nsub == 0) return RAZER_OK;
    const int sf = var_sf(sfmt), sh = bs_shift_of(bs);
    if (sf == kVarE3M3) launch_dequant_variant<kVarE3M3>(codes, scales, ts, nsub, K / 16, sh, V, out, dt, st);
    else if (sf == kVarE4M3) launch_dequant_variant<kVarE4M3>(codes, scales, ts, nsub, K / 16, sh, V, out, dt, st);
    else launch_dequant_variant<kVarF16>(codes, scales, ts, nsub, K / 16, sh, V, out, dt, st);
    return last_launch_status();
}

// ---------------------------------------------------------------------------
// Two-term 16-bit copy of a weight tensor with FP16 scale words, for the
// prefill GEMM: v = q*s*2^11 (exact in binary32: at most 5 + 11 significant
// bits; in [2^-14, 38912] for every nonzero q and scale word, inside fp16's
// normal range), hi = RN16(v), lo = RN16(v - hi) (v - hi is exact in binary32
// and at most half a 16-bit ulp of hi).  Row n of the [N, 2 K] output holds hi
// in columns [0, K) and lo in [K, 2 K), so a GEMM over 2 K columns against
// [X | X] sums x * (hi + lo).  bf16: hi keeps 8 of v's at most 16 significant
// bits and lo the other at most 8, so hi + lo == v exactly.  fp16: exact
// unless lo falls below fp16's normal range (v < 2^-3), and then off by at
// most 2^-25 -- where one fp16 term would be off by up to 2^-11 relative.
// One thread per 16-element sub-block.
// ---------------------------------------------------------------------------
template <bool BF>
__global__ void __launch_bounds__(256) decode_f16w_split_kernel(const uint2 *__restrict__ codes, const uint8_t *__restrict__ scales,
                                                                int64_t nsub, int64_t sub_per_row, int bs_shift, VariantV V,
                                                                uint4 *__restrict__ out)
{
    pdl_wait();
    const int64_t per_row = sub_per_row >> bs_shift;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nsub; b += stride) {
        const int64_t r = b / sub_per_row, u = b - r * sub_per_row;
        const unsigned sw = reinterpret_cast<const unsigned short *>(scales)[r * per_row + (u >> bs_shift)];
        const float s = __half2float(__ushort_as_half((unsigned short)(sw & 0x3FFFu)));
        const unsigned meta = sw >> 14;
        const float v = meta == 0 ? V.v[0] : (meta == 1 ? V.v[1] : (meta == 2 ? V.v[2] : V.v[3]));
        const uint2 c = codes[b];
        unsigned hw[8], lw[8];
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
            float hv[2], lv[2];
#pragma unroll
            for (int e = 0; e < 2; e++) {
                const unsigned code = ((j + e < 8 ? c.x : c.y) >> (4 * ((j + e) & 7))) & 15u;
                float q;
                if (code == 8u) q = V.nv > 0 ? v : 0.0f;
                else q = (code & 8u) ? -fp4_mag(code & 7u) : fp4_mag(code & 7u);
                const float w = __fmul_rn(__fmul_rn(q, s), 2048.0f);
                const float h = BF ? __bfloat162float(__float2bfloat16_rn(w)) : __half2float(__float2half_rn(w));
                hv[e] = w;
                lv[e] = __fsub_rn(w, h);
            }
            if constexpr (BF) {
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(hv[0], hv[1]), l2 = __floats2bfloat162_rn(lv[0], lv[1]);
                hw[j / 2] = *reinterpret_cast<const unsigned *>(&h2);
                lw[j / 2] = *reinterpret_cast<const unsigned *>(&l2);
            } else {
                const __half2 h2 = __floats2half2_rn(hv[0], hv[1]), l2 = __floats2half2_rn(lv[0], lv[1]);
                hw[j / 2] = *reinterpret_cast<const unsigned *>(&h2);
                lw[j / 2] = *reinterpret_cast<const unsigned *>(&l2);
            }
        }
        // sub-block u of row r: 16 halves at column 16 u of the hi and lo halves
        uint4 *oh = out + r * (sub_per_row * 4) + 2 * u;
        uint4 *ol = oh + sub_per_row * 2;
        oh[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        oh[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
        ol[0] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        ol[1] = make_uint4(lw[4], lw[5], lw[6], lw[7]);
    }
}

razer_status run_decode_f16w_split(const uint8_t *codes, const uint8_t *scales, int64_t N, int64_t K, int bs, const VariantV &V, void *out,
                                   bool bf16, cudaStream_t st)
{
    const int64_t nsub = N * K / 16;
    if (nsub == 0) return RAZER_OK;
    int64_t g = (nsub + 255) / 256;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (g > cap) g = cap;
    if (launch_pdl(bf16 ? decode_f16w_split_kernel<true> : decode_f16w_split_kernel<false>, (unsigned)g, 256u, 0, st,
                   reinterpret_cast<const uint2 *>(codes), scales, nsub, K / 16, bs_shift_of(bs), V, reinterpret_cast<uint4 *>(out)) !=
        cudaSuccess)
        return RAZER_ERR_CUDA;
    return RAZER_OK;
}

}  // namespace razer
