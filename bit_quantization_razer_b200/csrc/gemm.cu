// RaZeR W4A16 GEMM on the tcgen05 tensor cores (sm_100a).
//
//   Y[m, n] = ts * sum_k X[m, k] * (q*s)[n, k]
//
// (RaZeR notes 关键设计 3: weight-only kernels that decode the remapped codes
// on the fly; gist.science summary 2.3.)  The contraction is dense, so it runs
// on the 5th-generation tensor cores, by one of two kernels:
//   * gemm_kernel (below): each CTA decodes its weight tile into shared memory
//     every k-step -- for small M, where that decode is not repeated often;
//   * gemm_tma_kernel (further down): the weights are decoded once into a
//     16-bit copy in HBM and a persistent kernel multiplies two TMA-fed
//     operands -- for large M, and for M >= 256 on small weight matrices.
// gemm_kernel:
//   * CTA tile 256 (M) x 256 (N), k-step 64.  Two UMMA instructions of
//     M = 128 share one decoded weight tile, so every weight is decoded once
//     per 256 activation rows (half the decode work per SM of a 128-row tile).
//   * warp 0: TMA producer of the X tiles (K-major, 128-byte swizzle);
//     warp 1: TMEM allocator and the single MMA-issuing thread;
//     warps 2-9: decoders, one weight row per thread, two warps per
//     scheduler -- they stream the packed codes and scale bytes with
//     128-bit loads (two k-steps ahead, in registers), decode to 16-bit q*s
//     and write the
//     UMMA canonical K-major 128B-swizzled layout with 16-byte stores; after
//     the k loop they are the epilogue (tcgen05.ld, * ts, convert, store).
//   * fp32 accumulators: two 128 x 256 tiles = all 512 TMEM columns.
//   * 3-stage mbarrier pipeline; every wait is bounded (~2 s of globaltimer):
//     on expiry the kernel records RAZER_ERR_TIMEOUT in the device status word,
//     the other roles stop at their next wait, in-flight TMA loads are waited
//     for (bounded), and the TMEM is freed before the CTA exits.
// Decode exactness: q (E2M1 with the redundant zero replaced by v) is exact in
// fp16; q*s*2^-8 (E3M3) or q*s*2^-4 (E4M3) is an exact fp16 product in the
// normal range, which converts exactly to bf16 (at most 7 significant bits)
// for bf16 activations.
#include <cuda.h>
#include <algorithm>
#include <cstdlib>

#include "razer_internal.cuh"
#include "sm100_async.cuh"
#include "variant.cuh"

namespace razer {
namespace gemm {

#ifndef RAZER_GEMM_BM
#define RAZER_GEMM_BM 256
#endif
#ifndef RAZER_GEMM_BN
#define RAZER_GEMM_BN 256
#endif
#ifndef RAZER_GEMM_STAGES
#define RAZER_GEMM_STAGES 3
#endif
// CTA tile BM x BN x 64: BM / 128 UMMAs of M = 128 share each decoded BN-row
// weight tile (every weight is decoded once per BM activation rows); the
// accumulators fill (BM / 128) * BN = 512 TMEM columns.
constexpr int BM = RAZER_GEMM_BM, BN = RAZER_GEMM_BN, BK = 64, STAGES = RAZER_GEMM_STAGES;
constexpr int kMBlocks = BM / 128;
static_assert(kMBlocks * BN == 512, "the accumulators fill the 512 TMEM columns");
#ifndef RAZER_GEMM_DECODE_WARPS
#define RAZER_GEMM_DECODE_WARPS 8
#endif
constexpr int kDecodeWarps = RAZER_GEMM_DECODE_WARPS;  // 8: a row per thread; 16: half a row per thread
constexpr int kThreadsPerRow = 32 * kDecodeWarps / BN;   // decoder threads per weight row (1 or 2)
constexpr int kHalvesPerThread = 2 / kThreadsPerRow;     // 32-code halves of a k-step per thread
static_assert(kThreadsPerRow >= 1 && kThreadsPerRow <= 2, "one or two decoder threads per row");
constexpr int kFirstDecodeWarp = 2;  // warp 0: X TMA, 1: MMA
constexpr int kThreads = 32 * kFirstDecodeWarp + 32 * kDecodeWarps;
constexpr uint32_t A_HALF_BYTES = 128 * BK * 2;                      // 16 KB: one 128-row block of X
constexpr uint32_t B_BYTES = BN * BK * 2;                            // decoded weights
constexpr uint32_t STAGE_BYTES = kMBlocks * A_HALF_BYTES + B_BYTES;  // 64 KB (256x256) / 80 KB (512x128)
constexpr uint32_t BAR_BYTES = 256;
constexpr uint32_t SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;  // + alignment slack
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// UMMA shared-memory descriptor of a K-major, 128B-swizzled tile whose
// 8-row groups are 1024 bytes apart (rows of 128 bytes).
__device__ __forceinline__ uint64_t smem_desc_k128(uint32_t addr)
{
    uint64_t d = 0;
    d |= (uint64_t)((addr & 0x3FFFFu) >> 4);  // start address
    d |= (uint64_t)1 << 16;                   // leading byte offset (unused for 128B swizzle)
    d |= (uint64_t)(1024 >> 4) << 32;         // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1 << 46;                   // descriptor version for sm_100
    d |= (uint64_t)2 << 61;                   // 128-byte swizzle
    return d;
}

// kind::f16 instruction descriptor: fp32 accumulate, K-major A and B.
__host__ __device__ constexpr uint32_t idesc_f16(bool bf16, int M, int N)
{
    return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t dtmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(dtmem), "l"(adesc),
        "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,"
        "%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]),
          "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
          "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; i++) v[i] = __uint_as_float(r[i]);
}

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
__device__ __forceinline__ unsigned hmul2(unsigned a, unsigned b)
{
    unsigned r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ unsigned hfma2(unsigned a, unsigned b, unsigned c)
{
    unsigned r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}

// Per-block decode constants of one scale byte (fp16 pairs).
struct BlockK {
    unsigned s2;   // s * 2^-bias
    unsigned vs2;  // v * s * 2^-bias (0 when the format has no remap)
};

template <int FMT>
__device__ __forceinline__ BlockK block_consts(unsigned sb)
{
    BlockK k;
    const unsigned s16 = scale_f16_bits<FMT>(sb);        // s * 2^-12 (E3M3) or s * 2^-8 (E4M3)
    k.s2 = hmul2(s16 | (s16 << 16), 0x4C004C00u);       // * 16 (exact): keeps q*s in the fp16 normal range
    if constexpr (Fmt<FMT>::kSpecials > 0) {
        const unsigned meta = sb >> Fmt<FMT>::kMetaShift;
        const unsigned v16 = ((meta & 2u) ? 0x4800u : 0x4500u) | ((meta & 1u) << 15);
        k.vs2 = hmul2(v16 | (v16 << 16), k.s2);
    } else {
        k.vs2 = 0u;
    }
    return k;
}

// Decode one 32-bit word (8 codes of one block) into 4 packed 16-bit pairs of
// q*s*2^-bias.  The redundant-zero codes (converted to -0) receive v*s through
// the convert of an indicator word (code of 1.0 where the code is 0b1000)
// folded in with a packed FMA.
template <int FMT, bool BF16>
__device__ __forceinline__ uint4 decode_word(unsigned w, const BlockK &k)
{
    unsigned p[4] = {cvt_lane<0>(w), cvt_lane<1>(w), cvt_lane<2>(w), cvt_lane<3>(w)};
    if constexpr (Fmt<FMT>::kSpecials > 0) {
        const unsigned t = (w & 0x77777777u) + 0x77777777u;
        const unsigned ind = __umulhi(w & ~t & 0x88888888u, 0x40000000u);  // nibble 0b0010 where the code is 0b1000
        const unsigned i[4] = {cvt_lane<0>(ind), cvt_lane<1>(ind), cvt_lane<2>(ind), cvt_lane<3>(ind)};
#pragma unroll
        for (int b = 0; b < 4; b++) p[b] = hfma2(i[b], k.vs2, hmul2(p[b], k.s2));
    } else {
#pragma unroll
        for (int b = 0; b < 4; b++) p[b] = hmul2(p[b], k.s2);
    }
    if constexpr (BF16) {
#pragma unroll
        for (int b = 0; b < 4; b++) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&p[b]));
            __nv_bfloat162 h2 = __floats2bfloat162_rn(f.x, f.y);  // exact
            p[b] = *reinterpret_cast<unsigned *>(&h2);
        }
    }
    return make_uint4(p[0], p[1], p[2], p[3]);
}

// The fused kernel: the decoder warps write each k-step's weight tile into
// shared memory (the decode-once path runs gemm_tma_kernel instead).
template <int FMT, bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint8_t *__restrict__ codes,
                const uint8_t *__restrict__ scales, const float *__restrict__ ts_p, float unbias, int M, int N, int K,
                void *Y, int out_dt, int kb0, int nkb, const float *addend, int inject_stall)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *bars = smem + STAGES * STAGE_BYTES;
    const uint32_t full_a = smem_addr(bars);              // STAGES x 8
    const uint32_t full_b = full_a + 8 * STAGES;          // STAGES x 8
    const uint32_t empty = full_b + 8 * STAGES;           // STAGES x 8
    const uint32_t acc_full = empty + 8 * STAGES;         // 8
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(bars + 192);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 200);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BN, m0 = blockIdx.y * BM;
    // this launch covers k-steps [kb0, kb0 + nkb) of the K / 64; a previous
    // chunk's fp32 result (already scaled) is added in the epilogue.  With
    // gridDim.z > 1 the range is split further: split z takes its own part and
    // writes its scaled fp32 sum to slice z of Y ([gridDim.z, M, N] fp32).
    const int kbs = kb0 + (int)((int64_t)blockIdx.z * nkb / gridDim.z);
    const int KB = kb0 + (int)((int64_t)(blockIdx.z + 1) * nkb / gridDim.z) - kbs;
    if (gridDim.z > 1) Y = reinterpret_cast<float *>(Y) + (size_t)blockIdx.z * (size_t)M * (size_t)N;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; s++) {
            mbar_init(full_a + 8 * s, 1);
            mbar_init(full_b + 8 * s, kDecodeWarps);  // one arrival per decoder warp
            mbar_init(empty + 8 * s, 1);
        }
        mbar_init(acc_full, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_addr((const void *)tmem_slot)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer (X tiles) ----------------
        if (lane == 0) {
            int issued = 0;
            for (int kb = 0; kb < KB; kb++) {
                const int s = kb % STAGES;
                const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
                if (!mbar_wait(empty + 8 * s, ph ^ 1u, abort_flag)) break;
                const uint32_t a0 = smem_addr(smem + s * STAGE_BYTES);
                mbar_expect_tx(full_a + 8 * s, kMBlocks * A_HALF_BYTES);
#pragma unroll
                for (int a = 0; a < kMBlocks; a++) tma_load_2d(a0 + a * A_HALF_BYTES, &tmap_x, (kbs + kb) * BK, m0 + 128 * a, full_a + 8 * s);
                issued = kb + 1;
            }
            if (*abort_flag) {
                // let the loads already issued land before the CTA exits (bounded)
                const uint64_t t0 = globaltimer();
                for (int kb = (issued > STAGES ? issued - STAGES : 0); kb < issued; kb++) {
                    const int s = kb % STAGES;
                    const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
                    while (!mbar_try_wait(full_a + 8 * s, ph) && globaltimer() - t0 < kTimeoutNs) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idesc = idesc_f16(BF16, 128, BN);
            bool ok = true;
            for (int kb = 0; kb < KB && ok; kb++) {
                const int s = kb % STAGES;
                const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
                ok = mbar_wait(full_a + 8 * s, ph, abort_flag) && mbar_wait(full_b + 8 * s, ph, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a0 = smem_addr(smem + s * STAGE_BYTES);
                const uint32_t b0 = a0 + kMBlocks * A_HALF_BYTES;
#pragma unroll
                for (int k = 0; k < BK / 16; k++) {
                    const uint64_t bd = smem_desc_k128(b0 + 32 * k);
                    const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
#pragma unroll
                    for (int a = 0; a < kMBlocks; a++)
                        umma_f16(tmem + a * BN, smem_desc_k128(a0 + a * A_HALF_BYTES + 32 * k), bd, idesc, acc);
                }
                umma_commit(empty + 8 * s);
            }
            umma_commit(acc_full);
            if (!ok) {
                // stopped early: let the MMAs already issued finish (bounded)
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(acc_full, 0) && globaltimer() - t0 < kTimeoutNs) {
                }
            }
        }
    } else {
        // ---------------- decoders, then epilogue ----------------
        const int dt = threadIdx.x - 32 * kFirstDecodeWarp;  // 0 .. 32*kDecodeWarps-1
        const int row = dt & (BN - 1);                                // weight row of the tile
        const int hk0 = kHalvesPerThread == 1 ? (dt / BN) : 0;        // first 32-element half of the k-step
        const int n = n0 + row;
        const bool valid = n < N;
        const uint8_t *crow = codes + (size_t)(valid ? n : (N - 1)) * (K >> 1) + 16 * hk0;
        const uint8_t *srow = scales + (size_t)(valid ? n : (N - 1)) * (K >> 4) + 2 * hk0;
        // codes and scale bytes of the next two k-steps are in flight in
        // registers, so a global-load latency is covered by two decode steps
        struct Regs {
            uint4 c[kHalvesPerThread];
            unsigned s;
        };
        auto load_stage = [&](int kb, Regs &r) {
#pragma unroll
            for (int h = 0; h < kHalvesPerThread; h++) r.c[h] = ldg_stream(crow + (size_t)(kbs + kb) * 32 + 16 * h);
            r.s = kHalvesPerThread == 1 ? (unsigned)*reinterpret_cast<const unsigned short *>(srow + (size_t)(kbs + kb) * 4)
                                        : *reinterpret_cast<const unsigned *>(srow + (size_t)(kbs + kb) * 4);
        };
        Regs r0, r1;
        bool ok = true;
        load_stage(0, r0);
        if (KB > 1) load_stage(1, r1);
        for (int kb = 0; kb < KB; kb++) {
            const int s = kb % STAGES;
            const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
            uint4 c0[kHalvesPerThread];
#pragma unroll
            for (int h = 0; h < kHalvesPerThread; h++) c0[h] = r0.c[h];
            const unsigned cs = valid ? r0.s : 0u;
            r0 = r1;
            if (kb + 2 < KB) load_stage(kb + 2, r1);
            // the decoded tile goes into B slot s once the MMAs released it
            if (!mbar_wait_warp(empty + 8 * s, ph ^ 1u, abort_flag)) {
                ok = false;
                break;
            }
            uint8_t *rbase = smem + s * STAGE_BYTES + kMBlocks * A_HALF_BYTES + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
            for (int h = 0; h < kHalvesPerThread; h++) {
                const unsigned words[4] = {c0[h].x, c0[h].y, c0[h].z, c0[h].w};
#pragma unroll
                for (int blk = 0; blk < 2; blk++) {
                    const BlockK kc = block_consts<FMT>((cs >> (8 * (2 * h + blk))) & 0xFFu);
#pragma unroll
                    for (int e = 0; e < 2; e++) {
                        const int j = 4 * (hk0 + h) + 2 * blk + e;  // 16-byte chunk = 8 elements
                        const uint4 v = decode_word<FMT, BF16>(words[2 * blk + e], kc);
                        *reinterpret_cast<uint4 *>(rbase + ((j ^ (row & 7)) << 4)) = v;
                    }
                }
            }
            fence_proxy_async();
            __syncwarp();
            // fault injection (tests only): a decoder warp that never arrives
            // makes the MMA thread's bounded wait run out
            if (lane == 0 && !(inject_stall && warp == kFirstDecodeWarp)) mbar_arrive(full_b + 8 * s);
        }

        // epilogue: TMEM lanes 32*(warp%4) .. +31; the warps of a lane quarter
        // split the 256 columns of each accumulator
        if (ok && mbar_wait_warp(acc_full, 0, abort_flag) && !*abort_flag) {
            tc_fence_after();
            const int q = warp & 3;
            const int cbeg = ((warp - kFirstDecodeWarp) >> 2) * (BN * 4 / kDecodeWarps);
            const float scale = __fmul_rn(*ts_p, unbias);
#pragma unroll 1
            for (int half = 0; half < kMBlocks; half++) {
                const int m = m0 + half * 128 + q * 32 + lane;
#pragma unroll 1
                for (int c0 = cbeg; c0 < cbeg + BN * 4 / kDecodeWarps; c0 += 32) {
                    float v[32];
                    tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(half * BN + c0), v);
                    const int n = n0 + c0;
                    if (m < M && n < N) {
                        const int cnt = min(32, N - n);
                        // 16-byte vector accesses need rows of N % 4 (fp32) / N % 8 (16-bit) elements
                        const bool vec = out_dt == RAZER_F32 ? (N & 3) == 0 : (N & 7) == 0;
                        const float *add = addend ? addend + (size_t)m * N + n : nullptr;
                        if (add && cnt == 32 && (N & 3) == 0) {
#pragma unroll
                            for (int i = 0; i < 8; i++) {
                                const float4 t = reinterpret_cast<const float4 *>(add)[i];
                                v[4 * i] = __fmaf_rn(v[4 * i], scale, t.x);
                                v[4 * i + 1] = __fmaf_rn(v[4 * i + 1], scale, t.y);
                                v[4 * i + 2] = __fmaf_rn(v[4 * i + 2], scale, t.z);
                                v[4 * i + 3] = __fmaf_rn(v[4 * i + 3], scale, t.w);
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; i++) v[i] = (add && i < cnt) ? __fmaf_rn(v[i], scale, add[i]) : v[i] * scale;
                        }
                        if (cnt < 32 || !vec) {
                            for (int i = 0; i < cnt; i++) {
                                const float a = v[i];
                                if (out_dt == RAZER_F32) reinterpret_cast<float *>(Y)[(size_t)m * N + n + i] = a;
                                else if (out_dt == RAZER_BF16) reinterpret_cast<__nv_bfloat16 *>(Y)[(size_t)m * N + n + i] = __float2bfloat16_rn(a);
                                else reinterpret_cast<__half *>(Y)[(size_t)m * N + n + i] = __float2half_rn(a);
                            }
                        } else if (out_dt == RAZER_F32) {
                            float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(Y) + (size_t)m * N + n);
#pragma unroll
                            for (int i = 0; i < 8; i++) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                        } else {
                            uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(Y) + (size_t)m * N + n);
#pragma unroll
                            for (int i = 0; i < 4; i++) {
                                unsigned p[4];
#pragma unroll
                                for (int e = 0; e < 4; e++) {
                                    const float a = v[8 * i + 2 * e], b = v[8 * i + 2 * e + 1];
                                    if (out_dt == RAZER_BF16) {
                                        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
                                        p[e] = *reinterpret_cast<unsigned *>(&h);
                                    } else {
                                        __half2 h = __floats2half2_rn(a, b);
                                        p[e] = *reinterpret_cast<unsigned *>(&h);
                                    }
                                }
                                dst[i] = make_uint4(p[0], p[1], p[2], p[3]);
                            }
                        }
                    }
                }
            }
        }
        tc_fence_before();
    }

    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
    }
}

// ---------------------------------------------------------------------------
// Persistent GEMM on two bulk-tensor-loaded 16-bit operands (the decode-once
// path, and the W4A4 product): Y[m, n] = ts * unbias * sum_k X[m, k] Wd[n, k].
// One CTA per SM walks the work units u = blockIdx.x, + gridDim.x, ... of the
// (256 x 256 output tile, K split) grid, m-tile fastest so that consecutive
// units share their weight tile in L2:
//   * warp 0, lane 0: the bulk-tensor producer.  It runs ahead across units:
//     while the epilogue drains one unit's accumulator it fills the stages
//     of the next;
//   * warp 1, lane 0: the MMA issuer (two M = 128 UMMAs per k-substep share
//     the B tile); it returns each stage to the producer and hands each
//     finished accumulator to the epilogue;
//   * warps 2-9: the epilogue.  Each warp drains its TMEM lane quarter in
//     32-column chunks, scales them, stages each chunk in shared memory
//     (16-byte units XOR-swizzled by row, conflict-free both ways) and reads it
//     back row-contiguous, so every warp store writes whole row segments of
//     four rows (128 bytes per row in fp32, 64 in 16-bit) instead of sixteen
//     bytes in each of 32 rows.  The accumulator goes back to the MMA issuer
//     as soon as every warp has read its last chunk.
// Every wait is bounded as in gemm_kernel; a timeout stops all roles.
// ---------------------------------------------------------------------------
constexpr int kEpiWarps = 8;
constexpr int kTmaThreads = 32 * (2 + kEpiWarps);
// the tile is 256 x TBN with TBN = 256 or 224: the host takes the width whose
// rounds of tiles over the SMs cost least (4096 x 14336: 896 tiles of 256 are
// 7 rounds, the last with 8 tiles; 1024 tiles of 224 are 7 full rounds)
__host__ __device__ constexpr uint32_t tma_stage_bytes(int tbn) { return 2 * A_HALF_BYTES + (uint32_t)tbn * BK * 2; }  // X 256 x 64 + W tbn x 64
constexpr uint32_t kEpiStageBytes = 32 * 128;                                  // one warp's 32 x 32 fp32 chunk
__host__ __device__ constexpr uint32_t tma_smem_bytes(int tbn) { return STAGES * tma_stage_bytes(tbn) + kEpiWarps * kEpiStageBytes + BAR_BYTES + 1024; }
static_assert(tma_smem_bytes(256) <= 232448, "shared memory of the persistent GEMM");

struct TmaUnit {
    int m0, n0, kbs, nk, z;
};
__device__ __forceinline__ TmaUnit tma_unit(int u, int mt, int T, int S, int kb0, int nkb, int tbn)
{
    TmaUnit w;
    w.z = u / T;
    const int t = u - w.z * T;
    w.m0 = (t % mt) * 256;
    w.n0 = (t / mt) * tbn;
    w.kbs = kb0 + (int)((int64_t)w.z * nkb / S);
    w.nk = kb0 + (int)((int64_t)(w.z + 1) * nkb / S) - w.kbs;
    return w;
}

template <typename TOut>
__device__ __forceinline__ void store4(TOut *p, float4 a);
template <> __device__ __forceinline__ void store4<float>(float *p, float4 a) { *reinterpret_cast<float4 *>(p) = a; }
template <> __device__ __forceinline__ void store4<__half>(__half *p, float4 a)
{
    __half2 lo = __floats2half2_rn(a.x, a.y), hi = __floats2half2_rn(a.z, a.w);
    *reinterpret_cast<uint2 *>(p) = make_uint2(*reinterpret_cast<unsigned *>(&lo), *reinterpret_cast<unsigned *>(&hi));
}
template <> __device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16 *p, float4 a)
{
    __nv_bfloat162 lo = __floats2bfloat162_rn(a.x, a.y), hi = __floats2bfloat162_rn(a.z, a.w);
    *reinterpret_cast<uint2 *>(p) = make_uint2(*reinterpret_cast<unsigned *>(&lo), *reinterpret_cast<unsigned *>(&hi));
}
template <typename TOut> __device__ __forceinline__ void store1(TOut *p, float a);
template <> __device__ __forceinline__ void store1<float>(float *p, float a) { *p = a; }
template <> __device__ __forceinline__ void store1<__half>(__half *p, float a) { *p = __float2half_rn(a); }
template <> __device__ __forceinline__ void store1<__nv_bfloat16>(__nv_bfloat16 *p, float a) { *p = __float2bfloat16_rn(a); }

// One epilogue warp's row-contiguous write of a staged 32 x 32 chunk whose
// top-left output element is (m, n): lane l writes 4 elements of row
// 4 p + l / 8, for p = 0..7.
template <typename TOut>
__device__ __forceinline__ void epi_write(const uint8_t *stage, int lane, int m, int n, int M, int N, TOut *Y, const float *addend)
{
    const int u = lane & 7;
    const bool vec = (N & 3) == 0;  // rows of whole 4-element groups: 16-byte (fp32) / 8-byte (16-bit) aligned
#pragma unroll
    for (int p = 0; p < 8; p++) {
        const int r = 4 * p + (lane >> 3);
        float4 a = *reinterpret_cast<const float4 *>(stage + r * 128 + ((u ^ (r & 7)) << 4));
        const int mm = m + r, nn = n + 4 * u;
        if (mm >= M || nn >= N) continue;
        const size_t off = (size_t)mm * (size_t)N + (size_t)nn;
        if (vec && nn + 4 <= N) {
            if (addend) {
                const float4 t = *reinterpret_cast<const float4 *>(addend + off);
                a.x += t.x;
                a.y += t.y;
                a.z += t.z;
                a.w += t.w;
            }
            store4<TOut>(Y + off, a);
        } else {
            const float e[4] = {a.x, a.y, a.z, a.w};
            for (int i = 0; i < 4 && nn + i < N; i++) store1<TOut>(Y + off + i, addend ? e[i] + addend[off + i] : e[i]);
        }
    }
}

template <bool BF16, typename TOut, int TBN>
__global__ void __launch_bounds__(kTmaThreads, 1)
    gemm_tma_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w, const float *__restrict__ ts_p,
                    float unbias, int M, int N, int mt, int T, int S, int kb0, int nkb, TOut *Y, const float *addend, int inject_stall,
                    int kx_wrap)
{
    constexpr uint32_t kTmaStageBytes = tma_stage_bytes(TBN);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *epi = smem + STAGES * kTmaStageBytes;
    uint8_t *bars = epi + kEpiWarps * kEpiStageBytes;
    const uint32_t full = smem_addr(bars);       // STAGES x 8
    const uint32_t empty = full + 8 * STAGES;     // STAGES x 8
    const uint32_t acc_full = empty + 8 * STAGES;  // 8
    const uint32_t acc_empty = acc_full + 8;       // 8
    const uint32_t drained = acc_empty + 8;        // 8: the MMA issuer's own wait after a timeout
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(bars + 192);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 200);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int U = T * S, G = gridDim.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; s++) {
            mbar_init(full + 8 * s, 1);
            mbar_init(empty + 8 * s, 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kEpiWarps);
        mbar_init(drained, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_addr((const void *)tmem_slot)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();  // the decoded operands come from earlier kernels in the stream

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- bulk-tensor producer ----------------
            uint32_t g = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < U && ok; u += G) {
                const TmaUnit w = tma_unit(u, mt, T, S, kb0, nkb, TBN);
                for (int kb = 0; kb < w.nk; kb++, g++) {
                    const uint32_t s = g % STAGES, ph = (g / STAGES) & 1u;
                    if (!mbar_wait(empty + 8 * s, ph ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    // fault injection (tests only): CTA 0 never fills its first stage
                    if (inject_stall && blockIdx.x == 0 && g == 0) continue;
                    const uint32_t a0 = smem_addr(smem + s * kTmaStageBytes);
                    // kx_wrap > 0: the weight operand has kx_wrap k-steps per X pass
                    // ([W_hi | W_lo] against [X | X])
                    const int kx = kx_wrap > 0 ? (w.kbs + kb) % kx_wrap : w.kbs + kb;
                    mbar_expect_tx(full + 8 * s, kTmaStageBytes);
                    tma_load_2d(a0, &tmap_x, kx * BK, w.m0, full + 8 * s);
                    tma_load_2d(a0 + A_HALF_BYTES, &tmap_x, kx * BK, w.m0 + 128, full + 8 * s);
                    tma_load_2d(a0 + 2 * A_HALF_BYTES, &tmap_w, (w.kbs + kb) * BK, w.n0, full + 8 * s);
                }
            }
            if (!ok) {
                // let the loads already issued land before the CTA exits (bounded)
                const uint64_t t0 = globaltimer();
                for (uint32_t gg = g > (uint32_t)STAGES ? g - STAGES : 0u; gg < g; gg++) {
                    if (inject_stall && blockIdx.x == 0 && gg == 0) continue;
                    while (!mbar_try_wait(full + 8 * (gg % STAGES), (gg / STAGES) & 1u) && globaltimer() - t0 < kTimeoutNs) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            const uint32_t idesc = idesc_f16(BF16, 128, TBN);
            uint32_t g = 0, ti = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < U && ok; u += G, ti++) {
                const TmaUnit w = tma_unit(u, mt, T, S, kb0, nkb, TBN);
                // the epilogue has drained the previous unit's accumulator
                if (!mbar_wait(acc_empty, (ti & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kb = 0; kb < w.nk; kb++, g++) {
                    const uint32_t s = g % STAGES, ph = (g / STAGES) & 1u;
                    if (!mbar_wait(full + 8 * s, ph, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_addr(smem + s * kTmaStageBytes);
                    const uint32_t b0 = a0 + 2 * A_HALF_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / 16; k++) {
                        const uint64_t bd = smem_desc_k128(b0 + 32 * k);
                        const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
                        umma_f16(tmem, smem_desc_k128(a0 + 32 * k), bd, idesc, acc);
                        umma_f16(tmem + TBN, smem_desc_k128(a0 + A_HALF_BYTES + 32 * k), bd, idesc, acc);
                    }
                    umma_commit(empty + 8 * s);
                }
                if (ok) umma_commit(acc_full);
            }
            // every MMA issued has completed before the TMEM is freed (bounded)
            umma_commit(drained);
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(drained, 0) && globaltimer() - t0 < kTimeoutNs) {
            }
        }
    } else {
        // ---------------- epilogue ----------------
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        // the two warps of a quarter split each half's columns: [0, 128) and [128, TBN)
        const int wb = (warp - 2) >> 2, cbeg = wb * 128, nch = (wb ? TBN - 128 : 128) / 32;
        uint8_t *stage = epi + (warp - 2) * kEpiStageBytes;
        const float scale = __fmul_rn(*ts_p, unbias);
        TOut *Yz = Y;
        uint32_t ti = 0;
        for (int u = blockIdx.x; u < U; u += G, ti++) {
            const TmaUnit w = tma_unit(u, mt, T, S, kb0, nkb, TBN);
            if (!mbar_wait_warp(acc_full, ti & 1u, abort_flag)) break;
            tc_fence_after();
            Yz = Y + (S > 1 ? (size_t)w.z * (size_t)M * (size_t)N : 0);
#pragma unroll 1
            for (int c = 0; c < 2 * nch; c++) {
                const int half = c / nch, col = cbeg + 32 * (c % nch);
                float v[32];
                tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(half * TBN + col), v);
                if (c == 2 * nch - 1) {
                    // this warp has read the whole accumulator: hand it back
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(acc_empty);
                }
                // an empty K range leaves the accumulator unwritten: its sum is 0
                if (w.nk == 0) {
#pragma unroll
                    for (int i = 0; i < 32; i++) v[i] = 0.0f;
                }
                // stage row `lane` (16-byte unit j at j ^ (lane & 7))
#pragma unroll
                for (int j = 0; j < 8; j++)
                    *reinterpret_cast<float4 *>(stage + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                        make_float4(v[4 * j] * scale, v[4 * j + 1] * scale, v[4 * j + 2] * scale, v[4 * j + 3] * scale);
                __syncwarp();
                epi_write<TOut>(stage, lane, w.m0 + half * 128 + q * 32, w.n0 + col, M, N, Yz, S > 1 ? nullptr : addend);
                __syncwarp();
            }
        }
        tc_fence_before();
    }

    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
    }
}

// Decodes the packed weights once into a [N, K] 16-bit copy holding
// q*s*2^-bias (the exact values the fused kernel writes to shared memory);
// one thread per 16-element block.
template <int FMT, bool BF16>
__global__ void __launch_bounds__(256) decode_weights_kernel(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scales,
                                                             int64_t nblk, uint4 *__restrict__ out)
{
    pdl_wait();
    pdl_trigger();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk; b += stride) {
        const uint2 c = ldg_stream_u2(reinterpret_cast<const uint2 *>(codes) + b);
        const BlockK kc = block_consts<FMT>(scales[b]);
        out[2 * b] = decode_word<FMT, BF16>(c.x, kc);
        out[2 * b + 1] = decode_word<FMT, BF16>(c.y, kc);
    }
}

// Online activation quantizer that also writes the decoded operand of the
// W4A4 product: each block goes through the same block quantizer as
// razer_quantize_acts (codes and scale byte, stored only when the caller asks
// for them) and its codes are decoded at once to q*s*2^-bias in fp16 (exact),
// so the activations are read once and the product needs no separate decode.
template <int FMT, typename TIn, bool FAST, bool HIST>
__device__ __forceinline__ void quantize_decode_loop(const TIn *__restrict__ x, int64_t nblk, const ScaleCtx &k, uint8_t *__restrict__ codes,
                                                     uint8_t *__restrict__ scales, uint4 *__restrict__ dec, unsigned (&cnt)[4])
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const uint4 *p = reinterpret_cast<const uint4 *>(x);
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk; b += stride) {
        const uint4 v0 = ldg_stream(p + 2 * b), v1 = ldg_stream(p + 2 * b + 1);
        const unsigned wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        float xv[16];
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const float2 f = In16<TIn>::to_f2(wv[i]);
            xv[2 * i] = f.x;
            xv[2 * i + 1] = f.y;
        }
        const BlockOut o = quantize_block<FMT, FAST, std::is_same<TIn, __half>::value>(xv, k);
        if (codes) reinterpret_cast<uint2 *>(codes)[b] = o.packed;
        if (scales) scales[b] = (uint8_t)o.sbyte;
        const BlockK kc = block_consts<FMT>(o.sbyte);
        dec[2 * b] = decode_word<FMT, false>(o.packed.x, kc);
        dec[2 * b + 1] = decode_word<FMT, false>(o.packed.y, kc);
        if constexpr (HIST) {
            const unsigned m1 = o.meta & 1u, e = o.effective ? 1u : 0u;
            cnt[0] += 1u - m1;
            cnt[1] += m1;
            cnt[2] += e & (1u - m1);
            cnt[3] += e & m1;
        }
    }
}

template <int FMT, typename TIn, bool HIST>
__global__ void __launch_bounds__(256) quantize_decode_kernel(const TIn *__restrict__ x, int64_t nblk, const float *__restrict__ ts_src,
                                                             int ts_is_amax, uint8_t *__restrict__ codes, uint8_t *__restrict__ scales,
                                                             unsigned long long *__restrict__ hist, uint4 *__restrict__ dec)
{
    using F = Fmt<FMT>;
    pdl_wait();
    pdl_trigger();
    const float tv = *ts_src;
    const float ts = ts_is_amax ? __fdiv_rn(tv, F::kC) : tv;
    __shared__ float tab_d[F::kMagMask + 1], tab_y[F::kMagMask + 1];
    const ScaleCtx k = make_ctx<FMT>(ts, tab_d, tab_y);
    __syncthreads();
    unsigned cnt[4] = {0u, 0u, 0u, 0u};
    if (fast_ts(ts)) quantize_decode_loop<FMT, TIn, true, HIST>(x, nblk, k, codes, scales, dec, cnt);
    else quantize_decode_loop<FMT, TIn, false, HIST>(x, nblk, k, codes, scales, dec, cnt);
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

// ts_a * ts_w (one binary32 rounding) for the epilogue of the W4A4 product
__global__ void ts_product_kernel(const float *__restrict__ a, const float *__restrict__ b, float *__restrict__ out)
{
    pdl_wait();
    pdl_trigger();
    *out = __fmul_rn(*a, *b);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
// decode once and run the persistent 16-bit GEMM when M is large enough that
// the fused kernel would decode every weight many times (M / BM), and for
// M >= 256 when the weight matrix is small enough that its decoded copy is
// cheap: measured on a B200 (bf16 out), M = 512: 4096 x 4096 47.1 -> 37.6 us,
// but 14336 x 4096 83.2 -> 92.7 us and 28672 x 8192 292 -> 342 us; M = 256:
// 4096 x 4096 38.4 -> 32.5 us, 14336 x 4096 63.1 -> 77.2 us
constexpr int64_t kDecodedMinM = 1024;
constexpr int64_t kDecodedSmallMinM = 256;
constexpr int64_t kDecodedSmallMaxNK = int64_t(1) << 25;

// Longest K one tensor-memory accumulation chain covers. The tcgen05 fp32
// accumulator loses precision over long chains (measured on B200 with
// decoded E3M3 weights: relative error ~5e-4 at K = 7168 but ~2.5e-3 at
// K = 28672), so a longer K runs as equal chunks whose scaled partial sums
// are added in fp32: as parallel splits with one [M, N] slice each in
// razer_gemm, through one [M, N] buffer chunk after chunk in the W4A4 product.
#ifndef RAZER_GEMM_CHAIN_K
#define RAZER_GEMM_CHAIN_K 16384
#endif
constexpr int64_t kMaxChainK = RAZER_GEMM_CHAIN_K;
static_assert(kMaxChainK % BK == 0, "chain length must be whole k-steps");

static int64_t num_chunks(int64_t K) { return (K + kMaxChainK - 1) / kMaxChainK; }
// Shapes the fused decoders cannot stream (K % 64 != 0: a row's last k-step
// is partial; N % 16 != 0) take the decode-once path: the bulk-tensor copies
// zero-fill past K and past N, so the k-steps simply run to ceil(K / 64).
static bool gemm_generic(int64_t N, int64_t K) { return K % BK != 0 || N % 16 != 0; }
static size_t decoded_bytes(int64_t M, int64_t N, int64_t K)
{
    const bool small_w = M >= kDecodedSmallMinM && N * K <= kDecodedSmallMaxNK;
    return (M >= kDecodedMinM || small_w || gemm_generic(N, K)) ? (size_t)N * (size_t)K * 2 : 0;
}
static size_t partial_bytes(int64_t M, int64_t N, int64_t K) { return num_chunks(K) > 1 ? (size_t)M * (size_t)N * 4 : 0; }

// Parallel K splits of razer_gemm: at least the number of accumulation chains
// K needs, and more when the output tiles alone cannot occupy the SMs (each
// split keeps at least kMinSplitSteps k-steps).  Every split writes its scaled
// fp32 sum to its own [M, N] slice of the workspace; gemm_splits_reduce_kernel
// adds the slices in split order (deterministic) and converts.
constexpr int64_t kMinSplitSteps = 8;
static int gemm_splits(int64_t M, int64_t N, int64_t K)
{
    const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    int64_t s = num_chunks(K);
    const int64_t sm = sm_count();
    if (tiles > 0 && tiles < sm) s = std::max(s, std::min(sm / tiles, (K / BK) / kMinSplitSteps));
    return (int)std::max<int64_t>(s, 1);
}
static size_t split_bytes(int64_t M, int64_t N, int64_t K)
{
    const int s = gemm_splits(M, N, K);
    return s > 1 ? (size_t)s * (size_t)M * (size_t)N * 4 : 0;
}

template <typename TOut>
__global__ void __launch_bounds__(256) gemm_splits_reduce_kernel(const float4 *__restrict__ part, int S, int64_t n4, TOut *__restrict__ Y)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
        float4 a = part[i];
        for (int z = 1; z < S; z++) {
            const float4 b = part[(size_t)z * (size_t)n4 + (size_t)i];
            a.x += b.x;
            a.y += b.y;
            a.z += b.z;
            a.w += b.w;
        }
        if constexpr (sizeof(TOut) == 4) {
            reinterpret_cast<float4 *>(Y)[i] = a;
        } else if constexpr (std::is_same<TOut, __half>::value) {
            __half2 lo = __floats2half2_rn(a.x, a.y), hi = __floats2half2_rn(a.z, a.w);
            reinterpret_cast<uint2 *>(Y)[i] = make_uint2(*reinterpret_cast<unsigned *>(&lo), *reinterpret_cast<unsigned *>(&hi));
        } else {
            __nv_bfloat162 lo = __floats2bfloat162_rn(a.x, a.y), hi = __floats2bfloat162_rn(a.z, a.w);
            reinterpret_cast<uint2 *>(Y)[i] = make_uint2(*reinterpret_cast<unsigned *>(&lo), *reinterpret_cast<unsigned *>(&hi));
        }
    }
}

// the same for any element count (rows of N % 4 != 0 elements are not
// 16-byte aligned)
template <typename TOut>
__global__ void __launch_bounds__(256) gemm_splits_reduce1_kernel(const float *__restrict__ part, int S, int64_t n, TOut *__restrict__ Y)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        float a = part[i];
        for (int z = 1; z < S; z++) a += part[(size_t)z * (size_t)n + (size_t)i];
        if constexpr (sizeof(TOut) == 4) Y[i] = a;
        else if constexpr (std::is_same<TOut, __half>::value) Y[i] = __float2half_rn(a);
        else Y[i] = __float2bfloat16_rn(a);
    }
}

template <int FMT, bool BF16>
static razer_status launch(const CUtensorMap &map, const uint8_t *codes, const uint8_t *scales, const float *ts,
                           float unbias, int M, int N, int K, void *Y, razer_dtype out_dt, int kb0, int nkb, const float *addend,
                           cudaStream_t st, int splits = 1)
{
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(gemm_kernel<FMT, BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES) !=
            cudaSuccess)
            return RAZER_ERR_CUDA;
        attr_set[dev] = true;
    }
    const unsigned nt = (unsigned)((N + BN - 1) / BN), mt = (unsigned)((M + BM - 1) / BM);
    const dim3 grid(nt, mt, (unsigned)splits);
    // fault injection (tests only) withholds one decoder warp's arrivals so
    // that the kernel's bounded waits expire (RAZER_ERR_TIMEOUT)
    const int inject = fault_injection_enabled() ? 1 : 0;
    gemm_kernel<FMT, BF16><<<grid, kThreads, SMEM_BYTES, st>>>(map, codes, scales, ts, unbias, M, N, K, Y, (int)out_dt, kb0, nkb, addend,
                                                             inject);
    return last_launch_status();
}

// tile width of the persistent GEMM: the candidate whose rounds of units over
// the SMs (each round as long as one tile of that width) cost least
static int choose_tbn(int64_t M, int64_t N, int S)
{
    const int64_t sm = sm_count(), mt = (M + 255) / 256;
    int best = 256;
    int64_t best_cost = 0;
    for (int c : {256, 224}) {
        const int64_t units = mt * ((N + c - 1) / c) * S, cost = (units + sm - 1) / sm * c;
        if (c == 256 || cost < best_cost) {
            best = c;
            best_cost = cost;
        }
    }
    return best;
}

// the persistent GEMM on two decoded 16-bit operands; S > 1 writes fp32
// slices (out = the slice buffer, out_dt = RAZER_F32); wmap's box is tbn rows
template <bool BF16, typename TOut, int TBN>
static razer_status launch_tma_t(const CUtensorMap &map, const CUtensorMap &wmap, const float *ts, float unbias, int M, int N, TOut *out,
                                 int kb0, int nkb, const float *addend, cudaStream_t st, int S, int kx_wrap)
{
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(gemm_tma_kernel<BF16, TOut, TBN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)tma_smem_bytes(TBN)) != cudaSuccess)
            return RAZER_ERR_CUDA;
        attr_set[dev] = true;
    }
    const int mt = (M + 255) / 256, nt = (N + TBN - 1) / TBN, T = mt * nt;
    const int G = (int)std::min<int64_t>((int64_t)T * S, sm_count());
    // fault injection (tests only): CTA 0 leaves its first stage unfilled so
    // that the kernel's bounded waits expire (RAZER_ERR_TIMEOUT)
    const int inject = fault_injection_enabled() ? 1 : 0;
    if (launch_pdl(gemm_tma_kernel<BF16, TOut, TBN>, (unsigned)G, (unsigned)kTmaThreads, (size_t)tma_smem_bytes(TBN), st, map, wmap, ts,
                   unbias, M, N, mt, T, S, kb0, nkb, out, addend, inject, kx_wrap) != cudaSuccess)
        return RAZER_ERR_CUDA;
    return RAZER_OK;
}

template <bool BF16, typename TOut>
static razer_status launch_tma_w(const CUtensorMap &map, const CUtensorMap &wmap, int tbn, const float *ts, float unbias, int M, int N,
                                 TOut *out, int kb0, int nkb, const float *addend, cudaStream_t st, int S, int kx_wrap)
{
    if (tbn == 224) return launch_tma_t<BF16, TOut, 224>(map, wmap, ts, unbias, M, N, out, kb0, nkb, addend, st, S, kx_wrap);
    return launch_tma_t<BF16, TOut, 256>(map, wmap, ts, unbias, M, N, out, kb0, nkb, addend, st, S, kx_wrap);
}

template <bool BF16>
static razer_status launch_tma(const CUtensorMap &map, const CUtensorMap &wmap, int tbn, const float *ts, float unbias, int M, int N,
                               void *out, razer_dtype out_dt, int kb0, int nkb, const float *addend, cudaStream_t st, int S,
                               int kx_wrap = 0)
{
    if (out_dt == RAZER_F32)
        return launch_tma_w<BF16, float>(map, wmap, tbn, ts, unbias, M, N, reinterpret_cast<float *>(out), kb0, nkb, addend, st, S, kx_wrap);
    if (out_dt == RAZER_F16)
        return launch_tma_w<BF16, __half>(map, wmap, tbn, ts, unbias, M, N, reinterpret_cast<__half *>(out), kb0, nkb, addend, st, S, kx_wrap);
    return launch_tma_w<BF16, __nv_bfloat16>(map, wmap, tbn, ts, unbias, M, N, reinterpret_cast<__nv_bfloat16 *>(out), kb0, nkb, addend, st,
                                             S, kx_wrap);
}

static razer_status reduce_splits(const float *slices, int S, int M, int N, void *Y, razer_dtype out_dt, cudaStream_t st);

template <int FMT, bool BF16>
static razer_status launch_fmt(const CUtensorMap &map, const CUtensorMap &wmap, int tbn, bool decoded, const uint8_t *codes,
                               const uint8_t *scales, const float *ts, float unbias, int M, int N, int K, void *Y, razer_dtype out_dt,
                               void *wdec, float *slices, cudaStream_t st)
{
    if (decoded) {
        const int64_t nblk = (int64_t)N * K / 16;
        const int64_t g = std::min<int64_t>((nblk + 255) / 256, (int64_t)sm_count() * 8);
        if (launch_pdl(decode_weights_kernel<FMT, BF16>, (unsigned)g, 256u, 0, st, codes, scales, nblk, reinterpret_cast<uint4 *>(wdec)) !=
            cudaSuccess)
            return RAZER_ERR_CUDA;
    }
    const int KB = (K + BK - 1) / BK;  // the last k-step of a generic K is zero-filled past K
    const int S = gemm_splits(M, N, K);
    void *out = S > 1 ? static_cast<void *>(slices) : Y;
    const razer_dtype odt = S > 1 ? RAZER_F32 : out_dt;
    const razer_status r = decoded ? launch_tma<BF16>(map, wmap, tbn, ts, unbias, M, N, out, odt, 0, KB, nullptr, st, S)
                                   : launch<FMT, BF16>(map, codes, scales, ts, unbias, M, N, K, out, odt, 0, KB, nullptr, st, S);
    if (r != RAZER_OK || S == 1) return r;
    return reduce_splits(slices, S, M, N, Y, out_dt, st);
}

// adds the S fp32 [M, N] slices in split order and converts to out_dt
static razer_status reduce_splits(const float *slices, int S, int M, int N, void *Y, razer_dtype out_dt, cudaStream_t st)
{
    if (N % 4 != 0) {
        const int64_t n1 = (int64_t)M * N;
        const int64_t g = std::max<int64_t>(1, std::min<int64_t>((n1 + 255) / 256, (int64_t)sm_count() * 8));
        if (out_dt == RAZER_F32) gemm_splits_reduce1_kernel<float><<<(unsigned)g, 256, 0, st>>>(slices, S, n1, reinterpret_cast<float *>(Y));
        else if (out_dt == RAZER_F16) gemm_splits_reduce1_kernel<__half><<<(unsigned)g, 256, 0, st>>>(slices, S, n1, reinterpret_cast<__half *>(Y));
        else gemm_splits_reduce1_kernel<__nv_bfloat16><<<(unsigned)g, 256, 0, st>>>(slices, S, n1, reinterpret_cast<__nv_bfloat16 *>(Y));
        return last_launch_status();
    }
    const int64_t n4 = (int64_t)M * N / 4;  // N % 4 == 0
    const int64_t g = std::max<int64_t>(1, std::min<int64_t>((n4 + 255) / 256, (int64_t)sm_count() * 8));
    const float4 *part = reinterpret_cast<const float4 *>(slices);
    if (out_dt == RAZER_F32) gemm_splits_reduce_kernel<float><<<(unsigned)g, 256, 0, st>>>(part, S, n4, reinterpret_cast<float *>(Y));
    else if (out_dt == RAZER_F16) gemm_splits_reduce_kernel<__half><<<(unsigned)g, 256, 0, st>>>(part, S, n4, reinterpret_cast<__half *>(Y));
    else gemm_splits_reduce_kernel<__nv_bfloat16><<<(unsigned)g, 256, 0, st>>>(part, S, n4, reinterpret_cast<__nv_bfloat16 *>(Y));
    return last_launch_status();
}

// decoded q*s*2^-bias of a packed [R, K] tensor into out (16-bit, [R, K])
template <bool BF16>
static razer_status decode_into(razer_format fmt, const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t K, void *out,
                                cudaStream_t st)
{
    const int64_t nblk = rows * K / 16;
    const int64_t g = std::min<int64_t>((nblk + 255) / 256, (int64_t)sm_count() * 8);
    uint4 *o = reinterpret_cast<uint4 *>(out);
    cudaError_t e;
    if (fmt == RAZER_FMT_WEIGHT) e = launch_pdl(decode_weights_kernel<RAZER_FMT_WEIGHT, BF16>, (unsigned)g, 256u, 0, st, codes, scales, nblk, o);
    else if (fmt == RAZER_FMT_ACT) e = launch_pdl(decode_weights_kernel<RAZER_FMT_ACT, BF16>, (unsigned)g, 256u, 0, st, codes, scales, nblk, o);
    else e = launch_pdl(decode_weights_kernel<RAZER_FMT_NVFP4, BF16>, (unsigned)g, 256u, 0, st, codes, scales, nblk, o);
    return e == cudaSuccess ? RAZER_OK : RAZER_ERR_CUDA;
}

// 2^bias carried by the decoded q*s of a format (E3M3: 2^-8, E4M3: 2^-4)
static float decode_unbias(razer_format fmt) { return fmt == RAZER_FMT_WEIGHT ? 256.0f : 16.0f; }

static size_t w4a4_decoded_a_bytes(int64_t M, int64_t K) { return (size_t)M * (size_t)K * 2; }

}  // namespace gemm

size_t gemm_w4a4_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    // decoded A [M, K] and W [N, K] (fp16), the fp32 partial sums when K spans
    // several accumulation chains, then ts_a * ts_w
    return gemm::w4a4_decoded_a_bytes(M, K) + (size_t)N * (size_t)K * 2 + gemm::partial_bytes(M, N, K) + 16;
}

// W4A4 product of two RaZeR-packed operands: both decoded exactly to fp16
// (q*s*2^-bias) and multiplied on the tcgen05 pipeline of the decode-once
// path; the epilogue applies ts_a * ts_w and both unbias factors.
// The product half of the W4A4 path: the decoded A (fp16) sits at the start
// of the workspace, written earlier on the stream; ts_a is the activations'
// tensor scale (device).
static razer_status w4a4_product(const float *ts_a, razer_format afmt, int64_t M, const uint8_t *codes_w,
                                 const uint8_t *scales_w, const float *ts_w, razer_format wfmt, int64_t N, int64_t K, void *Y,
                                 razer_dtype out_dt, void *workspace, cudaStream_t st)
{
    using namespace gemm;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return RAZER_ERR_CUDA;
    uint8_t *base = static_cast<uint8_t *>(workspace);
    uint8_t *wa = base, *ww = base + w4a4_decoded_a_bytes(M, K);
    uint8_t *after_w = ww + (size_t)N * (size_t)K * 2;
    float *partial = partial_bytes(M, N, K) ? reinterpret_cast<float *>(after_w) : nullptr;
    float *tsp = reinterpret_cast<float *>(after_w + partial_bytes(M, N, K));
    if (launch_pdl(ts_product_kernel, 1u, 1u, 0, st, ts_a, ts_w, tsp) != cudaSuccess) return RAZER_ERR_CUDA;
    razer_status r = decode_into<false>(wfmt, codes_w, scales_w, N, K, ww, st);
    if (r != RAZER_OK) return r;
    CUtensorMap amap, wmap;
    const cuuint32_t estr[2] = {1u, 1u};
    {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {(cuuint32_t)BK, 128u};
        if (enc(&amap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, wa, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return RAZER_ERR_CUDA;
    }
    const int tbn = choose_tbn(M, N, 1);
    {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)N};
        const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)tbn};
        if (enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, ww, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return RAZER_ERR_CUDA;
    }
    const float unbias = decode_unbias(afmt) * decode_unbias(wfmt);  // a power of two: exact
    const int m = (int)M, n = (int)N, k = (int)K, KB = (k + BK - 1) / BK, nc = (int)num_chunks(K);
    for (int c = 0; c < nc; c++) {
        const int kb0 = (int)((int64_t)c * KB / nc), kb1 = (int)((int64_t)(c + 1) * KB / nc);
        const bool last = c == nc - 1;
        r = launch_tma<false>(amap, wmap, tbn, tsp, unbias, m, n, last ? Y : partial, last ? out_dt : RAZER_F32, kb0, kb1 - kb0,
                              c > 0 ? partial : nullptr, st, 1);
        if (r != RAZER_OK) return r;
    }
    return RAZER_OK;
}

// W4A4 product of two RaZeR-packed operands: both decoded exactly to fp16
// (q*s*2^-bias) and multiplied on the tcgen05 pipeline of the decode-once
// path; the epilogue applies ts_a * ts_w and both unbias factors.
razer_status run_gemm_w4a4(const uint8_t *codes_a, const uint8_t *scales_a, const float *ts_a, razer_format afmt, int64_t M,
                           const uint8_t *codes_w, const uint8_t *scales_w, const float *ts_w, razer_format wfmt, int64_t N, int64_t K,
                           void *Y, razer_dtype out_dt, void *workspace, cudaStream_t st)
{
    using namespace gemm;
    if (K == 0) {
        const size_t esz = out_dt == RAZER_F32 ? 4 : 2;
        return cudaMemsetAsync(Y, 0, (size_t)M * (size_t)N * esz, st) == cudaSuccess ? RAZER_OK : RAZER_ERR_CUDA;
    }
    uint8_t *wa = static_cast<uint8_t *>(workspace);
    const razer_status r = decode_into<false>(afmt, codes_a, scales_a, M, K, wa, st);
    if (r != RAZER_OK) return r;
    return w4a4_product(ts_a, afmt, M, codes_w, scales_w, ts_w, wfmt, N, K, Y, out_dt, workspace, st);
}

// Online W4A4: the activations X are quantized (dynamic tensor scale when
// ts_in is NULL, as razer_quantize_acts) by the fused quantize + decode
// kernel, then multiplied as in run_gemm_w4a4.  codes_a / scales_a / hist may
// be NULL; ts_a_out receives the activations' tensor scale.
template <int FMT, typename TIn>
static razer_status quantize_decode_t(const void *X, int64_t nblk, const float *ts_src, int is_amax, uint8_t *codes, uint8_t *scales,
                                      unsigned long long *hist, void *dec, cudaStream_t st)
{
    const unsigned grid = (unsigned)std::min<int64_t>((nblk + 255) / 256, (int64_t)sm_count() * 8);
    cudaError_t e;
    if (hist && Fmt<FMT>::kSpecials > 0)
        e = launch_pdl(gemm::quantize_decode_kernel<FMT, TIn, true>, grid, 256u, 0, st, reinterpret_cast<const TIn *>(X), nblk, ts_src,
                       is_amax, codes, scales, hist, reinterpret_cast<uint4 *>(dec));
    else
        e = launch_pdl(gemm::quantize_decode_kernel<FMT, TIn, false>, grid, 256u, 0, st, reinterpret_cast<const TIn *>(X), nblk, ts_src,
                       is_amax, codes, scales, (unsigned long long *)nullptr, reinterpret_cast<uint4 *>(dec));
    return e == cudaSuccess ? RAZER_OK : RAZER_ERR_CUDA;
}

razer_status run_gemm_w4a4_online(const void *X, razer_dtype x_dt, int64_t M, const float *ts_in, razer_format afmt, uint8_t *codes_a,
                                  uint8_t *scales_a, float *ts_a_out, unsigned long long *hist, const uint8_t *codes_w,
                                  const uint8_t *scales_w, const float *ts_w, razer_format wfmt, int64_t N, int64_t K, void *Y,
                                  razer_dtype out_dt, void *workspace, cudaStream_t st)
{
    const int64_t n = M * K, nblk = n / 16;
    const float C = afmt == RAZER_FMT_WEIGHT ? Fmt<RAZER_FMT_WEIGHT>::kC : Fmt<RAZER_FMT_ACT>::kC;
    if (hist || !ts_in) {
        if (launch_pdl(quant_init_kernel, 1u, 32u, 0, st, hist, ts_in ? (unsigned *)nullptr : reinterpret_cast<unsigned *>(ts_a_out),
                   (unsigned *)nullptr) !=
            cudaSuccess)
            return RAZER_ERR_CUDA;
    }
    const float *ts_src = ts_in;
    int is_amax = 0;
    if (!ts_in) {
        if (n > 0) {
            if (x_dt == RAZER_F16) launch_amax<__half>(X, n, reinterpret_cast<unsigned *>(ts_a_out), st);
            else launch_amax<__nv_bfloat16>(X, n, reinterpret_cast<unsigned *>(ts_a_out), st);
        }
        ts_src = ts_a_out;
        is_amax = 1;
    }
    uint8_t *wa = static_cast<uint8_t *>(workspace);
    if (nblk > 0) {
        const bool h = x_dt == RAZER_F16;
        razer_status r;
        if (afmt == RAZER_FMT_ACT)
            r = h ? quantize_decode_t<RAZER_FMT_ACT, __half>(X, nblk, ts_src, is_amax, codes_a, scales_a, hist, wa, st)
                  : quantize_decode_t<RAZER_FMT_ACT, __nv_bfloat16>(X, nblk, ts_src, is_amax, codes_a, scales_a, hist, wa, st);
        else
            r = h ? quantize_decode_t<RAZER_FMT_NVFP4, __half>(X, nblk, ts_src, is_amax, codes_a, scales_a, hist, wa, st)
                  : quantize_decode_t<RAZER_FMT_NVFP4, __nv_bfloat16>(X, nblk, ts_src, is_amax, codes_a, scales_a, hist, wa, st);
        if (r != RAZER_OK) return r;
    }
    if (!ts_in) {
        if (launch_pdl(finalize_ts_kernel, 1u, 1u, 0, st, ts_a_out, C) != cudaSuccess) return RAZER_ERR_CUDA;
    } else if (ts_a_out != ts_in) {
        if (launch_pdl(copy_ts_kernel, 1u, 1u, 0, st, ts_in, ts_a_out) != cudaSuccess) return RAZER_ERR_CUDA;
    }
    if (K == 0) {
        const size_t esz = out_dt == RAZER_F32 ? 4 : 2;
        return cudaMemsetAsync(Y, 0, (size_t)M * (size_t)N * esz, st) == cudaSuccess ? RAZER_OK : RAZER_ERR_CUDA;
    }
    return w4a4_product(ts_a_out, afmt, M, codes_w, scales_w, ts_w, wfmt, N, K, Y, out_dt, workspace, st);
}

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    // the decoded weight copy when the decode-once path applies, then one fp32
    // [M, N] slice per parallel K split when there is more than one
    return gemm::decoded_bytes(M, N, K) + gemm::split_bytes(M, N, K);
}

razer_status run_gemm(const void *X, razer_dtype act_dt, int64_t M, const uint8_t *codes, const uint8_t *scales, const float *ts,
                      razer_format wfmt, int64_t N, int64_t K, void *Y, razer_dtype out_dt, void *workspace, cudaStream_t st)
{
    using namespace gemm;
    if (K == 0) {
        const size_t esz = out_dt == RAZER_F32 ? 4 : 2;
        return cudaMemsetAsync(Y, 0, (size_t)M * (size_t)N * esz, st) == cudaSuccess ? RAZER_OK : RAZER_ERR_CUDA;
    }
    EncodeTiledFn enc = encode_fn();
    if (!enc) return RAZER_ERR_CUDA;
    const bool bf = act_dt == RAZER_BF16;
    CUtensorMap map;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)BK, 128u};
    const cuuint32_t estr[2] = {1u, 1u};
    if (enc(&map, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(X), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return RAZER_ERR_CUDA;
    // the decoded q*s carries 2^-8 (E3M3) / 2^-4 (E4M3); undone in the epilogue
    const float unbias = wfmt == RAZER_FMT_WEIGHT ? 256.0f : 16.0f;
    const bool decoded = decoded_bytes(M, N, K) > 0;
    float *slices = split_bytes(M, N, K) ? reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + decoded_bytes(M, N, K)) : nullptr;
    CUtensorMap wmap = map;  // unused by the fused kernel
    const int tbn = choose_tbn(M, N, gemm_splits(M, N, K));
    if (decoded) {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)N};
        const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)tbn};
        const cuuint32_t estr[2] = {1u, 1u};
        if (enc(&wmap, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, workspace, dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return RAZER_ERR_CUDA;
    }
    const int m = (int)M, n = (int)N, k = (int)K;
    if (wfmt == RAZER_FMT_WEIGHT)
        return bf ? launch_fmt<RAZER_FMT_WEIGHT, true>(map, wmap, tbn, decoded, codes, scales, ts, unbias, m, n, k, Y, out_dt, workspace, slices, st)
                  : launch_fmt<RAZER_FMT_WEIGHT, false>(map, wmap, tbn, decoded, codes, scales, ts, unbias, m, n, k, Y, out_dt, workspace, slices, st);
    if (wfmt == RAZER_FMT_ACT)
        return bf ? launch_fmt<RAZER_FMT_ACT, true>(map, wmap, tbn, decoded, codes, scales, ts, unbias, m, n, k, Y, out_dt, workspace, slices, st)
                  : launch_fmt<RAZER_FMT_ACT, false>(map, wmap, tbn, decoded, codes, scales, ts, unbias, m, n, k, Y, out_dt, workspace, slices, st);
    return bf ? launch_fmt<RAZER_FMT_NVFP4, true>(map, wmap, tbn, decoded, codes, scales, ts, unbias, m, n, k, Y, out_dt, workspace, slices, st)
              : launch_fmt<RAZER_FMT_NVFP4, false>(map, wmap, tbn, decoded, codes, scales, ts, unbias, m, n, k, Y, out_dt, workspace, slices, st);
}


// ---------------------------------------------------------------------------
// Prefill GEMM on a format-variant weight tensor (blocks of 16-128 elements, a
// caller-chosen special-value set, or the pages' FP16-scale words; RaZeR
// notes, 关键设计 3 and 训练策略).  The weights are decoded once into a 16-bit
// copy and the persistent tcgen05 GEMM multiplies it, applying ts in the
// epilogue.
//   * byte scales: the decoder of razer_dequant_variant, given a device 1.0
//     in place of ts, writes round16(q*s) -- exact: q*s has at most 5 + 4
//     significant bits and lies in [2^-10, 4256], inside fp16's normal range;
//     in bf16 as well unless +-9.5 is in the set (refused by the caller);
//   * FP16 scale words: q*s has up to 16 significant bits, more than a 16-bit
//     operand holds, so the copy is two 16-bit terms of q*s*2^11 side by side
//     ([N, 2 K]: hi, then lo; see decode_f16w_split_kernel) and the GEMM runs
//     over 2 K with the activations' k-steps taken twice, then scales by
//     ts * 2^-11.  Twice the MMA work of the byte-scale formats, for a
//     product within fp32 accumulation of the exact one (bf16: hi + lo is
//     q*s*2^11 exactly; fp16: to within 2^-25 where lo is subnormal).
// ---------------------------------------------------------------------------
razer_status run_dequant_variant(const uint8_t *codes, const uint8_t *scales, const float *ts, int64_t R, int64_t K, int bs,
                                 razer_format sfmt, const VariantV &V, void *out, razer_dtype dt, cudaStream_t st);
razer_status run_decode_f16w_split(const uint8_t *codes, const uint8_t *scales, int64_t N, int64_t K, int bs, const VariantV &V, void *out,
                                   bool bf16, cudaStream_t st);

namespace gemm {
__global__ void unit_scale_kernel(float *p) { *p = 1.0f; }
}  // namespace gemm

size_t gemm_variant_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    // sized for the FP16-word layout (two terms, 2 K columns; the byte-scale
    // formats use the first half): the decoded copy, the fp32 slices of the
    // parallel K splits, one float
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    return (size_t)N * (size_t)K * 4 + gemm::split_bytes(M, N, 2 * K) + 16;
}

razer_status run_gemm_variant(const void *X, razer_dtype act_dt, int64_t M, const uint8_t *codes, const uint8_t *scales, const float *ts,
                              int block, razer_format sfmt, const VariantV &V, int64_t N, int64_t K, void *Y, razer_dtype out_dt,
                              void *workspace, cudaStream_t st)
{
    using namespace gemm;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return RAZER_ERR_CUDA;
    const bool bf = act_dt == RAZER_BF16, two = sfmt == RAZER_SCALE_F16;
    const int64_t Kw = two ? 2 * K : K;  // columns of the weight copy
    uint8_t *base = static_cast<uint8_t *>(workspace);
    const size_t dec = (size_t)N * (size_t)Kw * 2, sb = split_bytes(M, N, Kw);
    float *slices = sb ? reinterpret_cast<float *>(base + dec) : nullptr;
    razer_status r;
    if (two) {
        r = run_decode_f16w_split(codes, scales, N, K, block, V, base, bf, st);
    } else {
        float *one = reinterpret_cast<float *>(base + dec + sb);
        unit_scale_kernel<<<1, 1, 0, st>>>(one);
        r = run_dequant_variant(codes, scales, one, N, K, block, sfmt, V, base, bf ? RAZER_BF16 : RAZER_F16, st);
    }
    if (r != RAZER_OK) return r;
    CUtensorMap map, wmap;
    const cuuint32_t estr[2] = {1u, 1u};
    const CUtensorMapDataType tdt = bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {(cuuint32_t)BK, 128u};
        if (enc(&map, tdt, 2, const_cast<void *>(X), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return RAZER_ERR_CUDA;
    }
    const int tbn = choose_tbn(M, N, gemm_splits(M, N, Kw));
    {
        const cuuint64_t dims[2] = {(cuuint64_t)Kw, (cuuint64_t)N};
        const cuuint64_t strides[1] = {(cuuint64_t)Kw * 2};
        const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)tbn};
        if (enc(&wmap, tdt, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return RAZER_ERR_CUDA;
    }
    // two terms: K % 64 == 0 (checked by the caller), so the hi and lo halves
    // are whole k-steps and X's k-steps repeat after KB
    const int m = (int)M, n = (int)N, KB = (int)((K + BK - 1) / BK), KBw = two ? 2 * KB : KB;
    const int S = gemm_splits(M, N, Kw);
    const float unbias = two ? 1.0f / 2048.0f : 1.0f;  // a power of two: exact
    void *out = S > 1 ? static_cast<void *>(slices) : Y;
    const razer_dtype odt = S > 1 ? RAZER_F32 : out_dt;
    r = bf ? launch_tma<true>(map, wmap, tbn, ts, unbias, m, n, out, odt, 0, KBw, nullptr, st, S, two ? KB : 0)
           : launch_tma<false>(map, wmap, tbn, ts, unbias, m, n, out, odt, 0, KBw, nullptr, st, S, two ? KB : 0);
    if (r != RAZER_OK || S == 1) return r;
    return reduce_splits(slices, S, m, n, Y, out_dt, st);
}

}  // namespace razer
