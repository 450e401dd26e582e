// RaZeR W4A16 GEMV / skinny GEMM (1 <= B <= 32), bulk-tensor pipeline for
// sm_100a; taken when K % 256 == 0 (the scale rows are then 16-byte strided,
// as a tensor map requires) and the scale pointer is 16-byte aligned.
//
// y[b, n] = ts * sum_k x[b, k] * (q*s)[n, k]     (RaZeR notes 关键设计 3:
// weight-only kernels that decode the remapped codes in registers, and
// split-K sized for the machine -- here one persistent CTA per SM.)
//
//   * Work = 128-row tiles x 128-k half-units, flattened tile-major and cut
//     into one contiguous range per CTA ("stream-K"): every SM streams the
//     same number of weight bytes, whatever N and K, and there is no tail
//     wave.
//   * Warp 0 (one lane) is the TMA producer.  Per 256-k stage it loads the
//     code tile (128 rows x 128 B, 128-byte swizzle), the scale tile
//     (128 x 16 B) and the B activation rows (B x 512 B) into an S-deep
//     shared-memory ring guarded by full / empty mbarriers.
//   * The consumer warps each own 16 * kMT rows of the tile and one 128-k half
//     of every stage; they run the register decode and warp-level m16n8k16
//     MMAs of the split-K kernel (the kMT row tiles share the activation
//     fragments).  The MMA rows g = 2p and 2p+1 (one 128-bit shared-load
//     phase) map to tile rows p and p+4, whose swizzled 16-byte chunks sit in
//     opposite halves of the banks, so the code loads are conflict-free.
//   * When a CTA finishes its part of a tile, the consumers drop their fp32
//     partials into one of two shared-memory hand-over buffers and go on with
//     the next tile at once.  Warp 1 (the epilogue warp) adds the two k-halves
//     and either writes y (the CTA covered the whole tile) or stores the sum in
//     slot (cta + tile) of the workspace -- the slot index grows along the
//     flattened order, so it is unique.  A small second kernel, launched as a
//     programmatic dependent of the first (it is resident and waiting while
//     the first drains), sums the slots of the shared tiles in CTA order --
//     deterministic --, applies ts and converts.  Both kernels wait on their
//     predecessor in the stream (griddepcontrol.wait) before reading memory it
//     may have written.
//   * Every mbarrier wait is bounded; on expiry the CTA records
//     RAZER_ERR_TIMEOUT, stops waiting, keeps its control flow (and its
//     arrivals) uniform, and the producer lets its in-flight loads land
//     before it exits.
#include <algorithm>
#include <cstring>
#include <vector>

#include "razer_internal.cuh"
#include "sm100_async.cuh"

namespace razer {
namespace gemv_tma {

constexpr int kTileRows = 128;
constexpr int kFirstConsumer = 2;                   // warp 0: TMA producer, warp 1: epilogue
constexpr int kCodeBytes = kTileRows * 128;         // 128 rows x 256 codes
constexpr int kScaleBytes = kTileRows * 16;         // 128 rows x 16 blocks
constexpr int kMaxStages = 8;
constexpr int kBarBytes = 256;
constexpr int kTableBytes = 2048;                   // 256 (s, v*s) fp32 pairs, one per scale byte
constexpr int kSmemLimit = 227 * 1024;
// consumer warps: one per (group of 16 * MT rows of the tile, 128-k half of a stage)
__host__ __device__ constexpr int consumer_warps(int MT) { return 2 * (kTileRows / (16 * MT)); }
__host__ __device__ constexpr int cta_threads(int MT) { return 32 * (kFirstConsumer + consumer_warps(MT)); }

__host__ __device__ constexpr int stage_bytes(int B) { return (kCodeBytes + kScaleBytes + B * 512 + 1023) / 1024 * 1024; }
// two hand-over buffers of [k-half][B][128 rows] fp32 partials
__host__ __device__ constexpr int part_bytes(int B) { return 2 * 2 * B * kTileRows * 4; }
// dynamic shared memory: 2 KB alignment slack | scale table | stages | hand-over | barriers
__host__ __device__ constexpr int fixed_bytes(int B) { return 2047 + kTableBytes + part_bytes(B) + kBarBytes; }
__host__ __device__ constexpr int num_stages(int B)
{
    return (kSmemLimit - fixed_bytes(B)) / stage_bytes(B) > kMaxStages ? kMaxStages : (kSmemLimit - fixed_bytes(B)) / stage_bytes(B);
}
__host__ __device__ constexpr int smem_bytes(int B) { return num_stages(B) * stage_bytes(B) + fixed_bytes(B); }

// A batch of independent problems y_i = ts_i * x_i * deq(W_i)^T (same
// formats, same output type) run as one stream-K pass: their tiles are
// concatenated in problem order, so one launch (one pipeline fill, one drain,
// one reduction) serves all of them.  Problem i covers the global half-units
// [unit0[i], unit0[i + 1]) and the global tiles [tile0[i], tile0[i + 1]).
constexpr int kMaxProblems = 8;
struct BatchInfo {
    int count;
    int B[kMaxProblems], N[kMaxProblems], UK2[kMaxProblems];
    int unit0[kMaxProblems + 1], tile0[kMaxProblems + 1];
    const float *ts[kMaxProblems];
    void *y[kMaxProblems];
};
struct Batch {
    CUtensorMap map[kMaxProblems][3];  // codes, scales and x of problem i
    BatchInfo info;
};

// the problem whose half-units contain global half-unit p
__device__ __forceinline__ int problem_of(const BatchInfo &I, int p)
{
    int i = 0;
    while (i + 1 < I.count && p >= I.unit0[i + 1]) i++;
    return i;
}

// first half-unit of CTA c's range
__host__ __device__ __forceinline__ int range_start(int c, int U, int G) { return (int)((int64_t)c * U / G); }
// the CTA whose range holds half-unit p (ranges are never empty: G <= U)
__host__ __device__ __forceinline__ int range_owner(int p, int U, int G) { return (int)(((int64_t)(p + 1) * G - 1) / U); }

// tile row of MMA row g (and g + 8 -> +8): rows 2p, 2p+1 -> p, p+4
__device__ __forceinline__ int tile_row(int g) { return (g >> 1) | ((g & 1) << 2); }

__device__ __forceinline__ uint4 lds128(uint32_t a)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ unsigned lds16(uint32_t a)
{
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ void store_out(void *y, int out_dt, size_t i, float v)
{
    if (out_dt == RAZER_F32) reinterpret_cast<float *>(y)[i] = v;
    else if (out_dt == RAZER_F16) reinterpret_cast<__half *>(y)[i] = __float2half_rn(v);
    else reinterpret_cast<__nv_bfloat16 *>(y)[i] = __float2bfloat16_rn(v);
}

// wait that returns at once when the phase is complete (the common case)
__device__ __forceinline__ void wait_phase(uint32_t bar, uint32_t ph, volatile int *flags)
{
    if (!mbar_try_wait(bar, ph)) (void)mbar_wait(bar, ph, flags);  // on abort: carry on, results are void
}

// ---------------------------------------------------------------------------
// Block-column decode (B <= 4, fp16 activations).
//
// The per-element decode is reduced to one hardware E2M1 convert per code
// pair: neither the block scale nor the special value is applied to the
// decoded operand.
//   * The 8 output columns of each m16n8k16 MMA carry (block, batch row)
//     pairs instead of batch rows: the activation operand is block-diagonal
//     (column n only sees the k of its block), so after the MMAs of one group
//     column n holds the unscaled dot product of one 16-element block.  The
//     block scale s is then applied once per (row, block) with an fp32 FMA on
//     the MMA output.  BP = padded batch (1, 2 or 4); a group of 8 / BP MMAs
//     covers 8 / BP blocks.
//   * The redundant-zero codes (0b1000) convert to -0, so the plain MMA adds
//     nothing for them.  A second MMA multiplies a 0/1 indicator operand
//     (the E2M1 code of 1.0 exactly where the code is 0b1000, found with
//     three integer operations per 8 codes) by the same activations; its
//     output, times v*s, is the special values' share of the block
//     (RaZeR notes 关键设计 2: the -0 code carries the special value).
//   * s and v*s of every scale byte come from a 256-entry fp32 table in
//     shared memory built at kernel start (one 8-byte load per block).
// Each fp32 product s*(q.x) equals the exact sum up to the MMA's fp32
// accumulation, and q*x, v*x are exact in the MMA, so the result carries
// the same rounding as decoding q*s first.
// ---------------------------------------------------------------------------

// E2M1 pair -> f16x2 of byte lane L of w (L a compile-time constant after unrolling)
__device__ __forceinline__ unsigned cvt_byte(unsigned w, int L)
{
    unsigned r;
    if (L == 0) asm("{ .reg .b8 b0, b1, b2, b3; mov.b32 {b0, b1, b2, b3}, %1; cvt.rn.f16x2.e2m1x2 %0, b0; }" : "=r"(r) : "r"(w));
    else if (L == 1) asm("{ .reg .b8 b0, b1, b2, b3; mov.b32 {b0, b1, b2, b3}, %1; cvt.rn.f16x2.e2m1x2 %0, b1; }" : "=r"(r) : "r"(w));
    else if (L == 2) asm("{ .reg .b8 b0, b1, b2, b3; mov.b32 {b0, b1, b2, b3}, %1; cvt.rn.f16x2.e2m1x2 %0, b2; }" : "=r"(r) : "r"(w));
    else asm("{ .reg .b8 b0, b1, b2, b3; mov.b32 {b0, b1, b2, b3}, %1; cvt.rn.f16x2.e2m1x2 %0, b3; }" : "=r"(r) : "r"(w));
    return r;
}

// E2M1 codes of 1.0 (0b0010) exactly where a nibble of w is 0b1000, 0 elsewhere
__device__ __forceinline__ unsigned indicator_codes(unsigned w)
{
    const unsigned t = (w & 0x77777777u) + 0x77777777u;  // bit 3 set where the magnitude bits are non-zero
    const unsigned is8 = w & ~t & 0x88888888u;           // bit 3 set where the code is 0b1000
    return __umulhi(is8, 0x40000000u);                   // >> 2 on the multiply pipe
}

// not volatile: a pure function of its operands, so the compiler may
// interleave the MMAs of independent row tiles and groups
__device__ __forceinline__ void mma_f16(float (&d)[4], unsigned a0, unsigned a1, unsigned a2, unsigned a3, unsigned b0, unsigned b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// (s, v*s) of byte lane L of w
__device__ __forceinline__ float2 table_entry(unsigned w, int L, const float2 *tbl) { return tbl[(w >> (8 * L)) & 0xFFu]; }

// Shared-memory loads as plain C++ loads (not volatile asm): the compiler
// schedules them freely between the pipeline-barrier waits, whose asm
// carries a memory clobber, so no load moves above the wait for its stage.
template <typename T> __device__ __forceinline__ T sld(const uint8_t *p) { return *reinterpret_cast<const T *>(p); }

// MMA row g of a 16-row tile -> tile row (0..7), chosen so that the code
// loads of one shared-memory phase hit distinct banks under the 128-byte swizzle
template <int BP> __device__ __forceinline__ int bc_row(int g) { return BP == 2 ? (((g & 3) << 1) | (g >> 2)) : tile_row(g); }

// One 128-k slice of one 16-row tile: the codes of rows r and r + 8 (tile
// rows; r & 7 == pr) through the block-column MMAs, accumulated into acc
// (BP = 1: [row g, row g+8]; BP = 2, 4: [row g: 2 batch columns, row g+8: 2]).
template <int FMT, int BP>
__device__ __forceinline__ void bc_tile(const uint8_t *st, const uint8_t *scl, const float2 *tbl, int r, int pr, int kh, int t,
                                        const unsigned (&xb0)[16], const unsigned (&xb1)[16], float (&acc)[4])
{
    constexpr bool kSpecial = Fmt<FMT>::kSpecials > 0;
    const uint8_t *rowA = st + r * 128, *rowB = rowA + 8 * 128;
    // this half's 8 scale bytes of rows r and r + 8
    const uint2 sA = sld<uint2>(scl + r * 16 + 8 * kh), sB = sld<uint2>(scl + (r + 8) * 16 + 8 * kh);
    if constexpr (BP == 1) {
        // lane t: blocks 2t, 2t+1 (16 bytes, one swizzled chunk); MMA i takes pair i of both
        const int off = ((4 * kh + t) ^ pr) << 4;
        const uint4 cA = sld<uint4>(rowA + off), cB = sld<uint4>(rowB + off);
        const unsigned wA[4] = {cA.x, cA.y, cA.z, cA.w}, wB[4] = {cB.x, cB.y, cB.z, cB.w};
        unsigned iA[4], iB[4];
        if constexpr (kSpecial) {
#pragma unroll
            for (int k = 0; k < 4; k++) {
                iA[k] = indicator_codes(wA[k]);
                iB[k] = indicator_codes(wB[k]);
            }
        }
        float dq[4] = {0.f, 0.f, 0.f, 0.f}, di[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const int lo = i >> 2, hi = 2 + (i >> 2), L = i & 3;
            mma_f16(dq, cvt_byte(wA[lo], L), cvt_byte(wB[lo], L), cvt_byte(wA[hi], L), cvt_byte(wB[hi], L), xb0[i], xb1[i]);
            if constexpr (kSpecial)
                mma_f16(di, cvt_byte(iA[lo], L), cvt_byte(iB[lo], L), cvt_byte(iA[hi], L), cvt_byte(iB[hi], L), xb0[i], xb1[i]);
        }
        // scale bytes 2t, 2t+1 of the half: word t >> 1, byte lanes 2(t & 1), +1
        const unsigned wsA = (t >> 1) ? sA.y : sA.x, wsB = (t >> 1) ? sB.y : sB.x;
        const unsigned shA = wsA >> (16 * (t & 1)), shB = wsB >> (16 * (t & 1));
        const float2 e0 = (table_entry(shA, 0, tbl)), e1 = (table_entry(shA, 1, tbl));
        const float2 e2 = (table_entry(shB, 0, tbl)), e3 = (table_entry(shB, 1, tbl));
        acc[0] = fmaf(e0.x, dq[0], acc[0]);
        acc[0] = fmaf(e1.x, dq[1], acc[0]);
        acc[1] = fmaf(e2.x, dq[2], acc[1]);
        acc[1] = fmaf(e3.x, dq[3], acc[1]);
        if constexpr (kSpecial) {
            acc[0] = fmaf(e0.y, di[0], acc[0]);
            acc[0] = fmaf(e1.y, di[1], acc[0]);
            acc[1] = fmaf(e2.y, di[2], acc[1]);
            acc[1] = fmaf(e3.y, di[3], acc[1]);
        }
    } else if constexpr (BP == 2) {
        // group gm (blocks 4gm .. 4gm+3): lane t decodes block 4gm + t (8 bytes);
        // MMA i takes its pairs 2i, 2i+1
#pragma unroll
        for (int gm = 0; gm < 2; gm++) {
            const int off = (((4 * kh + 2 * gm + (t >> 1)) ^ pr) << 4) + 8 * (t & 1);
            const uint2 cA = sld<uint2>(rowA + off), cB = sld<uint2>(rowB + off);
            const unsigned wA[2] = {cA.x, cA.y}, wB[2] = {cB.x, cB.y};
            unsigned iA[2], iB[2];
            if constexpr (kSpecial) {
#pragma unroll
                for (int k = 0; k < 2; k++) {
                    iA[k] = indicator_codes(wA[k]);
                    iB[k] = indicator_codes(wB[k]);
                }
            }
            float dq[4] = {0.f, 0.f, 0.f, 0.f}, di[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const int w = i >> 1, L0 = 2 * (i & 1), L1 = L0 + 1;
                mma_f16(dq, cvt_byte(wA[w], L0), cvt_byte(wB[w], L0), cvt_byte(wA[w], L1), cvt_byte(wB[w], L1), xb0[4 * gm + i],
                        xb1[4 * gm + i]);
                if constexpr (kSpecial)
                    mma_f16(di, cvt_byte(iA[w], L0), cvt_byte(iB[w], L0), cvt_byte(iA[w], L1), cvt_byte(iB[w], L1), xb0[4 * gm + i],
                            xb1[4 * gm + i]);
            }
            // scale byte 4gm + t of the half: word gm, byte lane t
            const unsigned wsA = gm ? sA.y : sA.x, wsB = gm ? sB.y : sB.x;
            const unsigned shA = wsA >> (8 * t), shB = wsB >> (8 * t);
            const float2 ea = (table_entry(shA, 0, tbl)), eb = (table_entry(shB, 0, tbl));
            // columns 2t, 2t+1 = (block t, batch 0), (block t, batch 1)
            acc[0] = fmaf(ea.x, dq[0], acc[0]);
            acc[1] = fmaf(ea.x, dq[1], acc[1]);
            acc[2] = fmaf(eb.x, dq[2], acc[2]);
            acc[3] = fmaf(eb.x, dq[3], acc[3]);
            if constexpr (kSpecial) {
                acc[0] = fmaf(ea.y, di[0], acc[0]);
                acc[1] = fmaf(ea.y, di[1], acc[1]);
                acc[2] = fmaf(eb.y, di[2], acc[2]);
                acc[3] = fmaf(eb.y, di[3], acc[3]);
            }
        }
    } else {
        // group gm (blocks 2gm, 2gm+1): lane t decodes word t & 1 of block
        // 2gm + (t >> 1); MMA i takes its byte lanes 2i, 2i+1
#pragma unroll
        for (int gm = 0; gm < 4; gm++) {
            const int off = (((4 * kh + gm) ^ pr) << 4) + 4 * t;
            const unsigned wA = sld<unsigned>(rowA + off), wB = sld<unsigned>(rowB + off);
            unsigned iA = 0u, iB = 0u;
            if constexpr (kSpecial) {
                iA = indicator_codes(wA);
                iB = indicator_codes(wB);
            }
            float dq[4] = {0.f, 0.f, 0.f, 0.f}, di[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 2; i++) {
                mma_f16(dq, cvt_byte(wA, 2 * i), cvt_byte(wB, 2 * i), cvt_byte(wA, 2 * i + 1), cvt_byte(wB, 2 * i + 1), xb0[2 * gm + i],
                        xb1[2 * gm + i]);
                if constexpr (kSpecial)
                    mma_f16(di, cvt_byte(iA, 2 * i), cvt_byte(iB, 2 * i), cvt_byte(iA, 2 * i + 1), cvt_byte(iB, 2 * i + 1),
                            xb0[2 * gm + i], xb1[2 * gm + i]);
            }
            // scale byte 2gm + (t >> 1) of the half: word gm >> 1, byte lane 2(gm & 1) + (t >> 1)
            const unsigned wsA = (gm >> 1) ? sA.y : sA.x, wsB = (gm >> 1) ? sB.y : sB.x;
            const int L = 2 * (gm & 1);
            const unsigned shA = wsA >> (8 * (t >> 1)), shB = wsB >> (8 * (t >> 1));
            const float2 ea = (table_entry(shA, L, tbl)), eb = (table_entry(shB, L, tbl));
            // columns 2t, 2t+1 = (block t >> 1, batch 2(t & 1)), (.., batch 2(t & 1) + 1)
            acc[0] = fmaf(ea.x, dq[0], acc[0]);
            acc[1] = fmaf(ea.x, dq[1], acc[1]);
            acc[2] = fmaf(eb.x, dq[2], acc[2]);
            acc[3] = fmaf(eb.x, dq[3], acc[3]);
            if constexpr (kSpecial) {
                acc[0] = fmaf(ea.y, di[0], acc[0]);
                acc[1] = fmaf(ea.y, di[1], acc[1]);
                acc[2] = fmaf(eb.y, di[2], acc[2]);
                acc[3] = fmaf(eb.y, di[3], acc[3]);
            }
        }
    }
}

// The activation operand of one 128-k slice for the block-column MMAs:
// lanes that hold a (block, batch row) column load its values, every other
// lane holds zeros.  xs = shared address of batch row 0 of this k-half.
template <int BP>
__device__ __forceinline__ void bc_activations(const uint8_t *xs, int g, int t, int B, unsigned (&xb0)[16], unsigned (&xb1)[16])
{
#pragma unroll
    for (int i = 0; i < 16; i++) xb0[i] = xb1[i] = 0u;
    if constexpr (BP == 1) {
        // column g = block g: kk-pair t is block 2t, kk-pair t+4 block 2t+1
        if (t == (g >> 1)) {
            const uint4 v0 = sld<uint4>(xs + 32 * g), v1 = sld<uint4>(xs + 32 * g + 16);
            const unsigned xr[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
            for (int i = 0; i < 8; i++) {
                if (g & 1) xb1[i] = xr[i];
                else xb0[i] = xr[i];
            }
        }
    } else if constexpr (BP == 2) {
        // column g = (block g >> 1 of the group, batch row g & 1)
        const int b = g & 1;
        if (t == (g >> 1) && b < B) {
#pragma unroll
            for (int gm = 0; gm < 2; gm++) {
                const uint8_t *a = xs + 512 * b + 32 * (4 * gm + t);
                const uint4 v0 = sld<uint4>(a), v1 = sld<uint4>(a + 16);
                const unsigned xr[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    xb0[4 * gm + i] = xr[2 * i];
                    xb1[4 * gm + i] = xr[2 * i + 1];
                }
            }
        }
    } else {
        // column g = (block g >> 2 of the group, batch row g & 3)
        const int b = g & 3;
        if ((t >> 1) == (g >> 2) && b < B) {
#pragma unroll
            for (int gm = 0; gm < 4; gm++) {
                const uint4 v = sld<uint4>(xs + 512 * b + 32 * (2 * gm + (t >> 1)) + 16 * (t & 1));
                xb0[2 * gm] = v.x;
                xb1[2 * gm] = v.y;
                xb0[2 * gm + 1] = v.z;
                xb1[2 * gm + 1] = v.w;
            }
        }
    }
}

// BP = 0: the per-element decode of the split-K kernel (scale and special
// value folded into the MMA operand; every B <= 32, fp16 or bf16).
// BP = 1, 2, 4: the block-column decode above (B <= BP, fp16).
template <int FMT, bool BF16, int NB, int BP, int MT>
__global__ void __launch_bounds__(cta_threads(MT), 1)
    gemv_tma_kernel(const __grid_constant__ Batch A, int U, int stages, int stage_sz, int slot_elems, float *__restrict__ ws,
                    float unbias, int out_dt, int inject_stall)
{
    constexpr int kConsumerWarps = consumer_warps(MT);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 2047) & ~uintptr_t(2047));
    float2 *table = reinterpret_cast<float2 *>(base);
    uint8_t *smem = base + kTableBytes;
    const BatchInfo &I = A.info;
    float *part = reinterpret_cast<float *>(smem + stages * stage_sz);  // [2 buffers][2 k-halves][Bmax][128]
    uint8_t *bars = smem + stages * stage_sz + 2 * 2 * slot_elems * 4;
    const uint32_t full = smem_addr(bars), empty = full + 8 * kMaxStages;
    const uint32_t pfull = empty + 8 * kMaxStages, pempty = pfull + 16;
    volatile int *flags = reinterpret_cast<volatile int *>(bars + 16 * kMaxStages + 32);  // [0] abort
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, c = blockIdx.x;
    const int p_begin = range_start(c, U, G), p_end = range_start(c + 1, U, G);

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; s++) {
            mbar_init(full + 8 * s, 1);
            mbar_init(empty + 8 * s, kConsumerWarps);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(pfull + 8 * b, kConsumerWarps);
            mbar_init(pempty + 8 * b, 1);
        }
        flags[0] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if constexpr (BP > 0) {
        // (s, v * s) of every scale byte: exact binary32 values
        if (threadIdx.x < 256) {
            const unsigned code = threadIdx.x;
            const float s = decode_scale<FMT>(code);
            float vs = 0.0f;
            if constexpr (Fmt<FMT>::kSpecials > 0) vs = special_value((int)(code >> Fmt<FMT>::kMetaShift)) * s;
            table[code] = make_float2(s, vs);
        }
    }
    __syncthreads();
    // the reduction kernel may be scheduled now (it waits for this grid to finish)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == 0) {
        // ------------------------- TMA producer -------------------------
        if (lane == 0) {
            // the tensor maps are kernel parameters: fetch them while the
            // previous kernel in the stream may still run; its outputs (which
            // may be our inputs) are read only after griddepcontrol.wait
            for (int pi = problem_of(I, p_begin); pi <= problem_of(I, p_end - 1); pi++)
#pragma unroll
                for (int m = 0; m < 3; m++) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&A.map[pi][m])) : "memory");
            asm volatile("griddepcontrol.wait;" ::: "memory");
            int s = 0, issued = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int p = p_begin; p < p_end && ok;) {
                const int pi = problem_of(I, p), UK2 = I.UK2[pi], u0 = I.unit0[pi];
                const int r = (p - u0) / UK2;
                const int pe = min(p_end, u0 + (r + 1) * UK2);
                const int h0 = p - u0 - r * UK2, h1 = pe - u0 - r * UK2;
                const uint32_t tx = (uint32_t)(kCodeBytes + kScaleBytes + I.B[pi] * 512);
                const CUtensorMap *tm_codes = &A.map[pi][0], *tm_scales = &A.map[pi][1], *tm_x = &A.map[pi][2];
                for (int j = h0 >> 1; j < (h1 + 1) >> 1; j++) {
                    if (!mbar_wait(empty + 8 * s, ph ^ 1u, flags)) {
                        ok = false;
                        break;
                    }
                    // fault injection (tests only): CTA 0 never fills its second
                    // stage, so its consumers' bounded waits expire
                    if (inject_stall && c == 0 && issued == 1) {
                        inject_stall = 0;
                        issued++;  // the ring position is used (the drain's bounded wait on it expires)
                        if (++s == stages) {
                            s = 0;
                            ph ^= 1u;
                        }
                        continue;
                    }
                    const uint32_t dst = smem_addr(smem + s * stage_sz);
                    mbar_expect_tx(full + 8 * s, tx);
                    tma_load_2d(dst, tm_codes, j * 128, r * kTileRows, full + 8 * s);
                    tma_load_2d(dst + kCodeBytes, tm_scales, j * 16, r * kTileRows, full + 8 * s);
                    tma_load_2d(dst + kCodeBytes + kScaleBytes, tm_x, j * 256, 0, full + 8 * s);
                    issued++;
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                p = pe;
            }
            // the loads issued last into each stage land before this warp (and,
            // on an abort, the CTA) goes away
            for (int i = issued > stages ? issued - stages : 0; i < issued; i++) {
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(full + 8 * (i % stages), (uint32_t)(i / stages) & 1u) && globaltimer() - t0 < kTimeoutNs) {
                }
            }
        }
        return;
    }

    if (warp == 1) {
        // ------------------------- epilogue -------------------------
        asm volatile("griddepcontrol.wait;" ::: "memory");
        int q = 0;
        for (int p = p_begin; p < p_end; q++) {
            const int pi = problem_of(I, p), UK2 = I.UK2[pi], u0 = I.unit0[pi], B = I.B[pi], N = I.N[pi];
            void *y = I.y[pi];
            const float oscale = __fmul_rn(*I.ts[pi], unbias);
            const int r = (p - u0) / UK2;
            const int pe = min(p_end, u0 + (r + 1) * UK2);
            const int buf = q & 1;
            wait_phase(pfull + 8 * buf, (uint32_t)(q >> 1) & 1u, flags);
            const float *h0p = part + buf * 2 * slot_elems, *h1p = h0p + slot_elems;
            const int c_first = range_owner(u0 + r * UK2, U, G), c_last = range_owner(u0 + (r + 1) * UK2 - 1, U, G);
            const int row_base = r * kTileRows;
            // lane owns float4 e4 = lane + 32 i (i < B) of the [B][128] tile
            const float4 *h0v = reinterpret_cast<const float4 *>(h0p), *h1v = reinterpret_cast<const float4 *>(h1p);
            if (c_first == c_last) {
                for (int i = 0; i < B; i++) {
                    const int e4 = lane + 32 * i;
                    const float4 a = h0v[e4], b4 = h1v[e4];
                    const float v[4] = {a.x + b4.x, a.y + b4.y, a.z + b4.z, a.w + b4.w};
                    const int b = e4 >> 5, row = row_base + 4 * (e4 & 31);
#pragma unroll
                    for (int u = 0; u < 4; u++)
                        if (row + u < N) store_out(y, out_dt, (size_t)b * N + row + u, __fmul_rn(v[u], oscale));
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(pempty + 8 * buf);
            } else {
                float4 *slot = reinterpret_cast<float4 *>(ws + (size_t)(c + I.tile0[pi] + r) * slot_elems);
                for (int i = 0; i < B; i++) {
                    const int e4 = lane + 32 * i;
                    const float4 a = h0v[e4], b4 = h1v[e4];
                    slot[e4] = make_float4(a.x + b4.x, a.y + b4.y, a.z + b4.z, a.w + b4.w);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(pempty + 8 * buf);
            }
            p = pe;
        }
        return;
    }

    // ------------------------- consumers -------------------------
    // warp (rg, kh): rows 16 MT rg .. 16 MT (rg + 1) - 1 of the tile, k-half kh
    // of every 256-k stage
    const int cw = warp - kFirstConsumer, rg = cw >> 1, kh = cw & 1, g = lane >> 2, t = lane & 3;
    const uint32_t sbase = smem_addr(smem);
    int s = 0, q = 0;  // ring position of the next stage, hand-over count (no divisions in the loop)
    uint32_t ph = 0;
    uint32_t st = sbase;

    if constexpr (BP > 0) {
        const int pr = bc_row<BP>(g);
        const int R0 = 16 * MT * rg + pr;  // tile row of MMA row g of the first 16-row tile
        const float2 *tbl = table;
        float acc[MT][4];
        unsigned xb0[16], xb1[16];
        const uint8_t *sp = smem;  // generic pointer of the current stage
        for (int p = p_begin; p < p_end; q++) {
            const int pi = problem_of(I, p), UK2 = I.UK2[pi], u0 = I.unit0[pi], B = I.B[pi];
            const int r = (p - u0) / UK2;
            const int pe = min(p_end, u0 + (r + 1) * UK2);
            const int h0 = p - u0 - r * UK2, h1 = pe - u0 - r * UK2;
            const int ja = (h0 - kh + 1) >> 1, jb = (h1 - 1 - kh) >> 1;
#pragma unroll
            for (int m = 0; m < MT; m++) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.0f;

            for (int j = h0 >> 1; j < (h1 + 1) >> 1; j++) {
                wait_phase(full + 8 * s, ph, flags);
                if (j >= ja && j <= jb) {
                    bc_activations<BP>(sp + kCodeBytes + kScaleBytes + 256 * kh, g, t, B, xb0, xb1);
#pragma unroll
                    for (int m = 0; m < MT; m++)
                        bc_tile<FMT, BP>(sp, sp + kCodeBytes, tbl, R0 + 16 * m, pr, kh, t, xb0, xb1, acc[m]);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty + 8 * s);
                sp += stage_sz;
                if (++s == stages) {
                    s = 0;
                    ph ^= 1u;
                    sp = smem;
                }
            }

            // hand the partial of this tile to the epilogue warp and go on
            const int buf = q & 1;
            wait_phase(pempty + 8 * buf, ((uint32_t)(q >> 1) & 1u) ^ 1u, flags);
            float *dst = part + (buf * 2 + kh) * slot_elems;
#pragma unroll
            for (int m = 0; m < MT; m++) {
                const int row = R0 + 16 * m;
                if constexpr (BP == 1) {
                    float a0 = acc[m][0], a1 = acc[m][1];
                    a0 += __shfl_xor_sync(0xffffffffu, a0, 1);
                    a1 += __shfl_xor_sync(0xffffffffu, a1, 1);
                    a0 += __shfl_xor_sync(0xffffffffu, a0, 2);
                    a1 += __shfl_xor_sync(0xffffffffu, a1, 2);
                    if (t == 0) {
                        dst[row] = a0;
                        dst[row + 8] = a1;
                    }
                } else {
                    float a[4] = {acc[m][0], acc[m][1], acc[m][2], acc[m][3]};
#pragma unroll
                    for (int u = 0; u < 4; u++) {
                        if (BP == 2) a[u] += __shfl_xor_sync(0xffffffffu, a[u], 1);
                        a[u] += __shfl_xor_sync(0xffffffffu, a[u], 2);
                    }
                    // BP = 2: lane t = 0 holds batch rows 0, 1; BP = 4: lanes t = 0, 1 hold 2t, 2t+1
                    if ((BP == 2 && t == 0) || (BP == 4 && t < 2)) {
                        const int b0 = BP == 2 ? 0 : 2 * t;
                        if (b0 < B) {
                            dst[b0 * kTileRows + row] = a[0];
                            dst[b0 * kTileRows + row + 8] = a[2];
                        }
                        if (b0 + 1 < B) {
                            dst[(b0 + 1) * kTileRows + row] = a[1];
                            dst[(b0 + 1) * kTileRows + row + 8] = a[3];
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(pfull + 8 * buf);
            p = pe;
        }
        return;
    } else {
        const int pr = tile_row(g);
        const int cc = t + 4 * kh;  // this lane's 16-byte chunk of the 128-byte code row
        const int R0 = 16 * MT * rg + pr;  // tile row of MMA row g of the first 16-row tile
        const uint32_t offA = (uint32_t)(R0 * 128 + ((cc ^ pr) << 4));  // + 1024 for row g + 8, + 2048 per 16-row tile
        const uint32_t offS = (uint32_t)(kCodeBytes + R0 * 16 + 2 * cc);  // + 128 for row g + 8, + 256 per tile
        const uint32_t offX = (uint32_t)(kCodeBytes + kScaleBytes + g * 512 + 64 * cc);

        float acc[MT][NB][4];
        unsigned xw[NB][16];
#pragma unroll
        for (int j = 0; j < NB; j++)
#pragma unroll
            for (int i = 0; i < 16; i++) xw[j][i] = 0u;

        for (int p = p_begin; p < p_end; q++) {
            const int pi = problem_of(I, p), UK2 = I.UK2[pi], u0 = I.unit0[pi], B = I.B[pi];
            const bool xrow = g < B;
            const int r = (p - u0) / UK2;
            const int pe = min(p_end, u0 + (r + 1) * UK2);
            const int h0 = p - u0 - r * UK2, h1 = pe - u0 - r * UK2;
            // stages j whose half-unit 2j + kh lies in [h0, h1)
            const int ja = (h0 - kh + 1) >> 1, jb = (h1 - 1 - kh) >> 1;
#pragma unroll
            for (int m = 0; m < MT; m++)
#pragma unroll
                for (int j = 0; j < NB; j++) acc[m][j][0] = acc[m][j][1] = acc[m][j][2] = acc[m][j][3] = 0.0f;

            for (int j = h0 >> 1; j < (h1 + 1) >> 1; j++) {
                wait_phase(full + 8 * s, ph, flags);
                if (j >= ja && j <= jb) {
                    uint4 ca[MT], cb[MT];
                    unsigned sA[MT], sB[MT];
#pragma unroll
                    for (int m = 0; m < MT; m++) {
                        ca[m] = lds128(st + offA + 2048 * m);
                        cb[m] = lds128(st + offA + 2048 * m + 1024);
                        sA[m] = lds16(st + offS + 256 * m);
                        sB[m] = lds16(st + offS + 256 * m + 128);
                    }
#pragma unroll
                    for (int jj = 0; jj < NB; jj++) {
                        if (8 * jj + g < B && (NB > 1 || xrow)) {
#pragma unroll
                            for (int i = 0; i < 4; i++) {
                                const uint4 v = lds128(st + offX + (uint32_t)(jj * 8 * 512 + 16 * i));
                                xw[jj][4 * i] = v.x;
                                xw[jj][4 * i + 1] = v.y;
                                xw[jj][4 * i + 2] = v.z;
                                xw[jj][4 * i + 3] = v.w;
                            }
                        }
                    }
#pragma unroll
                    for (int m = 0; m < MT; m++) slice_mma<FMT, BF16, NB>(ca[m], cb[m], sA[m], sB[m], xw, acc[m]);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty + 8 * s);
                st += (uint32_t)stage_sz;
                if (++s == stages) {
                    s = 0;
                    ph ^= 1u;
                    st = sbase;
                }
            }

            // hand the partial of this tile to the epilogue warp and go on
            const int buf = q & 1;
            wait_phase(pempty + 8 * buf, ((uint32_t)(q >> 1) & 1u) ^ 1u, flags);
            float *dst = part + (buf * 2 + kh) * slot_elems;
#pragma unroll
            for (int m = 0; m < MT; m++) {
#pragma unroll
                for (int jj = 0; jj < NB; jj++) {
                    const int b0 = 8 * jj + 2 * t;
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        const int b = b0 + (i & 1), row = R0 + 16 * m + ((i & 2) ? 8 : 0);
                        if (b < B) dst[b * kTileRows + row] = acc[m][jj][i];
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(pfull + 8 * buf);
            p = pe;
        }
    }
}

// Sums the workspace slots of the tiles shared by several CTAs, in CTA order.
// Launched as a programmatic dependent of gemv_tma_kernel: it may become
// resident early and waits here until that grid has completed.
__global__ void __launch_bounds__(256) gemv_tma_reduce_kernel(const float *__restrict__ ws, const BatchInfo I, int slot_elems, int U,
                                                              int G, float unbias, int out_dt)
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // the next call may become resident
    const int64_t total = (int64_t)I.tile0[I.count] * slot_elems;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
        const int R = (int)(t / slot_elems), e = (int)(t - (int64_t)R * slot_elems);
        int pi = 0;
        while (pi + 1 < I.count && R >= I.tile0[pi + 1]) pi++;
        const int r = R - I.tile0[pi], UK2 = I.UK2[pi], u0 = I.unit0[pi], N = I.N[pi];
        const int c_first = range_owner(u0 + r * UK2, U, G), c_last = range_owner(u0 + (r + 1) * UK2 - 1, U, G);
        const int row = r * kTileRows + (e & (kTileRows - 1)), b = e >> 7;
        if (c_first == c_last || row >= N || b >= I.B[pi]) continue;  // whole tiles were written by the main kernel
        // slot (cta + global tile) holds that CTA's part of the tile
        const float *src = ws + (size_t)R * slot_elems + e;
        float sum = 0.0f;
        for (int k = c_first; k <= c_last; k++) sum += __ldcg(src + (size_t)k * slot_elems);
        store_out(I.y[pi], out_dt, (size_t)b * N + row, __fmul_rn(sum, __fmul_rn(*I.ts[pi], unbias)));
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
struct Problem {
    const void *x;
    int64_t B;
    const uint8_t *codes, *scales;
    const float *ts;
    int64_t N, K;
    void *y;
};

struct Plan {
    int64_t T, U, G, Bmax;  // tiles, half-units, CTAs, largest batch of the group
    size_t total;           // workspace: one [Bmax][128] fp32 slot per (CTA, tile) pair
};

static Plan plan(const Problem *P, int n)
{
    Plan p = {0, 0, 0, 0, 0};
    for (int i = 0; i < n; i++) {
        const int64_t T = (P[i].N + kTileRows - 1) / kTileRows;
        p.T += T;
        p.U += T * (P[i].K / 128);
        p.Bmax = std::max<int64_t>(p.Bmax, P[i].B);
    }
    p.G = std::min<int64_t>(sm_count(), p.U);
    p.total = (size_t)(p.G + p.T - 1) * (size_t)p.Bmax * kTileRows * sizeof(float);
    return p;
}

// Launch classes: problems of one class share a launch.  With fp16
// activations, B = 1, B = 2 and B = 3..4 take the block-column kernels
// (padded batch 1, 2, 4); every other case takes the per-element decode
// with 1, 2 or 4 n8 MMA tiles (B <= 8, <= 16, <= 32).
enum { kClassBC1 = 0, kClassBC2, kClassBC4, kClassNB1, kClassNB2, kClassNB4, kNumClasses };
static int launch_class(int64_t B, bool bc)
{
    if (bc && B <= 4) return B == 1 ? kClassBC1 : (B == 2 ? kClassBC2 : kClassBC4);
    return B <= 8 ? kClassNB1 : (B <= 16 ? kClassNB2 : kClassNB4);
}

template <int FMT, bool BF16, int NB, int BP, int MT>
static razer_status launch(const Batch &A, const Plan &pl, float *ws, float unbias, razer_dtype out_dt, cudaStream_t st)
{
    const int Bmax = (int)pl.Bmax;
    const int stages = num_stages(Bmax), sz = stage_bytes(Bmax), smem = smem_bytes(Bmax), slot_elems = Bmax * kTileRows;
    static bool attr_done[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(gemv_tma_kernel<FMT, BF16, NB, BP, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) !=
            cudaSuccess)
            return RAZER_ERR_CUDA;
        attr_done[dev] = true;
    }
    const int U = (int)pl.U, G = (int)pl.G;
    // fault injection (tests only): one stage is never filled, so the
    // kernel's bounded waits expire (RAZER_ERR_TIMEOUT)
    const int inject = fault_injection_enabled() ? 1 : 0;
    if (launch_pdl(gemv_tma_kernel<FMT, BF16, NB, BP, MT>, (unsigned)G, (unsigned)cta_threads(MT), (size_t)smem, st, A, U, stages, sz,
                   slot_elems, ws, unbias, (int)out_dt, inject) != cudaSuccess)
        return RAZER_ERR_CUDA;
    // tiles shared by several CTAs exist unless every CTA range is whole tiles
    const BatchInfo &I = A.info;
    bool shared = false;
    for (int pi = 0; pi < I.count && !shared; pi++)
        for (int r = 0; r < I.tile0[pi + 1] - I.tile0[pi] && !shared; r++)
            shared = range_owner(I.unit0[pi] + r * I.UK2[pi], U, G) != range_owner(I.unit0[pi] + (r + 1) * I.UK2[pi] - 1, U, G);
    if (!shared) return RAZER_OK;
    const int64_t total = pl.T * slot_elems;
    const unsigned rgrid = (unsigned)std::min<int64_t>((total + 255) / 256, (int64_t)sm_count() * 4);
    if (launch_pdl(gemv_tma_reduce_kernel, rgrid, 256u, 0, st, (const float *)ws, I, slot_elems, U, G, unbias, (int)out_dt) != cudaSuccess)
        return RAZER_ERR_CUDA;
    return RAZER_OK;
}

#ifndef RAZER_GEMV_BC_MT
#define RAZER_GEMV_BC_MT 2
#endif
constexpr int kLegacyMT = 2;             // per-element decode: 2 row tiles per consumer warp
constexpr int kBcMT = RAZER_GEMV_BC_MT;  // block-column decode

template <int FMT, bool BF16>
static razer_status launch_class_fmt(int cls, const Batch &A, const Plan &pl, float *ws, razer_format wfmt, razer_dtype out_dt,
                                     cudaStream_t st)
{
    // the per-element decode carries q*s*2^-bias; the block-column one exact s
    const float unbias = wfmt == RAZER_FMT_WEIGHT ? scale_f16_unbias<RAZER_FMT_WEIGHT>() : scale_f16_unbias<RAZER_FMT_ACT>();
    if constexpr (!BF16) {
        if (cls == kClassBC1) return launch<FMT, false, 1, 1, kBcMT>(A, pl, ws, 1.0f, out_dt, st);
        if (cls == kClassBC2) return launch<FMT, false, 1, 2, kBcMT>(A, pl, ws, 1.0f, out_dt, st);
        if (cls == kClassBC4) return launch<FMT, false, 1, 4, kBcMT>(A, pl, ws, 1.0f, out_dt, st);
    }
    if (cls == kClassNB1) return launch<FMT, BF16, 1, 0, kLegacyMT>(A, pl, ws, unbias, out_dt, st);
    if (cls == kClassNB2) return launch<FMT, BF16, 2, 0, kLegacyMT>(A, pl, ws, unbias, out_dt, st);
    if (cls == kClassNB4) return launch<FMT, BF16, 4, 0, kLegacyMT>(A, pl, ws, unbias, out_dt, st);
    return RAZER_ERR_UNSUPPORTED;
}

// The three tensor maps of one problem: codes [N, K/2] u8 in 128 x 128-byte
// boxes (128-byte swizzle), scales [N, K/16] u8 in 128 x 16-byte boxes, x
// [B, K] 16-bit in B x 256 boxes.
static bool encode_problem(EncodeTiledFn enc, const Problem &P, CUtensorMap *m)
{
    const cuuint32_t estr[2] = {1u, 1u};
    {
        const cuuint64_t dims[2] = {(cuuint64_t)(P.K / 2), (cuuint64_t)P.N};
        const cuuint64_t strides[1] = {(cuuint64_t)(P.K / 2)};
        const cuuint32_t box[2] = {128u, (cuuint32_t)kTileRows};
        if (enc(&m[0], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(P.codes), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)(P.K / 16), (cuuint64_t)P.N};
        const cuuint64_t strides[1] = {(cuuint64_t)(P.K / 16)};
        const cuuint32_t box[2] = {16u, (cuuint32_t)kTileRows};
        if (enc(&m[1], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(P.scales), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)P.K, (cuuint64_t)P.B};
        const cuuint64_t strides[1] = {(cuuint64_t)P.K * 2};
        const cuuint32_t box[2] = {256u, (cuuint32_t)P.B};
        if (enc(&m[2], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void *>(P.x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    return true;
}

// Calls fn(class, group, n) for the launches of a batch: problems of the
// same launch class, in their order, at most kMaxProblems per launch.
template <typename Fn> static razer_status for_each_group(const Problem *P, int n, bool bc, Fn fn)
{
    for (int cls = 0; cls < kNumClasses; cls++) {
        Problem g[kMaxProblems];
        int k = 0;
        for (int i = 0; i <= n; i++) {
            if (i < n && launch_class(P[i].B, bc) == cls) g[k++] = P[i];
            if (k > 0 && (k == kMaxProblems || i == n)) {
                const razer_status r = fn(cls, g, k);
                if (r != RAZER_OK) return r;
                k = 0;
            }
        }
    }
    return RAZER_OK;
}

}  // namespace gemv_tma

bool gemv_tma_eligible(int64_t B, int64_t N, int64_t K)
{
    // half-unit indices are 32-bit
    return B >= 1 && B <= 32 && N >= 1 && K >= 256 && K % 256 == 0 && ((N + 127) / 128) * (K / 128) < (int64_t)INT32_MAX;
}

size_t gemv_tma_batch_workspace_bytes(const gemv_tma::Problem *P, int n)
{
    // the grouping depends on the activation type: size for both
    size_t need = 0;
    for (int bc = 0; bc < 2; bc++)
        gemv_tma::for_each_group(P, n, bc != 0, [&](int, const gemv_tma::Problem *g, int k) {
            need = std::max(need, gemv_tma::plan(g, k).total);
            return RAZER_OK;
        });
    return need;
}

size_t gemv_tma_workspace_bytes(int64_t B, int64_t N, int64_t K)
{
    gemv_tma::Problem P = {nullptr, B, nullptr, nullptr, nullptr, N, K, nullptr};
    return gemv_tma_batch_workspace_bytes(&P, 1);
}

// Runs the problems (each gemv_tma_eligible, scales 16-byte aligned) in as few
// launches as their n-tile classes allow; the launches reuse one workspace
// (each waits for its predecessor in the stream before writing it).
razer_status run_gemv_tma_batch(const gemv_tma::Problem *P, int n, razer_dtype act_dt, razer_format wfmt, razer_dtype out_dt,
                                void *workspace, cudaStream_t st)
{
    using namespace gemv_tma;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return RAZER_ERR_CUDA;
    float *ws = reinterpret_cast<float *>(workspace);
    const bool bf = act_dt == RAZER_BF16;
    return for_each_group(P, n, !bf, [&](int cls, const Problem *g, int k) {
        Batch A;
        memset(&A, 0, sizeof(A));
        BatchInfo &I = A.info;
        I.count = k;
        for (int i = 0; i < k; i++) {
            if (!encode_problem(enc, g[i], A.map[i])) return RAZER_ERR_CUDA;
            const int T = (int)((g[i].N + kTileRows - 1) / kTileRows), UK2 = (int)(g[i].K / 128);
            I.B[i] = (int)g[i].B;
            I.N[i] = (int)g[i].N;
            I.UK2[i] = UK2;
            I.unit0[i + 1] = I.unit0[i] + T * UK2;
            I.tile0[i + 1] = I.tile0[i] + T;
            I.ts[i] = g[i].ts;
            I.y[i] = g[i].y;
        }
        const Plan pl = plan(g, k);
        if (wfmt == RAZER_FMT_WEIGHT)
            return bf ? launch_class_fmt<RAZER_FMT_WEIGHT, true>(cls, A, pl, ws, wfmt, out_dt, st)
                      : launch_class_fmt<RAZER_FMT_WEIGHT, false>(cls, A, pl, ws, wfmt, out_dt, st);
        if (wfmt == RAZER_FMT_ACT)
            return bf ? launch_class_fmt<RAZER_FMT_ACT, true>(cls, A, pl, ws, wfmt, out_dt, st)
                      : launch_class_fmt<RAZER_FMT_ACT, false>(cls, A, pl, ws, wfmt, out_dt, st);
        return bf ? launch_class_fmt<RAZER_FMT_NVFP4, true>(cls, A, pl, ws, wfmt, out_dt, st)
                  : launch_class_fmt<RAZER_FMT_NVFP4, false>(cls, A, pl, ws, wfmt, out_dt, st);
    });
}

razer_status run_gemv_tma(const void *x, razer_dtype act_dt, int64_t B, const uint8_t *codes, const uint8_t *scales, const float *ts,
                          razer_format wfmt, int64_t N, int64_t K, void *y, razer_dtype out_dt, void *workspace, cudaStream_t st)
{
    const gemv_tma::Problem P = {x, B, codes, scales, ts, N, K, y};
    return run_gemv_tma_batch(&P, 1, act_dt, wfmt, out_dt, workspace, st);
}

// --- razer_gemv_batch: the bulk-tensor batch for every problem it can take,
// the single-problem path for the rest (after it), empty problems handled
// here.  Arguments were validated by the caller.
static bool batch_tma_ok(const razer_gemv_problem &p)
{
    return p.N > 0 && p.K > 0 && gemv_tma_eligible(p.B, p.N, p.K) && (reinterpret_cast<uintptr_t>(p.scales) & 15) == 0;
}

size_t gemv_batch_workspace_bytes(int count, const razer_gemv_problem *P)
{
    std::vector<gemv_tma::Problem> t;
    size_t other = 0;
    for (int i = 0; i < count; i++) {
        const razer_gemv_problem &p = P[i];
        if (p.N == 0 || p.K == 0) continue;
        if (batch_tma_ok(p)) t.push_back({p.x, p.B, p.codes, p.scales, p.ts, p.N, p.K, p.y});
        else other = std::max(other, gemv_workspace_bytes(p.B, p.N, p.K));
    }
    return std::max(other, t.empty() ? (size_t)0 : gemv_tma_batch_workspace_bytes(t.data(), (int)t.size()));
}

razer_status run_gemv_batch(int count, const razer_gemv_problem *P, razer_dtype act_dt, razer_format wfmt, razer_dtype out_dt,
                            void *workspace, cudaStream_t st)
{
    std::vector<gemv_tma::Problem> t;
    for (int i = 0; i < count; i++) {
        const razer_gemv_problem &p = P[i];
        if (p.N > 0 && p.K > 0 && batch_tma_ok(p)) t.push_back({p.x, p.B, p.codes, p.scales, p.ts, p.N, p.K, p.y});
    }
    if (!t.empty()) {
        const razer_status r = run_gemv_tma_batch(t.data(), (int)t.size(), act_dt, wfmt, out_dt, workspace, st);
        if (r != RAZER_OK) return r;
    }
    for (int i = 0; i < count; i++) {
        const razer_gemv_problem &p = P[i];
        if (p.N == 0) continue;
        if (p.K == 0) {  // empty sums: y = 0
            if (cudaMemsetAsync(p.y, 0, (size_t)p.B * (size_t)p.N * (out_dt == RAZER_F32 ? 4 : 2), st) != cudaSuccess) return RAZER_ERR_CUDA;
            continue;
        }
        if (batch_tma_ok(p)) continue;
        const razer_status r = run_gemv(p.x, act_dt, p.B, p.codes, p.scales, p.ts, wfmt, p.N, p.K, p.y, out_dt, workspace, st);
        if (r != RAZER_OK) return r;
    }
    return RAZER_OK;
}

}  // namespace razer
