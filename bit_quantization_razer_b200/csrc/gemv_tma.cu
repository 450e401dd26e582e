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
constexpr int kFirstConsumer = 2;  // warp 0: TMA producer, warp 1: epilogue
// Consumer layout per n8 activation tile count NB: B <= 8 (NB = 1) runs 16
// consumer warps of one 16-row MMA tile each (more warps to hide the decode's
// latencies: the three 8B projections at B = 1 / 4 took 30.3 / 32.3 us
// against 32.0 / 34.1 us with 8 warps); larger B runs 8 warps of two tiles
// that share the activation fragments (16 warps: 51.8 against 46.8 us at
// B = 16, and spills at B = 32).
template <int NB> struct Cfg {
    static constexpr int MT = NB == 1 ? 1 : 2;                   // 16-row MMA tiles per consumer warp
    static constexpr int RowGroups = kTileRows / (16 * MT);      // consumer warps per k-half
    static constexpr int ConsumerWarps = 2 * RowGroups;          // one per (row group, 128-k half of a stage)
    static constexpr int Threads = 32 * (kFirstConsumer + ConsumerWarps);
};
constexpr int kCodeBytes = kTileRows * 128;         // 128 rows x 256 codes
constexpr int kScaleBytes = kTileRows * 16;         // 128 rows x 16 blocks
constexpr int kMaxStages = 8;
constexpr int kBarBytes = 256;
constexpr int kSmemLimit = 227 * 1024;

__host__ __device__ constexpr int stage_bytes(int B) { return (kCodeBytes + kScaleBytes + B * 512 + 1023) / 1024 * 1024; }
// two hand-over buffers of [k-half][B][128 rows] fp32 partials
__host__ __device__ constexpr int part_bytes(int B) { return 2 * 2 * B * kTileRows * 4; }
__host__ __device__ constexpr int num_stages(int B)
{
    return (kSmemLimit - 1024 - kBarBytes - part_bytes(B)) / stage_bytes(B) > kMaxStages
               ? kMaxStages
               : (kSmemLimit - 1024 - kBarBytes - part_bytes(B)) / stage_bytes(B);
}
__host__ __device__ constexpr int smem_bytes(int B) { return num_stages(B) * stage_bytes(B) + part_bytes(B) + kBarBytes + 1024; }

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

template <int FMT, bool BF16, int NB>
__global__ void __launch_bounds__(Cfg<NB>::Threads, 1)
    gemv_tma_kernel(const __grid_constant__ Batch A, int U, int stages, int stage_sz, int slot_elems, float *__restrict__ ws,
                    float unbias, int out_dt, int inject_stall)
{
    constexpr int kMT = Cfg<NB>::MT, kConsumerWarps = Cfg<NB>::ConsumerWarps;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
    // warp (rg, kh): rows 16 kMT rg .. 16 kMT (rg + 1) - 1 of the tile, k-half kh
    // of every 256-k stage
    const int cw = warp - kFirstConsumer, rg = cw >> 1, kh = cw & 1, g = lane >> 2, t = lane & 3;
    const int pr = tile_row(g);
    const int cc = t + 4 * kh;  // this lane's 16-byte chunk of the 128-byte code row
    const int R0 = 16 * kMT * rg + pr;  // tile row of MMA row g of the first 16-row tile
    const uint32_t sbase = smem_addr(smem);
    const uint32_t offA = (uint32_t)(R0 * 128 + ((cc ^ pr) << 4));  // + 1024 for row g + 8, + 2048 per 16-row tile
    const uint32_t offS = (uint32_t)(kCodeBytes + R0 * 16 + 2 * cc);  // + 128 for row g + 8, + 256 per tile
    const uint32_t offX = (uint32_t)(kCodeBytes + kScaleBytes + g * 512 + 64 * cc);

    float acc[kMT][NB][4];
    unsigned xw[NB][16];
#pragma unroll
    for (int j = 0; j < NB; j++)
#pragma unroll
        for (int i = 0; i < 16; i++) xw[j][i] = 0u;

    int s = 0, q = 0;  // ring position of the next stage, hand-over count (no divisions in the loop)
    uint32_t ph = 0;
    uint32_t st = sbase;
    for (int p = p_begin; p < p_end; q++) {
        const int pi = problem_of(I, p), UK2 = I.UK2[pi], u0 = I.unit0[pi], B = I.B[pi];
        const bool xrow = g < B;
        const int r = (p - u0) / UK2;
        const int pe = min(p_end, u0 + (r + 1) * UK2);
        const int h0 = p - u0 - r * UK2, h1 = pe - u0 - r * UK2;
        // stages j whose half-unit 2j + kh lies in [h0, h1)
        const int ja = (h0 - kh + 1) >> 1, jb = (h1 - 1 - kh) >> 1;
#pragma unroll
        for (int m = 0; m < kMT; m++)
#pragma unroll
            for (int j = 0; j < NB; j++) acc[m][j][0] = acc[m][j][1] = acc[m][j][2] = acc[m][j][3] = 0.0f;

        for (int j = h0 >> 1; j < (h1 + 1) >> 1; j++) {
            wait_phase(full + 8 * s, ph, flags);
            if (j >= ja && j <= jb) {
                uint4 ca[kMT], cb[kMT];
                unsigned sA[kMT], sB[kMT];
#pragma unroll
                for (int m = 0; m < kMT; m++) {
                    ca[m] = lds128(st + offA + 2048 * m);
                    cb[m] = lds128(st + offA + 2048 * m + 1024);
                    sA[m] = lds16(st + offS + 256 * m);
                    sB[m] = lds16(st + offS + 256 * m + 128);
                }
                {
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
                    for (int m = 0; m < kMT; m++) slice_mma<FMT, BF16, NB>(ca[m], cb[m], sA[m], sB[m], xw, acc[m]);
                }
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
        for (int m = 0; m < kMT; m++) {
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

// Sums the workspace slots of the tiles shared by several CTAs, in CTA order.
// Launched as a programmatic dependent of gemv_tma_kernel: it may become
// resident early and waits here until that grid has completed.
__global__ void __launch_bounds__(kTileRows) gemv_tma_reduce_kernel(const float *__restrict__ ws, const BatchInfo I, int slot_elems, int U,
                                                                    int G, float unbias, int out_dt)
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // the next call may become resident
    // CTA R: global tile R (thread = tile row); its contributing CTAs are
    // found once per tile, and whole tiles were written by the main kernel
    const int R = blockIdx.x;
    int pi = 0;
    while (pi + 1 < I.count && R >= I.tile0[pi + 1]) pi++;
    const int r = R - I.tile0[pi], UK2 = I.UK2[pi], u0 = I.unit0[pi], N = I.N[pi], B = I.B[pi];
    const int c_first = range_owner(u0 + r * UK2, U, G), c_last = range_owner(u0 + (r + 1) * UK2 - 1, U, G);
    const int row = r * kTileRows + threadIdx.x;
    if (c_first == c_last || row >= N) return;
    const float oscale = __fmul_rn(*I.ts[pi], unbias);
    for (int b = 0; b < B; b++) {
        // slot (cta + global tile) holds that CTA's part of the tile; the slots
        // are loaded eight at a time (independent loads) and added in CTA order
        const float *src = ws + (size_t)R * slot_elems + b * kTileRows + threadIdx.x;
        float sum = 0.0f;
        for (int k0 = c_first; k0 <= c_last; k0 += 8) {
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; i++) v[i] = k0 + i <= c_last ? __ldcg(src + (size_t)(k0 + i) * slot_elems) : 0.0f;
#pragma unroll
            for (int i = 0; i < 8; i++)
                if (k0 + i <= c_last) sum += v[i];
        }
        store_out(I.y[pi], out_dt, (size_t)b * N + row, __fmul_rn(sum, oscale));
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

// n-tiles of 8 columns the MMA needs for batch B
static int nb_class(int64_t B) { return B <= 8 ? 1 : (B <= 16 ? 2 : 4); }

template <int FMT, bool BF16, int NB>
static razer_status launch(const Batch &A, const Plan &pl, float *ws, float unbias, razer_dtype out_dt, cudaStream_t st)
{
    const int Bmax = (int)pl.Bmax;
    const int stages = num_stages(Bmax), sz = stage_bytes(Bmax), smem = smem_bytes(Bmax), slot_elems = Bmax * kTileRows;
    static bool attr_done[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(gemv_tma_kernel<FMT, BF16, NB>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) != cudaSuccess)
            return RAZER_ERR_CUDA;
        attr_done[dev] = true;
    }
    const int U = (int)pl.U, G = (int)pl.G;
    // fault injection (tests only): one stage is never filled, so the
    // kernel's bounded waits expire (RAZER_ERR_TIMEOUT)
    const int inject = fault_injection_enabled() ? 1 : 0;
    if (launch_pdl(gemv_tma_kernel<FMT, BF16, NB>, (unsigned)G, (unsigned)Cfg<NB>::Threads, (size_t)smem, st, A, U, stages, sz, slot_elems, ws, unbias,
                   (int)out_dt, inject) != cudaSuccess)
        return RAZER_ERR_CUDA;
    // tiles shared by several CTAs exist unless every CTA range is whole tiles
    const BatchInfo &I = A.info;
    bool shared = false;
    for (int pi = 0; pi < I.count && !shared; pi++)
        for (int r = 0; r < I.tile0[pi + 1] - I.tile0[pi] && !shared; r++)
            shared = range_owner(I.unit0[pi] + r * I.UK2[pi], U, G) != range_owner(I.unit0[pi] + (r + 1) * I.UK2[pi] - 1, U, G);
    if (!shared) return RAZER_OK;
    if (launch_pdl(gemv_tma_reduce_kernel, (unsigned)pl.T, (unsigned)kTileRows, 0, st, (const float *)ws, I, slot_elems, U, G, unbias,
                   (int)out_dt) != cudaSuccess)
        return RAZER_ERR_CUDA;
    return RAZER_OK;
}

template <int FMT, bool BF16>
static razer_status launch_nb(int nb, const Batch &A, const Plan &pl, float *ws, float unbias, razer_dtype out_dt, cudaStream_t st)
{
    if (nb == 1) return launch<FMT, BF16, 1>(A, pl, ws, unbias, out_dt, st);
    if (nb == 2) return launch<FMT, BF16, 2>(A, pl, ws, unbias, out_dt, st);
    return launch<FMT, BF16, 4>(A, pl, ws, unbias, out_dt, st);
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

// Calls fn(group, n) for the launches of a batch: problems of the same
// n-tile class, in their order, at most kMaxProblems per launch.
template <typename Fn> static razer_status for_each_group(const Problem *P, int n, Fn fn)
{
    for (int nb = 1; nb <= 4; nb *= 2) {
        Problem g[kMaxProblems];
        int k = 0;
        for (int i = 0; i <= n; i++) {
            if (i < n && nb_class(P[i].B) == nb) g[k++] = P[i];
            if (k > 0 && (k == kMaxProblems || i == n)) {
                const razer_status r = fn(nb, g, k);
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
    size_t need = 0;
    gemv_tma::for_each_group(P, n, [&](int, const gemv_tma::Problem *g, int k) {
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
    const float unbias = wfmt == RAZER_FMT_WEIGHT ? scale_f16_unbias<RAZER_FMT_WEIGHT>() : scale_f16_unbias<RAZER_FMT_ACT>();
    const bool bf = act_dt == RAZER_BF16;
    return for_each_group(P, n, [&](int nb, const Problem *g, int k) {
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
            return bf ? launch_nb<RAZER_FMT_WEIGHT, true>(nb, A, pl, ws, unbias, out_dt, st)
                      : launch_nb<RAZER_FMT_WEIGHT, false>(nb, A, pl, ws, unbias, out_dt, st);
        if (wfmt == RAZER_FMT_ACT)
            return bf ? launch_nb<RAZER_FMT_ACT, true>(nb, A, pl, ws, unbias, out_dt, st)
                      : launch_nb<RAZER_FMT_ACT, false>(nb, A, pl, ws, unbias, out_dt, st);
        return bf ? launch_nb<RAZER_FMT_NVFP4, true>(nb, A, pl, ws, unbias, out_dt, st)
                  : launch_nb<RAZER_FMT_NVFP4, false>(nb, A, pl, ws, unbias, out_dt, st);
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
