// razer_gemv_noalloc: the GEMV with its split-K scratch in a fixed,
// library-owned device array instead of a caller-provided workspace.
//
// For callers that cannot allocate device memory at all -- for example a
// runtime that hands every byte of the GPU to its own pool up front, or code
// running under a fixed static memory budget -- and so cannot provide the
// workspace that razer_gemv requires.
//
// The scratch is one file-scope array of kGemvNoAllocScratchBytes bytes.
// Every GPU that loads this library holds it until the process exits.  All
// calls on a device share it and it keeps the previous call's contents; the
// GEMV writes every partial it later reads, so nothing needs clearing, but
// two calls whose kernels overlap on the GPU (different streams, no ordering)
// race on it.
#include <cuda.h>

#include <mutex>

#include "razer_internal.cuh"

namespace razer {

constexpr size_t kGemvNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB

static __device__ __align__(256) unsigned char g_gemv_noalloc_scratch[kGemvNoAllocScratchBytes];

size_t gemv_workspace_bytes(int64_t B, int64_t N, int64_t K);
razer_status run_gemv(const void *x, razer_dtype act_dt, int64_t B, const uint8_t *codes, const uint8_t *scales, const float *ts,
                      razer_format wfmt, int64_t N, int64_t K, void *y, razer_dtype out_dt, void *workspace, cudaStream_t st);

// Device address of the scratch array: looked up with the device current
// (host code cannot use the array's name as an address) and cached per
// device together with the id of the CUDA context it belongs to.  A new
// context on the device (e.g. after cudaDeviceReset) reloads the module, so
// the address is looked up again; the mutex makes the cache safe to use from
// several host threads.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

static unsigned long long current_context_id()
{
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

static void *noalloc_scratch_ptr()
{
    struct Slot {
        unsigned long long ctx;
        void *ptr;
    };
    static Slot slots[64] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    const unsigned long long ctx = current_context_id();
    if (slots[dev].ptr && ctx != 0 && slots[dev].ctx == ctx) return slots[dev].ptr;
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_gemv_noalloc_scratch) != cudaSuccess) return nullptr;
    slots[dev].ptr = p;
    slots[dev].ctx = current_context_id();  // the lookup made the device's context current
    return p;
}

}  // namespace razer

extern "C" size_t razer_gemv_noalloc_max_scratch(void) { return razer::kGemvNoAllocScratchBytes; }

extern "C" razer_status razer_gemv_noalloc(const void *x, razer_dtype act_dt, int64_t B, const uint8_t *codes,
                                           const uint8_t *scales, const float *ts, razer_format wfmt, int64_t N, int64_t K,
                                           void *y, razer_dtype out_dt, razer_stream_t stream)
{
    using namespace razer;
    // the same checks, in the same order, as razer_gemv
    if (!ts || (!x && K > 0) || (!y && N > 0)) return RAZER_ERR_INVALID_ARG;
    if (wfmt != RAZER_FMT_WEIGHT && wfmt != RAZER_FMT_ACT && wfmt != RAZER_FMT_NVFP4) return RAZER_ERR_INVALID_ARG;
    if (act_dt != RAZER_F16 && act_dt != RAZER_BF16 && act_dt != RAZER_F32) return RAZER_ERR_INVALID_ARG;
    if (out_dt != RAZER_F16 && out_dt != RAZER_BF16 && out_dt != RAZER_F32) return RAZER_ERR_INVALID_ARG;
    if (act_dt == RAZER_F32) return RAZER_ERR_DTYPE;
    if (N < 0 || K < 0 || K % 16 != 0) return RAZER_ERR_SHAPE;
    if (N * K > 0) {
        if (!codes || !scales) return RAZER_ERR_INVALID_ARG;
        if (reinterpret_cast<uintptr_t>(codes) % 16 || reinterpret_cast<uintptr_t>(scales) % 4) return RAZER_ERR_ALIGN;
    }
    if (B < 1 || B > 32 || N > INT32_MAX || K > INT32_MAX) return RAZER_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) % 16 || reinterpret_cast<uintptr_t>(ts) % 4)
        return RAZER_ERR_ALIGN;
    if (N == 0) return RAZER_OK;
    if (K == 0)  // empty sums: y = 0
        return cudaMemsetAsync(y, 0, (size_t)B * (size_t)N * (out_dt == RAZER_F32 ? 4 : 2), (cudaStream_t)stream) == cudaSuccess
                   ? RAZER_OK
                   : RAZER_ERR_CUDA;
    if (gemv_workspace_bytes(B, N, K) > kGemvNoAllocScratchBytes) return RAZER_ERR_WORKSPACE;
    void *scratch = noalloc_scratch_ptr();
    if (!scratch) return RAZER_ERR_CUDA;
    return run_gemv(x, act_dt, B, codes, scales, ts, wfmt, N, K, y, out_dt, scratch, (cudaStream_t)stream);
}
