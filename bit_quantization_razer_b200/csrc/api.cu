// extern "C" surface of the RaZeR library: argument validation, then the
// launches of the kernels in quantize.cu / dequant.cu / gemv.cu / gemm.cu.
// No call allocates memory or synchronises (razer_get_device_status excepted).
#include <atomic>
#include <cmath>
#include <cstdlib>

#include "razer_internal.cuh"
#include "variant.cuh"

namespace razer {

int sm_count()
{
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

razer_status last_launch_status() { return cudaGetLastError() == cudaSuccess ? RAZER_OK : RAZER_ERR_CUDA; }

// Off unless razer_debug_set_fault_injection turns it on; the environment
// variable RAZER_FAULT_INJECT_STALL=1 sets the initial value, read once when
// the library is loaded.
static std::atomic<int> g_fault_injection{[] {
    const char *v = getenv("RAZER_FAULT_INJECT_STALL");
    return (v && v[0] == '1') ? 1 : 0;
}()};
bool fault_injection_enabled() { return g_fault_injection.load(std::memory_order_relaxed) != 0; }

razer_status run_quantize(const void *x, razer_dtype dt, int64_t R, int64_t K, const float *ts_in, uint8_t *codes,
                          uint8_t *scales, float *ts_out, unsigned long long *hist, razer_format fmt, cudaStream_t st);
razer_status run_quantize_46(const void *x, razer_dtype dt, int64_t R, int64_t K, uint8_t *codes, uint8_t *scales, float *ts_out,
                             unsigned long long *n_four, cudaStream_t st);
razer_status run_quant_sse(const void *x, razer_dtype dt, int64_t R, int64_t K, const uint8_t *codes, const uint8_t *scales,
                           const float *ts, razer_format fmt, double *out, cudaStream_t st);
razer_status run_quantize_variant(const void *x, razer_dtype dt, int64_t R, int64_t K, int bs, razer_format sfmt, const VariantV &V,
                                  uint8_t *codes, uint8_t *scales, float *ts_out, cudaStream_t st);
razer_status run_quant_sse_variant(const void *x, razer_dtype dt, int64_t R, int64_t K, int bs, razer_format sfmt, const VariantV &V,
                                   const uint8_t *codes, const uint8_t *scales, const float *ts, double *out, cudaStream_t st);
razer_status run_dequant_variant(const uint8_t *codes, const uint8_t *scales, const float *ts, int64_t R, int64_t K, int bs,
                                 razer_format sfmt, const VariantV &V, void *out, razer_dtype dt, cudaStream_t st);
razer_status run_gemv_variant(const void *x, razer_dtype act_dt, int64_t B, const uint8_t *codes, const uint8_t *scales, const float *ts,
                              int bs, razer_format sfmt, const VariantV &V, int64_t N, int64_t K, void *y, razer_dtype out_dt,
                              void *workspace, cudaStream_t st);
size_t gemv_variant_workspace_bytes(int64_t B, int64_t N, int64_t K);
razer_status run_quantize_batch(int count, const void *const *W, razer_dtype dt, const int64_t *R, const int64_t *K,
                                uint8_t *const *codes, uint8_t *const *scales, float *ts, razer_format fmt, cudaStream_t st);
razer_status run_dequant(const uint8_t *codes, const uint8_t *scales, const float *ts, razer_format fmt, int64_t R, int64_t K,
                         void *out, razer_dtype dt, cudaStream_t st);
razer_status run_gemv(const void *x, razer_dtype act_dt, int64_t B, const uint8_t *codes, const uint8_t *scales, const float *ts,
                      razer_format wfmt, int64_t N, int64_t K, void *y, razer_dtype out_dt, void *workspace, cudaStream_t st);
size_t gemv_workspace_bytes(int64_t B, int64_t N, int64_t K);
razer_status run_gemv_batch(int count, const razer_gemv_problem *P, razer_dtype act_dt, razer_format wfmt, razer_dtype out_dt,
                            void *workspace, cudaStream_t st);
size_t gemv_batch_workspace_bytes(int count, const razer_gemv_problem *P);
razer_status run_gemm(const void *X, razer_dtype act_dt, int64_t M, const uint8_t *codes, const uint8_t *scales, const float *ts,
                      razer_format wfmt, int64_t N, int64_t K, void *Y, razer_dtype out_dt, void *workspace, cudaStream_t st);
size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);
razer_status run_gemm_w4a4(const uint8_t *codes_a, const uint8_t *scales_a, const float *ts_a, razer_format afmt, int64_t M,
                           const uint8_t *codes_w, const uint8_t *scales_w, const float *ts_w, razer_format wfmt, int64_t N, int64_t K,
                           void *Y, razer_dtype out_dt, void *workspace, cudaStream_t st);
size_t gemm_w4a4_workspace_bytes(int64_t M, int64_t N, int64_t K);
size_t gemm_variant_workspace_bytes(int64_t M, int64_t N, int64_t K);
razer_status run_gemm_variant(const void *X, razer_dtype act_dt, int64_t M, const uint8_t *codes, const uint8_t *scales, const float *ts,
                              int block, razer_format sfmt, const VariantV &V, int64_t N, int64_t K, void *Y, razer_dtype out_dt,
                              void *workspace, cudaStream_t st);
razer_status run_gemm_w4a4_online(const void *X, razer_dtype x_dt, int64_t M, const float *ts_in, razer_format afmt, uint8_t *codes_a,
                                  uint8_t *scales_a, float *ts_a_out, unsigned long long *hist, const uint8_t *codes_w,
                                  const uint8_t *scales_w, const float *ts_w, razer_format wfmt, int64_t N, int64_t K, void *Y,
                                  razer_dtype out_dt, void *workspace, cudaStream_t st);

static bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
static bool valid_fmt(int f) { return f == RAZER_FMT_WEIGHT || f == RAZER_FMT_ACT || f == RAZER_FMT_NVFP4; }
static bool valid_dt(int d) { return d == RAZER_F16 || d == RAZER_BF16 || d == RAZER_F32; }
static bool in16(int d) { return d == RAZER_F16 || d == RAZER_BF16; }

// Shared checks of a [R, K] packed tensor.
static razer_status check_packed(const uint8_t *codes, const uint8_t *scales, int64_t R, int64_t K)
{
    if (R < 0 || K < 0 || (K % 16) != 0) return RAZER_ERR_SHAPE;
    if (R * K == 0) return RAZER_OK;  // empty: pointers may be null
    if (!codes || !scales) return RAZER_ERR_INVALID_ARG;
    if (!aligned(codes, 16) || !aligned(scales, 4)) return RAZER_ERR_ALIGN;
    return RAZER_OK;
}

}  // namespace razer

using namespace razer;

extern "C" {

razer_status razer_quantize_weights(const void *W, razer_dtype in_dt, int64_t N, int64_t K, uint8_t *codes, uint8_t *scales,
                                    float *tensor_scale, razer_format fmt, razer_stream_t stream)
{
    if (!tensor_scale || (!W && N * K > 0)) return RAZER_ERR_INVALID_ARG;
    if (fmt != RAZER_FMT_WEIGHT && fmt != RAZER_FMT_NVFP4 && fmt != RAZER_FMT_FOUR_OVER_SIX)
        return valid_fmt(fmt) ? RAZER_ERR_UNSUPPORTED : RAZER_ERR_INVALID_ARG;
    if (!valid_dt(in_dt)) return RAZER_ERR_INVALID_ARG;
    if (!in16(in_dt)) return RAZER_ERR_DTYPE;
    razer_status st = check_packed(codes, scales, N, K);
    if (st != RAZER_OK) return st;
    if (!aligned(W, 16) || !aligned(tensor_scale, 4)) return RAZER_ERR_ALIGN;
    if (fmt == RAZER_FMT_FOUR_OVER_SIX)
        return run_quantize_46(W, in_dt, N, K, codes, scales, tensor_scale, nullptr, (cudaStream_t)stream);
    return run_quantize(W, in_dt, N, K, nullptr, codes, scales, tensor_scale, nullptr, fmt, (cudaStream_t)stream);
}

razer_status razer_quantize_weights_batch(int count, const void *const *W, razer_dtype in_dt, const int64_t *N, const int64_t *K,
                                          uint8_t *const *codes, uint8_t *const *scales, float *tensor_scales, razer_format fmt,
                                          razer_stream_t stream)
{
    if (count < 0) return RAZER_ERR_INVALID_ARG;
    if (count == 0) return RAZER_OK;
    if (!W || !N || !K || !codes || !scales || !tensor_scales) return RAZER_ERR_INVALID_ARG;
    if (fmt != RAZER_FMT_WEIGHT && fmt != RAZER_FMT_NVFP4) return valid_fmt(fmt) ? RAZER_ERR_UNSUPPORTED : RAZER_ERR_INVALID_ARG;
    if (!valid_dt(in_dt)) return RAZER_ERR_INVALID_ARG;
    if (!in16(in_dt)) return RAZER_ERR_DTYPE;
    if (!aligned(tensor_scales, 4)) return RAZER_ERR_ALIGN;
    for (int i = 0; i < count; i++) {
        if (!W[i] && N[i] * K[i] > 0) return RAZER_ERR_INVALID_ARG;
        razer_status st = check_packed(codes[i], scales[i], N[i], K[i]);
        if (st != RAZER_OK) return st;
        if (!aligned(W[i], 16)) return RAZER_ERR_ALIGN;
    }
    return run_quantize_batch(count, W, in_dt, N, K, codes, scales, tensor_scales, fmt, (cudaStream_t)stream);
}

razer_status razer_quantize_acts(const void *X, razer_dtype in_dt, int64_t M, int64_t K, const float *ts_in, uint8_t *codes,
                                 uint8_t *scales, float *ts_out, unsigned long long *meta_hist, razer_format fmt,
                                 razer_stream_t stream)
{
    if (!ts_out || (!X && M * K > 0)) return RAZER_ERR_INVALID_ARG;
    if (fmt != RAZER_FMT_ACT && fmt != RAZER_FMT_NVFP4) return valid_fmt(fmt) ? RAZER_ERR_UNSUPPORTED : RAZER_ERR_INVALID_ARG;
    if (!valid_dt(in_dt)) return RAZER_ERR_INVALID_ARG;
    if (!in16(in_dt)) return RAZER_ERR_DTYPE;
    razer_status st = check_packed(codes, scales, M, K);
    if (st != RAZER_OK) return st;
    if (!aligned(X, 16) || !aligned(ts_out, 4) || (ts_in && !aligned(ts_in, 4)) || (meta_hist && !aligned(meta_hist, 8)))
        return RAZER_ERR_ALIGN;
    return run_quantize(X, in_dt, M, K, ts_in, codes, scales, ts_out, meta_hist, fmt, (cudaStream_t)stream);
}

razer_status razer_dequant(const uint8_t *codes, const uint8_t *scales, const float *ts, razer_format fmt, int64_t R, int64_t K,
                           void *out, razer_dtype out_dt, razer_stream_t stream)
{
    if (!ts || (!out && R * K > 0)) return RAZER_ERR_INVALID_ARG;
    if (!valid_fmt(fmt) || !valid_dt(out_dt)) return RAZER_ERR_INVALID_ARG;
    razer_status st = check_packed(codes, scales, R, K);
    if (st != RAZER_OK) return st;
    if (!aligned(out, 16) || !aligned(ts, 4)) return RAZER_ERR_ALIGN;
    return run_dequant(codes, scales, ts, fmt, R, K, out, out_dt, (cudaStream_t)stream);
}

size_t razer_workspace_size(razer_op op, int64_t M_or_B, int64_t N, int64_t K)
{
    if (op == RAZER_OP_GEMV) return gemv_workspace_bytes(M_or_B, N, K);
    if (op == RAZER_OP_GEMM) return gemm_workspace_bytes(M_or_B, N, K);
    if (op == RAZER_OP_GEMM_W4A4) return M_or_B > 0 && N > 0 && K > 0 ? gemm_w4a4_workspace_bytes(M_or_B, N, K) : 0;
    if (op == RAZER_OP_GEMM_VARIANT) return gemm_variant_workspace_bytes(M_or_B, N, K);
    return 0;
}

razer_status razer_gemv(const void *x, razer_dtype act_dt, int64_t B, const uint8_t *codes, const uint8_t *scales, const float *ts,
                        razer_format wfmt, int64_t N, int64_t K, void *y, razer_dtype out_dt, void *workspace, size_t ws_bytes,
                        razer_stream_t stream)
{
    if (!ts || (!x && K > 0) || (!y && N > 0)) return RAZER_ERR_INVALID_ARG;
    if (!valid_fmt(wfmt) || !valid_dt(act_dt) || !valid_dt(out_dt)) return RAZER_ERR_INVALID_ARG;
    if (!in16(act_dt)) return RAZER_ERR_DTYPE;
    razer_status st = check_packed(codes, scales, N, K);
    if (st != RAZER_OK) return st;
    if (B < 1 || B > 32 || N > INT32_MAX || K > INT32_MAX) return RAZER_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(ts, 4)) return RAZER_ERR_ALIGN;
    if (N == 0) return RAZER_OK;
    if (K == 0)  // empty sums: y = 0
        return cudaMemsetAsync(y, 0, (size_t)B * (size_t)N * (out_dt == RAZER_F32 ? 4 : 2), (cudaStream_t)stream) == cudaSuccess
                   ? RAZER_OK
                   : RAZER_ERR_CUDA;
    const size_t need = gemv_workspace_bytes(B, N, K);
    if (need) {
        if (!workspace || ws_bytes < need) return RAZER_ERR_WORKSPACE;
        if (!aligned(workspace, 16)) return RAZER_ERR_ALIGN;
    }
    return run_gemv(x, act_dt, B, codes, scales, ts, wfmt, N, K, y, out_dt, workspace, (cudaStream_t)stream);
}

size_t razer_gemv_batch_workspace_size(int count, const razer_gemv_problem *problems)
{
    if (count <= 0 || !problems) return 0;
    return gemv_batch_workspace_bytes(count, problems);
}

razer_status razer_gemv_batch(int count, const razer_gemv_problem *problems, razer_dtype act_dt, razer_format wfmt, razer_dtype out_dt,
                              void *workspace, size_t ws_bytes, razer_stream_t stream)
{
    if (count < 0 || (count > 0 && !problems)) return RAZER_ERR_INVALID_ARG;
    if (count == 0) return RAZER_OK;
    if (!valid_fmt(wfmt) || !valid_dt(act_dt) || !valid_dt(out_dt)) return RAZER_ERR_INVALID_ARG;
    if (!in16(act_dt)) return RAZER_ERR_DTYPE;
    for (int i = 0; i < count; i++) {  // each problem as razer_gemv checks its arguments
        const razer_gemv_problem &p = problems[i];
        if (!p.ts || (!p.x && p.K > 0) || (!p.y && p.N > 0)) return RAZER_ERR_INVALID_ARG;
        razer_status st = check_packed(p.codes, p.scales, p.N, p.K);
        if (st != RAZER_OK) return st;
        if (p.B < 1 || p.B > 32 || p.N > INT32_MAX || p.K > INT32_MAX) return RAZER_ERR_SHAPE;
        if (!aligned(p.x, 16) || !aligned(p.y, 16) || !aligned(p.ts, 4)) return RAZER_ERR_ALIGN;
    }
    const size_t need = gemv_batch_workspace_bytes(count, problems);
    if (need) {
        if (!workspace || ws_bytes < need) return RAZER_ERR_WORKSPACE;
        if (!aligned(workspace, 16)) return RAZER_ERR_ALIGN;
    }
    return run_gemv_batch(count, problems, act_dt, wfmt, out_dt, workspace, (cudaStream_t)stream);
}

razer_status razer_gemm(const void *X, razer_dtype act_dt, int64_t M, const uint8_t *codes, const uint8_t *scales, const float *ts,
                        razer_format wfmt, int64_t N, int64_t K, void *Y, razer_dtype out_dt, void *workspace, size_t ws_bytes,
                        razer_stream_t stream)
{
    if (!ts || (!X && M * K > 0) || (!Y && M * N > 0)) return RAZER_ERR_INVALID_ARG;
    if (!valid_fmt(wfmt) || !valid_dt(act_dt) || !valid_dt(out_dt)) return RAZER_ERR_INVALID_ARG;
    if (!in16(act_dt)) return RAZER_ERR_DTYPE;
    razer_status st = check_packed(codes, scales, N, K);
    if (st != RAZER_OK) return st;
    if (M < 0 || M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return RAZER_ERR_SHAPE;
    if (!aligned(X, 16) || !aligned(Y, 16) || !aligned(ts, 4)) return RAZER_ERR_ALIGN;
    if (M == 0 || N == 0) return RAZER_OK;
    const size_t need = gemm_workspace_bytes(M, N, K);
    if (need) {
        if (!workspace || ws_bytes < need) return RAZER_ERR_WORKSPACE;
        if (!aligned(workspace, 16)) return RAZER_ERR_ALIGN;
    }
    return run_gemm(X, act_dt, M, codes, scales, ts, wfmt, N, K, Y, out_dt, workspace, (cudaStream_t)stream);
}

razer_status razer_gemm_w4a4(const uint8_t *codes_a, const uint8_t *scales_a, const float *ts_a, razer_format afmt, int64_t M,
                             const uint8_t *codes_w, const uint8_t *scales_w, const float *ts_w, razer_format wfmt, int64_t N,
                             int64_t K, void *Y, razer_dtype out_dt, void *workspace, size_t ws_bytes, razer_stream_t stream)
{
    if (!ts_a || !ts_w || (!Y && M * N > 0)) return RAZER_ERR_INVALID_ARG;
    if (!valid_fmt(afmt) || !valid_fmt(wfmt) || !valid_dt(out_dt)) return RAZER_ERR_INVALID_ARG;
    razer_status st = check_packed(codes_a, scales_a, M, K);
    if (st != RAZER_OK) return st;
    st = check_packed(codes_w, scales_w, N, K);
    if (st != RAZER_OK) return st;
    if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return RAZER_ERR_SHAPE;
    if (!aligned(Y, 16) || !aligned(ts_a, 4) || !aligned(ts_w, 4)) return RAZER_ERR_ALIGN;
    if (M == 0 || N == 0) return RAZER_OK;
    const size_t need = K > 0 ? gemm_w4a4_workspace_bytes(M, N, K) : 0;
    if (need) {
        if (!workspace || ws_bytes < need) return RAZER_ERR_WORKSPACE;
        if (!aligned(workspace, 16)) return RAZER_ERR_ALIGN;
    }
    return run_gemm_w4a4(codes_a, scales_a, ts_a, afmt, M, codes_w, scales_w, ts_w, wfmt, N, K, Y, out_dt, workspace,
                         (cudaStream_t)stream);
}

razer_status razer_gemm_w4a4_online(const void *X, razer_dtype x_dt, int64_t M, const float *ts_in, razer_format afmt,
                                    uint8_t *codes_a, uint8_t *scales_a, float *ts_a_out, unsigned long long *meta_hist,
                                    const uint8_t *codes_w, const uint8_t *scales_w, const float *ts_w, razer_format wfmt, int64_t N,
                                    int64_t K, void *Y, razer_dtype out_dt, void *workspace, size_t ws_bytes, razer_stream_t stream)
{
    if (!ts_a_out || !ts_w || (!X && M * K > 0) || (!Y && M * N > 0)) return RAZER_ERR_INVALID_ARG;
    if (afmt != RAZER_FMT_ACT && afmt != RAZER_FMT_NVFP4) return valid_fmt(afmt) ? RAZER_ERR_UNSUPPORTED : RAZER_ERR_INVALID_ARG;
    if (!valid_fmt(wfmt) || !valid_dt(x_dt) || !valid_dt(out_dt)) return RAZER_ERR_INVALID_ARG;
    if (!in16(x_dt)) return RAZER_ERR_DTYPE;
    if ((codes_a == nullptr) != (scales_a == nullptr)) return RAZER_ERR_INVALID_ARG;
    razer_status st = codes_a ? check_packed(codes_a, scales_a, M, K) : RAZER_OK;
    if (st != RAZER_OK) return st;
    st = check_packed(codes_w, scales_w, N, K);
    if (st != RAZER_OK) return st;
    if (M < 0 || M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return RAZER_ERR_SHAPE;
    if (!aligned(X, 16) || !aligned(Y, 16) || !aligned(ts_a_out, 4) || !aligned(ts_w, 4) || (ts_in && !aligned(ts_in, 4)) ||
        (meta_hist && !aligned(meta_hist, 8)))
        return RAZER_ERR_ALIGN;
    if (M == 0 || N == 0) return RAZER_OK;
    const size_t need = K > 0 ? gemm_w4a4_workspace_bytes(M, N, K) : 0;
    if (need) {
        if (!workspace || ws_bytes < need) return RAZER_ERR_WORKSPACE;
        if (!aligned(workspace, 16)) return RAZER_ERR_ALIGN;
    }
    return run_gemm_w4a4_online(X, x_dt, M, ts_in, afmt, codes_a, scales_a, ts_a_out, meta_hist, codes_w, scales_w, ts_w, wfmt, N, K, Y,
                                out_dt, workspace, (cudaStream_t)stream);
}

// checks of a format variant; fills V (scale format RAZER_FMT_ACT and NVFP4
// both mean E4M3 with a 1-bit meta)
static razer_status check_variant(int64_t R, int64_t K, int block, razer_format sfmt, const float *vals, int nv, VariantV &V)
{
    if (block != 16 && block != 32 && block != 64 && block != 128) return RAZER_ERR_SHAPE;
    if (R < 0 || K < 0 || K % block != 0) return RAZER_ERR_SHAPE;
    if (!valid_fmt(sfmt) && sfmt != RAZER_SCALE_F16) return RAZER_ERR_INVALID_ARG;
    const int max_nv = (sfmt == RAZER_FMT_WEIGHT || sfmt == RAZER_SCALE_F16) ? 4 : 2;
    if (nv < 0 || nv > max_nv || (nv > 0 && !vals)) return RAZER_ERR_INVALID_ARG;
    V.nv = nv;
    for (int i = 0; i < 4; i++) V.v[i] = 0.0f;
    for (int i = 0; i < nv; i++) {
        const float a = fabsf(vals[i]), h = a * 2.0f;
        // a multiple of 0.5 in [2.5, 9.5], not an E2M1 magnitude (3, 4, 6)
        if (!(a >= 2.5f && a <= 9.5f) || h != floorf(h) || a == 3.0f || a == 4.0f || a == 6.0f) return RAZER_ERR_INVALID_ARG;
        V.v[i] = vals[i];
    }
    return RAZER_OK;
}

razer_status razer_quantize_variant(const void *X, razer_dtype in_dt, int64_t R, int64_t K, int block, razer_format scale_fmt,
                                    const float *special_values, int n_special, uint8_t *codes, uint8_t *scales, float *ts_out,
                                    razer_stream_t stream)
{
    VariantV V;
    razer_status st = check_variant(R, K, block, scale_fmt, special_values, n_special, V);
    if (st != RAZER_OK) return st;
    if (!ts_out || (!X && R * K > 0) || (R * K > 0 && (!codes || !scales))) return RAZER_ERR_INVALID_ARG;
    if (!valid_dt(in_dt)) return RAZER_ERR_INVALID_ARG;
    if (!in16(in_dt)) return RAZER_ERR_DTYPE;
    if (!aligned(X, 16) || !aligned(codes, 16) || !aligned(ts_out, 4) || (scale_fmt == RAZER_SCALE_F16 && !aligned(scales, 2)))
        return RAZER_ERR_ALIGN;
    return run_quantize_variant(X, in_dt, R, K, block, scale_fmt, V, codes, scales, ts_out, (cudaStream_t)stream);
}

razer_status razer_quant_error_variant(const void *X, razer_dtype in_dt, int64_t R, int64_t K, int block, razer_format scale_fmt,
                                       const float *special_values, int n_special, const uint8_t *codes, const uint8_t *scales,
                                       const float *ts, double *sse, razer_stream_t stream)
{
    VariantV V;
    razer_status st = check_variant(R, K, block, scale_fmt, special_values, n_special, V);
    if (st != RAZER_OK) return st;
    if (!ts || !sse || (!X && R * K > 0) || (R * K > 0 && (!codes || !scales))) return RAZER_ERR_INVALID_ARG;
    if (!valid_dt(in_dt)) return RAZER_ERR_INVALID_ARG;
    if (!in16(in_dt)) return RAZER_ERR_DTYPE;
    if (!aligned(X, 16) || !aligned(codes, 8) || !aligned(ts, 4) || !aligned(sse, 8) ||
        (scale_fmt == RAZER_SCALE_F16 && !aligned(scales, 2)))
        return RAZER_ERR_ALIGN;
    return run_quant_sse_variant(X, in_dt, R, K, block, scale_fmt, V, codes, scales, ts, sse, (cudaStream_t)stream);
}

razer_status razer_dequant_variant(const uint8_t *codes, const uint8_t *scales, const float *ts, int64_t R, int64_t K, int block,
                                   razer_format scale_fmt, const float *special_values, int n_special, void *out, razer_dtype out_dt,
                                   razer_stream_t stream)
{
    VariantV V;
    razer_status st = check_variant(R, K, block, scale_fmt, special_values, n_special, V);
    if (st != RAZER_OK) return st;
    if (!ts || (R * K > 0 && (!codes || !scales || !out))) return RAZER_ERR_INVALID_ARG;
    if (!valid_dt(out_dt)) return RAZER_ERR_INVALID_ARG;
    if (!aligned(codes, 8) || !aligned(out, 16) || !aligned(ts, 4) || (scale_fmt == RAZER_SCALE_F16 && !aligned(scales, 2)))
        return RAZER_ERR_ALIGN;
    return run_dequant_variant(codes, scales, ts, R, K, block, scale_fmt, V, out, out_dt, (cudaStream_t)stream);
}

// whether v * s can need more than the 8 significant bits of bf16 for some
// scale: the odd part of 2|v| times every scale significand (1..15, the
// E3M3 / E4M3 mantissa with its leading bit, or a subnormal one) must stay
// below 256.  Of the allowed values only 9.5 (19 * 15 = 285) fails.
static bool rounds_in_bf16(const VariantV &V)
{
    for (int i = 0; i < V.nv; i++) {
        int h = (int)(fabsf(V.v[i]) * 2.0f);
        while (h > 0 && (h & 1) == 0) h >>= 1;
        for (int m = 1; m <= 15; m++) {
            int p = h * m;
            while (p > 0 && (p & 1) == 0) p >>= 1;
            if (p >= 256) return true;
        }
    }
    return false;
}

razer_status razer_gemm_variant(const void *X, razer_dtype act_dt, int64_t M, const uint8_t *codes, const uint8_t *scales, const float *ts,
                                int block, razer_format scale_fmt, const float *special_values, int n_special, int64_t N, int64_t K,
                                void *Y, razer_dtype out_dt, void *workspace, size_t ws_bytes, razer_stream_t stream)
{
    VariantV V;
    razer_status st = check_variant(N, K, block, scale_fmt, special_values, n_special, V);
    if (st != RAZER_OK) return st;
    if (!ts || (!X && M * K > 0) || (!Y && M * N > 0) || (N * K > 0 && (!codes || !scales))) return RAZER_ERR_INVALID_ARG;
    if (!valid_dt(act_dt) || !valid_dt(out_dt)) return RAZER_ERR_INVALID_ARG;
    if (!in16(act_dt)) return RAZER_ERR_DTYPE;
    if (M < 0 || M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return RAZER_ERR_SHAPE;
    // the 16-bit weight copy must hold q*s: bf16 holds it exactly for byte
    // scales without +-9.5 (FP16 scale words take two terms in either type)
    if (act_dt == RAZER_BF16 && scale_fmt != RAZER_SCALE_F16 && rounds_in_bf16(V)) return RAZER_ERR_UNSUPPORTED;
    if (scale_fmt == RAZER_SCALE_F16 && K % 64 != 0) return RAZER_ERR_UNSUPPORTED;  // the two-term copy takes whole k-steps
    if (!aligned(X, 16) || !aligned(Y, 16) || !aligned(ts, 4) || !aligned(codes, 8) || (scale_fmt == RAZER_SCALE_F16 && !aligned(scales, 2)))
        return RAZER_ERR_ALIGN;
    if (M == 0 || N == 0) return RAZER_OK;
    if (K == 0)  // empty sums: Y = 0
        return cudaMemsetAsync(Y, 0, (size_t)M * (size_t)N * (out_dt == RAZER_F32 ? 4 : 2), (cudaStream_t)stream) == cudaSuccess
                   ? RAZER_OK
                   : RAZER_ERR_CUDA;
    const size_t need = gemm_variant_workspace_bytes(M, N, K);
    if (!workspace || ws_bytes < need) return RAZER_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return RAZER_ERR_ALIGN;
    return run_gemm_variant(X, act_dt, M, codes, scales, ts, block, scale_fmt, V, N, K, Y, out_dt, workspace, (cudaStream_t)stream);
}

razer_status razer_gemv_variant(const void *x, razer_dtype act_dt, int64_t B, const uint8_t *codes, const uint8_t *scales, const float *ts,
                                int block, razer_format scale_fmt, const float *special_values, int n_special, int64_t N, int64_t K,
                                void *y, razer_dtype out_dt, void *workspace, size_t ws_bytes, razer_stream_t stream)
{
    VariantV V;
    razer_status st = check_variant(N, K, block, scale_fmt, special_values, n_special, V);
    if (st != RAZER_OK) return st;
    if (!ts || (!x && K > 0) || (!y && N > 0) || (N * K > 0 && (!codes || !scales))) return RAZER_ERR_INVALID_ARG;
    if (!valid_dt(act_dt) || !valid_dt(out_dt)) return RAZER_ERR_INVALID_ARG;
    if (!in16(act_dt)) return RAZER_ERR_DTYPE;
    if (B < 1 || B > 32 || K % 128 != 0 || N > INT32_MAX || K > INT32_MAX) return RAZER_ERR_SHAPE;
    if (scale_fmt == RAZER_SCALE_F16 && block != 128) return RAZER_ERR_UNSUPPORTED;
    if (scale_fmt != RAZER_SCALE_F16 && act_dt == RAZER_BF16 && rounds_in_bf16(V)) return RAZER_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(ts, 4) || !aligned(codes, 16) ||
        (scale_fmt == RAZER_SCALE_F16 && !aligned(scales, 2)))
        return RAZER_ERR_ALIGN;
    if (N == 0) return RAZER_OK;
    if (K == 0)  // empty sums: y = 0
        return cudaMemsetAsync(y, 0, (size_t)B * (size_t)N * (out_dt == RAZER_F32 ? 4 : 2), (cudaStream_t)stream) == cudaSuccess
                   ? RAZER_OK
                   : RAZER_ERR_CUDA;
    const size_t need = gemv_variant_workspace_bytes(B, N, K);
    if (need) {
        if (!workspace || ws_bytes < need) return RAZER_ERR_WORKSPACE;
        if (!aligned(workspace, 16)) return RAZER_ERR_ALIGN;
    }
    return run_gemv_variant(x, act_dt, B, codes, scales, ts, block, scale_fmt, V, N, K, y, out_dt, workspace, (cudaStream_t)stream);
}

razer_status razer_quant_error(const void *X, razer_dtype in_dt, int64_t R, int64_t K, const uint8_t *codes, const uint8_t *scales,
                               const float *ts, razer_format fmt, double *sse, razer_stream_t stream)
{
    if (!ts || !sse || (!X && R * K > 0)) return RAZER_ERR_INVALID_ARG;
    if (!valid_fmt(fmt) || !valid_dt(in_dt)) return RAZER_ERR_INVALID_ARG;
    if (!in16(in_dt)) return RAZER_ERR_DTYPE;
    razer_status st = check_packed(codes, scales, R, K);
    if (st != RAZER_OK) return st;
    if (!aligned(X, 16) || !aligned(ts, 4) || !aligned(sse, 8)) return RAZER_ERR_ALIGN;
    return run_quant_sse(X, in_dt, R, K, codes, scales, ts, fmt, sse, (cudaStream_t)stream);
}

razer_status razer_get_device_status(razer_stream_t stream)
{
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return RAZER_ERR_CUDA;
    unsigned v = 0u, zero = 0u;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) return RAZER_ERR_CUDA;
    if (v && cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess) return RAZER_ERR_CUDA;
    return (razer_status)v;
}

const char *razer_status_string(razer_status s)
{
    switch (s) {
    case RAZER_OK: return "ok";
    case RAZER_ERR_INVALID_ARG: return "invalid argument";
    case RAZER_ERR_SHAPE: return "unsupported shape";
    case RAZER_ERR_ALIGN: return "misaligned pointer";
    case RAZER_ERR_DTYPE: return "unsupported element type";
    case RAZER_ERR_WORKSPACE: return "workspace too small";
    case RAZER_ERR_UNSUPPORTED: return "unsupported request";
    case RAZER_ERR_TIMEOUT: return "device-side wait timed out";
    case RAZER_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

int razer_version(void) { return 200; }

int razer_set_quantize_path(int path)
{
    if (path != RAZER_QPATH_TWO_PASS && path != RAZER_QPATH_SINGLE_PASS) return -1;
    return set_single_pass_quantizer(path == RAZER_QPATH_SINGLE_PASS) ? RAZER_QPATH_SINGLE_PASS : RAZER_QPATH_TWO_PASS;
}

int razer_debug_set_fault_injection(int on)
{
    return g_fault_injection.exchange(on ? 1 : 0, std::memory_order_relaxed);
}

}  // extern "C"
