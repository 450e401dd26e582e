// RaZeR W4A16 GEMM on the tcgen05 tensor cores (sm_100a).
#include "razer_internal.cuh"

namespace razer {

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    (void)M; (void)N; (void)K;
    return 0;
}

razer_status run_gemm(const void *X, razer_dtype act_dt, int64_t M, const uint8_t *codes, const uint8_t *scales, const float *ts,
                      razer_format wfmt, int64_t N, int64_t K, void *Y, razer_dtype out_dt, void *workspace, cudaStream_t st)
{
    (void)X; (void)act_dt; (void)M; (void)codes; (void)scales; (void)ts; (void)wfmt; (void)N; (void)K; (void)Y; (void)out_dt;
    (void)workspace; (void)st;
    return RAZER_ERR_UNSUPPORTED;
}

}  // namespace razer
