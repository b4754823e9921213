// Block-scaled FP4 GEMM entry points (tcgen05 kernel in progress).
#include <cuda_runtime.h>
#include <stdint.h>

#include "mx.h"

extern "C" {

int64_t mx_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    (void)M; (void)N; (void)K;
    return 0;
}

int mx_gemm(const mx_config *ca, const mx_config *cb, const void *Aq, const uint8_t *Asf,
            const void *Bq, const uint8_t *Bsf, const float *tsA, const float *tsB, int64_t M,
            int64_t N, int64_t K, void *C, int32_t c_dtype, void *stream)
{
    (void)ca; (void)cb; (void)Aq; (void)Asf; (void)Bq; (void)Bsf; (void)tsA; (void)tsB;
    (void)M; (void)N; (void)K; (void)C; (void)c_dtype; (void)stream;
    return MX_ERR_UNSUPPORTED;
}

int mx_gemm_qsnr(const mx_config *ca, const mx_config *cb, const void *A, const void *B, int64_t M,
                 int64_t N, int64_t K, const void *Aq, const uint8_t *Asf, const void *Bq,
                 const uint8_t *Bsf, const float *tsA, const float *tsB, double *stats,
                 void *workspace, int64_t workspace_bytes, void *stream)
{
    (void)ca; (void)cb; (void)A; (void)B; (void)M; (void)N; (void)K; (void)Aq; (void)Asf;
    (void)Bq; (void)Bsf; (void)tsA; (void)tsB; (void)stats; (void)workspace;
    (void)workspace_bytes; (void)stream;
    return MX_ERR_UNSUPPORTED;
}

int mx_device_status(void *stream, int32_t *status)
{
    (void)stream;
    if (status) *status = 0;
    return MX_OK;
}

}  // extern "C"
