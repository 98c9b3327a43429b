#include "sgemm.cuh"

namespace gq {

gptq_status sgemm_launch(const SgemmArgs& a, bool b_trans, int epi, cudaStream_t s) {
    if (a.M <= 0 || a.N <= 0) return GPTQ_OK;
    if (a.K % 4 || a.N % 4 || a.lda % 4 || a.ldb % 4 ||
        (epi == EPI_STORE && a.ldc % 4) || (epi == EPI_DOT && a.ldd % 4))
        return GPTQ_ERR_ARG;
    const dim3 grid((a.N + sg::BN - 1) / sg::BN, (a.M + sg::BM - 1) / sg::BM);
    if (grid.y > 65535) return GPTQ_ERR_ARG;
    if (b_trans) {
        if (epi == EPI_STORE) sgemm_kernel<true, EPI_STORE><<<grid, sg::THREADS, 0, s>>>(a);
        else sgemm_kernel<true, EPI_DOT><<<grid, sg::THREADS, 0, s>>>(a);
    } else {
        if (epi == EPI_STORE) sgemm_kernel<false, EPI_STORE><<<grid, sg::THREADS, 0, s>>>(a);
        else sgemm_kernel<false, EPI_DOT><<<grid, sg::THREADS, 0, s>>>(a);
    }
    GPTQ_LAUNCHED();
    return GPTQ_OK;
}

}  // namespace gq
