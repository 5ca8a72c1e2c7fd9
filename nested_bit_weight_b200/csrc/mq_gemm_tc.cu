// Batched path (M >= 9).  Interim version: runs the GEMV over 8-row slices
// of X; the tcgen05 tensor-core kernel replaces it.
#include "mq_common.cuh"

namespace mq {

size_t gemm_tc_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
    (void)M;
    return gemv_workspace_bytes(kGemvMaxM, N, K, r);
}

mq_status launch_gemm_tc(const uint16_t *X, const mq_weights *w, int64_t M, uint16_t *Y,
                         void *ws, size_t ws_bytes, cudaStream_t st) {
    for (int64_t m0 = 0; m0 < M; m0 += kGemvMaxM) {
        const int64_t mc = (M - m0) < kGemvMaxM ? (M - m0) : kGemvMaxM;
        mq_status s = launch_gemv(X + m0 * w->K, w, mc, Y + m0 * w->N, ws, ws_bytes, st);
        if (s != MQ_OK) return s;
    }
    return MQ_OK;
}

}  // namespace mq
