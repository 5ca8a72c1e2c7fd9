// C-ABI entry points of libmq that are not kernels: argument checks, the
// O(1) slice, sizes, dispatch between the GEMV and the tensor-core GEMM, and
// error reporting.
#include <stdarg.h>
#include <string.h>

#include "mq_common.cuh"

namespace mq {

static thread_local mq_status g_last = MQ_OK;
static int g_gemv_variant = MQ_GEMV_TC;    // process-wide kernel choice for M <= 8
static thread_local char g_msg[512] = "no error";

void set_error(mq_status s, const char *fmt, ...) {
    g_last = s;
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
}

mq_status cuda_fail(cudaError_t e, const char *where) {
    set_error(MQ_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
    return MQ_ERR_CUDA;
}

// Driver calls reached through the runtime's entry-point query, so the library
// has no link-time dependency on libcuda (it loads on machines without a GPU).
typedef int (*CtxGetCurrentFn)(void **);
typedef int (*CtxGetDeviceFn)(int *);

static int current_context_device() {
    static CtxGetCurrentFn get_ctx = nullptr;
    static CtxGetDeviceFn get_dev = nullptr;
    static bool looked_up = false;
    if (!looked_up) {
        cudaDriverEntryPointQueryResult q;
        cudaGetDriverEntryPoint("cuCtxGetCurrent", (void **)&get_ctx, cudaEnableDefault, &q);
        cudaGetDriverEntryPoint("cuCtxGetDevice", (void **)&get_dev, cudaEnableDefault, &q);
        looked_up = true;
    }
    void *ctx = nullptr;
    int dev = -1;
    if (!get_ctx || !get_dev || get_ctx(&ctx) != 0 || !ctx || get_dev(&dev) != 0) return -1;
    return dev;
}

mq_status bind_device(cudaStream_t st) {
    static thread_local cudaStream_t last_stream = nullptr;
    if (st != nullptr && st == last_stream) return MQ_OK;
    int dev = -1;
    if (st != nullptr) {
        cudaError_t e = cudaStreamGetDevice(st, &dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaStreamGetDevice");
    } else {
        dev = current_context_device();   // legacy stream: the caller's context
        if (dev < 0) return MQ_OK;
    }
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess || cur != dev) {
        cudaError_t e = cudaSetDevice(dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
    }
    last_stream = st;
    return MQ_OK;
}

mq_status check_weights(const mq_weights *w, int64_t N, int64_t K) {
    if (!w) return fail(MQ_ERR_INVALID_ARG, "weights view is NULL");
    if (!w->planes || !w->scales)
        return fail(MQ_ERR_INVALID_ARG, "weights view has a NULL buffer");
    if (w->r < 1 || w->r > 8) return fail(MQ_ERR_INVALID_ARG, "r must be in 1..8");
    if (w->group != kGroup) return fail(MQ_ERR_INVALID_ARG, "group must be 128");
    if (w->N != N || w->K != K)
        return fail(MQ_ERR_INVALID_ARG, "weights view shape differs from (N, K)");
    if (N < 1 || K < kGroup || K % kGroup)
        return fail(MQ_ERR_INVALID_ARG, "need N >= 1 and K a positive multiple of 128");
    if (!aligned16(w->planes) || !aligned16(w->scales) || (w->zeros && !aligned16(w->zeros)))
        return fail(MQ_ERR_MISALIGNED, "planes, scales and zero points must be 16-byte aligned");
    return MQ_OK;
}

// M <= 8 dispatch, from the measured crossover of the two kernels on the
// Llama-3.1-8B shapes (CUDA-graph back-to-back launches over L2-cold
// weights): the GEMV is ahead up to M = 3 on every shape, at M = 4 on the
// q/o-size shapes and below, and at M = 5..6 only on the k/v-size shapes;
// from there the GEMM (whose time barely grows with M) is ahead.
bool small_m_uses_gemv(int64_t M, int64_t N, int64_t K, int r) {
    if (__atomic_load_n(&g_gemv_variant, __ATOMIC_RELAXED) != MQ_GEMV_TC) return false;
    const int64_t weights = N * K;
    const bool gemv_ahead = M <= 3 || (M == 4 && weights < (int64_t)32 << 20) ||
                            (M <= 6 && weights <= (int64_t)8 << 20);
    return gemv_ahead && gemv_tc_supported(M, N, K, r);
}

mq_status launch_small_m(const uint16_t *X, const mq_weights *w, int64_t M, uint16_t *Y,
                         void *ws, size_t ws_bytes, cudaStream_t st) {
    // the asymmetric variant runs on the GEMM for every M
    if (!w->zeros && small_m_uses_gemv(M, w->N, w->K, w->r))
        return launch_gemv_tc(X, w, M, Y, ws, ws_bytes, st);
    return launch_gemm_tc(X, w, M, Y, ws, ws_bytes, st);
}

// fail() with a formatted message.
template <class... A>
mq_status failf(mq_status s, const char *fmt, A... args) {
    set_error(s, fmt, args...);
    return s;
}

}  // namespace mq

using namespace mq;

extern "C" {

size_t mq_plane_bytes(int64_t N, int64_t K, int r) {
    if (N < 1 || K < kGroup || K % kGroup || r < 1 || r > 8) return 0;
    return (size_t)r * (size_t)((N + 127) / 128 * 128) * (size_t)K / 8;
}

size_t mq_scale_bytes(int64_t N, int64_t K, int group) {
    if (N < 1 || K < kGroup || K % kGroup || group != kGroup) return 0;
    return 2 * (size_t)((N + 127) / 128 * 128) * (size_t)(K / group);
}

mq_status mq_slice(const mq_weights *parent, int r, mq_weights *out) {
    if (!parent || !out) return fail(MQ_ERR_INVALID_ARG, "NULL argument to mq_slice");
    if (r < 1 || r > 8) return fail(MQ_ERR_INVALID_ARG, "r must be in 1..8");
    if (parent->r < r)
        return fail(MQ_ERR_INVALID_ARG, "cannot slice to more bits than the parent has");
    mq_status s = check_weights(parent, parent->N, parent->K);
    if (s != MQ_OK) return s;
    *out = *parent;   // same buffer: the first r planes are the r-bit model
    out->r = r;
    return MQ_OK;
}

size_t mq_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
    if (M < 1 || N < 1 || K < kGroup || K % kGroup || r < 1 || r > 8) return 0;
    if (M <= kGemvMaxM) {
        const size_t a = gemv_tc_workspace_bytes(M, N, K, r), b = gemm_tc_workspace_bytes(M, N, K, r);
        return a > b ? a : b;
    }
    return gemm_tc_workspace_bytes(M, N, K, r);
}

mq_status mq_gemm(const uint16_t *X, const mq_weights *w, int64_t M, int64_t N,
                  int64_t K, uint16_t *Y, void *workspace, size_t workspace_bytes,
                  void *stream) {
    mq_status s = check_weights(w, N, K);
    if (s != MQ_OK) return s;
    if (M < 0) return fail(MQ_ERR_INVALID_ARG, "M must be >= 0");
    if (M == 0) return MQ_OK;
    if (!X || !Y) return fail(MQ_ERR_INVALID_ARG, "X or Y is NULL");
    if (!aligned16(X) || !aligned16(Y) || (workspace && !aligned16(workspace)))
        return fail(MQ_ERR_MISALIGNED, "X, Y and workspace must be 16-byte aligned");
    size_t need = mq_gemm_workspace_bytes(M, N, K, w->r);
    if (need && (!workspace || workspace_bytes < need))
        return fail(MQ_ERR_WORKSPACE, "workspace smaller than mq_gemm_workspace_bytes");
    cudaStream_t st = (cudaStream_t)stream;
    if ((s = bind_device(st)) != MQ_OK) return s;
    if (M <= kGemvMaxM) return launch_small_m(X, w, M, Y, workspace, workspace_bytes, st);
    return launch_gemm_tc(X, w, M, Y, workspace, workspace_bytes, st);
}

mq_status mq_gemm_chain(const mq_call *calls, int n, void *workspace, size_t workspace_bytes,
                        void *stream) {
    if (n < 0 || (n > 0 && !calls)) return fail(MQ_ERR_INVALID_ARG, "bad chain (n < 0 or calls NULL)");
    if (workspace && !aligned16(workspace)) return fail(MQ_ERR_MISALIGNED, "workspace must be 16-byte aligned");
    // validate every call before launching any
    for (int i = 0; i < n; ++i) {
        const mq_call &c = calls[i];
        if (!c.w) return failf(MQ_ERR_INVALID_ARG, "chain call %d: weights are NULL", i);
        mq_status s = check_weights(c.w, c.w->N, c.w->K);
        if (s != MQ_OK) return s;
        if (c.M < 0) return failf(MQ_ERR_INVALID_ARG, "chain call %d: M must be >= 0", i);
        if (c.M == 0) continue;
        if (!c.X || !c.Y) return failf(MQ_ERR_INVALID_ARG, "chain call %d: X or Y is NULL", i);
        if (!aligned16(c.X) || !aligned16(c.Y))
            return failf(MQ_ERR_MISALIGNED, "chain call %d: X and Y must be 16-byte aligned", i);
        const size_t need = mq_gemm_workspace_bytes(c.M, c.w->N, c.w->K, c.w->r);
        if (need && (!workspace || workspace_bytes < need))
            return failf(MQ_ERR_WORKSPACE, "chain call %d: workspace smaller than mq_gemm_workspace_bytes", i);
    }
    cudaStream_t st = (cudaStream_t)stream;
    mq_status s = bind_device(st);
    if (s != MQ_OK) return s;
    for (int i = 0; i < n; ++i) {
        const mq_call &c = calls[i];
        if (c.M == 0) continue;
        s = c.M <= kGemvMaxM ? launch_small_m(c.X, c.w, c.M, c.Y, workspace, workspace_bytes, st)
                             : launch_gemm_tc(c.X, c.w, c.M, c.Y, workspace, workspace_bytes, st);
        if (s != MQ_OK) return s;
    }
    return MQ_OK;
}

mq_status mq_set_gemv_variant(int variant) {
    if (variant != MQ_GEMV_TC && variant != MQ_GEMV_VIA_GEMM)
        return fail(MQ_ERR_INVALID_ARG, "unknown GEMV variant");
    __atomic_store_n(&g_gemv_variant, variant, __ATOMIC_RELAXED);
    return MQ_OK;
}

int mq_get_gemv_variant(void) { return __atomic_load_n(&g_gemv_variant, __ATOMIC_RELAXED); }

int mq_gemm_kernel(int64_t M, int64_t N, int64_t K, int r) {
    if (M < 1 || N < 1 || K < kGroup || K % kGroup || r < 1 || r > 8) return 0;
    return M <= kGemvMaxM && small_m_uses_gemv(M, N, K, r) ? MQ_KERNEL_GEMV : MQ_KERNEL_GEMM;
}

mq_status mq_last_error(void) { return g_last; }

mq_status mq_device_status(void) {
    const cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    bool a = false, b = false;
    if (!gemv_tc_take_timeout(&a) || !gemm_tc_take_timeout(&b))
        return fail(MQ_ERR_CUDA, "device timeout flags not readable");
    if (a || b) return fail(MQ_ERR_TIMEOUT, "a bounded device-side wait expired in an earlier launch");
    return MQ_OK;
}
const char *mq_last_error_string(void) { return g_msg; }

const char *mq_status_string(mq_status s) {
    switch (s) {
        case MQ_OK: return "ok";
        case MQ_ERR_INVALID_ARG: return "invalid argument";
        case MQ_ERR_UNSUPPORTED: return "unsupported";
        case MQ_ERR_MISALIGNED: return "misaligned pointer";
        case MQ_ERR_CUDA: return "CUDA error";
        case MQ_ERR_TIMEOUT: return "device wait timed out";
        case MQ_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

const char *mq_version(void) { return "0.1.0"; }

}  // extern "C"
