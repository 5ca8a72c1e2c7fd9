// Internal helpers shared by the libmq translation units (not installed).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stdio.h>

#include <exception>
#include <new>

#include "../../include/mq.h"

namespace mq {

constexpr int kGroup = 128;          // columns per scale
constexpr int kPlanes = 8;           // planes in a parent buffer
// Split-K arrival tickets live in the first kTicketBytes of every workspace;
// each call returns the tickets it used to zero.
constexpr size_t kTicketBytes = 64 * 1024;

// Per-host-thread record of the last failure (mq_last_error*).
void set_error(mq_status s, const char *fmt, ...);
inline mq_status fail(mq_status s, const char *what) {
    set_error(s, "%s", what);
    return s;
}
mq_status cuda_fail(cudaError_t e, const char *where);

// f() for the host-only entry points that allocate or start threads: no C++
// exception crosses the C ABI (host memory exhausted, or threads refused,
// returns MQ_ERR_UNSUPPORTED with the reason).
template <class F>
mq_status host_guarded(F &&f) {
    try {
        return f();
    } catch (const std::bad_alloc &) {
        return fail(MQ_ERR_UNSUPPORTED, "out of host memory");
    } catch (const std::exception &e) {
        return fail(MQ_ERR_UNSUPPORTED, e.what());
    } catch (...) {
        return fail(MQ_ERR_UNSUPPORTED, "host error");
    }
}

inline bool aligned16(const void *p) {
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

// Make the stream's device current for this library's runtime (the library
// links its own CUDA runtime, whose current device is not the caller's).
mq_status bind_device(cudaStream_t st);

// Validate a weight view against (N, K); returns MQ_OK or the failing status.
mq_status check_weights(const mq_weights *w, int64_t N, int64_t K);

// Kernel launchers (each returns MQ_OK or MQ_ERR_CUDA after the launch).
bool gemv_tc_supported(int64_t M, int64_t N, int64_t K, int r);
// Read and clear the device flag of a timed-out wait (false: device not readable).
bool gemv_tc_take_timeout(bool *set);
bool gemm_tc_take_timeout(bool *set);
size_t gemv_tc_workspace_bytes(int64_t M, int64_t N, int64_t K, int r);
mq_status launch_gemv_tc(const uint16_t *X, const mq_weights *w, int64_t M,
                         uint16_t *Y, void *ws, size_t ws_bytes, cudaStream_t st);
size_t gemm_tc_workspace_bytes(int64_t M, int64_t N, int64_t K, int r);
mq_status launch_gemm_tc(const uint16_t *X, const mq_weights *w, int64_t M,
                         uint16_t *Y, void *ws, size_t ws_bytes, cudaStream_t st);
// Whether an M <= 8 call takes the tensor-core GEMV (variant and shape).
bool small_m_uses_gemv(int64_t M, int64_t N, int64_t K, int r);
// The M <= 8 product with the kernel chosen by mq_set_gemv_variant.
mq_status launch_small_m(const uint16_t *X, const mq_weights *w, int64_t M,
                         uint16_t *Y, void *ws, size_t ws_bytes, cudaStream_t st);

// Largest M served by the GEMV kernels; larger M runs the tcgen05 GEMM.
constexpr int kGemvMaxM = 8;

}  // namespace mq
