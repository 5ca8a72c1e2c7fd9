// mq_gemv_noalloc: the M <= 8 product without a caller-supplied workspace.
//
// Some callers cannot allocate device memory at the point where they run a
// layer: plugins embedded in a host application that owns all device memory
// and exposes no allocator, serving processes that hand the whole GPU to
// their own pool at start-up, and latency-critical loops that cannot take
// cudaMalloc's implicit device synchronisation.  They can still call this
// entry point: its scratch (the X operand of the call, and for the GEMM route
// the split-K partial sums and arrival tickets) lives in a fixed array
// compiled into the library instead of a workspace they would have to
// provide.
#include "mq_common.cuh"

namespace mq {
namespace {

// The scratch: 16 MiB of device memory per GPU that loads the library, held
// until the process exits.  Host code must not use the symbol's host address
// directly; the device address comes from cudaGetSymbolAddress below.
constexpr size_t kNoAllocBytes = (size_t)16 << 20;
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices];        // device address of the array, per device

}  // namespace
}  // namespace mq

using namespace mq;

extern "C" mq_status mq_gemv_noalloc(const uint16_t *X, const mq_weights *w, int64_t M,
                                     int64_t N, int64_t K, uint16_t *Y, void *stream) {
    mq_status s = check_weights(w, N, K);
    if (s != MQ_OK) return s;
    if (M < 0 || M > kGemvMaxM) return fail(MQ_ERR_INVALID_ARG, "mq_gemv_noalloc serves 0 <= M <= 8");
    if (M == 0) return MQ_OK;
    if (!X || !Y) return fail(MQ_ERR_INVALID_ARG, "X or Y is NULL");
    if (!aligned16(X) || !aligned16(Y))
        return fail(MQ_ERR_MISALIGNED, "X and Y must be 16-byte aligned");
    // the kernel this call will run, and the scratch that kernel needs (the
    // tensor-core GEMV: its X operand; the GEMM: its split-K partial sums,
    // its X operand and its arrival tickets)
    cudaStream_t st = (cudaStream_t)stream;
    if ((s = bind_device(st)) != MQ_OK) return s;
    const bool gemv = !w->zeros && small_m_uses_gemv(M, N, K, w->r);
    const size_t need = gemv ? gemv_tc_workspace_bytes(M, N, K, w->r)
                             : gemm_tc_workspace_bytes(M, N, K, w->r);
    if (need > kNoAllocBytes)
        return fail(MQ_ERR_WORKSPACE,
                    "problem needs more scratch than the 16 MiB built into mq_gemv_noalloc; "
                    "use mq_gemm with a workspace");
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(MQ_ERR_UNSUPPORTED, "device index out of range");
    void *scratch = __atomic_load_n(&g_scratch_addr[dev], __ATOMIC_ACQUIRE);
    if (!scratch) {
        // once per device, with that device current: the array's device address
        e = cudaGetSymbolAddress(&scratch, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
        __atomic_store_n(&g_scratch_addr[dev], scratch, __ATOMIC_RELEASE);
    }
    // the tensor-core GEMV keeps the X operand of the call in the scratch
    if (gemv) return launch_gemv_tc(X, w, M, Y, scratch, kNoAllocBytes, st);
    // the GEMM's arrival tickets must start at zero whatever an earlier call
    // (or one that gave up on a wait) left there
    e = cudaMemsetAsync(scratch, 0, kTicketBytes, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    return launch_gemm_tc(X, w, M, Y, scratch, kNoAllocBytes, st);
}
