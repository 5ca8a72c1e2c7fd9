/*
 * libmq -- nested (Matryoshka) r-bit weight GEMM for NVIDIA B200 (sm_100a).
 *
 * One 8-bit parent checkpoint serves every bit-width r = 1..8: the r-bit
 * model is the top r bits of each parent code ("MatGPTQ: Efficient and
 * Accurate Inference over Nested Quantized Models", abstract: lower-precision
 * models are read from the parent by reading fewer bits, and the refined
 * representation makes an r-bit model read exactly r bits; "MatGPTQ:
 * Accurate and Efficient Post-Training Matryoshka Quantization", abstract:
 * the most significant bits are sliced at inference time, with kernels for
 * slicing and mixed-precision execution).
 *
 * Definitions used by every call:
 *   q      parent code, uint8, N x K row-major (N output features, K inputs)
 *   q_r    = q >> (8 - r)                               (top r bits)
 *   v_r    = 2^(8-r) * q_r + 2^(7-r) - 128              (dequantized level)
 *   s      per-group scale, one per 128 consecutive k, stored as fp16
 *   W_r    [n, k] = s[n, k / 128] * v_r[n, k]
 *   Y      = X . W_r^T, X is M x K bf16 row-major, Y is M x N bf16 row-major
 *
 * Storage ("bit planes", the library's own layout; the pages fix none):
 * rows are padded with zero rows to N128 = 128 * ceil(N / 128).  The buffer
 * holds 8 planes of N128 * K / 32 uint32 words; plane p holds bit (7 - p) of
 * q (most significant plane first), so the r-bit model is the prefix made of
 * the first r planes (r * N128 * K / 8 bytes) and reads exactly r bits per
 * stored weight.  Inside a plane, the 128-row x 128-column block (row tile
 * t, column group g) is 512 contiguous words at (t * G + g) * 512, G = K/128;
 * row i of the block is the 4 words at 4 i, and bit j of word w holds the
 * code of column 128 g + 32 w + j.  The fp16 scales follow the same block
 * order: the 128 rows of block (t, g) at (t * G + g) * 128 (padding rows 0).
 * A run of consecutive (t, g) blocks is therefore one contiguous stream per
 * plane.
 *
 * Conventions:
 *   - All pointers named *_dev are device pointers; the caller owns every
 *     buffer and every stream.  The library allocates no device memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy stream).
 *   - Calls are asynchronous on `stream` unless stated otherwise.  Argument
 *     errors are returned before anything is launched.  Launch failures
 *     return MQ_ERR_CUDA; the CUDA error text is kept for mq_last_error_string.
 *   - fp16 and bf16 values are passed as their uint16_t bit patterns.
 *   - No C++ exception crosses this interface.
 */
#ifndef MQ_H_
#define MQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MQ_API __attribute__((visibility("default")))
#else
#define MQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MQ_OK = 0,
    MQ_ERR_INVALID_ARG = 1,   /* null pointer, bad size, r or group out of range */
    MQ_ERR_UNSUPPORTED = 2,   /* valid request the library does not serve (e.g. a scale that overflows fp16) */
    MQ_ERR_MISALIGNED = 3,    /* pointer not 16-byte aligned */
    MQ_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    MQ_ERR_TIMEOUT = 5,       /* a bounded device-side wait expired */
    MQ_ERR_WORKSPACE = 6      /* workspace missing or smaller than mq_gemm_workspace_bytes */
} mq_status;

/* A view of an r-bit weight set inside a bit-plane buffer (no ownership). */
typedef struct {
    const uint32_t *planes;   /* device: plane 0 of the buffer; first r planes are read */
    const uint16_t *scales;   /* device: fp16 scales in the tiled block order (see above) */
    int64_t N;                /* output features (rows of W) */
    int64_t K;                /* input features, multiple of 128 */
    int32_t group;            /* columns per scale; must be 128 */
    int32_t r;                /* bits per weight, 1..8 */
    const uint16_t *zeros;    /* device: fp16 zero points in the scales' order (mq_pack_zeros),
                                 or NULL for the symmetric format (the zero point 128) */
} mq_weights;

/*
 * Bytes of the first r planes: r * N128 * K / 8 (0 on invalid arguments),
 * N128 = N rounded up to a multiple of 128.  An r-bit model reads exactly r
 * bits per weight ("MatGPTQ: Efficient and Accurate Inference over Nested
 * Quantized Models", abstract, and Table 1, "Exact r-bit loading"): these are
 * the bytes one mq_gemm call at width r streams for its planes.
 */
MQ_API size_t mq_plane_bytes(int64_t N, int64_t K, int r);

/*
 * Bytes of the stored fp16 scales: 2 * N128 * (K / group) (0 on invalid
 * arguments); one scale per row and 128-column group, shared by every r of
 * the nested model (the single multi-precision checkpoint of the MatGPTQ
 * abstract).  The zero points of the asymmetric variant take the same size.
 */
MQ_API size_t mq_scale_bytes(int64_t N, int64_t K, int group);

/*
 * Pack parent codes into the 8 bit planes and round the scales to fp16.
 * Follows the exact-r-bit storage of the MatGPTQ abstract (Table 1, "Exact
 * r-bit loading"; "single multi-precision checkpoint").
 *   codes_dev   uint8 N x K (row-major), the 8-bit parent codes
 *   scales_dev  fp32 N x (K/group), the per-group scales
 *   planes_out  the 8 tiled planes (mq_plane_bytes(N, K, 8) bytes)
 *   scales_out  fp16 bits in the tiled block order (mq_scale_bytes(N, K, 128)
 *               bytes), round-to-nearest-even of scales_dev
 * Preconditions: N >= 1, K >= 128, K % 128 == 0, group == 128, all four
 * pointers 16-byte aligned, buffers do not overlap.
 * Synchronous: returns after the work on `stream` has finished, because it
 * reports MQ_ERR_UNSUPPORTED when any scale is negative, NaN or rounds to an
 * fp16 infinity (the outputs are then unspecified).
 */
MQ_API mq_status mq_pack(const uint8_t *codes_dev, const float *scales_dev,
                  int64_t N, int64_t K, int group,
                  uint32_t *planes_out, uint16_t *scales_out, void *stream);

/*
 * Asymmetric variant (MatGPTQ paper page, captions of Tables 4-7: asymmetric
 * MatGPTQ): a zero point z per 128-column group, real, in units of the 8-bit
 * code, shared by every r; the weight is s * (2^(8-r) q_r + 2^(7-r) - z)
 * (z = 128 is the symmetric format).  Round the fp32 zero points to fp16 in
 * the tiled block order of the scales.
 *   zeros_dev  fp32 N x (K/group)
 *   zeros_out  fp16 bits, mq_scale_bytes(N, K, 128) bytes (padding rows 0)
 * Preconditions as mq_pack; synchronous, MQ_ERR_UNSUPPORTED when a zero
 * point is NaN or rounds to an fp16 infinity.  Set the result as
 * mq_weights.zeros of the parent (mq_slice keeps it).
 */
MQ_API mq_status mq_pack_zeros(const float *zeros_dev, int64_t N, int64_t K, int group,
                               uint16_t *zeros_out, void *stream);

/*
 * Select the r-bit model of a parent: host-only, O(1), no device work and no
 * copy.  `out` refers to the first r planes of `parent`'s buffer and to the
 * same scales, so it lives as long as the parent's buffers.  MSB slicing per
 * the MatGPTQ author-page abstract.  parent->r must be >= r (slicing is
 * nested: the slice of a slice is the slice of the parent).
 */
MQ_API mq_status mq_slice(const mq_weights *parent, int r, mq_weights *out);

/*
 * Bytes of device workspace mq_gemm needs for this problem (0 if none).
 * The workspace holds the M >= 9 GEMM's arrival counters (first 64 KiB) and
 * the fp32 partial sums of the output tiles whose K range is split between
 * CTAs.  The M <= 8 kernel uses none (tiles shared between CTAs are summed
 * inside thread-block clusters), but for M <= 8 the size still covers the
 * GEMM, which serves shapes the GEMV cannot take and the MQ_GEMV_VIA_GEMM
 * variant.
 */
MQ_API size_t mq_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int r);

/*
 * Y = X . W_r^T (MatGPTQ abstract: kernels for the nested format that serve
 * batch sizes beyond one).  Small batches run the tcgen05 GEMV (decoded
 * weights in tensor memory; see mq_set_gemv_variant): M <= 3 on every shape,
 * M = 4 when N * K < 2^25, M = 5..6 when N * K <= 2^23, where it is measured
 * faster; every other call runs the tcgen05 GEMM (mq_gemm_kernel tells
 * which).
 *   X_dev      bf16 M x K row-major
 *   w          r-bit view (from mq_slice, or a parent with r = 8)
 *   Y_dev      bf16 M x N row-major (written, not accumulated)
 *   workspace  device buffer of at least mq_gemm_workspace_bytes(M, N, K, r)
 *              bytes whose first 64 KiB (arrival tickets) are zero-filled
 *              before its first use; every call leaves those 64 KiB zero
 *              again, so one workspace serves calls of any shape in stream
 *              order.  May be NULL when the size is 0.  Calls that run
 *              concurrently must not share a workspace.
 * Preconditions: M >= 1, w->N >= 1, w->K == K, K % 128 == 0, w->group == 128,
 * 1 <= w->r <= 8, X/Y/planes/scales/workspace 16-byte aligned, Y does not
 * overlap the inputs.  M == 0 is accepted and does nothing.
 * The fp32 accumulation order is fixed, so results are deterministic.
 *
 * Stream order.  Both kernels are launched with programmatic dependent
 * launch: a call may start while the preceding kernel on the stream is still
 * running, and it begins streaming the weights (planes and scales) before it
 * waits for that kernel; X is read, and Y and the workspace are written, only
 * after the preceding kernel has completed and its writes are visible.  So
 * the weights must not be written by the immediately preceding kernel on the
 * same stream if that kernel lets its dependents launch early
 * (griddepcontrol.launch_dependents or its CUDA equivalent).  Kernels that
 * never do so -- mq_pack, torch's kernels, cudaMemcpy -- are safe: their
 * dependents start only after they have completed.  mq_gemm's own kernels
 * do trigger early, so weights produced by an mq_gemm call need a
 * cudaStreamSynchronize or an event wait on another stream first (outputs Y
 * used as the next call's X are fine).
 */
MQ_API mq_status mq_gemm(const uint16_t *X_dev, const mq_weights *w,
                  int64_t M, int64_t N, int64_t K, uint16_t *Y_dev,
                  void *workspace, size_t workspace_bytes, void *stream);

/* One product of a chain: Y = X . W_r^T with N = w->N, K = w->K. */
typedef struct mq_call {
    const uint16_t *X;       /* bf16 M x K, device */
    const mq_weights *w;     /* r-bit view */
    int64_t M;               /* rows of X (>= 0) */
    uint16_t *Y;             /* bf16 M x N, device */
} mq_call;

/*
 * A chain of products, such as the linear layers of one decoder layer (the
 * fused q|k|v, o, fused gate|up and down projections at their own bit widths:
 * MatGPTQ author page, abstract: heterogeneous per-layer bit-widths served as
 * one mixed-precision model), enqueued back to back on one stream in array
 * order.  Consecutive launches overlap through programmatic dependent launch
 * (see mq_gemm, Stream order): a call may read the previous call's Y as its
 * X.  Each call follows mq_gemm's preconditions; the workspace must hold
 * mq_gemm_workspace_bytes of every call (they run in stream order, so one
 * workspace serves all).  Validation of every call happens before the first
 * launch: on an error nothing is enqueued.  n == 0 does nothing.
 */
MQ_API mq_status mq_gemm_chain(const mq_call *calls, int n, void *workspace,
                               size_t workspace_bytes, void *stream);

/* One candidate bit width of one layer for mq_bitwidth_search. */
typedef struct mq_choice {
    int32_t r;              /* bit width (informational; returned through the index) */
    uint64_t bytes;         /* storage the layer costs at this width (e.g. mq_plane_bytes) */
    double error;           /* the layer's error at this width (e.g. its output error
                               against the parent on calibration inputs), >= 0 */
} mq_choice;

/*
 * Budget-aware per-layer bit-width search (MatGPTQ author page, abstract:
 * "budget-aware search for heterogeneous per-layer bit-widths"): choose one
 * candidate per layer so that the summed bytes stay within budget_bytes and
 * the summed error is least (a multiple-choice knapsack, solved exactly by
 * dynamic programming over the bytes in units of their greatest common
 * divisor).  Host only, no device work.
 *   choices     n_layers x n_choices candidates, layer-major
 *   choice_out  n_layers indices into each layer's candidates
 *   error_out   the summed error of the choice (may be NULL)
 * Ties: least error, then fewest bytes, then the lowest candidate indices.
 * Returns MQ_ERR_INVALID_ARG for bad sizes or a negative / non-finite error,
 * MQ_ERR_UNSUPPORTED when no choice fits the budget, the dynamic program
 * would need more than 2^26 (layer, budget unit) cells, or host memory runs
 * out.
 */
MQ_API mq_status mq_bitwidth_search(const mq_choice *choices, int n_layers, int n_choices,
                                    uint64_t budget_bytes, int *choice_out, double *error_out);

/*
 * One-shot multi-precision quantizer (host, offline): the parent codes and
 * scales of the nested format from float weights W (N x K, row-major) and a
 * layer's Hessian proxy H (K x K, e.g. X^T X of calibration inputs), by
 * GPTQ's column loop with MatGPTQ's multi-precision objective ("MatGPTQ:
 * Efficient and Accurate Inference over Nested Quantized Models", abstract:
 * bit-slicing and cross-bit error compensation; Tables 6-7: the lambda
 * weighting of the widths).  All pointers are host memory.
 *   mq_matgptq_prepare: U_out (K x K) upper triangular with
 *     U^T U = (H + damp * mean(diag H) * I)^-1, by one blocked Cholesky
 *     factorisation and one blocked triangular inverse (threads; AVX-512 or
 *     AVX2 with FMA when the CPU has them, else portable loops; in the
 *     environment MQ_PORTABLE_HOST=1 forces the portable loops and
 *     MQ_NO_AVX512=1 stops at AVX2: the paths round differently, within
 *     ~1e-15 relative).  Holds one K x K work buffer besides U_out.
 *   mq_matgptq_quantize: per 128-column group, when its first column is
 *     reached, a row's scale is alpha * max|w| / 127.5 over the group's
 *     current weights (alpha from `alphas`, the least lambda-weighted group
 *     error; ties: the first); each code minimises
 *     sum_i lambdas[i] (w - s v_rs[i](q))^2 over the nested levels (ties: the
 *     smallest code); the lambda-weighted mean of the slice errors e is
 *     carried to the later columns of the row, w_j -= e / U[k][k] * U[k][j].
 *     codes_out N x K uint8, scales_out N x (K/128) fp32 (inputs of mq_pack).
 *     threads <= 0: one per hardware thread.  fp64 in a fixed order, so the
 *     result does not depend on the thread count (in the default
 *     floating-point environment: round to nearest even).
 * Errors: MQ_ERR_INVALID_ARG for bad sizes, widths, lambdas (all zero, or
 * negative) or alphas, a non-finite weight, or a zero on U's diagonal;
 * MQ_ERR_UNSUPPORTED when the damped Hessian is not positive definite (or
 * too ill-conditioned to invert), or when host memory or threads run out (no
 * C++ exception leaves the library).  The caller owns every buffer; nothing
 * is written to codes_out or scales_out on an argument error.
 */
MQ_API mq_status mq_matgptq_prepare(const double *H, int64_t K, double damp, double *U_out);
MQ_API mq_status mq_matgptq_quantize(const float *W, int64_t N, int64_t K, const double *U,
                                     const int32_t *rs, const double *lambdas, int n_r,
                                     const double *alphas, int n_alpha, int threads,
                                     uint8_t *codes_out, float *scales_out);

/*
 * The same with the asymmetric levels u_r = 2^(8-r) q_r + 2^(7-r) - z (the
 * variant the pages evaluate: "MatGPTQ: Efficient and Accurate Inference over
 * Nested Quantized Models", captions of Tables 5-7).  Per group and alpha the
 * grid spans alpha times the group's current range [lo, hi], centred on it:
 * s = alpha (hi - lo) / 255, z = 128 - (hi + lo) / (2 s), z rounded as stored
 * (to fp32, then fp16, nearest-even); a group of zero range, or whose z is no
 * finite fp16, takes the symmetric grid (s = alpha max|w| / 127.5, z = 128).
 * zeros_out N x (K/128) fp32 holds those fp16 values (the input of
 * mq_pack_zeros); the rest as mq_matgptq_quantize.
 */
MQ_API mq_status mq_matgptq_quantize_asym(const float *W, int64_t N, int64_t K, const double *U,
                                          const int32_t *rs, const double *lambdas, int n_r,
                                          const double *alphas, int n_alpha, int threads,
                                          uint8_t *codes_out, float *scales_out, float *zeros_out);

/* Kernels for M <= 8 (both compute the same Y within the stated tolerance). */
enum {
    MQ_GEMV_TC = 0,        /* default: 128 rows per tensor-core MMA, int8 operands,
                              decoded weights stored in tensor memory */
    MQ_GEMV_VIA_GEMM = 1   /* the M >= 9 tcgen05 GEMM (bf16 operands), X rows padded to 32 */
};

/*
 * Choose the M <= 8 kernel for later mq_gemm calls in this process (host
 * only, no device work).  Returns MQ_ERR_INVALID_ARG for an unknown value.
 * Both variants follow the same definition of Y (MatGPTQ abstract: kernels
 * for slicing and mixed-precision execution); shapes whose operands do not
 * fit the GEMV's shared memory always take the GEMM.
 */
MQ_API mq_status mq_set_gemv_variant(int variant);

/* The M <= 8 kernel in use (MQ_GEMV_TC or MQ_GEMV_VIA_GEMM). */
MQ_API int mq_get_gemv_variant(void);

/* Kernels that serve an mq_gemm call. */
enum {
    MQ_KERNEL_GEMV = 1,    /* the M <= 8 tensor-core GEMV */
    MQ_KERNEL_GEMM = 2     /* the tcgen05 GEMM */
};

/*
 * Which kernel mq_gemm(M, N, K, r) would run under the current variant for
 * symmetric weights (host only, no device work): MQ_KERNEL_GEMV or
 * MQ_KERNEL_GEMM, 0 for an invalid problem (M < 1, N < 1, K not a positive
 * multiple of 128, r outside 1..8).  Weights with zero points always run the
 * GEMM.  Lets a caller or a benchmark label its timings; it has no effect on
 * the call itself.
 */
MQ_API int mq_gemm_kernel(int64_t M, int64_t N, int64_t K, int r);

/*
 * Test helper: codes_out[n, k] = q_r[n, k] read back from the first r planes
 * (uint8 N x K row-major, device): the r-bit model as the top r bits of the
 * parent code ("MatGPTQ: Accurate and Efficient Post-Training Matryoshka
 * Quantization", author-page abstract: the most significant bits are sliced
 * at inference time).  Same preconditions as mq_gemm on `w`.
 */
MQ_API mq_status mq_unpack(const mq_weights *w, uint8_t *codes_out, void *stream);

/*
 * mq_gemv_noalloc: Y = X . W_r^T for 1 <= M <= 8 without a workspace.  For
 * callers that cannot call cudaMalloc where they run the layer: a plugin
 * whose host application owns all device memory and offers no allocator, a
 * server that hands the whole GPU to its own memory pool at start-up, or a
 * latency-critical loop that must not take cudaMalloc's implicit device
 * synchronisation.  The paper has no counterpart: this is a calling
 * convention, not part of the method.
 *   Arguments and results are those of mq_gemm without the workspace.
 *   Scratch: a 16 MiB array compiled into the library, resident on every GPU
 *   that loads it until the process exits.  The call runs the kernel
 *   mq_gemm would run for M <= 8: the tensor-core GEMV needs no scratch; the
 *   GEMM (shapes the GEMV does not take, or the MQ_GEMV_VIA_GEMM variant)
 *   keeps its split-K partial sums, its X operand and its arrival tickets in
 *   the array.  A problem whose kernel needs more than 16 MiB of scratch
 *   returns MQ_ERR_WORKSPACE; M > 8 returns MQ_ERR_INVALID_ARG.  Both checks
 *   happen before any launch.  The first call on a device that takes the
 *   GEMM looks up the array's device address (once per device, with that
 *   device current); make that first call before any stream capture.  Each
 *   call that takes the GEMM clears the array's arrival tickets (one
 *   cudaMemsetAsync on `stream`) and overwrites the rest.
 *   All calls share the one array, which keeps the last call's contents:
 *   calls that can overlap on the GPU (other streams, other host threads)
 *   race and must be serialised by the caller.
 *   Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
MQ_API mq_status mq_gemv_noalloc(const uint16_t *X_dev, const mq_weights *w, int64_t M,
                                 int64_t N, int64_t K, uint16_t *Y_dev, void *stream);

/* Status of the most recent failing call on this host thread (MQ_OK if none). */
MQ_API mq_status mq_last_error(void);

/*
 * Device-side failures of earlier launches on the current device: every wait
 * inside the kernels gives up after about one second of GPU time (a copy or
 * an MMA that never completes), records the fact in a device flag and returns
 * instead of hanging.  This call synchronises the current device, reads and
 * clears the flags, and returns MQ_ERR_TIMEOUT if any was set (MQ_OK
 * otherwise; MQ_ERR_CUDA if the device cannot be read).  The Y of a launch
 * that timed out is unspecified.  No counterpart in the paper (a robustness
 * hook of this library).
 */
MQ_API mq_status mq_device_status(void);

/* Text of the most recent failure on this host thread (never NULL). */
MQ_API const char *mq_last_error_string(void);

/* Fixed description of a status code (never NULL). */
MQ_API const char *mq_status_string(mq_status s);

/* Library version, e.g. "0.1.0". */
MQ_API const char *mq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MQ_H_ */
