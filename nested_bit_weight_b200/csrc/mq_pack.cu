// Bit-plane packer and its inverse (exact-r-bit storage of the MatGPTQ
// abstract and Table 1, "Exact r-bit loading").
//
// Layout (include/mq.h): rows padded to a multiple of 128; each plane is a
// sequence of 2 KB blocks, one per (128-row tile t, 128-column group g) in
// t-major order; row i of a block is 4 words (16 bytes), bit j of word w
// holding column 128g + 32w + j.  Scales use the same block order, 128
// fp16 values per block.
//
// pack: a warp turns 32 consecutive codes of a row into one word of each of
// the 8 planes with warp ballots (lane j votes bit j of its code).
#include "mq_common.cuh"

namespace mq {

__device__ unsigned int g_pack_bad;   // set when a scale is not storable

__global__ void __launch_bounds__(256)
pack_kernel(const uint8_t *__restrict__ codes, int64_t N, int64_t K,
            uint32_t *__restrict__ planes) {
    // one warp per (row, block of 32 words): chunk c's ballots land in lane c,
    // so each plane's 32 words leave as one coalesced 128-byte store
    const int lane = threadIdx.x & 31;
    const int64_t W = K / 32;                        // words per plane row
    const int64_t blocks_per_row = (W + 31) / 32;
    const int64_t total = N * blocks_per_row;
    const int64_t plane_words = (N + 127) / 128 * 128 * W;
    int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t i = warp; i < total; i += nwarps) {
        const int64_t n = i / blocks_per_row, w0 = (i % blocks_per_row) * 32;
        uint32_t mine[kPlanes] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int c = 0; c < 32 && w0 + c < W; ++c) {
            const unsigned q = codes[n * K + 32 * (w0 + c) + lane];
#pragma unroll
            for (int p = 0; p < kPlanes; ++p) {
                const uint32_t word = __ballot_sync(0xffffffffu, (q >> (7 - p)) & 1u);
                if (lane == c) mine[p] = word;
            }
        }
        if (w0 + lane < W) {
            const int64_t w = w0 + lane;
            const int64_t at = ((n / 128) * (W / 4) + w / 4) * 512 + (n % 128) * 4 + (w % 4);
#pragma unroll
            for (int p = 0; p < kPlanes; ++p) planes[(int64_t)p * plane_words + at] = mine[p];
        }
    }
}

// fp32 [N, G] -> fp16 RNE in the tiled block order; `signed_ok` admits
// negative values (zero points) and refuses only NaN and fp16 overflow.
__global__ void __launch_bounds__(256)
scales_kernel(const float *__restrict__ s, int64_t N, int64_t G, __half *__restrict__ out,
              bool signed_ok) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < N * G;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = i / G, g = i - n * G;
        const float v = s[i];
        const __half h = __float2half_rn(v);
        if (!(signed_ok ? v == v : v >= 0.0f) || __hisinf(h)) atomicOr(&g_pack_bad, 1u);
        out[((n / 128) * G + g) * 128 + n % 128] = h;
    }
}

// codes_out[n, k] = q_r read from the first r planes.
__global__ void __launch_bounds__(256)
unpack_kernel(const uint32_t *__restrict__ planes, int64_t N, int64_t K, int r,
              uint8_t *__restrict__ out) {
    const int64_t W = K / 32;
    const int64_t plane_words = (N + 127) / 128 * 128 * W;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < N * W;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = i / W, w = i - n * W;
        const int64_t at = ((n / 128) * (W / 4) + w / 4) * 512 + (n % 128) * 4 + (w % 4);
        uint32_t P[kPlanes];
        for (int p = 0; p < r; ++p) P[p] = planes[(int64_t)p * plane_words + at];
        uint32_t packed[8];
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            uint32_t v = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int bit = 4 * b + j;
                uint32_t q = 0;
                for (int p = 0; p < r; ++p) q = (q << 1) | ((P[p] >> bit) & 1u);
                v |= q << (8 * j);
            }
            packed[b] = v;
        }
        uint4 *dst = reinterpret_cast<uint4 *>(out + i * 32);
        dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    }
}

static int grid_for(int64_t work, int per_block) {
    int64_t g = (work + per_block - 1) / per_block;
    if (g > 148 * 32) g = 148 * 32;
    return (int)(g < 1 ? 1 : g);
}

}  // namespace mq

using namespace mq;

extern "C" mq_status mq_pack(const uint8_t *codes, const float *scales, int64_t N,
                             int64_t K, int group, uint32_t *planes_out,
                             uint16_t *scales_out, void *stream) {
    if (!codes || !scales || !planes_out || !scales_out)
        return fail(MQ_ERR_INVALID_ARG, "NULL pointer passed to mq_pack");
    if (N < 1 || K < kGroup || K % kGroup)
        return fail(MQ_ERR_INVALID_ARG, "need N >= 1 and K a positive multiple of 128");
    if (group != kGroup) return fail(MQ_ERR_INVALID_ARG, "group must be 128");
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(planes_out) ||
        !aligned16(scales_out))
        return fail(MQ_ERR_MISALIGNED, "mq_pack pointers must be 16-byte aligned");
    cudaStream_t st = (cudaStream_t)stream;
    mq_status bs = bind_device(st);
    if (bs != MQ_OK) return bs;
    const unsigned zero = 0;
    cudaError_t e = cudaMemcpyToSymbolAsync(g_pack_bad, &zero, sizeof(zero), 0,
                                            cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "mq_pack reset");
    if (N % 128) {
        // padding rows of the last tile: zero bits and zero scales
        e = cudaMemsetAsync(planes_out, 0, mq_plane_bytes(N, K, 8), st);
        if (e == cudaSuccess) e = cudaMemsetAsync(scales_out, 0, mq_scale_bytes(N, K, kGroup), st);
        if (e != cudaSuccess) return cuda_fail(e, "mq_pack padding");
    }
    pack_kernel<<<grid_for(N * ((K / 32 + 31) / 32) * 32, 256), 256, 0, st>>>(codes, N, K, planes_out);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "pack_kernel");
    const int64_t ns = N * (K / kGroup);
    scales_kernel<<<grid_for(ns, 256), 256, 0, st>>>(scales, N, K / kGroup,
                                                     reinterpret_cast<__half *>(scales_out), false);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "scales_kernel");
    unsigned bad = 0;
    e = cudaMemcpyFromSymbolAsync(&bad, g_pack_bad, sizeof(bad), 0,
                                  cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "mq_pack");
    if (bad) return fail(MQ_ERR_UNSUPPORTED,
                         "a scale is negative, NaN, or overflows fp16");
    return MQ_OK;
}

extern "C" mq_status mq_pack_zeros(const float *zeros, int64_t N, int64_t K, int group,
                                   uint16_t *zeros_out, void *stream) {
    if (!zeros || !zeros_out) return fail(MQ_ERR_INVALID_ARG, "NULL pointer passed to mq_pack_zeros");
    if (N < 1 || K < kGroup || K % kGroup)
        return fail(MQ_ERR_INVALID_ARG, "need N >= 1 and K a positive multiple of 128");
    if (group != kGroup) return fail(MQ_ERR_INVALID_ARG, "group must be 128");
    if (!aligned16(zeros) || !aligned16(zeros_out))
        return fail(MQ_ERR_MISALIGNED, "mq_pack_zeros pointers must be 16-byte aligned");
    cudaStream_t st = (cudaStream_t)stream;
    mq_status bs = bind_device(st);
    if (bs != MQ_OK) return bs;
    const unsigned zero = 0;
    cudaError_t e = cudaMemcpyToSymbolAsync(g_pack_bad, &zero, sizeof(zero), 0,
                                            cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "mq_pack_zeros reset");
    if (N % 128 && (e = cudaMemsetAsync(zeros_out, 0, mq_scale_bytes(N, K, kGroup), st)) != cudaSuccess)
        return cuda_fail(e, "mq_pack_zeros padding");
    const int64_t ns = N * (K / kGroup);
    scales_kernel<<<grid_for(ns, 256), 256, 0, st>>>(zeros, N, K / kGroup,
                                                     reinterpret_cast<__half *>(zeros_out), true);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "scales_kernel (zeros)");
    unsigned bad = 0;
    e = cudaMemcpyFromSymbolAsync(&bad, g_pack_bad, sizeof(bad), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "mq_pack_zeros");
    if (bad) return fail(MQ_ERR_UNSUPPORTED, "a zero point is NaN or overflows fp16");
    return MQ_OK;
}

extern "C" mq_status mq_unpack(const mq_weights *w, uint8_t *codes_out, void *stream) {
    if (!w) return fail(MQ_ERR_INVALID_ARG, "weights view is NULL");
    mq_status s = check_weights(w, w->N, w->K);
    if (s != MQ_OK) return s;
    if (!codes_out) return fail(MQ_ERR_INVALID_ARG, "codes_out is NULL");
    if (!aligned16(codes_out)) return fail(MQ_ERR_MISALIGNED, "codes_out must be 16-byte aligned");
    cudaStream_t st = (cudaStream_t)stream;
    if ((s = bind_device(st)) != MQ_OK) return s;
    const int64_t words = w->N * (w->K / 32);
    unpack_kernel<<<grid_for(words, 256), 256, 0, st>>>(w->planes, w->N, w->K, w->r,
                                                        codes_out);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "unpack_kernel");
    return MQ_OK;
}
