// Batched path (M >= 9): tcgen05 tensor-core GEMM over decoded r-bit tiles.
//
// The r-bit levels v_r = 2^(8-r) q_r + 2^(7-r) - 128 are exact in bf16 (at
// most 8 significant bits), so the MMA operands are exact:
//     D_g[n, m] = sum_{k in group g} v_r[n, k] * x[m, k]     (fp32, in TMEM)
//     Y[m, n]   = sum_g s[n, g] * D_g[n, m]                  (fp32 registers)
// One CTA owns 128 weight rows and BM rows of X.  Per 128-column group it
// decodes its rows' r planes into a 128 x 128 bf16 tile (K-major, 128-byte
// swizzle) in shared memory, stages the matching X tile, issues eight
// 128 x BM x 16 MMAs from one thread, and folds the group into fp32
// accumulators with the group's scale.  Decoding emits columns within each
// 32-column word in the order 4e + j <- k = 8j + e, so X is first copied into
// the workspace in that order (prep kernel); the contraction is unchanged.
#include "mq_common.cuh"
#include "mq_sm100.cuh"

namespace mq {
namespace {

using namespace sm100;

constexpr int kTcThreads = 128;
constexpr int kTileN = 128;

__device__ unsigned int g_tc_timeout;      // set when a bounded wait gave up

// Stage A/B/C transposition (same network as the GEMV): byte j of out[e] is
// q_r << (8 - r) of column 8 j + e.
template <int R>
__device__ __forceinline__ void tc_planes_to_bytes(const uint32_t (&P)[8], uint32_t (&out)[8]) {
    uint32_t A[4][2];
#pragma unroll
    for (int pp = 0; pp < 4; ++pp) {
        const uint32_t a = (2 * pp < R) ? P[2 * pp] : 0u;
        const uint32_t b = (2 * pp + 1 < R) ? P[2 * pp + 1] : 0u;
        A[pp][1] = (a & 0xAAAAAAAAu) | ((b >> 1) & 0x55555555u);
        A[pp][0] = ((a << 1) & 0xAAAAAAAAu) | (b & 0x55555555u);
    }
    uint32_t Bq[2][4];
#pragma unroll
    for (int qd = 0; qd < 2; ++qd)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint32_t x = A[2 * qd][c], y = A[2 * qd + 1][c];
            Bq[qd][c] = ((x << 2) & 0xCCCCCCCCu) | (y & 0x33333333u);
            Bq[qd][2 + c] = (x & 0xCCCCCCCCu) | ((y >> 2) & 0x33333333u);
        }
#pragma unroll
    for (int d = 0; d < 4; ++d) {
        const uint32_t x = Bq[0][d], y = Bq[1][d];
        out[d] = ((x << 4) & 0xF0F0F0F0u) | (y & 0x0F0F0F0Fu);
        out[4 + d] = (x & 0xF0F0F0F0u) | ((y >> 4) & 0x0F0F0F0Fu);
    }
}

// Two bf16 levels (bytes j0 and j0+1 of E, E's bytes hold q_r << (8 - r)).
template <int R>
__device__ __forceinline__ uint32_t levels_bf16x2(uint32_t E, int j0) {
    if constexpr (R <= 6) {
        // bf16 bits 0x4380 | (b >> 1) encode 256 + b (b even): one byte
        // permute builds two of them, one exact subtraction centres them
        // (384 - 2^(7-r) is exact in bf16 for r <= 6).
        const uint32_t F = ((E >> 1) & 0x7F7F7F7Fu) | 0x80808080u;
        const uint32_t h = __byte_perm(F, 0x43434343u, j0 == 0 ? 0x4140 : 0x4342);
        const float c = 384.0f - (float)(1 << (7 - R));
        const __nv_bfloat162 off = __floats2bfloat162_rn(c, c);
        __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162 *>(&h);
        v = __hsub2(v, off);
        return *reinterpret_cast<uint32_t *>(&v);
    } else {
        // through fp32: 2^22 + b has a 0.5 ulp, so subtracting
        // 2^22 + 128 - 2^(7-r) is exact and leaves v_r
        constexpr float c = 4194432.0f - (R == 8 ? 0.5f : 1.0f);
        const uint32_t b0 = (E >> (8 * j0)) & 0xFFu, b1 = (E >> (8 * j0 + 8)) & 0xFFu;
        const float f0 = __uint_as_float(0x4A800000u | (b0 << 1)) - c;
        const float f1 = __uint_as_float(0x4A800000u | (b1 << 1)) - c;
        __nv_bfloat162 v = __floats2bfloat162_rn(f0, f1);
        return *reinterpret_cast<uint32_t *>(&v);
    }
}

// X rows, each 32-column block permuted to the decode order 4e + j <- 8j + e;
// rows M..Mp-1 are zero.
__global__ void __launch_bounds__(256)
x_permute_kernel(const uint16_t *__restrict__ X, int M, int Mp, int64_t K,
                 uint16_t *__restrict__ Xp) {
    const int64_t blocks = (int64_t)Mp * (K / 32);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < blocks;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t m = i / (K / 32), b = i % (K / 32);
        uint16_t in[32], out[32];
        if (m < M) {
            const uint4 *src = reinterpret_cast<const uint4 *>(X + m * K + b * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v) *reinterpret_cast<uint4 *>(in + 8 * v) = src[v];
        } else {
#pragma unroll
            for (int v = 0; v < 32; ++v) in[v] = 0;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e)
#pragma unroll
            for (int j = 0; j < 4; ++j) out[4 * e + j] = in[8 * j + e];
        uint4 *dst = reinterpret_cast<uint4 *>(Xp + m * K + b * 32);
#pragma unroll
        for (int v = 0; v < 4; ++v) dst[v] = *reinterpret_cast<uint4 *>(out + 8 * v);
    }
}

template <int R, int BM>
__global__ void __launch_bounds__(kTcThreads)
gemm_tc_kernel(const uint16_t *__restrict__ Xp, const uint32_t *__restrict__ planes,
               const __half *__restrict__ scales, int M, int64_t N, int64_t K,
               int groups_per_split, int KS, float *__restrict__ part,
               unsigned *__restrict__ tickets, __nv_bfloat16 *__restrict__ Y) {
    constexpr int kCols = BM < 32 ? 32 : BM;                // TMEM columns (power of 2)
    constexpr uint32_t kIdesc = idesc_bf16_f32(kTileN, BM);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // align the base by an offset so the compiler keeps the shared address space
    uint8_t *base = smem_raw + ((1024u - (static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw)) & 1023u)) & 1023u);
    uint8_t *sA = base;
    uint8_t *sB = base + 2 * kTileN * 128;
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int s_last;

    const int t = threadIdx.x, warp = t >> 5;
    const int64_t G = K / kGroup;
    const int64_t n0 = (int64_t)blockIdx.x * kTileN;
    const int m0 = blockIdx.y * BM;
    const int64_t gbeg = (int64_t)blockIdx.z * groups_per_split;
    const int64_t gend = (gbeg + groups_per_split < G) ? gbeg + groups_per_split : G;

    if (warp == 0) { tmem_alloc(&tmem_slot, kCols); tmem_relinquish(); }
    if (t == 0) { mbar_init(&bar, 1); fence_mbar_init(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t taddr = tmem_slot;

    const int64_t n = n0 + t;
    const bool row_ok = n < N;
    const int64_t plane_words = (N + 127) / 128 * 128 * (K / 32);   // tiled planes
    float y[BM];
#pragma unroll
    for (int c = 0; c < BM; ++c) y[c] = 0.f;
    uint32_t phase = 0;
    bool ok = true;

    // The next group's plane words, scale and X chunks are loaded into
    // registers while the current group is decoded and multiplied (the loop
    // is otherwise bound by the global-load latency of every group).
    constexpr bool kPrefetch = R * 8 + BM <= 96;
    constexpr int kXv = BM * 16 / kTcThreads;            // X chunks per thread (BM <= 32)
    uint4 pvn[R];
    float sn = 0.f;
    uint4 xvn[kXv > 0 && BM <= 32 ? kXv : 1];
    auto load_group = [&](int64_t g) {
#pragma unroll
        for (int p = 0; p < R; ++p)
            pvn[p] = *reinterpret_cast<const uint4 *>(planes + p * plane_words +
                                                      ((int64_t)blockIdx.x * G + g) * 512 + t * 4);
        sn = __half2float(scales[((int64_t)blockIdx.x * G + g) * 128 + t]);
        if constexpr (BM <= 32) {
#pragma unroll
            for (int i = 0; i < kXv; ++i) {
                const int idx = t + i * kTcThreads, row = idx >> 4, c = idx & 15;
                xvn[i] = *reinterpret_cast<const uint4 *>(Xp + (int64_t)(m0 + row) * K + g * kGroup + c * 8);
            }
        }
    };
    if (kPrefetch && gbeg < gend) load_group(gbeg);

    for (int64_t g = gbeg; g < gend; ++g) {
        // ---- decode this thread's row of the A tile
        uint4 pv[R];
        float s;
        uint4 xv[kXv > 0 && BM <= 32 ? kXv : 1];
        if constexpr (kPrefetch) {
#pragma unroll
            for (int p = 0; p < R; ++p) pv[p] = pvn[p];
            s = sn;
            if constexpr (BM <= 32) {
#pragma unroll
                for (int i = 0; i < kXv; ++i) xv[i] = xvn[i];
            }
            if (g + 1 < gend) load_group(g + 1);
        } else {
#pragma unroll
            for (int p = 0; p < R; ++p)
                pv[p] = *reinterpret_cast<const uint4 *>(planes + p * plane_words +
                                                         ((int64_t)blockIdx.x * G + g) * 512 + t * 4);
            s = __half2float(scales[((int64_t)blockIdx.x * G + g) * 128 + t]);
        }
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            uint32_t P[8], E[8];
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const uint4 &v = pv[p < R ? p : 0];
                P[p] = p < R ? (w == 0 ? v.x : w == 1 ? v.y : w == 2 ? v.z : v.w) : 0u;
            }
            tc_planes_to_bytes<R>(P, E);
#pragma unroll
            for (int cq = 0; cq < 4; ++cq) {              // 8 columns: words 2cq, 2cq+1
                uint4 chunk;
                chunk.x = levels_bf16x2<R>(E[2 * cq], 0);
                chunk.y = levels_bf16x2<R>(E[2 * cq], 2);
                chunk.z = levels_bf16x2<R>(E[2 * cq + 1], 0);
                chunk.w = levels_bf16x2<R>(E[2 * cq + 1], 2);
                const int c = 4 * w + cq;                 // 16-byte chunk of the row
                *reinterpret_cast<uint4 *>(sA + (c >> 3) * (kTileN * 128) +
                                           sw128_offset(t, c & 7)) = chunk;
            }
        }
        // ---- stage the X tile (already in decode order)
        if constexpr (kPrefetch && BM <= 32) {
#pragma unroll
            for (int i = 0; i < kXv; ++i) {
                const int idx = t + i * kTcThreads, row = idx >> 4, c = idx & 15;
                *reinterpret_cast<uint4 *>(sB + (c >> 3) * (BM * 128) + sw128_offset(row, c & 7)) = xv[i];
            }
        } else {
            for (int idx = t; idx < BM * 16; idx += kTcThreads) {
                const int row = idx >> 4, c = idx & 15;
                const uint4 v = *reinterpret_cast<const uint4 *>(
                    Xp + (int64_t)(m0 + row) * K + g * kGroup + c * 8);
                *reinterpret_cast<uint4 *>(sB + (c >> 3) * (BM * 128) + sw128_offset(row, c & 7)) = v;
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- eight K=16 MMAs into TMEM, one issuing thread
        if (t == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int h = ks >> 2, kk = ks & 3;
                const uint64_t ad = smem_desc_sw128(smem_u32(sA + h * (kTileN * 128) + kk * 32));
                const uint64_t bd = smem_desc_sw128(smem_u32(sB + h * (BM * 128) + kk * 32));
                mma_bf16(taddr, ad, bd, kIdesc, ks > 0 ? 1u : 0u);
            }
            mma_commit(&bar);
        }
        const bool mine = mbar_wait_bounded(&bar, phase);
        phase ^= 1u;
        if (!__syncthreads_and(mine)) { ok = false; break; }
        tc_fence_after();

        // ---- fold this group in: y[m] += s[n, g] * D_g[n, m]
#pragma unroll
        for (int cb = 0; cb < BM / 16; ++cb) {
            float v[16];
            { uint32_t u[16]; tmem_ld16(taddr + ((uint32_t)(32 * warp) << 16) + cb * 16, u); for (int q = 0; q < 16; ++q) v[q] = __uint_as_float(u[q]); }
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) y[cb * 16 + i] = fmaf(s, v[i], y[cb * 16 + i]);
        }
        tc_fence_before();
        __syncthreads();
    }

    if (!ok) {
        if (t == 0) atomicOr(&g_tc_timeout, 1u);
    } else if (KS == 1) {
        if (row_ok)
#pragma unroll
            for (int c = 0; c < BM; ++c)
                if (m0 + c < M) Y[(int64_t)(m0 + c) * N + n] = __float2bfloat16_rn(y[c]);
    } else {
        if (row_ok) {
#pragma unroll
            for (int c = 0; c < BM; ++c)
                if (m0 + c < M) part[((int64_t)blockIdx.z * M + m0 + c) * N + n] = y[c];
            __threadfence();
        }
        __syncthreads();
        const unsigned tk = blockIdx.y * gridDim.x + blockIdx.x;
        if (t == 0) s_last = atomicAdd(&tickets[tk], 1u) == (unsigned)KS - 1;
        __syncthreads();
        if (s_last) {
            __threadfence();
            if (row_ok)
                for (int c = 0; c < BM && m0 + c < M; ++c) {
                    float a = 0.f;
                    for (int z = 0; z < KS; ++z)
                        a += __ldcg(part + ((int64_t)z * M + m0 + c) * N + n);
                    Y[(int64_t)(m0 + c) * N + n] = __float2bfloat16_rn(a);
                }
            if (t == 0) tickets[tk] = 0u;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) { tc_fence_after(); tmem_dealloc(taddr, kCols); }
}

struct TcPlan {
    int BM, tiles_m, Mp, KS, gps;
    int64_t tiles_n;
    size_t part_off, xp_off, ws_bytes, smem;
};

TcPlan tc_plan(int64_t M, int64_t N, int64_t K) {
    TcPlan p{};
    p.BM = M <= 16 ? 16 : 32;                 // more CTAs beat larger X tiles (measured)
    p.tiles_m = (int)((M + p.BM - 1) / p.BM);
    p.Mp = p.tiles_m * p.BM;
    p.tiles_n = (N + kTileN - 1) / kTileN;
    const int64_t G = K / kGroup;
    int64_t ks = (2 * 148 + p.tiles_n * p.tiles_m - 1) / (p.tiles_n * p.tiles_m);
    if (ks < 1) ks = 1;
    if (ks > G) ks = G;
    p.gps = (int)((G + ks - 1) / ks);
    p.KS = (int)((G + p.gps - 1) / p.gps);
    p.part_off = kTicketBytes;
    const size_t part = p.KS > 1 ? (size_t)p.KS * M * N * sizeof(float) : 0;
    p.xp_off = (p.part_off + part + 1023) & ~(size_t)1023;
    p.ws_bytes = p.xp_off + (size_t)p.Mp * K * sizeof(uint16_t);
    p.smem = 1024 + 2 * kTileN * 128 + 2 * (size_t)p.BM * 128;
    return p;
}

using TcFn = void (*)(const uint16_t *, const uint32_t *, const __half *, int, int64_t, int64_t,
                      int, int, float *, unsigned *, __nv_bfloat16 *);

template <int R>
TcFn tc_pick_bm(int BM) {
    switch (BM) {
        case 16: return gemm_tc_kernel<R, 16>;
        case 32: return gemm_tc_kernel<R, 32>;
        case 64: return gemm_tc_kernel<R, 64>;
        default: return gemm_tc_kernel<R, 128>;
    }
}

TcFn tc_pick(int r, int BM) {
    switch (r) {
        case 1: return tc_pick_bm<1>(BM);
        case 2: return tc_pick_bm<2>(BM);
        case 3: return tc_pick_bm<3>(BM);
        case 4: return tc_pick_bm<4>(BM);
        case 5: return tc_pick_bm<5>(BM);
        case 6: return tc_pick_bm<6>(BM);
        case 7: return tc_pick_bm<7>(BM);
        default: return tc_pick_bm<8>(BM);
    }
}

}  // namespace

size_t gemm_tc_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
    (void)r;
    return tc_plan(M, N, K).ws_bytes;
}

mq_status launch_gemm_tc(const uint16_t *X, const mq_weights *w, int64_t M, uint16_t *Y,
                         void *ws, size_t ws_bytes, cudaStream_t st) {
    const TcPlan p = tc_plan(M, w->N, w->K);
    if (p.ws_bytes > ws_bytes) return fail(MQ_ERR_WORKSPACE, "GEMM workspace too small");
    if (p.tiles_n * p.tiles_m > (int64_t)(kTicketBytes / sizeof(unsigned)))
        return fail(MQ_ERR_UNSUPPORTED, "too many output tiles for the ticket region");
    char *wsb = static_cast<char *>(ws);
    uint16_t *Xp = reinterpret_cast<uint16_t *>(wsb + p.xp_off);
    const int64_t blocks = (int64_t)p.Mp * (w->K / 32);
    int grid = (int)((blocks + 255) / 256);
    if (grid > 148 * 16) grid = 148 * 16;
    x_permute_kernel<<<grid, 256, 0, st>>>(X, (int)M, p.Mp, w->K, Xp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "x_permute_kernel");
    TcFn fn = tc_pick(w->r, p.BM);
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    dim3 g3((unsigned)p.tiles_n, (unsigned)p.tiles_m, (unsigned)p.KS);
    fn<<<g3, kTcThreads, p.smem, st>>>(
        Xp, w->planes, reinterpret_cast<const __half *>(w->scales), (int)M, w->N, w->K,
        p.gps, p.KS, reinterpret_cast<float *>(wsb + p.part_off),
        reinterpret_cast<unsigned *>(wsb), reinterpret_cast<__nv_bfloat16 *>(Y));
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "gemm_tc_kernel");
    return MQ_OK;
}

bool gemm_tc_take_timeout(bool *set) {
    unsigned v = 0, z = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc_timeout, sizeof(v)) != cudaSuccess) return false;
    if (v && cudaMemcpyToSymbol(g_tc_timeout, &z, sizeof(z)) != cudaSuccess) return false;
    *set = v != 0;
    return true;
}

}  // namespace mq
