// Split-K CUDA-core GEMV for the nested r-bit format, batch M <= 8.
//
// Work item: one thread owns one 128-column group g of RT consecutive rows.
// For each row it loads exactly r 16-byte vectors (one per plane: the r-bit
// model reads r bits per weight, MatGPTQ abstract), rebuilds the r-bit codes
// in registers, and accumulates  sum_k x[m,k] * f_k  in fp32, where
//     f_k = 1 + (q_r + 1/2) / 2^r   (exact in fp32; its bits are 0x3F8 | code)
//     v_r = 2^(8-r) q_r + 2^(7-r) - 128 = 256 (f_k - 3/2),
// so a group contributes  s_g * 256 * (sum_k x f_k - 3/2 sum_k x).
// The Gc threads of a row block sit in consecutive lanes: their plane loads
// are contiguous 16-byte vectors and their partial sums meet in warp
// shuffles.  K slices (blockIdx.y) are combined in fixed order by the last
// CTA of each row tile to arrive (atomic ticket, no waiting).
#include "mq_common.cuh"

namespace mq {
namespace {

constexpr int kThreads = 256;
constexpr int kXPad = 4;                 // floats of padding per staged group

struct GemvPlan {
    int MB, Gc, RT, KS, B;               // B = row blocks per CTA
    int64_t tiles;                       // CTAs along N
    size_t part_bytes, ws_bytes;          // part_bytes: offset of the partial sums
};

int pow2_floor(int64_t v) { int p = 1; while ((int64_t)p * 2 <= v) p *= 2; return p; }

GemvPlan make_plan(int64_t M, int64_t N, int64_t K, int r) {
    GemvPlan p{};
    p.MB = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8;
    const int64_t G = K / kGroup;
    int cap = 32 / p.MB;                               // staged x stays <= 17 KB
    int g2 = 1;                                        // largest 2^i dividing G
    while (g2 < cap && G % (g2 * 2) == 0) g2 *= 2;
    p.Gc = (g2 >= 4 || G <= cap) ? g2 : cap;
    if (p.Gc < 4 && G >= 4) p.Gc = 4;
    if (p.Gc > G) p.Gc = pow2_floor(G);
    p.KS = (int)((G + p.Gc - 1) / p.Gc);
    p.B = kThreads / p.Gc;
    const int rt_max = r >= 7 ? 2 : 4;
    p.RT = 1;
    for (int rt = rt_max; rt >= 1; rt /= 2) {
        const int64_t tiles = (N + (int64_t)p.B * rt - 1) / ((int64_t)p.B * rt);
        if (tiles * p.KS >= 2 * 148 || rt == 1) { p.RT = rt; break; }
    }
    p.tiles = (N + (int64_t)p.B * p.RT - 1) / ((int64_t)p.B * p.RT);
    if (p.KS > 1) {
        // tickets first, at a fixed place: a call with a different shape must
        // never find another call's partial sums where its tickets live
        p.part_bytes = kTicketBytes;
        p.ws_bytes = kTicketBytes + (((size_t)p.KS * M * N * sizeof(float) + 255) & ~(size_t)255);
    }
    return p;
}

// Stage A/B/C of a bit-matrix transpose by masked shifts: from the r plane
// words of 32 columns to 8 words of bytes; byte j of out[e] is the r-bit code
// of column 8 j + e, most significant plane in bit 7 (i.e. q_r << (8 - r)).
template <int R>
__device__ __forceinline__ void planes_to_bytes(const uint32_t (&P)[8], uint32_t (&out)[8]) {
    uint32_t A[4][2];                      // [plane pair][class c]: column 2i + c
#pragma unroll
    for (int pp = 0; pp < 4; ++pp) {
        const uint32_t a = (2 * pp < R) ? P[2 * pp] : 0u;
        const uint32_t b = (2 * pp + 1 < R) ? P[2 * pp + 1] : 0u;
        A[pp][1] = (a & 0xAAAAAAAAu) | ((b >> 1) & 0x55555555u);
        A[pp][0] = ((a << 1) & 0xAAAAAAAAu) | (b & 0x55555555u);
    }
    uint32_t Bq[2][4];                     // [plane quad][class d]: column 4j + d
#pragma unroll
    for (int qd = 0; qd < 2; ++qd) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint32_t x = A[2 * qd][c], y = A[2 * qd + 1][c];
            Bq[qd][c] = ((x << 2) & 0xCCCCCCCCu) | (y & 0x33333333u);
            Bq[qd][2 + c] = (x & 0xCCCCCCCCu) | ((y >> 2) & 0x33333333u);
        }
    }
#pragma unroll
    for (int d = 0; d < 4; ++d) {
        const uint32_t x = Bq[0][d], y = Bq[1][d];
        out[d] = ((x << 4) & 0xF0F0F0F0u) | (y & 0x0F0F0F0Fu);
        out[4 + d] = (x & 0xF0F0F0F0u) | ((y >> 4) & 0x0F0F0F0Fu);
    }
}

// f = 1 + (q_r + 1/2) / 2^r from a byte holding q_r << (8 - r).
template <int R>
__device__ __forceinline__ float level_f(uint32_t word, int j) {
    const uint32_t byte = (word >> (8 * j)) & 0xFFu;
    return __uint_as_float(0x3F800000u | (1u << (22 - R)) | (byte << 15));
}

__device__ __forceinline__ uint4 ld_stream(const uint32_t *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

template <int R, int MB, int RT>
__global__ void __launch_bounds__(kThreads)
gemv_kernel(const __nv_bfloat16 *__restrict__ X, const uint32_t *__restrict__ planes,
            const __half *__restrict__ scales, int M, int64_t N, int64_t K, int Gc, int KS,
            float *__restrict__ part, unsigned *__restrict__ tickets,
            __nv_bfloat16 *__restrict__ Y) {
    extern __shared__ float xs[];        // [MB][Gc][128 + kXPad], permuted columns
    __shared__ int s_last;
    const int tid = threadIdx.x;
    const int gl = tid % Gc, blk = tid / Gc;
    const int B = kThreads / Gc;
    const int64_t G = K / kGroup;
    const int ks = blockIdx.y;
    const int64_t g = (int64_t)ks * Gc + gl;
    const int gstride = kGroup + kXPad;

    // ---- stage this K slice of X as fp32, columns permuted to decode order
    const int64_t k0 = (int64_t)ks * Gc * kGroup;
    const int span = Gc * kGroup;
    for (int idx = tid * 8; idx < MB * span; idx += kThreads * 8) {
        const int m = idx / span, kk = idx % span;
        const int gg = kk / kGroup, within = kk % kGroup;
        const int w = within / 32, jj = (within % 32) / 8;   // 8 columns: e = 0..7
        float v[8];
        if (m < M && k0 + kk < K) {
            const uint4 raw = *reinterpret_cast<const uint4 *>(X + (int64_t)m * K + k0 + kk);
            const uint32_t r4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                v[2 * h] = __uint_as_float(r4[h] << 16);
                v[2 * h + 1] = __uint_as_float(r4[h] & 0xFFFF0000u);
            }
        } else {
#pragma unroll
            for (int h = 0; h < 8; ++h) v[h] = 0.f;
        }
        float *dst = xs + (m * Gc + gg) * gstride + w * 32 + jj;
#pragma unroll
        for (int e = 0; e < 8; ++e) dst[e * 4] = v[e];
    }
    __syncthreads();

    // ---- per-thread group sums of x (fixed order)
    float S[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) {
        const float4 *xr = reinterpret_cast<const float4 *>(xs + (m * Gc + gl) * gstride);
        float a = 0.f;
#pragma unroll 8
        for (int c = 0; c < 32; ++c) { const float4 t = xr[c]; a += (t.x + t.y) + (t.z + t.w); }
        S[m] = a;
    }

    // ---- load r plane vectors for RT rows (all in flight at once)
    const int64_t row0 = ((int64_t)blockIdx.x * B + blk) * RT;
    const int64_t plane_words = N * (K / 32);
    uint4 pv[RT][R];
    float sc[RT];
#pragma unroll
    for (int i = 0; i < RT; ++i) {
        const int64_t n = row0 + i;
        const bool ok = (n < N) && (g < G);
#pragma unroll
        for (int p = 0; p < R; ++p)
            pv[i][p] = ok ? ld_stream(planes + p * plane_words + n * (K / 32) + g * 4)
                          : make_uint4(0, 0, 0, 0);
        sc[i] = ok ? __half2float(scales[n * G + g]) : 0.f;
    }

    float acc[RT][MB];
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int m = 0; m < MB; ++m) acc[i][m] = 0.f;

#pragma unroll
    for (int w = 0; w < 4; ++w) {
        uint32_t by[RT][8];
#pragma unroll
        for (int i = 0; i < RT; ++i) {
            uint32_t P[8];
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const uint4 &v = pv[i][p < R ? p : 0];
                const uint32_t word = w == 0 ? v.x : w == 1 ? v.y : w == 2 ? v.z : v.w;
                P[p] = p < R ? word : 0u;
            }
            planes_to_bytes<R>(P, by[i]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
#pragma unroll
            for (int m = 0; m < MB; ++m) {
                const float4 x4 = *reinterpret_cast<const float4 *>(
                    xs + (m * Gc + gl) * gstride + w * 32 + e * 4);
#pragma unroll
                for (int i = 0; i < RT; ++i) {
                    acc[i][m] = fmaf(x4.x, level_f<R>(by[i][e], 0), acc[i][m]);
                    acc[i][m] = fmaf(x4.y, level_f<R>(by[i][e], 1), acc[i][m]);
                    acc[i][m] = fmaf(x4.z, level_f<R>(by[i][e], 2), acc[i][m]);
                    acc[i][m] = fmaf(x4.w, level_f<R>(by[i][e], 3), acc[i][m]);
                }
            }
        }
    }

    // ---- group scale, then sum the Gc groups of the slice across lanes
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int m = 0; m < MB; ++m) {
            float y = sc[i] * fmaf(-1.5f, S[m], acc[i][m]);
            for (int off = Gc / 2; off >= 1; off /= 2)
                y += __shfl_xor_sync(0xffffffffu, y, off);
            acc[i][m] = y;
        }

    if (KS == 1) {
        if (gl == 0) {
#pragma unroll
            for (int i = 0; i < RT; ++i)
#pragma unroll
                for (int m = 0; m < MB; ++m)
                    if (m < M && row0 + i < N)
                        Y[(int64_t)m * N + row0 + i] = __float2bfloat16_rn(256.f * acc[i][m]);
        }
        return;
    }

    // ---- split K: publish the partial, the last CTA of this row tile reduces
    if (gl == 0) {
#pragma unroll
        for (int i = 0; i < RT; ++i)
#pragma unroll
            for (int m = 0; m < MB; ++m)
                if (m < M && row0 + i < N)
                    part[((int64_t)ks * M + m) * N + row0 + i] = acc[i][m];
        __threadfence();
    }
    __syncthreads();
    if (tid == 0) {
        const unsigned t = atomicAdd(&tickets[blockIdx.x], 1u);
        s_last = (t == (unsigned)KS - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int rows = B * RT;
    const int64_t tile0 = (int64_t)blockIdx.x * rows;
    for (int idx = tid; idx < rows * M; idx += kThreads) {
        const int m = idx / rows;
        const int64_t n = tile0 + idx % rows;
        if (n >= N) continue;
        float y = 0.f;
        for (int s = 0; s < KS; ++s) y += __ldcg(part + ((int64_t)s * M + m) * N + n);
        Y[(int64_t)m * N + n] = __float2bfloat16_rn(256.f * y);
    }
    if (tid == 0) tickets[blockIdx.x] = 0u;   // leave the workspace zero-filled
}

}  // namespace

namespace {

using GemvFn = void (*)(const __nv_bfloat16 *, const uint32_t *, const __half *, int,
                        int64_t, int64_t, int, int, float *, unsigned *, __nv_bfloat16 *);

template <int R, int MB>
GemvFn pick_rt(int RT) {
    if (RT == 4) { if constexpr (R <= 6) return gemv_kernel<R, MB, 4>; }
    if (RT >= 2) return gemv_kernel<R, MB, 2>;
    return gemv_kernel<R, MB, 1>;
}

template <int R>
GemvFn pick_mb(int MB, int RT) {
    switch (MB) {
        case 1: return pick_rt<R, 1>(RT);
        case 2: return pick_rt<R, 2>(RT);
        case 4: return pick_rt<R, 4>(RT);
        default: return pick_rt<R, 8>(RT);
    }
}

GemvFn pick(int r, int MB, int RT) {
    switch (r) {
        case 1: return pick_mb<1>(MB, RT);
        case 2: return pick_mb<2>(MB, RT);
        case 3: return pick_mb<3>(MB, RT);
        case 4: return pick_mb<4>(MB, RT);
        case 5: return pick_mb<5>(MB, RT);
        case 6: return pick_mb<6>(MB, RT);
        case 7: return pick_mb<7>(MB, RT);
        default: return pick_mb<8>(MB, RT);
    }
}

}  // namespace

size_t gemv_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
    return make_plan(M, N, K, r).ws_bytes;
}

mq_status launch_gemv(const uint16_t *X, const mq_weights *w, int64_t M, uint16_t *Y,
                      void *ws, size_t ws_bytes, cudaStream_t st) {
    const GemvPlan p = make_plan(M, w->N, w->K, w->r);
    if (p.ws_bytes > ws_bytes) return fail(MQ_ERR_WORKSPACE, "GEMV workspace too small");
    if (p.KS > 1 && p.tiles > (int64_t)(kTicketBytes / sizeof(unsigned)))
        return fail(MQ_ERR_UNSUPPORTED, "too many row tiles for the split-K ticket region");
    unsigned *tickets = p.KS > 1 ? reinterpret_cast<unsigned *>(ws) : nullptr;
    float *part = p.KS > 1
        ? reinterpret_cast<float *>(static_cast<char *>(ws) + kTicketBytes) : nullptr;
    const size_t smem = (size_t)p.MB * p.Gc * (kGroup + kXPad) * sizeof(float);
    dim3 grid((unsigned)p.tiles, (unsigned)p.KS);
    GemvFn fn = pick(w->r, p.MB, p.RT);
    fn<<<grid, kThreads, smem, st>>>(
        reinterpret_cast<const __nv_bfloat16 *>(X), w->planes,
        reinterpret_cast<const __half *>(w->scales), (int)M, w->N, w->K, p.Gc, p.KS,
        part, tickets, reinterpret_cast<__nv_bfloat16 *>(Y));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "gemv_kernel");
    return MQ_OK;
}

}  // namespace mq
