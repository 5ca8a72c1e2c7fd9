// Batch M <= 8: bit planes -> bf16 operand fragments in registers -> mma.sync.
//
// Why not CUDA-core FMAs: turning a weight into a float costs integer/logic
// instructions, which B200 issues at half the fp32 rate, and the multiply-add
// then costs one more instruction per weight and batch row.  Here a single
// LOP3 builds two bf16 operands, and the warp-level MMA m16n8k16 (16 weight
// rows x 8 batch rows x 16 columns) does every multiply-add; its n = 8 covers
// M = 1..8 at the same cost.
//
// Operand construction.  Each lane owns one 32-column word of a 128-column
// group for weight rows g and g + 8 (g = lane / 4, word t = lane % 4), reads
// exactly r plane words per row (the r-bit model reads r bits per weight), and
// rearranges them into "field words" whose fields hold the r-bit code q (or
// 2q / a 4-bit part of it).  A field of width W at bit position p of a bf16
// mantissa gives the exact bf16 value
//          A = 1 + field * 2^(p - 7)          (bits 0x3F80 | field << p)
// and the matching X operand is x * 2^(7 - p) (exact power-of-two scaling),
// so A * B = x * 2^(7 - p) + x * field.  Per group g and batch row m:
//     D = C0 + 2^e sum_k x q,   C0 = sum of the B operands of the group,
//     sum_k x v_r = alpha (D - C0) + c_r S,  alpha = 2^(8 - r - e),
//     c_r = 2^(7 - r) - 128,  S = sum_k x,
// hence  y[n, m] += s[n, g] (alpha D - E[g, m]),  E = alpha C0 - c_r S.
// A prep kernel writes the B fragments and E for the call; the main kernel
// streams the planes, issues the MMAs and applies the group scales in fp32.
#include "mq_common.cuh"

namespace mq {
namespace {

// ----------------------------------------------------------- operand tables
// One register = two bf16 operands: field f of the low half and the field
// at the same place in the high half of field word `fw` after a right shift.
struct Entry { int fw, shift, p, f; };

template <int R> struct Layout;   // field words, registers per row, fields

// r = 1: the plane word itself, 1-bit fields, column k = f.
template <> struct Layout<1> {
    static constexpr int W = 1, NFW = 1, NREG = 16, E_EXP = 0;
    __host__ __device__ static constexpr Entry entry(int i) {
        return i < 7 ? Entry{0, 0, i, i} : i < 14 ? Entry{0, 7, i - 7, i} : Entry{0, 14, i - 14, i};
    }
    __host__ __device__ static constexpr int col(int fw, int f) { return f; }
    __host__ __device__ static constexpr int part(int fw) { return 0; }
};

// r = 2: 2-bit fields q; word 0 holds even columns (k = 2f), word 1 odd.
template <> struct Layout<2> {
    static constexpr int W = 2, NFW = 2, NREG = 16, E_EXP = 0;
    __host__ __device__ static constexpr Entry entry(int i) {
        const int w = i / 8, j = i % 8;
        return j < 3 ? Entry{w, 0, 2 * j, j} : j < 6 ? Entry{w, 6, 2 * (j - 3), j}
                                                 : Entry{w, 12, 2 * (j - 6), j};
    }
    __host__ __device__ static constexpr int col(int fw, int f) { return 2 * f + fw; }
    __host__ __device__ static constexpr int part(int fw) { return 0; }
};

// r = 3, 4: nibble fields (q, or 2q for r = 3); word d holds k = 4f + d.
// r >= 5: words 0..3 hold the top nibble of q << (8 - r), words 4..7 the
// bottom one (weighted 16 : 1 through the X operand).
template <int R> struct Layout {
    static constexpr int W = 4, NFW = R <= 4 ? 4 : 8, NREG = R <= 4 ? 16 : 32;
    static constexpr int E_EXP = R == 3 ? 1 : R >= 5 ? 8 - R : 0;
    __host__ __device__ static constexpr Entry entry(int i) {
        return Entry{i / 4, 4 * (i % 4), 0, i % 4};
    }
    __host__ __device__ static constexpr int col(int fw, int f) { return 4 * f + (fw & 3); }
    __host__ __device__ static constexpr int part(int fw) { return (R >= 5 && fw < 4) ? 1 : 0; }
};

template <int R> __host__ __device__ constexpr int fields_per_half() {
    return 16 / Layout<R>::W;
}

// Field words from the r plane words of one 32-column word.
template <int R>
__device__ __forceinline__ void field_words(const uint32_t (&P)[8], uint32_t (&F)[8]) {
    if constexpr (R == 1) {
        F[0] = P[0];
    } else if constexpr (R == 2) {
        F[0] = ((P[0] << 1) & 0xAAAAAAAAu) | (P[1] & 0x55555555u);
        F[1] = (P[0] & 0xAAAAAAAAu) | ((P[1] >> 1) & 0x55555555u);
    } else {
#pragma unroll
        for (int half = 0; half < (R <= 4 ? 1 : 2); ++half) {
            const uint32_t p0 = P[4 * half], p1 = 4 * half + 1 < R ? P[4 * half + 1] : 0u;
            const uint32_t p2 = 4 * half + 2 < R ? P[4 * half + 2] : 0u;
            const uint32_t p3 = 4 * half + 3 < R ? P[4 * half + 3] : 0u;
            const uint32_t x0 = ((p0 << 1) & 0xAAAAAAAAu) | (p1 & 0x55555555u);   // k even
            const uint32_t x1 = (p0 & 0xAAAAAAAAu) | ((p1 >> 1) & 0x55555555u);   // k odd
            const uint32_t y0 = ((p2 << 1) & 0xAAAAAAAAu) | (p3 & 0x55555555u);
            const uint32_t y1 = (p2 & 0xAAAAAAAAu) | ((p3 >> 1) & 0x55555555u);
            F[4 * half + 0] = ((x0 << 2) & 0xCCCCCCCCu) | (y0 & 0x33333333u);
            F[4 * half + 1] = ((x1 << 2) & 0xCCCCCCCCu) | (y1 & 0x33333333u);
            F[4 * half + 2] = (x0 & 0xCCCCCCCCu) | ((y0 >> 2) & 0x33333333u);
            F[4 * half + 3] = (x1 & 0xCCCCCCCCu) | ((y1 >> 2) & 0x33333333u);
        }
    }
}

// bf16 pair for register i: (field words >> shift) & mask | 1.0 (x2).
template <int R>
__device__ __forceinline__ uint32_t operand_reg(const uint32_t (&F)[8], int i) {
    constexpr int W = Layout<R>::W;
    const Entry e = Layout<R>::entry(i);
    const uint32_t fmask = ((1u << W) - 1u) << e.p;
    return ((F[e.fw] >> e.shift) & (fmask | (fmask << 16))) | 0x3F803F80u;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int R>
__host__ __device__ constexpr float level_offset() { return (float)(1 << 7 >> (R - 1)) * 0.5f - 128.0f; }

// ------------------------------------------------------------ prep kernel
// B fragments of every group (bf16 pairs, per lane in MMA order) and E[g, m].
template <int R>
__global__ void __launch_bounds__(256)
bfrag_kernel(const __nv_bfloat16 *__restrict__ X, int M, int64_t K,
             uint32_t *__restrict__ bfrag, float *__restrict__ Eg) {
    using L = Layout<R>;
    constexpr int NREG = L::NREG, FPH = fields_per_half<R>();
    const int64_t G = K / kGroup;
    const int64_t total = G * 32 * NREG;                       // one uint32 per thread
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int i = (int)(idx % NREG);                        // register (2s + half)
        const int lane = (int)((idx / NREG) % 32);
        const int64_t grp = idx / (NREG * 32);
        const int m = lane >> 2, t = lane & 3;
        const Entry e = L::entry(i);
        float v[2] = {0.f, 0.f};
        if (m < M) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int f = e.f + h * FPH;
                const int64_t k = grp * kGroup + 32 * t + L::col(e.fw, f);
                const float sc = (float)(1 << (7 - e.p)) * (L::part(e.fw) ? 16.f : 1.f);
                v[h] = __bfloat162float(X[(int64_t)m * K + k]) * sc;
            }
        }
        __nv_bfloat162 b = __floats2bfloat162_rn(v[0], v[1]);   // exact: power-of-two scale
        bfrag[idx] = *reinterpret_cast<uint32_t *>(&b);
    }
    // E[g, m] = alpha * C0 - c_r * S, with C0 the sum of the group's B operands
    constexpr float alpha = (float)(1 << (8 - R - L::E_EXP));
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < G * 8;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t grp = idx / 8;
        const int m = (int)(idx % 8);
        float c0 = 0.f, s = 0.f;
        if (m < M) {
            for (int t = 0; t < 4; ++t)
                for (int i = 0; i < NREG; ++i) {
                    const Entry e = L::entry(i);
                    for (int h = 0; h < 2; ++h) {
                        const int f = e.f + h * FPH;
                        const float x = __bfloat162float(
                            X[(int64_t)m * K + grp * kGroup + 32 * t + L::col(e.fw, f)]);
                        c0 += x * (float)(1 << (7 - e.p)) * (L::part(e.fw) ? 16.f : 1.f);
                        s += x;
                    }
                }
        }
        Eg[idx] = alpha * c0 - level_offset<R>() * s;
    }
}

// ------------------------------------------------------------- main kernel
constexpr int kMmaWarps = 4;
constexpr int kBatch = 2;               // groups loaded per pipeline stage

__device__ __forceinline__ uint32_t ld_plane(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// One warp: 16 weight rows x a range of groups.  Warp task w -> (tile, split).
template <int R>
__global__ void __launch_bounds__(kMmaWarps * 32)
gemv_mma_kernel(const uint32_t *__restrict__ planes, const __half *__restrict__ scales,
                const uint32_t *__restrict__ bfrag, const float *__restrict__ Eg,
                int M, int64_t N, int64_t K, int64_t tiles, int KS, int gpt,
                float *__restrict__ part, unsigned *__restrict__ tickets,
                __nv_bfloat16 *__restrict__ Y) {
    using L = Layout<R>;
    constexpr int NREG = L::NREG, STEPS = NREG / 2;
    constexpr float alpha = (float)(1 << (8 - R - L::E_EXP));
    const int lane = threadIdx.x & 31;
    const int64_t task = (int64_t)blockIdx.x * kMmaWarps + (threadIdx.x >> 5);
    if (task >= tiles * KS) return;
    const int64_t tile = task / KS;
    const int ks = (int)(task % KS);
    const int g = lane >> 2, t = lane & 3;
    const int64_t G = K / kGroup;
    const int64_t g0 = (int64_t)ks * gpt;
    const int64_t g1 = g0 + gpt < G ? g0 + gpt : G;
    const int64_t n_lo = tile * 16 + g, n_hi = n_lo + 8;
    const bool ok_lo = n_lo < N, ok_hi = n_hi < N;
    const int64_t plane_words = N * (K / 32);
    const uint32_t *row_lo = planes + (ok_lo ? n_lo : 0) * (K / 32) + t;
    const uint32_t *row_hi = planes + (ok_hi ? n_hi : 0) * (K / 32) + t;
    const bool bvalid = g < M;

    float y[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t w[2][kBatch][2][R];          // [buffer][group][row][plane]
    float sc[2][kBatch][2];

    auto load = [&](int buf, int64_t gb) {
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const int64_t gg = gb + j;
            const bool in = gg < g1;
#pragma unroll
            for (int p = 0; p < R; ++p) {
                w[buf][j][0][p] = (in && ok_lo) ? ld_plane(row_lo + p * plane_words + gg * 4) : 0u;
                w[buf][j][1][p] = (in && ok_hi) ? ld_plane(row_hi + p * plane_words + gg * 4) : 0u;
            }
            sc[buf][j][0] = (in && ok_lo) ? __half2float(scales[n_lo * G + gg]) : 0.f;
            sc[buf][j][1] = (in && ok_hi) ? __half2float(scales[n_hi * G + gg]) : 0.f;
        }
    };

    auto compute = [&](int buf, int64_t gb) {
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const int64_t gg = gb + j;
            if (gg >= g1) break;
            uint32_t F[2][8], P[8];
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
#pragma unroll
                for (int p = 0; p < 8; ++p) P[p] = p < R ? w[buf][j][rr][p] : 0u;
                field_words<R>(P, F[rr]);
            }
            const uint4 *bp = reinterpret_cast<const uint4 *>(bfrag + (gg * 32 + lane) * NREG);
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int q4 = 0; q4 < NREG / 4; ++q4) {
                const uint4 b = bvalid ? __ldg(bp + q4) : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int hs = 0; hs < 2; ++hs) {         // two MMA steps per uint4
                    const int s = 2 * q4 + hs;
                    uint32_t a[4];
                    a[0] = operand_reg<R>(F[0], 2 * s);
                    a[1] = operand_reg<R>(F[1], 2 * s);
                    a[2] = operand_reg<R>(F[0], 2 * s + 1);
                    a[3] = operand_reg<R>(F[1], 2 * s + 1);
                    mma_bf16_16816(d, a, hs ? b.z : b.x, hs ? b.w : b.y);
                }
            }
            const float2 e = *reinterpret_cast<const float2 *>(Eg + gg * 8 + 2 * t);
            y[0] = fmaf(sc[buf][j][0], fmaf(alpha, d[0], -e.x), y[0]);
            y[1] = fmaf(sc[buf][j][0], fmaf(alpha, d[1], -e.y), y[1]);
            y[2] = fmaf(sc[buf][j][1], fmaf(alpha, d[2], -e.x), y[2]);
            y[3] = fmaf(sc[buf][j][1], fmaf(alpha, d[3], -e.y), y[3]);
        }
    };

    // two register buffers, static indices: load one stage ahead
    load(0, g0);
    for (int64_t gb = g0; gb < g1; gb += 2 * kBatch) {
        if (gb + kBatch < g1) load(1, gb + kBatch);
        compute(0, gb);
        if (gb + kBatch >= g1) break;
        if (gb + 2 * kBatch < g1) load(0, gb + 2 * kBatch);
        compute(1, gb + kBatch);
    }
    (void)STEPS;

    // ---- outputs: lane holds rows (n_lo, n_hi) x batch rows (2t, 2t+1)
    const int m0 = 2 * t;
    if (KS == 1) {
        if (ok_lo && m0 < M) Y[(int64_t)m0 * N + n_lo] = __float2bfloat16_rn(y[0]);
        if (ok_lo && m0 + 1 < M) Y[(int64_t)(m0 + 1) * N + n_lo] = __float2bfloat16_rn(y[1]);
        if (ok_hi && m0 < M) Y[(int64_t)m0 * N + n_hi] = __float2bfloat16_rn(y[2]);
        if (ok_hi && m0 + 1 < M) Y[(int64_t)(m0 + 1) * N + n_hi] = __float2bfloat16_rn(y[3]);
        return;
    }
    float *pk = part + (int64_t)ks * M * N;
    if (ok_lo && m0 < M) pk[(int64_t)m0 * N + n_lo] = y[0];
    if (ok_lo && m0 + 1 < M) pk[(int64_t)(m0 + 1) * N + n_lo] = y[1];
    if (ok_hi && m0 < M) pk[(int64_t)m0 * N + n_hi] = y[2];
    if (ok_hi && m0 + 1 < M) pk[(int64_t)(m0 + 1) * N + n_hi] = y[3];
    __threadfence();
    __syncwarp();
    unsigned last = 0;
    if (lane == 0) last = atomicAdd(&tickets[tile], 1u) == (unsigned)KS - 1;
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) return;
    __threadfence();
    // the last warp of this tile sums the KS partials in fixed order
    for (int idx = lane; idx < 16 * M; idx += 32) {
        const int m = idx / 16;
        const int64_t n = tile * 16 + idx % 16;
        if (n >= N) continue;
        float a = 0.f;
        for (int z = 0; z < KS; ++z) a += __ldcg(part + ((int64_t)z * M + m) * N + n);
        Y[(int64_t)m * N + n] = __float2bfloat16_rn(a);
    }
    if (lane == 0) tickets[tile] = 0u;
}

struct MmaPlan {
    int KS, gpt;
    int64_t tiles, tasks;
    size_t part_off, bfrag_off, e_off, ws_bytes;
};

MmaPlan mma_plan(int64_t M, int64_t N, int64_t K, int r) {
    MmaPlan p{};
    const int64_t G = K / kGroup;
    p.tiles = (N + 15) / 16;
    const int64_t want = 148 * 16;                   // warp tasks to fill the GPU
    int64_t ks = (want + p.tiles - 1) / p.tiles;
    int64_t cap = G / 4 > 1 ? G / 4 : 1;
    if (ks > cap) ks = cap;
    if (ks < 1) ks = 1;
    p.gpt = (int)((G + ks - 1) / ks);
    p.KS = (int)((G + p.gpt - 1) / p.gpt);
    p.tasks = p.tiles * p.KS;
    const int nreg = r <= 4 ? 16 : 32;
    p.part_off = kTicketBytes;
    size_t off = p.part_off + (p.KS > 1 ? (size_t)p.KS * M * N * sizeof(float) : 0);
    p.bfrag_off = (off + 255) & ~(size_t)255;
    off = p.bfrag_off + (size_t)G * 32 * nreg * sizeof(uint32_t);
    p.e_off = (off + 255) & ~(size_t)255;
    p.ws_bytes = p.e_off + (size_t)G * 8 * sizeof(float);
    return p;
}

template <int R>
mq_status run_mma(const uint16_t *X, const mq_weights *w, int64_t M, uint16_t *Y, char *ws,
                  const MmaPlan &p, cudaStream_t st) {
    uint32_t *bfrag = reinterpret_cast<uint32_t *>(ws + p.bfrag_off);
    float *Eg = reinterpret_cast<float *>(ws + p.e_off);
    const int64_t G = w->K / kGroup;
    const int64_t work = G * 32 * Layout<R>::NREG;
    int grid = (int)((work + 255) / 256);
    if (grid > 148 * 8) grid = 148 * 8;
    bfrag_kernel<R><<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16 *>(X), (int)M,
                                          w->K, bfrag, Eg);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "bfrag_kernel");
    const unsigned blocks = (unsigned)((p.tasks + kMmaWarps - 1) / kMmaWarps);
    gemv_mma_kernel<R><<<blocks, kMmaWarps * 32, 0, st>>>(
        w->planes, reinterpret_cast<const __half *>(w->scales), bfrag, Eg, (int)M, w->N, w->K,
        p.tiles, p.KS, p.gpt, reinterpret_cast<float *>(ws + p.part_off),
        reinterpret_cast<unsigned *>(ws), reinterpret_cast<__nv_bfloat16 *>(Y));
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "gemv_mma_kernel");
    return MQ_OK;
}

}  // namespace

size_t gemv_mma_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
    return mma_plan(M, N, K, r).ws_bytes;
}

mq_status launch_gemv_mma(const uint16_t *X, const mq_weights *w, int64_t M, uint16_t *Y,
                          void *ws, size_t ws_bytes, cudaStream_t st) {
    const MmaPlan p = mma_plan(M, w->N, w->K, w->r);
    if (p.ws_bytes > ws_bytes) return fail(MQ_ERR_WORKSPACE, "GEMV workspace too small");
    if (p.KS > 1 && p.tiles > (int64_t)(kTicketBytes / sizeof(unsigned)))
        return fail(MQ_ERR_UNSUPPORTED, "too many row tiles for the split-K ticket region");
    char *b = static_cast<char *>(ws);
    switch (w->r) {
        case 1: return run_mma<1>(X, w, M, Y, b, p, st);
        case 2: return run_mma<2>(X, w, M, Y, b, p, st);
        case 3: return run_mma<3>(X, w, M, Y, b, p, st);
        case 4: return run_mma<4>(X, w, M, Y, b, p, st);
        case 5: return run_mma<5>(X, w, M, Y, b, p, st);
        case 6: return run_mma<6>(X, w, M, Y, b, p, st);
        case 7: return run_mma<7>(X, w, M, Y, b, p, st);
        default: return run_mma<8>(X, w, M, Y, b, p, st);
    }
}

}  // namespace mq
