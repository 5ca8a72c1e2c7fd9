// Batch M <= 8: bit planes -> u8 operand fragments in registers -> int8 MMA.
//
// Turning a weight into an operand costs integer/logic instructions, which
// B200 issues at half the fp32 rate; a CUDA-core FMA then costs one more
// instruction per weight and batch row.  Here one mask builds four u8
// operands (one per byte), and the warp MMA m16n8k32 (16 weight rows x 8
// columns x 32 inputs, u8 x s8 -> s32) does every multiply-add exactly.
//
// Weights: each lane owns one 32-column word of a 128-column group for rows g
// and g + 8 (g = lane / 4, word t = lane % 4), reads exactly r plane words per
// row, and builds eight u8x4 registers whose bytes are the r-bit codes q
// (times 2^e, e = 1 for r = 3 and 8 - r for r >= 5) of known columns.
//
// X: per batch row m and group g, x = 2^(E-6) (a1 + 2^-7 a2 + 2^-14 a3) with
// E = floor(log2 max|x|) and int8 slices a_j; bf16 x has 8 significant bits,
// so the three slices are exact for every x within 2^-13 of the group's
// largest (smaller ones keep an error below 2^(E-20)).  The slices are the MMA
// columns c = 3m + j, so M <= 8 needs at most three 8-column tiles.
//
// Per group:  D_c = sum_k a_j(m, k) * field_k  (exact int32), and
//   y[n, m] += s[n, g] * ( sum_j fac[g, c] D_c + c_r S[g, m] ),
//   fac = 2^(8 - r - e + E - 6 - 7j),  c_r = 2^(7-r) - 128,  S = sum_k x.
// A prep kernel writes the B fragments, fac and the c_r S terms; the main
// kernel streams the planes, issues the MMAs and applies scales in fp32.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <string.h>

#include "mq_common.cuh"
#include "mq_bits.cuh"

namespace mq {
namespace {

// ----------------------------------------------------------- operand layout
// Register i (0..7) of a row word; byte b holds column col_of<R>(i, b).
template <int R> __host__ __device__ constexpr int col_of(int i, int b) {
    return R == 1 ? 8 * b + i                                   // bit i of byte b
         : R == 2 ? 2 * (4 * b + (i & 3)) + (i >> 2)            // pair field 4b + j
         : R <= 4 ? 4 * (2 * b + (i & 1)) + (i >> 1)            // nibble 2b + j of class d
                  : 8 * b + i;                                   // byte word e = i
}
template <int R> __host__ __device__ constexpr int field_exp() {
    return R == 3 ? 1 : R >= 5 ? 8 - R : 0;
}

template <int R>
__device__ __forceinline__ void operand_bytes(const uint32_t (&P)[8], uint32_t (&A)[8]) {
    if constexpr (R == 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) A[i] = (P[0] >> i) & 0x01010101u;
    } else if constexpr (R == 2) {
        const uint32_t F[2] = {pair_even(P[0], P[1]), pair_odd(P[0], P[1])};
#pragma unroll
        for (int i = 0; i < 8; ++i) A[i] = (F[i >> 2] >> (2 * (i & 3))) & 0x03030303u;
    } else if constexpr (R <= 4) {
        uint32_t N[4];
        nibble_words<R>(P, 0, N);
#pragma unroll
        for (int i = 0; i < 8; ++i) A[i] = (N[i >> 1] >> (4 * (i & 1))) & 0x0F0F0F0Fu;
    } else {
        byte_words<R>(P, A);
    }
}

__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int R>
__host__ __device__ constexpr float level_offset() {   // c_r = 2^(7-r) - 128
    return (float)(128 >> (R - 1)) * 0.5f - 128.0f;
}

constexpr int kCols = 24;                 // 8 batch rows x 3 slices

// ------------------------------------------------------------ prep kernel
// One block (256 threads) per group.  Writes, for NT column tiles:
//   bq[g][nt][h][lane][4]  u32 B fragments (h: MMA steps 2h, 2h+1; b0, b1 each)
//   fac[g][24], off[g][24] floats (off = c_r S on slice-0 columns, else 0)
template <int R>
__global__ void __launch_bounds__(256)
xslice_kernel(const __nv_bfloat16 *__restrict__ X, int M, int64_t K, int NT,
              uint32_t *__restrict__ bq, float *__restrict__ fac, float *__restrict__ off) {
    __shared__ int8_t a[kCols][kGroup];       // slice j of batch row m at column k
    __shared__ int e_grp[8];
    __shared__ float s_grp[8];
    // the GEMV kernel may start now: it streams weights until it needs our output
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t grp = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // warp m: exponent, sum and the three slices of batch row m
    {
        const int m = warp;
        float x[4] = {0.f, 0.f, 0.f, 0.f};
        if (m < M) {
            const uint2 raw = *reinterpret_cast<const uint2 *>(X + (int64_t)m * K + grp * kGroup + 4 * lane);
            x[0] = __uint_as_float(raw.x << 16);
            x[1] = __uint_as_float(raw.x & 0xFFFF0000u);
            x[2] = __uint_as_float(raw.y << 16);
            x[3] = __uint_as_float(raw.y & 0xFFFF0000u);
        }
        float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
        float s = (x[0] + x[1]) + (x[2] + x[3]);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            s += __shfl_xor_sync(0xffffffffu, s, o);
        }
        // E = floor(log2 amax) from the exponent field (amax is a bf16 value)
        const int E = amax > 0.f ? (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127 : 0;
        if (lane == 0) { e_grp[m] = E; s_grp[m] = s; }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            // exact splitting: every step subtracts a representable multiple
            const float v1 = ldexpf(x[u], 6 - E);                    // |v1| < 128
            const float a1 = truncf(v1);
            const float v2 = (v1 - a1) * 128.f;
            const float a2 = truncf(v2);
            const float a3 = truncf((v2 - a2) * 128.f);
            a[3 * m + 0][4 * lane + u] = (int8_t)a1;
            a[3 * m + 1][4 * lane + u] = (int8_t)a2;
            a[3 * m + 2][4 * lane + u] = (int8_t)a3;
        }
    }
    __syncthreads();
    // B fragments: lane L = (column-in-tile cg, word t); step st uses the
    // bytes of registers 2 st (b0) and 2 st + 1 (b1)
    for (int idx = threadIdx.x; idx < NT * 2 * 32 * 4; idx += blockDim.x) {
        const int w = idx & 3, L = (idx >> 2) & 31, h = (idx >> 7) & 1, nt = idx >> 8;
        const int cg = L >> 2, t = L & 3;
        const int c = 8 * nt + cg;
        const int st = 2 * h + (w >> 1), reg = 2 * st + (w & 1);
        uint32_t v = 0;
        if (c < 3 * M) {
#pragma unroll
            for (int b = 0; b < 4; ++b)
                v |= (uint32_t)(uint8_t)a[c][32 * t + col_of<R>(reg, b)] << (8 * b);
        }
        bq[((grp * NT + nt) * 2 + h) * 128 + L * 4 + w] = v;
    }
    if (threadIdx.x < kCols) {
        const int c = threadIdx.x, m = c / 3, j = c % 3;
        float f = 0.f, o = 0.f;
        if (m < M) {
            f = ldexpf(1.f, 8 - R - field_exp<R>() + e_grp[m] - 6 - 7 * j);
            o = j == 0 ? level_offset<R>() * s_grp[m] : 0.f;
        }
        fac[grp * kCols + c] = f;
        off[grp * kCols + c] = o;
    }
}

// ------------------------------------------------------------- main kernel
// Persistent CTAs per K slice (blockIdx.y).  The CTA stages the slice's B
// fragments, fac and off once; each warp owns 16-row tiles and pulls a tile's
// plane bytes (16 rows x r planes x the slice's groups) into shared memory
// with bulk async copies issued by one lane, one tile ahead (two stages per
// warp), so a whole tile of HBM reads is in flight while it computes the last.
constexpr int kMmaWarps = 8;

// Groups per K slice: a tile row of one plane is 16 GPT bytes = one TMA
// swizzle span (128, 64 or 32 bytes).
template <int R> __host__ __device__ constexpr int slice_groups() { return R <= 2 ? 8 : R <= 4 ? 4 : 2; }


template <int R, int NT> struct MmaSmem {
    static constexpr int GPT = slice_groups<R>();
    static constexpr int ROWB = 16 * GPT;                 // bytes of one plane row of a tile
    static constexpr size_t stage_bytes = (size_t)R * 16 * ROWB;   // the TMA box
    static constexpr size_t stages = 0;                   // 1024-aligned (swizzle period)
    static constexpr size_t bq = stages + (size_t)kMmaWarps * 2 * ((stage_bytes + 256 + 1023) & ~(size_t)1023);
    static constexpr size_t fac = bq + (size_t)GPT * NT * 1024;
    static constexpr size_t off = fac + (size_t)GPT * kCols * 4;
    static constexpr size_t red = off + (size_t)GPT * kCols * 4;
    static constexpr size_t bars = red + (size_t)kMmaWarps * 16 * kCols * 4;
    static constexpr size_t stage_pitch = (stage_bytes + 256 + 1023) & ~(size_t)1023;
    static constexpr size_t total = bars + (1 + 2 * kMmaWarps) * 8 + 1024;   // + base alignment
};

__device__ unsigned int g_gemv_timeout;

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void bar_init(uint64_t *b, uint32_t n) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(b)), "r"(n));
}
__device__ __forceinline__ void bar_expect(uint64_t *b, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 ::"r"(smem_addr(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *b) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(b)) : "memory");
}
// One 3-D TMA box (words x rows x planes) of the plane tensor into shared memory.
__device__ __forceinline__ void tma_box3(void *dst, const CUtensorMap *map, int x, int y, int z,
                                         uint64_t *b) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(smem_addr(dst)), "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_addr(b)) : "memory");
}

// One 2-D TMA box (elements x rows) into shared memory.
__device__ __forceinline__ void tma_box2(void *dst, const CUtensorMap *map, int x, int y, uint64_t *b) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_addr(dst)), "l"(map), "r"(x), "r"(y), "r"(smem_addr(b)) : "memory");
}

// Arrival ticket: acquire-release add at GPU scope, returns the old value.
__device__ __forceinline__ unsigned ticket_add_acq_rel(unsigned *p) {
    unsigned old;
    asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
    return old;
}

// Bounded wait on an mbarrier phase (the hint lets the thread sleep).
__device__ __forceinline__ bool bar_wait(uint64_t *b, uint32_t parity) {
    for (uint32_t i = 0; i < (1u << 22); ++i) {
        uint32_t ok;
        asm volatile("{\n .reg .pred p;\n"
                     " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 1000000;\n"
                     " selp.u32 %0, 1, 0, p;\n}"
                     : "=r"(ok) : "r"(smem_addr(b)), "r"(parity) : "memory");
        if (ok) return true;
    }
    return false;
}

template <int R, int NT>
__global__ void __launch_bounds__(kMmaWarps * 32, 2)
gemv_i8_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap smap,
               int scales_tma, const __half *__restrict__ scales, const uint32_t *__restrict__ bq,
               const float *__restrict__ facg, const float *__restrict__ offg, int M, int64_t N,
               int64_t K, int64_t tiles, float *__restrict__ part, unsigned *__restrict__ tickets,
               __nv_bfloat16 *__restrict__ Y) {
    using S = MmaSmem<R, NT>;
    constexpr int GPT = S::GPT;
    constexpr int kStageWords = (int)(S::stage_pitch / 4);
    constexpr int ROWW = S::ROWB / 4;                       // words per tile row of a plane
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint4 *sB = reinterpret_cast<const uint4 *>(smem + S::bq);
    const float *sF = reinterpret_cast<const float *>(smem + S::fac);
    const float *sO = reinterpret_cast<const float *>(smem + S::off);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S::bars);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    float *red = reinterpret_cast<float *>(smem + S::red) + warp * 16 * kCols;
    const int KS = gridDim.y, ks = blockIdx.y;
    const int64_t G = K / kGroup;
    const int64_t g0 = (int64_t)ks * GPT;
    const int ng = (int)((g0 + GPT < G ? g0 + GPT : G) - g0);
    const int soff = (int)(g0 & 7);                         // first group inside the scale box
    uint32_t *const stage0 = reinterpret_cast<uint32_t *>(smem + S::stages + 2 * warp * S::stage_pitch);
    uint64_t *wbar = bars + 1 + 2 * warp;
    // 16-byte chunk of a row after the TMA swizzle (rows g and g + 8 agree)
    const int swz = GPT == 8 ? (g & 7) : GPT == 4 ? ((g >> 1) & 3) : ((g >> 2) & 1);

    if (threadIdx.x == 0) {
        bar_init(&bars[0], 1);
        for (int i = 0; i < 2 * kMmaWarps; ++i) bar_init(&bars[1 + i], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    // Tiles of this warp: blockIdx.x + gridDim.x * (warp + kMmaWarps * j), so
    // every CTA (and SM) gets the same number of tiles within one.
    const int64_t stride = (int64_t)gridDim.x * kMmaWarps;
    int64_t tile = blockIdx.x + (int64_t)gridDim.x * warp;

    // One tile into stage `st`: planes (and scales) by TMA from lane 0; rows
    // >= N and groups >= G arrive zero-filled.  Without a scale tensor map
    // (G not a multiple of 8) lanes 0..15 copy their row's scales.
    auto issue = [&](int st, int64_t tl) {
        uint32_t *dst = stage0 + st * kStageWords;
        if (lane == 0) {
            bar_expect(wbar + st, (uint32_t)S::stage_bytes + (scales_tma ? 256u : 0u));
            tma_box3(dst, &tmap, (int)(g0 * 4), (int)(tl * 16), 0, wbar + st);
            if (scales_tma)
                tma_box2(reinterpret_cast<uint8_t *>(dst) + S::stage_bytes, &smap,
                         (int)(g0 - soff), (int)(tl * 16), wbar + st);
        }
        if (!scales_tma && lane < 16) {
            const int64_t n = tl * 16 + lane;
            __half *sd = reinterpret_cast<__half *>(reinterpret_cast<uint8_t *>(dst) + S::stage_bytes);
#pragma unroll
            for (int grp = 0; grp < GPT; ++grp)
                sd[lane * 8 + soff + grp] = (n < N && grp < ng) ? scales[n * G + g0 + grp]
                                                                : __float2half(0.f);
        }
    };

    uint32_t phase_bits = 0u;
    bool ok = true;
    if (tile < tiles) issue(0, tile);
    // Everything above reads only the weights; X-derived operands come from
    // the preceding prep kernel of this call.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (threadIdx.x == 0) {
        const uint32_t bb = (uint32_t)ng * NT * 1024, fb = (uint32_t)ng * kCols * 4;
        bar_expect(&bars[0], bb + 2 * fb);
        bulk_g2s(smem + S::bq, bq + g0 * NT * 256, bb, &bars[0]);
        bulk_g2s(smem + S::fac, facg + g0 * kCols, fb, &bars[0]);
        bulk_g2s(smem + S::off, offg + g0 * kCols, fb, &bars[0]);
    }
    if (!bar_wait(&bars[0], 0)) ok = false;
    int st = 0;
    for (; tile < tiles && ok; tile += stride) {
        const int64_t next = tile + stride;
        __syncwarp();
        if (next < tiles) issue(st ^ 1, next);
        if (!bar_wait(wbar + st, (phase_bits >> st) & 1u)) { ok = false; break; }
        phase_bits ^= 1u << st;
        __syncwarp();
        const uint32_t *sw = stage0 + st * kStageWords;
        const __half *ss = reinterpret_cast<const __half *>(reinterpret_cast<const uint8_t *>(sw) + S::stage_bytes);

        float y[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) y[nt][i] = 0.f;
#pragma unroll
        for (int grp = 0; grp < GPT; ++grp) {
            if (grp >= ng) break;
            uint32_t A[2][8], P[8];
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
#pragma unroll
                for (int p = 0; p < 8; ++p)
                    P[p] = p < R ? sw[(p * 16 + g + 8 * hr) * ROWW + ((grp ^ swz) << 2) + t] : 0u;
                operand_bytes<R>(P, A[hr]);
            }
            const float s_lo = __half2float(ss[g * 8 + soff + grp]);
            const float s_hi = __half2float(ss[(g + 8) * 8 + soff + grp]);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                int d[4] = {0, 0, 0, 0};
                const uint4 b0 = sB[((grp * NT + nt) * 2 + 0) * 32 + lane];
                const uint4 b1 = sB[((grp * NT + nt) * 2 + 1) * 32 + lane];
                uint32_t a[4];
                a[0] = A[0][0]; a[1] = A[1][0]; a[2] = A[0][1]; a[3] = A[1][1];
                mma_u8s8(d, a, b0.x, b0.y);
                a[0] = A[0][2]; a[1] = A[1][2]; a[2] = A[0][3]; a[3] = A[1][3];
                mma_u8s8(d, a, b0.z, b0.w);
                a[0] = A[0][4]; a[1] = A[1][4]; a[2] = A[0][5]; a[3] = A[1][5];
                mma_u8s8(d, a, b1.x, b1.y);
                a[0] = A[0][6]; a[1] = A[1][6]; a[2] = A[0][7]; a[3] = A[1][7];
                mma_u8s8(d, a, b1.z, b1.w);
                const float2 f = *reinterpret_cast<const float2 *>(sF + grp * kCols + 8 * nt + 2 * t);
                const float2 o = *reinterpret_cast<const float2 *>(sO + grp * kCols + 8 * nt + 2 * t);
                y[nt][0] = fmaf(s_lo, fmaf(f.x, (float)d[0], o.x), y[nt][0]);
                y[nt][1] = fmaf(s_lo, fmaf(f.y, (float)d[1], o.y), y[nt][1]);
                y[nt][2] = fmaf(s_hi, fmaf(f.x, (float)d[2], o.x), y[nt][2]);
                y[nt][3] = fmaf(s_hi, fmaf(f.y, (float)d[3], o.y), y[nt][3]);
            }
        }
        st ^= 1;

        // ---- columns -> batch rows: Y[m, n] = sum_j column 3m + j
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int c = 8 * nt + 2 * t;
            red[g * kCols + c] = y[nt][0];
            red[g * kCols + c + 1] = y[nt][1];
            red[(g + 8) * kCols + c] = y[nt][2];
            red[(g + 8) * kCols + c + 1] = y[nt][3];
        }
        __syncwarp();
        float out[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {                      // 16 M <= 128 outputs
            const int idx = lane + 32 * q, rr = idx & 15, m = idx >> 4;
            out[q] = idx < 16 * M ? red[rr * kCols + 3 * m] + red[rr * kCols + 3 * m + 1] +
                                        red[rr * kCols + 3 * m + 2]
                                  : 0.f;
        }
        __syncwarp();
        if (KS == 1) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int idx = lane + 32 * q, rr = idx & 15, m = idx >> 4;
                const int64_t n = tile * 16 + rr;
                if (idx < 16 * M && n < N) Y[(int64_t)m * N + n] = __float2bfloat16_rn(out[q]);
            }
            continue;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int idx = lane + 32 * q, rr = idx & 15, m = idx >> 4;
            const int64_t n = tile * 16 + rr;
            if (idx < 16 * M && n < N) part[((int64_t)ks * M + m) * N + n] = out[q];
        }
        __syncwarp();                      // the warp's partials before lane 0's release
        unsigned last = 0;
        if (lane == 0) last = ticket_add_acq_rel(&tickets[tile]) == (unsigned)KS - 1;
        last = __shfl_sync(0xffffffffu, last, 0);
        if (!last) continue;
        __threadfence();
        for (int idx = lane; idx < 16 * M; idx += 32) {      // fixed-order sum
            const int rr = idx & 15, m = idx >> 4;
            const int64_t n = tile * 16 + rr;
            if (n >= N) continue;
            float acc = 0.f;
            for (int z = 0; z < KS; ++z) acc += __ldcg(part + ((int64_t)z * M + m) * N + n);
            Y[(int64_t)m * N + n] = __float2bfloat16_rn(acc);
        }
        if (lane == 0) tickets[tile] = 0u;
    }
    if (!ok && lane == 0) atomicOr(&g_gemv_timeout, 1u);
}

// Tensor map of the fp16 scales [N][G] with a 16 x 8 box; needs G % 8 == 0
// (row pitch a multiple of 16 bytes).
mq_status scale_map(const mq_weights *w, CUtensorMap *out, bool *ok) {
    const int64_t G = w->K / kGroup;
    *ok = (G % 8) == 0;
    if (!*ok) { memset(out, 0, sizeof(*out)); return MQ_OK; }
    struct Slot { const void *p; int64_t N, K; CUtensorMap map; };
    static thread_local Slot cache[32];
    static thread_local int next = 0;
    for (auto &c : cache)
        if (c.p == w->scales && c.N == w->N && c.K == w->K) { *out = c.map; return MQ_OK; }
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess || !fn)
        return fail(MQ_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    const cuuint64_t dims[2] = {(cuuint64_t)G, (cuuint64_t)w->N};
    const cuuint64_t strides[1] = {(cuuint64_t)(G * 2)};
    const cuuint32_t box[2] = {8u, 16u};
    const cuuint32_t estr[2] = {1u, 1u};
    CUtensorMap m;
    const CUresult res = encode(&m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t *>(w->scales),
                                dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (res != CUDA_SUCCESS) return fail(MQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the scales");
    cache[next] = Slot{w->scales, w->N, w->K, m};
    next = (next + 1) % 32;
    *out = m;
    return MQ_OK;
}

struct MmaPlan {
    int KS, NT;
    int64_t tiles, ctas_x;
    size_t part_off, bq_off, fac_off, off_off, ws_bytes;
};

int plan_gpt(int r) { return r <= 2 ? 8 : r <= 4 ? 4 : 2; }

// Tensor map of the r planes seen as [r][N][K/32] uint32, box (4 GPT words,
// 16 rows, r planes), swizzled so that a warp's operand reads are
// conflict-free.  Encoded through the runtime's driver entry point and cached
// per (buffer, shape, r).
mq_status plane_map(const mq_weights *w, int gpt, CUtensorMap *out) {
    struct Slot { const void *p; int64_t N, K; int r; CUtensorMap map; };
    static thread_local Slot cache[32];
    static thread_local int next = 0;
    for (auto &c : cache)
        if (c.p == w->planes && c.N == w->N && c.K == w->K && c.r == w->r) { *out = c.map; return MQ_OK; }
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        cudaDriverEntryPointQueryResult q;
        void *fn = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            !fn)
            return fail(MQ_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    const cuuint64_t dims[3] = {(cuuint64_t)(w->K / 32), (cuuint64_t)w->N, (cuuint64_t)w->r};
    const cuuint64_t strides[2] = {(cuuint64_t)(w->K / 8), (cuuint64_t)(w->N * (w->K / 8))};
    const cuuint32_t box[3] = {(cuuint32_t)(4 * gpt), 16u, (cuuint32_t)w->r};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    const CUtensorMapSwizzle sw = gpt == 8 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : gpt == 4 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
    CUtensorMap m;
    const CUresult res = encode(&m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t *>(w->planes),
                                dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (res != CUDA_SUCCESS) return fail(MQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the planes");
    cache[next] = Slot{w->planes, w->N, w->K, w->r, m};
    next = (next + 1) % 32;
    *out = m;
    return MQ_OK;
}

MmaPlan mma_plan(int64_t M, int64_t N, int64_t K, int r) {
    MmaPlan p{};
    const int64_t G = K / kGroup;
    const int gpt = plan_gpt(r);
    p.NT = (int)((3 * M + 7) / 8);
    p.tiles = (N + 15) / 16;
    p.KS = (int)((G + gpt - 1) / gpt);
    int64_t cap = (2 * 148) / p.KS;
    if (cap < 1) cap = 1;
    p.ctas_x = (p.tiles + kMmaWarps - 1) / kMmaWarps;
    if (p.ctas_x > cap) p.ctas_x = cap;
    p.part_off = kTicketBytes;
    size_t off = p.part_off + (p.KS > 1 ? (size_t)p.KS * M * N * sizeof(float) : 0);
    p.bq_off = (off + 255) & ~(size_t)255;
    off = p.bq_off + (size_t)G * p.NT * 1024;
    p.fac_off = (off + 255) & ~(size_t)255;
    off = p.fac_off + (size_t)G * kCols * sizeof(float);
    p.off_off = (off + 255) & ~(size_t)255;
    p.ws_bytes = p.off_off + (size_t)G * kCols * sizeof(float);
    return p;
}

template <int R, int NT>
mq_status run_i8(const uint16_t *X, const mq_weights *w, int64_t M, uint16_t *Y, char *ws,
                 const MmaPlan &p, cudaStream_t st) {
    uint32_t *bq = reinterpret_cast<uint32_t *>(ws + p.bq_off);
    float *fac = reinterpret_cast<float *>(ws + p.fac_off);
    float *off = reinterpret_cast<float *>(ws + p.off_off);
    const int64_t G = w->K / kGroup;
    xslice_kernel<R><<<(unsigned)G, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16 *>(X),
                                                  (int)M, w->K, NT, bq, fac, off);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "xslice_kernel");
    constexpr size_t smem = MmaSmem<R, NT>::total;
    static bool attr_set = false;
    if (!attr_set) {
        e = cudaFuncSetAttribute(gemv_i8_kernel<R, NT>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        attr_set = true;
    }
    CUtensorMap tmap, smap;
    bool stma = false;
    mq_status ms = plane_map(w, MmaSmem<R, NT>::GPT, &tmap);
    if (ms == MQ_OK) ms = scale_map(w, &smap, &stma);
    if (ms != MQ_OK) return ms;
    // programmatic dependent launch: the kernel starts streaming weights while
    // the prep kernel finishes, and waits for it before reading its output
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.ctas_x, (unsigned)p.KS);
    cfg.blockDim = dim3(kMmaWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, gemv_i8_kernel<R, NT>, tmap, smap, stma ? 1 : 0,
                           reinterpret_cast<const __half *>(w->scales),
                           (const uint32_t *)bq, (const float *)fac, (const float *)off, (int)M,
                           w->N, w->K, p.tiles, reinterpret_cast<float *>(ws + p.part_off),
                           reinterpret_cast<unsigned *>(ws), reinterpret_cast<__nv_bfloat16 *>(Y));
    if (e != cudaSuccess) return cuda_fail(e, "gemv_i8_kernel launch");
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "gemv_i8_kernel");
    return MQ_OK;
}

template <int R>
mq_status run_r(const uint16_t *X, const mq_weights *w, int64_t M, uint16_t *Y, char *ws,
                const MmaPlan &p, cudaStream_t st) {
    if (p.NT == 1) return run_i8<R, 1>(X, w, M, Y, ws, p, st);
    if (p.NT == 2) return run_i8<R, 2>(X, w, M, Y, ws, p, st);
    return run_i8<R, 3>(X, w, M, Y, ws, p, st);
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
    if (p.KS > 65535) return fail(MQ_ERR_UNSUPPORTED, "K too large");
    char *b = static_cast<char *>(ws);
    switch (w->r) {
        case 1: return run_r<1>(X, w, M, Y, b, p, st);
        case 2: return run_r<2>(X, w, M, Y, b, p, st);
        case 3: return run_r<3>(X, w, M, Y, b, p, st);
        case 4: return run_r<4>(X, w, M, Y, b, p, st);
        case 5: return run_r<5>(X, w, M, Y, b, p, st);
        case 6: return run_r<6>(X, w, M, Y, b, p, st);
        case 7: return run_r<7>(X, w, M, Y, b, p, st);
        default: return run_r<8>(X, w, M, Y, b, p, st);
    }
}

}  // namespace mq
