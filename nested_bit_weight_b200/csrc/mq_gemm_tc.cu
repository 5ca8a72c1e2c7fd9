// Batched path: tcgen05 tensor-core GEMM over decoded r-bit tiles (M >= 9,
// the small batches the dispatch gives it, and asymmetric weights for every
// M).
//
// The r-bit levels v_r = 2^(8-r) q_r + 2^(7-r) - 128 are exact in bf16 (at
// most 8 significant bits), so the MMA operands are exact:
//     D_g[n, m] = sum_{k in group g} v_r[n, k] * x[m, k]     (fp32, in TMEM)
//     Y[m, n]   = sum_g s[n, g] * D_g[n, m]                  (fp32 registers)
// (the fp16 scale is applied per 128-column group in fp32: folding s * v
// into one 16-bit operand rounds every weight, which the tolerance does not
// allow on large layers).  Asymmetric variant (a zero point z per group):
//     Y[m, n]   = sum_g s[n, g] * (D_g[n, m] + (128 - z[n, g]) * sum_{k in g} x[m, k])
// with the sums of X written by a small kernel before the GEMM.
//
// Work: items (X block mb, 128-row tile t, group g) in that order, cut into
// one contiguous range per CTA (about 148 CTAs, one per SM).  A tile whose
// groups are spread over several CTAs is summed by the CTA that delivers its
// last part, from the fp32 partial sums the others leave in the workspace,
// in CTA order (deterministic), with all its threads after its own range.
//
// Roles (warp-specialised; every hand-off an mbarrier; item i uses stage
// i mod kS of the A operand, the X operand and the accumulator):
//   decode warps    two groups of four taking alternate items (one group for
//                   BM = 128); a thread per weight row copies exactly its
//                   row's 16 bytes of each plane of the items ahead with
//                   L1-bypassing cp.async (up to 16 items, 96 KB per SM in
//                   flight), decodes each 32-column word to bf16 levels in
//                   natural column order and stores them to its TMEM lane of
//                   the A stage (tcgen05.st; the MMA reads A from TMEM);
//   X warp          one thread loads the group's BM x 128 block of X into
//                   the B stage with one 3-D tensor-map (TMA) copy in the
//                   MMA's K-major layout; rows beyond M read as zeros;
//   two MMA warps   one thread each (even / odd items) issues eight
//                   128 x BM x 16 MMAs per group into the stage's TMEM
//                   accumulator and commits once: the stage's A and B
//                   operands are free, its accumulator full;
//   fold warps      4 (BM <= 64) or 8 (BM = 128), one or two per TMEM lane
//                   quarter: y += s[n, g] * D_g, the tile's fp32 sums kept in
//                   registers until the tile ends; the scales (and zero
//                   points) arrive by per-thread cp.async eight items ahead.
// Launched with programmatic dependent launch: the decode warps stream the
// weights before the previous kernel of the stream has completed; X is read
// and Y and the workspace written only after griddepcontrol.wait.
// Every wait is bounded (about a second); a wait that gives up sets a CTA
// abort flag that ends the others at once, and a device flag read by
// mq_device_status.  The fold still runs every tile end, so arrival tickets
// always return to zero, also after a timeout (the output is then
// unspecified); copies, MMAs and barrier arrivals in flight land before the
// CTA exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <type_traits>

#include "mq_common.cuh"
#include "mq_bits.cuh"
#include "mq_sm100.cuh"

namespace mq {
namespace {

using namespace sm100;

constexpr int kTileN = 128;                  // weight rows per tile (MMA M)
constexpr int kMinItems = 4;                 // fewest items a CTA is given

// Per (r, BM) configuration.  15 warps, so 128 registers a thread: decode
// warps (two groups of four taking alternate items, or one group for
// BM = 128), fold warps, the X warp and two MMA warps.  Shared memory: kS X stages and a ring of kD items of plane
// words (the loads in flight that keep HBM busy).  Tensor memory (512
// columns): kS A stages of 64 columns and kS accumulators of BM columns, with
// kS = 4 for BM <= 64 (the decode, the MMA and the fold run up to three
// groups apart) and 2 for BM = 128.  Item i uses stage i % kS of all three,
// so one commit per item frees its A and X stages and fills its accumulator.
__host__ __device__ constexpr int ring_items(int r, int BM) {
    return (96 * 1024) / (r * 2048) < 16 ? (96 * 1024) / (r * 2048) : 16;
}
// Pipeline stages: item i uses A stage, X stage and accumulator i % stages.
__host__ __device__ constexpr int x_stages(int BM) { return BM == 128 ? 2 : 4; }
constexpr int kScaleAhead = 8;                // items of scales in flight per fold thread
__host__ __device__ constexpr size_t tc_smem_bytes(int r, int BM) {
    return 1024 + (size_t)x_stages(BM) * BM * 256 + (size_t)ring_items(r, BM) * r * 2048 +
           (size_t)2 * 256 * kScaleAhead * 4      // scale and zero-point rings of the fold
           + (size_t)x_stages(BM) * BM * 4           // sum of X per stage (asymmetric variant)
           + 512;
}

template <int R, int BM>
struct TcCfg {
    static constexpr int kDecW = BM == 128 ? 4 : 8;
    static constexpr int kFoldW = BM == 128 ? 8 : 4;
    static constexpr int kThreads = (kDecW + kFoldW + 3) * 32;  // + X warp + 2 MMA warps
    static constexpr int kGroups = kDecW / 4;                 // decode groups (alternate items)
    static constexpr int kS = x_stages(BM);
    static constexpr int kD = ring_items(R, BM) / kGroups;    // ring items per decode group
    static constexpr uint32_t kXStage = BM * 256;             // BM rows x 128 bf16
    static constexpr uint32_t kTmemCols = 512;
    static_assert(kS * 64 + kS * BM <= (int)kTmemCols, "TMEM columns");
    static constexpr uint32_t kSlot = R * 2048;               // plane words of one item
};

__device__ unsigned int g_tc_timeout;        // set when a bounded wait gave up

#ifdef MQ_TEST_HOOKS
// Test-hook builds only: while positive, the X warp of a CTA that takes a
// unit drops its first load and arrival, so that the MMA's bounded wait runs
// out (the timeout path, with no fault and no trap).
__device__ int g_test_drop_x;
#endif

// Wait of the decode and fold warps for their hand-offs.
#ifndef MQ_GEMM_WAIT
#define MQ_GEMM_WAIT mbar_wait_abortable
#endif

// The 16 A words of one 32-column plane word, before centring: word 4b + j
// holds columns 8b + 2j and 8b + 2j + 1 (low, high half), as bf16 256 + e
// for r <= 6 and as the bytes e0 | e1 << 8 for r >= 7 (e = q_r << (8 - r)).
template <int R>
__host__ __device__ __forceinline__ void word_pairs(const uint32_t (&P)[8], uint32_t (&v)[16]) {
    uint32_t E[8];
    if constexpr (R <= 6) {
        half_byte_words<R>(P, E);                      // byte b of E[e]: (column 8b + e) / 2
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int j = 0; j < 4; ++j) v[4 * b + j] = bf16_pair_from_halves(E[2 * j], E[2 * j + 1], b);
    } else {
        byte_words<R>(P, E);                           // byte b of E[e]: column 8b + e
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int j = 0; j < 4; ++j) v[4 * b + j] = byte_pair(E[2 * j], E[2 * j + 1], b);
    }
}

// Centre a word of word_pairs to the two bf16 levels v_r = e - 128 + 2^(7-r).
template <int R>
__device__ __forceinline__ uint32_t centre(uint32_t w) {
    if constexpr (R <= 6) {
        // one exact bf16 subtraction (384 - 2^(7-r) is exact in bf16 for r <= 6)
        const float c = 384.0f - (float)(1 << (7 - R));
        __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162 *>(&w);
        v = __hsub2(v, __floats2bfloat162_rn(c, c));
        return *reinterpret_cast<uint32_t *>(&v);
    } else {
        // through fp32: 2^22 + e has a 0.5 ulp, so subtracting
        // 2^22 + 128 - 2^(7-r) is exact and leaves v_r
        constexpr float c = 4194432.0f - (R == 8 ? 0.5f : 1.0f);
        const float f0 = __uint_as_float(0x4A800000u | ((w & 0xFFu) << 1)) - c;
        const float f1 = __uint_as_float(0x4A800000u | ((w >> 8) << 1)) - c;
        __nv_bfloat162 v = __floats2bfloat162_rn(f0, f1);
        return *reinterpret_cast<uint32_t *>(&v);
    }
}

// Kernel arguments.
struct GArgs {
    CUtensorMap xmap;           // X as (64 columns, M rows, K/64 halves), boxes 64 x BM x 2
    const uint32_t *planes;     // tiled planes
    const __half *scales;       // tiled fp16 scales
    const __half *zeros;        // tiled fp16 zero points (asymmetric variant) or null
    const float *sumx;          // [G][Mpad] sums of X over each group (asymmetric variant)
    int Mpad;                   // MB * BM
    __nv_bfloat16 *Y;           // M x N
    float *part;                // partial sums of shared tiles [tile * maxc + slot][BM][128]
    unsigned *tickets;          // one per (X block, tile)
    int64_t N, K;
    int M, T, G, MB, P, maxc;   // rows of X, row tiles, groups, X blocks, CTAs, CTAs per tile
    int64_t plane_words;        // uint32 words of one plane
};

__host__ __device__ inline int64_t range_first(int64_t b, int64_t W, int P) { return b * W / P; }
__host__ __device__ inline int cta_of(int64_t u, int64_t W, int P) { return (int)(((u + 1) * P - 1) / W); }

// Wait (bounded) for the last phase issued to every slot of a ring of n
// barriers that received `issued` phases in slot order.
__device__ __forceinline__ void drain_ring(uint64_t *bars, int n, int issued) {
    for (int s = 0; s < n && s < issued; ++s) {
        const int k = (issued - 1 - s) / n + 1;
        mbar_wait_bounded(bars + s, (uint32_t)(k - 1) & 1u);
    }
}

template <int R, int BM>
__global__ void __launch_bounds__(TcCfg<R, BM>::kThreads, 1)
gemm_tc_kernel(const __grid_constant__ GArgs a) {
    using C = TcCfg<R, BM>;
    constexpr int kDecW = C::kDecW, kFoldW = C::kFoldW, kS = C::kS, kD = C::kD;
    constexpr int kFoldW0 = kDecW, kXW = kDecW + kFoldW, kMmaW = kXW + 1;
    constexpr uint32_t kIdesc = idesc_bf16_f32(kTileN, BM);
    constexpr uint32_t kD0 = kS * 64;                          // TMEM: A stages, then the accumulators
    constexpr int kCW = BM * 4 / kFoldW;                       // columns per fold thread
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *sX = smem;                                        // [kS][2 halves][BM][128 B]
    uint8_t *ring = sX + kS * C::kXStage;                      // [group][kD][plane][128 rows][16 B]
    uint32_t *sring = reinterpret_cast<uint32_t *>(ring + C::kGroups * kD * C::kSlot);  // [fold thread][kScaleAhead]
    uint32_t *zring = sring + kFoldW * 32 * kScaleAhead;       // zero points, same shape
    float *sx = reinterpret_cast<float *>(zring + kFoldW * 32 * kScaleAhead);   // [kS][BM] sums of X
    uint64_t *bars = reinterpret_cast<uint64_t *>(sx + kS * BM);
    const bool asym = a.zeros != nullptr;                      // asymmetric variant (uniform)
    // afull: A stage decoded; xfull: X stage loaded; sempty: the stage's MMAs
    // done (A and X free, accumulator full); dempty: accumulator read
    uint64_t *afull = bars, *xfull = afull + kS, *sempty = xfull + kS, *dempty = sempty + kS;
    // [0] abort  [2], [9] last item + 1 issued by the even / odd MMA thread
    // [3] X items loaded  [4] tiles this CTA sums at the end  [5, 6] their
    // indices  [7, 8] their CTA counts
    volatile int *flags = reinterpret_cast<volatile int *>(dempty + kS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(dempty + kS) + 12;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // programmatic dependent launch: the next kernel of the stream may start
    // its prologue as SMs free up (it reads our output only after its own
    // wait, which returns once this grid has completed)
    if (threadIdx.x == 0) pdl_launch_dependents();
    const int64_t W = (int64_t)a.MB * a.T * a.G;
    const int64_t u0 = range_first(blockIdx.x, W, a.P), u1 = range_first(blockIdx.x + 1, W, a.P);
    const int L = (int)(u1 - u0);
    const int G = a.G, TG = a.T * a.G;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kS; ++i) {
            mbar_init(afull + i, 4);                           // the 4 warps of one decode group
            mbar_init(xfull + i, 1);
            mbar_init(sempty + i, 1);
            mbar_init(dempty + i, kFoldW);
        }
        for (int i = 0; i < 10; ++i) flags[i] = 0;     // [1] unused
        fence_mbar_init();
    }
    if (warp == kMmaW) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(tmem_slot);

    if (warp < kDecW) {
        // ------------------------------------------------------------ decode
        // group g (warps 4g .. 4g + 3) takes items g, g + kGroups, ...; thread
        // n of the group owns row n of the tile and copies exactly what it
        // decodes: 16 bytes (32 columns x 4 words) of each plane per item,
        // with L1-bypassing cp.async into the group's ring of kD items
        constexpr int kGroups = C::kGroups;
        const int n = threadIdx.x & (kTileN - 1);              // row of the tile
        const int g = threadIdx.x >> 7;                        // item group
        uint8_t *mine = ring + (size_t)g * kD * C::kSlot + n * 16;   // + slot, + plane
        int next_tg = (int)((u0 + g) % TG);                    // (tile, group) of the next item copied
        auto issue = [&](int j) {                              // the group's j-th item, in order
            const uint32_t *src = a.planes + (int64_t)next_tg * 512 + n * 4;
            uint8_t *dst = mine + (j % kD) * C::kSlot;
#pragma unroll
            for (int p = 0; p < R; ++p) cp_async_16(dst + p * 2048, src + p * a.plane_words);
            next_tg += kGroups;
            while (next_tg >= TG) next_tg -= TG;               // TG may be 1
        };
        const int Lg = L > g ? (L - g + kGroups - 1) / kGroups : 0;   // items of this group
#pragma unroll 1
        for (int j = 0; j < kD; ++j) {
            if (j < Lg) issue(j);
            cp_async_commit();
        }
        for (int j = 0; j < Lg; ++j) {
            const int i = g + j * kGroups;                     // item of the range
            const int st = i % kS;
            cp_async_wait<kD - 1>();                           // item i's words are in
            uint32_t pv[R][4];
            const uint8_t *src = mine + (j % kD) * C::kSlot;
#pragma unroll
            for (int p = 0; p < R; ++p) {
                const uint4 v = *reinterpret_cast<const uint4 *>(src + p * 2048);
                pv[p][0] = v.x; pv[p][1] = v.y; pv[p][2] = v.z; pv[p][3] = v.w;
            }
            if (j + kD < Lg) issue(j + kD);                    // refill the slot just read
            cp_async_commit();
            bool ok = i < kS || MQ_GEMM_WAIT(sempty + st, (uint32_t)(i / kS - 1) & 1u, flags);
            if (!__all_sync(0xFFFFFFFFu, ok)) break;
            tc_fence_after();
            // the row's four 32-column words -> 16 TMEM columns each of A stage st
            const uint32_t a_row = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(st * 64);
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                uint32_t P[8], v[16];
#pragma unroll
                for (int p = 0; p < 8; ++p) P[p] = p < R ? pv[p < R ? p : 0][w] : 0u;
                word_pairs<R>(P, v);
#pragma unroll
                for (int q = 0; q < 16; ++q) v[q] = centre<R>(v[q]);
                tmem_st16(a_row + (uint32_t)(16 * w), v);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(afull + st);
        }
        cp_async_wait<0>();                                    // no copy left in flight
    } else if (warp < kXW) {
        // -------------------------------------------------------------- fold
        const int f = warp - kFoldW0, q = f & 3, c0 = (f >> 2) * kCW;
        const int n = 32 * q + lane;                           // row of the tile
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        float y[kCW];
#pragma unroll
        for (int j = 0; j < kCW; ++j) y[j] = 0.f;
        // ok turns false for good once a wait of this warp gave up: the warp
        // then skips its waits and tensor-memory reads but still runs every
        // tile end, so the barriers below always match and every ticket is
        // taken (Y is then unspecified)
        bool ok = true;
        int gi = (int)(u0 % G);                                // group of item i inside its tile
        int64_t tu = u0 / G;                                   // tile of item i over (mb, t)
        int64_t tile_u0 = u0 - gi;                             // first item of that tile
        // the fp16 scales of the next kScaleAhead items in flight: each thread
        // copies the 4 bytes holding its row's scale (rows n & ~1 and n | 1)
        // into its own slots (cp.async groups are per thread: no barrier)
        uint32_t *slots = sring + (threadIdx.x - kFoldW0 * 32) * kScaleAhead;
        uint32_t *zslots = zring + (threadIdx.x - kFoldW0 * 32) * kScaleAhead;
        const uint16_t *sc = reinterpret_cast<const uint16_t *>(a.scales) + (n & ~1);
        const uint16_t *zc = asym ? reinterpret_cast<const uint16_t *>(a.zeros) + (n & ~1) : nullptr;
        int next_tg = (int)(u0 % TG);                          // (tile, group) of the next scale copied
        auto scale_issue = [&](int i) {
            cp_async_4(slots + i % kScaleAhead, sc + (int64_t)next_tg * 128);
            if (asym) cp_async_4(zslots + i % kScaleAhead, zc + (int64_t)next_tg * 128);
            if (++next_tg == TG) next_tg = 0;
        };
#pragma unroll 1
        for (int k = 0; k < kScaleAhead; ++k) {
            if (k < L) scale_issue(k);
            cp_async_commit();
        }
        pdl_wait();                                            // Y and the workspace: after the previous kernel
        for (int i = 0; i < L; ++i) {
            const int db = i % kS;
            cp_async_wait<kScaleAhead - 1>();                  // item i's scale is in
            const uint32_t sw = slots[i % kScaleAhead];
            const float s = __half2float(__ushort_as_half((unsigned short)((n & 1) ? sw >> 16 : sw & 0xFFFFu)));
            float cz = 0.f;                                    // 128 - z (asymmetric variant)
            if (asym) {
                const uint32_t zw = zslots[i % kScaleAhead];
                cz = 128.f - __half2float(__ushort_as_half((unsigned short)((n & 1) ? zw >> 16 : zw & 0xFFFFu)));
            }
            if (i + kScaleAhead < L) scale_issue(i + kScaleAhead);
            cp_async_commit();
            if (ok) ok = MQ_GEMM_WAIT(sempty + db, (uint32_t)(i / kS) & 1u, flags);
            // the stage's sums of X (asymmetric variant) land with its X tile
            if (asym && ok) ok = MQ_GEMM_WAIT(xfull + db, (uint32_t)(i / kS) & 1u, flags);
            ok = __all_sync(0xFFFFFFFFu, ok);                  // tcgen05.ld is warp-wide
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int cb = 0; cb < kCW; cb += 16) {
                    uint32_t v[16];
                    tmem_ld16(tmem + lane_base + kD0 + (uint32_t)(db * BM + c0 + cb), v);
                    tmem_ld_wait();
                    if (asym) {
                        // sum_k x w = s (D + (128 - z) sum_k x): the level
                        // measured from z instead of 128
                        const float4 *sxp = reinterpret_cast<const float4 *>(sx + db * BM + c0 + cb);
#pragma unroll
                        for (int j4 = 0; j4 < 4; ++j4) {
                            const float4 t = sxp[j4];
                            y[cb + 4 * j4 + 0] = fmaf(s, fmaf(cz, t.x, __uint_as_float(v[4 * j4 + 0])), y[cb + 4 * j4 + 0]);
                            y[cb + 4 * j4 + 1] = fmaf(s, fmaf(cz, t.y, __uint_as_float(v[4 * j4 + 1])), y[cb + 4 * j4 + 1]);
                            y[cb + 4 * j4 + 2] = fmaf(s, fmaf(cz, t.z, __uint_as_float(v[4 * j4 + 2])), y[cb + 4 * j4 + 2]);
                            y[cb + 4 * j4 + 3] = fmaf(s, fmaf(cz, t.w, __uint_as_float(v[4 * j4 + 3])), y[cb + 4 * j4 + 3]);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) y[cb + j] = fmaf(s, __uint_as_float(v[j]), y[cb + j]);
                    }
                }
                tc_fence_before();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(dempty + db);
            // the tile ends with this item (or the range does): write it out
            const bool tile_end = gi == G - 1 || i == L - 1;
            if (tile_end) {
                const int mb = (int)(tu / a.T), t = (int)(tu % a.T);
                const int64_t tn0 = tile_u0, tn1 = tile_u0 + G;    // the tile's items
                const int64_t nrow = (int64_t)t * kTileN + n;
                const int mlim = a.M - (mb * BM + c0);             // columns of this thread inside M
                const bool own = tn0 >= u0 && tn1 <= u1;           // the whole tile is in this range
                int cf = 0, cnt = 1;
                if (!own) {
                    cf = cta_of(tn0, W, a.P);
                    cnt = cta_of(tn1 - 1, W, a.P) - cf + 1;
                }
                // own tile: Y directly; shared tile: this CTA's fp32 partial
                // sums, as float4 (4 columns of one row) at [column / 4][row]
                float4 *pp = reinterpret_cast<float4 *>(a.part + ((size_t)tu * a.maxc + (own ? 0 : blockIdx.x - cf)) *
                                                                     (BM * kTileN)) + (c0 / 4) * kTileN + n;
                __nv_bfloat16 *yp = a.Y + (int64_t)(mb * BM + c0) * a.N + nrow;
                if (own ? nrow < a.N : true) {
#pragma unroll
                    for (int j = 0; j < kCW; j += 4) {
                        if (!own) {
                            pp[(j / 4) * kTileN] = make_float4(y[j], y[j + 1], y[j + 2], y[j + 3]);
                        } else {
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                if (j + q < mlim) yp[(int64_t)(j + q) * a.N] = __float2bfloat16_rn(y[j + q]);
                        }
                    }
                }
                if (!own) {
                    // take a ticket (one thread, after the fold warps' partial
                    // sums: the fence is cumulative over the barrier); the last
                    // CTA to arrive sums the tile after its own range (all
                    // threads of the CTA, in CTA order)
                    named_sync(3, kFoldW * 32);
                    if (f == 0 && lane == 0) {
                        __threadfence();
                        if (atomicAdd(a.tickets + tu, 1u) == (unsigned)(cnt - 1)) {
                            a.tickets[tu] = 0u;                // every part is in: reset for the next launch
                            const int k = flags[4];
                            flags[5 + k] = (int)tu;
                            flags[7 + k] = cnt;
                            flags[4] = k + 1;
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < kCW; ++j) y[j] = 0.f;
                tile_u0 += G;
            }
            if (++gi == G) {
                gi = 0;
                ++tu;
            }
        }
        cp_async_wait<0>();                                    // no scale copy left in flight
    } else if (warp == kXW) {
        // ----------------------------------------------------------------- X
        if (lane == 0) {
            pdl_wait();                                        // X may come from the previous kernel
            int mb = (int)(u0 / TG), g = (int)(u0 % G);        // X block and group of item i
            for (int i = 0; i < L; ++i) {
                const int xs = i % kS, kx = i / kS;
                // the stage is free once its MMAs are done; in the asymmetric
                // variant its sums of X also once the fold has read them
                if (kx > 0 && !mbar_wait_abortable(asym ? dempty + xs : sempty + xs, (uint32_t)(kx - 1) & 1u, flags))
                    break;
#ifdef MQ_TEST_HOOKS
                if (i == 0 && atomicSub(&g_test_drop_x, 1) > 0) {  // item 0 never arrives
                    if (++g == G) {
                        g = 0;
                        if ((int64_t)(i + 1 + u0) % TG == 0) ++mb;
                    }
                    continue;
                }
#endif
                mbar_expect_tx(xfull + xs, C::kXStage + (asym ? BM * 4 : 0));
                tma_load_3d(sX + xs * C::kXStage, &a.xmap, 0, mb * BM, 2 * g, xfull + xs);
                if (asym) bulk_g2s(sx + xs * BM, a.sumx + (int64_t)g * a.Mpad + mb * BM, BM * 4, xfull + xs);
                flags[3] = i + 1;
                if (++g == G) {
                    g = 0;
                    if ((int64_t)(i + 1 + u0) % TG == 0) ++mb;   // rare: once per pass over the tiles
                }
            }
        }
    } else {
        // --------------------------------------------------------------- MMA
        // two issuing threads (lane 0 of each MMA warp): parity p takes the
        // items p, p + 2, ..., so one thread's barrier waits overlap the
        // other's MMAs; within a round of kS items the stage of each item is
        // a constant, and every operand a constant offset from one base
        if (lane == 0) {
            const uint64_t bdesc0 = smem_desc_sw128(smem_u32(sX));
            auto run = [&](auto P) {
                constexpr int p = decltype(P)::value;
                for (int q = 0;; ++q) {                        // round q: items q * kS + s
                    bool more = true;
#pragma unroll
                    for (int e = 0; e < kS / 2; ++e) {
                        const int st = p + 2 * e, i = q * kS + st;
                        if (i >= L) { more = false; break; }
                        if (!mbar_wait_abortable(afull + st, (uint32_t)q & 1u, flags) ||
                            !mbar_wait_abortable(xfull + st, (uint32_t)q & 1u, flags) ||
                            (q > 0 && !mbar_wait_abortable(dempty + st, (uint32_t)(q - 1) & 1u, flags))) {
                            more = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks) {
                            const int h = ks >> 2, kk = ks & 3;
                            const uint64_t bd = bdesc0 + (uint64_t)((st * C::kXStage + h * (BM * 128) + kk * 32) >> 4);
                            mma_bf16_ts(tmem + kD0 + (uint32_t)(st * BM), tmem + (uint32_t)(st * 64 + 8 * ks), bd,
                                        kIdesc, ks > 0 ? 1u : 0u);
                        }
                        mma_commit(sempty + st);               // A, X free; accumulator full
                        flags[p ? 9 : 2] = i + 1;              // last item issued by this thread, + 1
                    }
                    if (!more) break;
                }
            };
            if (warp == kMmaW) run(std::integral_constant<int, 0>{});
            else run(std::integral_constant<int, 1>{});
        }
    }

    // ---- end: let the copies, MMAs and barrier arrivals issued land before
    // the CTA exits (already the case unless a wait gave up)
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
        // stage s is committed by the thread of parity s % 2, for its items
        // s, s + kS, ... below its last item issued
        for (int st = 0; st < kS; ++st) {
            const int last = flags[(st & 1) ? 9 : 2];
            if (last > st) mbar_wait_bounded(sempty + st, (uint32_t)((last - 1 - st) / kS) & 1u);
        }
        drain_ring(xfull, kS, flags[3]);
        if (flags[0]) atomicOr(&g_tc_timeout, 1u);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaW) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }

    // ---- shared tiles whose last part this CTA delivered: Y = sum of the
    // parts in CTA order, every thread of the CTA taking float4 positions
    if (flags[0]) return;
    __threadfence();
    for (int k = 0; k < flags[4]; ++k) {
        const int64_t tu = flags[5 + k];
        const int cnt = flags[7 + k];
        const int mb = (int)(tu / a.T), t = (int)(tu % a.T);
        const float4 *p0 = reinterpret_cast<const float4 *>(a.part + (size_t)tu * a.maxc * (BM * kTileN));
        constexpr int kPos = BM * kTileN / 4;                  // float4 positions of one part
        constexpr int kPer = (kPos + C::kThreads - 1) / C::kThreads;
        constexpr int kBatch = kPer <= 5 ? 2 : 1;              // parts loaded per round
        float4 acc[kPer];
#pragma unroll
        for (int e = 0; e < kPer; ++e) acc[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int sl = 0; sl < cnt; sl += kBatch) {
            float4 v[kBatch][kPer];
#pragma unroll
            for (int b = 0; b < kBatch; ++b)
#pragma unroll
                for (int e = 0; e < kPer; ++e) {
                    const int pos = threadIdx.x + e * C::kThreads;
                    v[b][e] = (sl + b < cnt && pos < kPos) ? __ldcg(p0 + (size_t)(sl + b) * kPos + pos)
                                                           : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
            for (int b = 0; b < kBatch; ++b)
#pragma unroll
                for (int e = 0; e < kPer; ++e) {
                    acc[e].x += v[b][e].x;
                    acc[e].y += v[b][e].y;
                    acc[e].z += v[b][e].z;
                    acc[e].w += v[b][e].w;
                }
        }
#pragma unroll
        for (int e = 0; e < kPer; ++e) {
            const int pos = threadIdx.x + e * C::kThreads;
            if (pos >= kPos) break;
            const int nn = pos % kTileN, m0 = mb * BM + (pos / kTileN) * 4;
            const int64_t nrow = (int64_t)t * kTileN + nn;
            if (nrow >= a.N) continue;
            const float vals[4] = {acc[e].x, acc[e].y, acc[e].z, acc[e].w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (m0 + q < a.M) a.Y[(int64_t)(m0 + q) * a.N + nrow] = __float2bfloat16_rn(vals[q]);
        }
    }
}

struct TcPlan {
    int BM, MB, T, G, P, maxc;
    size_t part_off, sumx_off, ws_bytes;
};

int tc_sm_count() {
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (!n) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

TcPlan tc_plan(int64_t M, int64_t N, int64_t K, int sms) {
    TcPlan p{};
    p.BM = M <= 32 ? 32 : M <= 64 ? 64 : 128;
    p.MB = (int)((M + p.BM - 1) / p.BM);
    p.T = (int)((N + kTileN - 1) / kTileN);
    p.G = (int)(K / kGroup);
    const int64_t W = (int64_t)p.MB * p.T * p.G;
    int64_t P = W / kMinItems;
    if (P > sms) P = sms;
    if (P < 1) P = 1;
    p.P = (int)P;
    // CTAs that can share one tile (its G items over ranges of >= floor(W/P))
    int maxc = 1;
    for (int64_t tu = 0; tu < (int64_t)p.MB * p.T; ++tu) {
        const int c = cta_of(tu * p.G + p.G - 1, W, p.P) - cta_of(tu * p.G, W, p.P) + 1;
        maxc = c > maxc ? c : maxc;
    }
    p.maxc = maxc;
    p.part_off = kTicketBytes;
    const size_t part = (size_t)p.MB * p.T * p.maxc * p.BM * kTileN * sizeof(float);
    p.sumx_off = p.part_off + part;                    // a multiple of 16 bytes
    // sums of X per (group, X row) for the asymmetric variant
    p.ws_bytes = p.sumx_off + (size_t)p.G * p.MB * p.BM * sizeof(float);
    return p;
}

// sumx[g][m] = sum over group g of X[m, k] (fp32), rows m in [M, Mpad) zero:
// the factor of the zero-point term of the asymmetric variant.
__global__ void __launch_bounds__(256)
sumx_kernel(const uint16_t *__restrict__ X, int M, int64_t K, int Mpad, float *__restrict__ sumx) {
    pdl_wait();                                        // X may come from the previous kernel
    pdl_launch_dependents();
    const int64_t G = K / kGroup;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < G * Mpad;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t g = i / Mpad;
        const int m = (int)(i - g * Mpad);
        float acc = 0.f;
        if (m < M) {
            const uint4 *p = reinterpret_cast<const uint4 *>(X + (int64_t)m * K + g * kGroup);
#pragma unroll 4
            for (int c = 0; c < kGroup / 8; ++c) {
                const uint4 v = __ldg(p + c);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    acc += __uint_as_float(w[e] << 16) + __uint_as_float(w[e] & 0xFFFF0000u);
            }
        }
        sumx[i] = acc;
    }
}

// cuTensorMapEncodeTiled from the driver (looked up once, no -lcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static std::atomic<void *> cached{nullptr};
    void *f = cached.load(std::memory_order_acquire);
    if (!f) {
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        cached.store(f, std::memory_order_release);
    }
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
}

// Tensor map of X (M x K bf16, row stride K) seen as (64 columns, M rows,
// K/64 halves): one box of 64 x BM x 2 is the BM x 128 block of one group,
// two halves of BM rows of 128 bytes in the 128-byte swizzle, the layout of
// the MMA's B operand; rows past M read as zeros.
bool encode_x_map(CUtensorMap *map, const uint16_t *X, int64_t M, int64_t K, int BM) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {64, (cuuint64_t)M, (cuuint64_t)(K / 64)};
    const cuuint64_t strides[2] = {(cuuint64_t)K * 2, 128};
    const cuuint32_t box[3] = {64, (cuuint32_t)BM, 2};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t *>(X), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

using TcFn = void (*)(GArgs);

template <int R>
TcFn tc_pick_bm(int BM) {
    switch (BM) {
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

// cudaFuncSetAttribute once per (kernel, device), safe from any host thread.
cudaError_t tc_smem_attr(TcFn fn, int r, int BM, size_t smem) {
    static std::atomic<uint64_t> done[8][3];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int bi = BM == 32 ? 0 : BM == 64 ? 1 : 2;
    const uint64_t bit = 1ull << (dev & 63);
    std::atomic<uint64_t> &d = done[r - 1][bi];
    if (d.load(std::memory_order_acquire) & bit) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(227 * 1024));
    (void)smem;
    if (e == cudaSuccess) d.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

}  // namespace

size_t gemm_tc_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
    (void)r;
    return tc_plan(M, N, K, tc_sm_count()).ws_bytes;
}

mq_status launch_gemm_tc(const uint16_t *X, const mq_weights *w, int64_t M, uint16_t *Y,
                         void *ws, size_t ws_bytes, cudaStream_t st) {
    const TcPlan p = tc_plan(M, w->N, w->K, tc_sm_count());
    if (!ws || p.ws_bytes > ws_bytes) return fail(MQ_ERR_WORKSPACE, "GEMM workspace too small");
    if ((int64_t)p.MB * p.T > (int64_t)(kTicketBytes / sizeof(unsigned)))
        return fail(MQ_ERR_UNSUPPORTED, "too many output tiles for the ticket region");
    TcFn fn = tc_pick(w->r, p.BM);
    const int threads = p.BM == 128 ? TcCfg<1, 128>::kThreads : TcCfg<1, 32>::kThreads;
    const size_t smem = tc_smem_bytes(w->r, p.BM);
    cudaError_t e = tc_smem_attr(fn, w->r, p.BM, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    char *wsb = static_cast<char *>(ws);
    GArgs a{};
    if (!encode_x_map(&a.xmap, X, M, w->K, p.BM)) return fail(MQ_ERR_CUDA, "cuTensorMapEncodeTiled (X)");
    a.planes = w->planes;
    a.scales = reinterpret_cast<const __half *>(w->scales);
    a.zeros = reinterpret_cast<const __half *>(w->zeros);
    a.sumx = reinterpret_cast<const float *>(wsb + p.sumx_off);
    a.Mpad = p.MB * p.BM;
    a.Y = reinterpret_cast<__nv_bfloat16 *>(Y);
    a.part = reinterpret_cast<float *>(wsb + p.part_off);
    a.tickets = reinterpret_cast<unsigned *>(wsb);
    a.N = w->N;
    a.K = w->K;
    a.M = (int)M;
    a.T = p.T;
    a.G = p.G;
    a.MB = p.MB;
    a.P = p.P;
    a.maxc = p.maxc;
    a.plane_words = (int64_t)p.T * kTileN * (w->K / 32);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    if (w->zeros) {
        // the asymmetric variant's sums of X, written before the GEMM reads them
        cudaLaunchConfig_t pc = {};
        const int64_t cells = (int64_t)p.G * a.Mpad;
        pc.gridDim = dim3((unsigned)((cells + 255) / 256 < 1184 ? (cells + 255) / 256 : 1184));
        pc.blockDim = dim3(256);
        pc.stream = st;
        pc.attrs = attr;
        pc.numAttrs = 1;
        e = cudaLaunchKernelEx(&pc, sumx_kernel, X, (int)M, (int64_t)w->K, a.Mpad,
                               reinterpret_cast<float *>(wsb + p.sumx_off));
        if (e != cudaSuccess) return cuda_fail(e, "sumx_kernel");
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.P);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, fn, a);
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

#ifdef MQ_TEST_HOOKS
// Test-hook builds only: make the next `n` GEMM CTAs drop one X arrival.
extern "C" __attribute__((visibility("default"))) int mq_test_drop_x_arrivals(int n) {
    return (int)cudaMemcpyToSymbol(mq::g_test_drop_x, &n, sizeof(n));
}
#endif
