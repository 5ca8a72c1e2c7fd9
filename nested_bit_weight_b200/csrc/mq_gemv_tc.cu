// Batch M <= 8: the nested r-bit product on the tcgen05 tensor cores, with the
// decoded weights as the MMA's A operand in tensor memory.
//
// The r-bit model is the first r bit planes of the parent ("MatGPTQ:
// Efficient and Accurate Inference over Nested Quantized Models", abstract:
// an r-bit model reads exactly r bits); its level is
//     v_r(q) = 2^(8-r) q + 2^(7-r) - 128,   w = s_g v_r(q),
// so per 128-column group g and batch row m
//     sum_k x_k w_k = s_g ( 2^(8-r) sum_k x_k q_k + (2^(7-r) - 128) S_g ),
// with S_g = sum_k x_k.  The tensor core computes sum_k x_k q_k exactly:
//
// * A (M = 128 weight rows x K = 128 columns of one group, unsigned 8-bit, in
//   TMEM).  Each thread of a 4-warp team owns one row: it reads the row's r
//   plane words of the group (16 bytes per plane), turns every 32-column word
//   into 8 registers whose bytes are fields q << sh(i) (one AND per register,
//   sh = the field's bit offset in its byte), and stores the 32 registers to
//   its TMEM lane with one tcgen05.st.  Byte b of register i of word t is
//   column 32t + 8b + i; TMEM column 8t + i holds it, so A's k = 32t + 4i + b.
// * B (N = 16 or 32 columns = 4 slices x M batch rows, signed 8-bit, shared
//   memory, K-major, 128-byte swizzle).  z_k = x_k 2^(-sh(k)) is cut into
//   four int8 slices relative to the group exponent Eg = max floor(log2|z|):
//       z_k = 2^(Eg-27) (a_1 2^21 + a_2 2^14 + a_3 2^7 + a_4),
//   exact for every x within 2^-20 of the group's largest; column 4m + j at
//   k = 32t + 4i + b holds slice j of z at column 32t + 8b + i.
// * D (128 x N, int32, TMEM) = exact per-group integer sums, read back with
//   tcgen05.ld and folded into fp32: y += s_g 2^(8-r) 2^(Eg-6) sum_j 2^(-7j) D_j
//   + s_g (2^(7-r) - 128) S_g.
//
// Work: the (128-row tile, group) items in tile order are cut into one
// contiguous range per CTA, row tiles being shared only by the CTAs of one
// thread-block cluster (shapes whose X operand does not fit in shared memory
// are left to the GEMM).  The packed format stores the 2 KB block of one
// (tile, group) contiguously per plane, items in this order, so a run of
// items is one contiguous stream per plane: a producer warp copies batches of
// items with bulk asynchronous copies into a ring of stages.  Three teams of
// four warps each take a pair of items per iteration: decode into registers,
// wait for the MMAs of their previous pair, store the new A to TMEM, read the
// previous D, meet at a team barrier, issue the MMAs and fold the previous
// pair.  Partial sums of a tile are combined in a fixed order; a tile shared
// by several CTAs of a cluster is summed by its owner from the parts the
// others write into its shared memory.
#include <string.h>

#include <atomic>
#include <mutex>

#include "mq_common.cuh"
#include "mq_bits.cuh"
#include "mq_sm100.cuh"

namespace mq {
namespace {

using namespace sm100;

constexpr int kTeams = 3;                    // teams of 4 warps (128 rows)
constexpr int kCW = 4 * kTeams;              // consumer warps
constexpr int kProd = kCW;                   // producer warp
constexpr int kThreads = (kCW + 1) * 32;
constexpr int kBatch = 2 * kTeams;           // items per bulk copy: one pair per team
constexpr int kSlices = 4;                   // int8 slices per x
constexpr int kHeadBatches = 2;              // batches streamed before X is requested
constexpr uint32_t kTmemCols = 512;          // TMEM columns per CTA (one CTA per SM)
constexpr size_t kSmemMax = 227 * 1024;      // shared memory of one CTA per SM

// ------------------------------------------------------------ operand decode
// Bit offset of register i's field inside each byte (the byte holds q << sh).
template <int R> __host__ __device__ constexpr int field_shift(int i) {
    return R == 1 ? i
         : R == 2 ? 2 * (i >> 1)
         : R == 3 ? 4 * (i >> 2) + 1
         : R == 4 ? 4 * (i >> 2)
                  : 8 - R;
}

// P[p] = plane p's word (planes >= R are 0) -> A[i]: byte b = field of column
// 8b + i, shifted by field_shift<R>(i).
template <int R>
__device__ __forceinline__ void field_operands(const uint32_t (&P)[8], uint32_t *A) {
    if constexpr (R == 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) A[i] = P[0] & (0x01010101u << i);
    } else if constexpr (R == 2) {
        const uint32_t e = pair_even(P[0], P[1]), o = pair_odd(P[0], P[1]);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            A[2 * s] = e & (0x03030303u << (2 * s));
            A[2 * s + 1] = o & (0x03030303u << (2 * s));
        }
    } else if constexpr (R <= 4) {
        uint32_t Nw[4];
        nibble_words<R>(P, 0, Nw);
#pragma unroll
        for (int d = 0; d < 4; ++d) {
            A[d] = Nw[d] & 0x0F0F0F0Fu;
            A[4 + d] = Nw[d] & 0xF0F0F0F0u;
        }
    } else {
        uint32_t B8[8];
        byte_words<R>(P, B8);
#pragma unroll
        for (int i = 0; i < 8; ++i) A[i] = B8[i];
    }
}

// ------------------------------------------------------ barriers and copies
// (mbarrier, bulk-copy, cluster and tcgen05 wrappers shared by every kernel
// of the library are in mq_sm100.cuh)
__device__ unsigned int g_gemv_timeout;     // set when a bounded wait gave up

// Suspending variant for the producer, which waits long and is not on the
// per-item critical path: the thread sleeps in try_wait instead of spinning
// (spinning would take issue slots from the decoding warps).
__device__ __forceinline__ bool bar_try_sleep(uint64_t *b, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n .reg .pred p;\n"
                 " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 2000;\n"
                 " selp.u32 %0, 1, 0, p;\n}"
                 : "=r"(ok) : "r"(smem_u32(b)), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool bar_wait_sleep(uint64_t *b, uint32_t parity) {
    const uint64_t t0 = global_ns();
    while (!bar_try_sleep(b, parity))
        if (global_ns() - t0 > kWaitNs) return false;
    return true;
}
// Wait for the phase of parity `parity` to complete by polling (a suspended
// try_wait can resume well after the phase completes, which the per-item
// hand-offs of this kernel cannot afford); gives up after about a second.
__device__ __forceinline__ bool bar_wait(uint64_t *b, uint32_t parity) { return mbar_wait_bounded(b, parity); }
__device__ __forceinline__ void st_release(int *p, int v) {
    asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}
// test_wait with cluster-scope acquire (parts written by other CTAs).
__device__ __forceinline__ bool bar_try_cluster(uint64_t *b, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n .reg .pred p;\n"
                 " mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
                 " selp.u32 %0, 1, 0, p;\n}"
                 : "=r"(ok) : "r"(smem_u32(b)), "r"(parity) : "memory");
    return ok != 0;
}

// ------------------------------------------------------------ decomposition
// Items u = 0 .. W-1, W = T * KC (T 128-row tiles, KC = K / 128 groups), in
// (tile, group) order; CTA b owns the contiguous items [first(b), first(b+1)).
// Clusters: the row tiles are cut into NC contiguous runs, one per cluster of
// CS CTAs; the items of a cluster's run are cut into CS contiguous ranges.  A
// row tile is therefore shared only by CTAs of one cluster, which sum it
// through distributed shared memory (CS = 1: every CTA owns whole tiles).
struct Work {
    int64_t T, KC;          // row tiles, groups per tile
    int NC, CS;             // clusters, CTAs per cluster
    // 32-bit arithmetic (T * KC < 2^31 and the products below stay under 2^32):
    // a 64-bit division costs hundreds of cycles on the GPU
    __host__ __device__ uint32_t tile_begin(uint32_t c) const {
        return (uint32_t)(c * (uint32_t)T) / (uint32_t)NC;
    }
    __host__ __device__ int64_t first(int64_t bb) const {
        const uint32_t b = (uint32_t)bb, c = b / (uint32_t)CS, k = b - c * (uint32_t)CS;
        const uint32_t t0 = tile_begin(c), t1 = tile_begin(c + 1);
        const uint32_t a = t0 * (uint32_t)KC, wc = (t1 - t0) * (uint32_t)KC;
        return (int64_t)(a + k * wc / (uint32_t)CS);
    }
    // CTA that holds item u
    __host__ __device__ int64_t cta_of(int64_t uu) const {
        const uint32_t u = (uint32_t)uu, t = u / (uint32_t)KC;
        const uint32_t c = ((t + 1) * (uint32_t)NC - 1) / (uint32_t)T;
        const uint32_t t0 = tile_begin(c), t1 = tile_begin(c + 1);
        const uint32_t a = t0 * (uint32_t)KC, wc = (t1 - t0) * (uint32_t)KC;
        return (int64_t)(c * (uint32_t)CS + ((u - a + 1) * (uint32_t)CS - 1) / wc);
    }
    __host__ __device__ int64_t ctas() const { return (int64_t)NC * CS; }
};

struct Range { int u0, u1, L; };
__host__ __device__ inline Range make_range(const Work &w, int64_t b) {
    Range r;
    r.u0 = (int)w.first(b);
    r.u1 = (int)w.first(b + 1);
    r.L = r.u1 - r.u0;
    return r;
}
// Group held by X slot `slot` of the CTA (slots count groups from the group
// of the CTA's first item, modulo KC).
__host__ __device__ inline int slot_chunk(const Work &w, const Range &r, int slot) {
    const int KC = (int)w.KC;
    const int c = r.u0 % KC + slot;
    return c >= KC ? c - KC : c;
}

// Kernel arguments (one struct, passed as a grid constant).
struct Args {
    const __nv_bfloat16 *X;
    const uint8_t *planes;  // tiled planes (2 KB per (tile, group) block per plane)
    const uint8_t *scales;  // tiled fp16 scales (256 B per block)
    __nv_bfloat16 *Y;
    Work w;
    int64_t N, K, G;
    int64_t plane_bytes;    // bytes of one plane
    int M, NB, S;           // batch rows, MMA N (16 or 32), ring stages (multiple of kBatch)
    // shared-memory offsets from the 1024-byte aligned base
    uint32_t o_ring, o_sring, o_b, o_pair, o_res, o_bar, o_red, o_misc;
};

// ------------------------------------------------------------- X operand
// Fixed-point value F = z 2^(27 - Ez), z = x 2^(-sh), truncated toward zero;
// x is given by its bf16 bits (zero and subnormal inputs give 0).
__device__ __forceinline__ int fixed_point(uint32_t h, int sh, int Ez) {
    const int e8 = (int)((h >> 7) & 0xFFu);
    const int mant = (int)((h & 0x7Fu) | 0x80u);
    const int sft = e8 - 107 - sh - Ez;                  // <= 20 for finite x
    int mag = sft >= 0 ? (mant << sft) : (sft > -9 ? (mant >> -sft) : 0);
    if (e8 == 0) mag = 0;
    return (h & 0x8000u) ? -mag : mag;
}

// Low bytes of four values -> one word (byte b from v_b).
__device__ __forceinline__ uint32_t pack_bytes(int v0, int v1, int v2, int v3) {
    const uint32_t lo = __byte_perm((uint32_t)v0, (uint32_t)v1, 0x0040);
    const uint32_t hi = __byte_perm((uint32_t)v2, (uint32_t)v3, 0x0040);
    return __byte_perm(lo, hi, 0x5410);
}

// X operand of the CTA's groups, built by the team warps.  Slot sl (the
// sl-th distinct group of the range) lives in B tile sl / gpb at position
// pos = sl % gpb (gpb = groups per tile): MMA column 4 (pos M + m) + j holds
// slice j of batch row m, K-major with the 128-byte swizzle; the pair
// {2^(8-r) 2^(Eg-6), S_g} of (slot, m) at pairs[sl * 8 + m].  X is staged
// first with one round of 16-byte copies (staging[sl][m][128 values]).
template <int R>
__device__ void build_x_operand(const Args &a, uint8_t *smem, const Work &w, const Range &rg,
                                int nslot, int *flags) {
    constexpr int kPrep = kCW * 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int M = a.M, gpb = a.NB == 16 ? (M == 1 ? 4 : M == 2 ? 2 : 1) : 1;
    const int t = lane >> 3, wi = lane & 7;
    const int sh = field_shift<R>(wi);
    float2 *pairs = reinterpret_cast<float2 *>(smem + a.o_pair);
    // the warp's tasks (slot, m) in chunks of 4: all loads of a chunk first
    const uint16_t *X = reinterpret_cast<const uint16_t *>(a.X);
    for (int t0 = warp; t0 < nslot * M; t0 += 4 * kCW) {
        uint32_t hv[4][4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int task = t0 + c * kCW;
            if (task < nslot * M) {
                const int sl = task / M, m = task - sl * M;
                const uint16_t *xr = X + (int64_t)m * a.K + (int64_t)slot_chunk(w, rg, sl) * kGroup + 32 * t + wi;
#pragma unroll
                for (int b = 0; b < 4; ++b) hv[c][b] = xr[8 * b];
            }
        }
        if (t0 == 0 && lane == 0) st_release(&flags[2], (int)(hv[0][0] | 1u));   // X fetched: stream the rest
        // the four tasks side by side (independent chains; absent tasks are
        // computed on zeros and not stored)
        int emax[4];
        float sum[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            emax[c] = -1000;
            sum[c] = 0.f;
            if (t0 + c * kCW >= nslot * M) {
#pragma unroll
                for (int b = 0; b < 4; ++b) hv[c][b] = 0u;
            }
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int e8 = (int)((hv[c][b] >> 7) & 0xFFu);
                const int v = e8 ? e8 - sh : -1000;
                emax[c] = v > emax[c] ? v : emax[c];
                sum[c] += __uint_as_float(hv[c][b] << 16);
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int other = __shfl_xor_sync(0xffffffffu, emax[c], o);
                emax[c] = other > emax[c] ? other : emax[c];
                sum[c] += __shfl_xor_sync(0xffffffffu, sum[c], o);
            }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int task = t0 + c * kCW;
            if (task >= nslot * M) break;
            const int sl = task / M, m = task - sl * M;
            const int Eg = emax[c] > -1000 ? emax[c] - 127 : 0;
            int F[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) F[b] = fixed_point(hv[c][b], sh, Eg);
            uint32_t wd[kSlices];
            wd[0] = pack_bytes(F[0] >> 21, F[1] >> 21, F[2] >> 21, F[3] >> 21);
            wd[1] = pack_bytes(F[0] >> 14, F[1] >> 14, F[2] >> 14, F[3] >> 14) & 0x7F7F7F7Fu;
            wd[2] = pack_bytes(F[0] >> 7, F[1] >> 7, F[2] >> 7, F[3] >> 7) & 0x7F7F7F7Fu;
            wd[3] = pack_bytes(F[0], F[1], F[2], F[3]) & 0x7F7F7F7Fu;
            uint8_t *tile = smem + a.o_b + (size_t)(sl / gpb) * a.NB * 128;
            const int chunk = 2 * t + (wi >> 2);           // 16-byte chunk of k = 32t + 4wi
#pragma unroll
            for (int j = 0; j < kSlices; ++j) {
                const int row = 4 * ((sl % gpb) * M + m) + j;
                *reinterpret_cast<uint32_t *>(tile + (row >> 3) * 1024 + (row & 7) * 128 +
                                              ((chunk ^ (row & 7)) << 4) + 4 * (wi & 3)) = wd[j];
            }
            if (lane == 0) {
                // 2^(8-r) 2^(Eg-6), clamped to the normal fp32 range
                int ex = 2 - R + Eg;
                ex = ex < -126 ? -126 : (ex > 127 ? 127 : ex);
                pairs[sl * 8 + m] = make_float2(__int_as_float((ex + 127) << 23), sum[c]);
            }
        }
    }
    // the tensor core reads B through the async proxy
    fence_proxy_async_smem();
    named_sync(1, kPrep);
}

// ------------------------------------------------------------------ kernel
// D columns of one item (4 slices per batch row, 4 MT registers) into registers.
template <int MT>
__device__ __forceinline__ void read_d(uint32_t taddr, int *d) {
    uint32_t *u = reinterpret_cast<uint32_t *>(d);
    if constexpr (MT == 1) tmem_ld4(taddr, u);
    else if constexpr (MT == 2) tmem_ld8(taddr, u);
    else if constexpr (MT == 4) tmem_ld16(taddr, u);
    else tmem_ld32(taddr, u);
}

// Fold one item's D into y (row `row` of the team's current tile); on a tile
// change the finished tile's sums go to res first.
#define FOLD_ITEM(D, SC, SLOT, LTILE)                                                      \
    do {                                                                                   \
        if ((LTILE) != cur) {                                                              \
            if (cur >= 0) {                                                                \
                _Pragma("unroll") for (int m = 0; m < MT; ++m) if (m < M)                  \
                    res[((team * ntile + cur) * M + m) * 128 + row] = y[m];                \
            }                                                                              \
            _Pragma("unroll") for (int m = 0; m < MT; ++m) y[m] = 0.f;                     \
            cur = (LTILE);                                                                 \
        }                                                                                  \
        _Pragma("unroll") for (int m = 0; m < MT; ++m) {                                   \
            if (m < M) {                                                                   \
                const float v = (float)(D)[4 * m] + 0x1p-7f * (float)(D)[4 * m + 1] +      \
                                0x1p-14f * (float)(D)[4 * m + 2] +                         \
                                0x1p-21f * (float)(D)[4 * m + 3];                          \
                const float2 ge = pairs[(SLOT) * 8 + m];                                   \
                y[m] = fmaf((SC) * ge.x, v, fmaf((SC) * kOffset, ge.y, y[m]));             \
            }                                                                              \
        }                                                                                  \
    } while (0)

// MT: batch class (M = 1, M = 2, M <= 4, M <= 8), fixing the MMA N (16 or 32)
// and the D columns read back per item.
template <int R, int MT>
__global__ void __launch_bounds__(kThreads, 1)
nested_gemv_tc_kernel(const __grid_constant__ Args a) {
    constexpr uint32_t kPlaneBlk = 2048;                // one (tile, group) block of one plane
    extern __shared__ uint8_t smem_raw[];
    // align the base by an offset so the compiler keeps the shared address space
    uint8_t *smem = smem_raw + ((1024u - (static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw)) & 1023u)) & 1023u);
    const Work &w = a.w;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Range rg = make_range(w, blockIdx.x);
    const int L = rg.L, S = a.S, M = a.M, G = (int)a.G;
    const int nbs = S / kBatch;                          // batch slots in the ring
    const int nbatch = (L + kBatch - 1) / kBatch;
    const int64_t tf = rg.u0 / G;                        // first tile of the range
    const int ntile = (int)((rg.u1 - 1) / G - tf + 1);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + a.o_bar);
    uint64_t *empty = full + nbs;
    uint64_t *dfull = empty + nbs;                       // [team]: the pair's MMAs done
    uint64_t *rbar = dfull + kTeams;                     // [tile]: parts of the tile received
    // parts of the split tiles this CTA owns: [tile][contributor][m][128]
    float *red = reinterpret_cast<float *>(smem + a.o_red);
    int *flags = reinterpret_cast<int *>(smem + a.o_misc);   // [0] error [1] batches issued [2] X asked
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + a.o_misc + 16);
    float *res = reinterpret_cast<float *>(smem + a.o_res);  // [team][tile][m][128]
    const int nslot = (int)(L < G ? L : G);

    // a batch of 4 items = one pair per team; each team warp frees it once
    if (threadIdx.x < 2 * nbs) mbar_init(full + threadIdx.x, threadIdx.x < nbs ? 1u : 4u * kTeams);
    // one commit per MMA issuer of a pair (kIssuers threads per team)
    if (threadIdx.x < kTeams) mbar_init(dfull + threadIdx.x, (uint32_t)(MT <= 2 ? 4 : 2));
    // The CTA holding a tile's first item owns it; if the tile continues in
    // later CTAs (of the same cluster), it waits for their parts.
    const int64_t tl = (rg.u1 - 1) / G;                  // last tile of the range
    const int64_t own_last = (tl * G >= rg.u0 && tl * G + G > rg.u1) ? tl : -1;
    const int own_nc = own_last >= 0 ? (int)(w.cta_of(own_last * G + G - 1) - blockIdx.x + 1) : 0;
    if (threadIdx.x == 0 && own_nc > 1) mbar_init(rbar + (own_last - tf), (uint32_t)(own_nc - 1));
    if (threadIdx.x == 0) { flags[0] = 0; flags[1] = 0; flags[2] = 0; }
    for (int i = threadIdx.x; i < kTeams * ntile * M * 128; i += kThreads) res[i] = 0.f;
    fence_mbar_init();
    __syncthreads();
    // every CTA of the cluster has initialised its barriers before any part is sent
    if (w.CS > 1) cluster_arrive();

    if (warp == kProd) {
        // ---------------------------------------------------------- producer
        // batch b = items [4b, 4b + 4): one bulk copy per plane and one for the
        // scales (consecutive items are consecutive blocks), into ring slot b % nbs
        if (lane == 0) {
            bool ok = true;
            for (int b = 0; b < nbatch && ok; ++b) {
                if (b == kHeadBatches) {
                    // the next call may start; and X should not queue behind the rest
                    pdl_launch_dependents();
                    const uint64_t t0 = global_ns();
                    while (ld_acquire(&flags[2]) == 0 && ok) {
                        if (global_ns() - t0 > kWaitNs) ok = false;
                        __nanosleep(128);
                    }
                    if (!ok) break;
                }
                const int bs = b % nbs;
                if (b >= nbs && !bar_wait_sleep(empty + bs, (uint32_t)((b / nbs) - 1) & 1u)) { ok = false; break; }
                const int i0 = b * kBatch, n = (L - i0) < kBatch ? (L - i0) : kBatch;
                const int64_t u = rg.u0 + i0;
                mbar_expect_tx(full + bs, (uint32_t)n * (kPlaneBlk * R + 256));
#pragma unroll
                for (int p = 0; p < R; ++p)
                    bulk_g2s(smem + a.o_ring + ((size_t)p * S + (size_t)bs * kBatch) * kPlaneBlk,
                             a.planes + p * a.plane_bytes + u * kPlaneBlk, (uint32_t)n * kPlaneBlk, full + bs);
                bulk_g2s(smem + a.o_sring + (size_t)bs * kBatch * 256, a.scales + u * 256,
                         (uint32_t)n * 256, full + bs);
                st_release(&flags[1], b + 1);
            }
            if (nbatch <= kHeadBatches) pdl_launch_dependents();
            if (!ok) { st_release(&flags[0], 1); atomicOr(&g_gemv_timeout, 1u); }
        }
    } else if (warp < kCW) {
        // ------------------------------------------------------------- teams
        // TMEM is taken here, off the producer's path
        if (warp == 0) {
            tmem_alloc(tmem_slot, kTmemCols);
            tmem_relinquish();
        }
        tc_fence_before();
        pdl_wait();                              // X comes from the previous kernel
        build_x_operand<R>(a, smem, w, rg, nslot, flags);       // ends with a team barrier
        tc_fence_after();
        const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(tmem_slot);
        const int team = warp >> 2, q = warp & 3, row = q * 32 + lane;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const uint32_t col0 = tmem + (uint32_t)team * 128;       // A0 A1 at +0 +32, D0 D1 at +64 +64+NB
        constexpr int gpb = MT <= 4 ? 4 / MT : 1;      // groups per B tile
        const float2 *pairs = reinterpret_cast<const float2 *>(smem + a.o_pair);
        constexpr float kOffset = (float)(128 >> (R - 1)) * 0.5f - 128.0f;   // 2^(7-r) - 128
        float y[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) y[m] = 0.f;
        int cur = -1;                                    // local tile of y
        // Iteration jj decodes the team's pair jj (items i0 = kBatch jj + 2 team and
        // i0 + 1) into registers, waits for the MMAs of pair jj - 1, stores
        // the new A, reads the old D, and folds pair jj - 1.  Indices advance
        // by kBatch items without divisions: ring stage, X slot, group and tile.
        const int Jp = (L - 2 * team + kBatch - 1) / kBatch;   // pairs of this team
        float sp[2] = {0.f, 0.f};                        // previous pair: scales, X slots, tiles
        int slp[2] = {0, 0}, ltp[2] = {0, 0}, np = 0;
        int st = 2 * team, fpar = 0;                     // ring stage of i0, parity of its fill
        int xslot = 2 * team, g = rg.u0 % G + 2 * team, lt = 0;
        while (xslot >= G) xslot -= G;
        while (g >= G) { g -= G; ++lt; }
        bool ok = true;
        constexpr int ND = 4 * MT;                       // D columns read per item
        const uint32_t idesc = idesc_u8s8(a.NB);
        constexpr int gsh = MT == 1 ? 2 : MT == 2 ? 1 : 0;   // log2 groups per B tile
        const uint32_t b0 = smem_u32(smem + a.o_b);
        // MMA issuers: for M <= 2 the first thread of each warp q issues K steps
        // 2(q&1), 2(q&1)+1 of item q>>1 into its own half of D; otherwise the
        // first thread of warp e < 2 issues all four steps of item e
        const bool issuer = lane == 0 && (MT <= 2 || q < 2);
        int issued = 0;                                  // pairs whose MMAs were issued
        for (int jj = 0; jj <= Jp; ++jj) {
            const bool have = jj < Jp, back = jj > 0;
            const int i0 = kBatch * jj + 2 * team;
            const int n = have ? (i0 + 1 < L ? 2 : 1) : 0;   // items in this pair
            uint32_t A0[32], A1[32];
            float sc[2] = {0.f, 0.f};
            bool good = ok;
            if (have && good) {
                const int bs = st / kBatch;              // ring slot of the batch
                good = __all_sync(0xffffffffu, bar_wait(full + bs, (uint32_t)fpar));
                if (good) {
                    uint4 pw[R];
#pragma unroll
                    for (int p = 0; p < R; ++p)
                        pw[p] = *reinterpret_cast<const uint4 *>(smem + a.o_ring + ((size_t)p * S + st) * kPlaneBlk + row * 16);
                    sc[0] = __half2float(*reinterpret_cast<const __half *>(smem + a.o_sring + (size_t)st * 256 + row * 2));
#pragma unroll
                    for (int t4 = 0; t4 < 4; ++t4) {
                        uint32_t P[8];
#pragma unroll
                        for (int p = 0; p < 8; ++p) {
                            const uint4 &v = pw[p < R ? p : 0];
                            P[p] = p < R ? (t4 == 0 ? v.x : t4 == 1 ? v.y : t4 == 2 ? v.z : v.w) : 0u;
                        }
                        field_operands<R>(P, A0 + 8 * t4);
                    }
                    if (n == 2) {
#pragma unroll
                        for (int p = 0; p < R; ++p)
                            pw[p] = *reinterpret_cast<const uint4 *>(smem + a.o_ring + ((size_t)p * S + st + 1) * kPlaneBlk + row * 16);
                        sc[1] = __half2float(*reinterpret_cast<const __half *>(smem + a.o_sring + (size_t)(st + 1) * 256 + row * 2));
#pragma unroll
                        for (int t4 = 0; t4 < 4; ++t4) {
                            uint32_t P[8];
#pragma unroll
                            for (int p = 0; p < 8; ++p) {
                                const uint4 &v = pw[p < R ? p : 0];
                                P[p] = p < R ? (t4 == 0 ? v.x : t4 == 1 ? v.y : t4 == 2 ? v.z : v.w) : 0u;
                            }
                            field_operands<R>(P, A1 + 8 * t4);
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(empty + bs);
                }
            }
            if (back && good) {
                // the MMAs of pair jj - 1 are done: A is free and D holds their sums
                good = __all_sync(0xffffffffu, bar_wait(dfull + team, (uint32_t)((jj - 1) & 1)));
                tc_fence_after();
            }
            int d0[ND], d1[ND];
            if (good) {
                if (have) {
                    tmem_st32(lane_base + col0, A0);
                    if (n == 2) tmem_st32(lane_base + col0 + 32, A1);
                }
                if (back) {
                    if constexpr (MT <= 2) {
                        // each item's D is two halves (K steps 0-1 and 2-3): add them
                        int h0[ND], h1[ND];
                        const uint32_t o0 = 4 * M * (slp[0] & (gpb - 1)), o1 = 4 * M * (slp[1] & (gpb - 1));
                        read_d<MT>(lane_base + col0 + 64 + o0, d0);
                        read_d<MT>(lane_base + col0 + 64 + 16 + o0, h0);
                        if (np == 2) {
                            read_d<MT>(lane_base + col0 + 96 + o1, d1);
                            read_d<MT>(lane_base + col0 + 112 + o1, h1);
                        }
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < ND; ++i) {
                            d0[i] += h0[i];
                            d1[i] += h1[i];
                        }
                    } else if constexpr (MT <= 4) {
                        read_d<MT>(lane_base + col0 + 64 + 4 * M * (slp[0] & (gpb - 1)), d0);
                        if (np == 2) read_d<MT>(lane_base + col0 + 64 + a.NB + 4 * M * (slp[1] & (gpb - 1)), d1);
                        tmem_ld_wait();
                    } else {
                        read_d<MT>(lane_base + col0 + 64 + 4 * M * (slp[0] & (gpb - 1)), d0);
                        tmem_ld_wait();
                        FOLD_ITEM(d0, sp[0], slp[0], ltp[0]);
                        if (np == 2) {
                            read_d<MT>(lane_base + col0 + 64 + a.NB + 4 * M * (slp[1] & (gpb - 1)), d1);
                            tmem_ld_wait();
                        }
                    }
                }
                if (have) tmem_st_wait();
            }
            tc_fence_before();
            // the whole team has stored A and read D (or a wait timed out)
            if (!named_sync_and(2 + team, 128, good)) { ok = false; break; }
            if (have && issuer) {
                // D[team][e] = A[team][e] . B(X slot of item e)^T, K = 128 in 4 steps;
                // every issuer commits (an empty commit arrives at once)
                tc_fence_after();
                if constexpr (MT <= 2) {
                    const int e = q >> 1, h = q & 1;
                    if (e < n) {
                        const int sl = xslot + e >= G ? xslot + e - G : xslot + e;
                        const uint32_t baddr = b0 + (uint32_t)((sl >> gsh) * a.NB * 128);
#pragma unroll
                        for (int k2 = 0; k2 < 2; ++k2) {
                            const int kk = 2 * h + k2;
                            mma_i8_ts(col0 + 64 + (uint32_t)(32 * e + 16 * h), col0 + 32 * e + 8 * kk,
                                      smem_desc_sw128(baddr + 32 * kk), idesc, k2 > 0 ? 1u : 0u);
                        }
                    }
                } else {
                    const int e = q;
                    if (e < n) {
                        const int sl = xslot + e >= G ? xslot + e - G : xslot + e;
                        const uint32_t baddr = b0 + (uint32_t)((sl >> gsh) * a.NB * 128);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_i8_ts(col0 + 64 + (uint32_t)(e * a.NB), col0 + 32 * e + 8 * kk,
                                      smem_desc_sw128(baddr + 32 * kk), idesc, kk > 0 ? 1u : 0u);
                    }
                }
                mma_commit(dfull + team);
            }
            if (have) ++issued;
            if (back) {
                if constexpr (MT <= 4) FOLD_ITEM(d0, sp[0], slp[0], ltp[0]);
                if (np == 2) FOLD_ITEM(d1, sp[1], slp[1], ltp[1]);
            }
            // this pair becomes the previous one; advance by kBatch items
            np = n;
            sp[0] = sc[0]; sp[1] = sc[1];
            slp[0] = xslot; ltp[0] = lt;
            slp[1] = xslot + 1 == G ? 0 : xslot + 1;
            ltp[1] = g + 1 == G ? lt + 1 : lt;
            st += kBatch;
            if (st >= S) { st -= S; fpar ^= 1; }
            xslot += kBatch;
            while (xslot >= G) xslot -= G;
            g += kBatch;
            while (g >= G) { g -= G; ++lt; }
        }
        if (cur >= 0) {
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (m < M) res[((team * ntile + cur) * M + m) * 128 + row] = y[m];
        }
        if (!ok && issued > 0) {
            // the team's last MMAs may still run: let them finish before TMEM is freed
            bar_wait(dfull + team, (uint32_t)((issued - 1) & 1));
        }
        if (!ok && lane == 0) { st_release(&flags[0], 1); atomicOr(&g_gemv_timeout, 1u); }
        named_sync(1, kCW * 32);
        // ---- combine the teams per tile (fixed order).  A tile inside this
        // CTA goes to Y; a tile this CTA owns but shares keeps its part in
        // slot 0 of `red`; the first tile, if it started in an earlier CTA of
        // the cluster, is sent to slot j of its owner (j = distance in CTAs).
        const int64_t ra0 = tf * G;
        const bool sends = ra0 < rg.u0;                  // the first tile started earlier
        const int64_t owner = sends ? w.cta_of(ra0) : -1;
        const int owner_rank = (int)owner % w.CS;
        const int owner_lt = sends ? (int)tf - (int)w.first(owner) / G : 0;
        const int jsend = (int)(blockIdx.x - owner);
        if (sends) cluster_wait();                       // the owner's barrier is initialised
        const uint32_t red_base = smem_u32(red);
        for (int idx = threadIdx.x; idx < ntile * M * 128; idx += kCW * 32) {
            const int lt = idx / (M * 128), rem = idx - lt * M * 128, m = rem >> 7, rr = rem & 127;
            float v = 0.f;
#pragma unroll
            for (int tm = 0; tm < kTeams; ++tm) v += res[((tm * ntile + lt) * M + m) * 128 + rr];
            const int64_t t = tf + lt, ra = t * G, rb = ra + G;
            if (ra >= rg.u0 && rb <= rg.u1) {
                const int64_t n = t * 128 + rr;
                if (n < a.N) a.Y[(int64_t)m * a.N + n] = __float2bfloat16_rn(v);
            } else if (ra >= rg.u0) {
                red[((size_t)lt * w.CS) * M * 128 + rem] = v;
            } else {
                const uint32_t off = (uint32_t)((((size_t)owner_lt * w.CS + jsend) * M * 128 + rem) * 4);
                st_cluster_f32(cluster_map(red_base + off, (uint32_t)owner_rank), v);
            }
        }
        named_sync(1, kCW * 32);
        if (sends && threadIdx.x == 0)
            mbar_arrive_remote(cluster_map(smem_u32(rbar + owner_lt), (uint32_t)owner_rank));
        if (own_nc > 1) {
            // the owned last tile: wait for the other parts, sum in CTA order
            const int lt = (int)(own_last - tf);
            bool got = true;
            if (threadIdx.x == 0) {
                const uint64_t t0 = global_ns();
                while (!bar_try_cluster(rbar + lt, 0u))
                    if (global_ns() - t0 > kWaitNs) { got = false; break; }
                if (!got) { st_release(&flags[0], 1); atomicOr(&g_gemv_timeout, 1u); }
            }
            named_sync(1, kCW * 32);
            for (int idx = threadIdx.x; idx < M * 128; idx += kCW * 32) {
                float v = 0.f;
                for (int j = 0; j < own_nc; ++j) v += red[((size_t)lt * w.CS + j) * M * 128 + idx];
                const int64_t n = own_last * 128 + (idx & 127);
                if (n < a.N) a.Y[(int64_t)(idx >> 7) * a.N + n] = __float2bfloat16_rn(v);
            }
        }
    }

    // after a timed-out wait, let the copies already issued land; then free TMEM
    tc_fence_before();
    __syncthreads();
    if (flags[0] && threadIdx.x == 0) {
        const int issued = flags[1];
        for (int bs = 0; bs < nbs && bs < issued; ++bs) {
            const int last = bs + ((issued - 1 - bs) / nbs) * nbs;
            bar_wait(full + bs, (uint32_t)(last / nbs) & 1u);
        }
    }
    // no CTA of a cluster leaves while another may still write into its
    // shared memory (a sender that was late when its owner gave up waiting):
    // every wait above is bounded, so every thread of the cluster gets here
    if (w.CS > 1) {
        const bool waited = warp < kCW && (int64_t)(rg.u0 / G) * G < rg.u0;   // senders waited above
        if (!waited) cluster_wait();
        cluster_arrive();
        cluster_wait();
    }
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(*reinterpret_cast<volatile uint32_t *>(tmem_slot), kTmemCols);
    }
}

// ---------------------------------------------------------------- host side
struct Plan {
    Work w;
    int NB, S, nslot, L, ntile;
    uint32_t o_ring, o_sring, o_b, o_pair, o_res, o_bar, o_red, o_misc;
    size_t smem;
    bool ok;
};

int sm_count() {
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (!n) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

inline uint32_t align_up(size_t x, size_t a) { return (uint32_t)((x + a - 1) / a * a); }

// Shared-memory layout for S stages; returns its size without slack.
size_t layout(Plan &p, int r, int M, int S) {
    const int gpb = p.NB == 16 ? (M == 1 ? 4 : M == 2 ? 2 : 1) : 1;
    size_t o = 0;
    p.o_ring = 0;
    o = (size_t)r * S * 2048;
    p.o_sring = align_up(o, 128);
    o = p.o_sring + (size_t)S * 256;
    p.o_b = align_up(o, 1024);
    o = p.o_b + (size_t)((p.nslot + gpb - 1) / gpb) * p.NB * 128;
    p.o_pair = align_up(o, 16);
    o = p.o_pair + (size_t)p.nslot * 8 * 8;
    p.o_res = align_up(o, 16);
    o = p.o_res + (size_t)kTeams * p.ntile * M * 128 * 4;
    p.o_bar = align_up(o, 16);
    o = p.o_bar + (size_t)(2 * (S / kBatch) + kTeams + p.ntile) * 8;
    p.o_red = align_up(o, 16);
    o = p.o_red + (p.w.CS > 1 ? (size_t)p.ntile * p.w.CS * M * 128 * 4 : 0);
    p.o_misc = align_up(o, 16);
    o = p.o_misc + 64;                                     // flags, TMEM address
    return o;
}

// Ranges, ring and shared memory for one (clusters, CTAs per cluster) split.
Plan plan_for(const Work &w, int64_t M, int r) {
    Plan p{};
    p.w = w;
    p.NB = M <= 4 ? 16 : 32;
    const int64_t G = w.KC;
    int64_t L = 0, nt = 0;
    for (int64_t b = 0; b < w.ctas(); ++b) {
        const int64_t u0 = w.first(b), u1 = w.first(b + 1);
        if (u1 <= u0) return p;                            // an empty CTA: not a valid split
        L = u1 - u0 > L ? u1 - u0 : L;
        const int64_t tt = (u1 - 1) / G - u0 / G + 1;
        nt = tt > nt ? tt : nt;
    }
    p.L = (int)L;
    p.ntile = (int)nt;
    p.nslot = (int)(L < G ? L : G);
    const size_t stage = (size_t)2048 * r + 256;
    const size_t fixed = layout(p, r, (int)M, 0);
    const int need = (int)((L + kBatch - 1) / kBatch) * kBatch;   // stages for the whole range
    const int want = need < kBatch ? need : kBatch;                // fewest stages accepted (one batch)
    if (fixed + (size_t)want * stage + 1024 > kSmemMax) return p;
    int S = (int)((kSmemMax - 1024 - fixed) / stage) / kBatch * kBatch;
    if (S > need) S = need;
    // the ring's barriers and alignment come on top of `fixed`
    while (S > want && layout(p, r, (int)M, S) + 1024 > kSmemMax) S -= kBatch;
    p.S = S;
    p.smem = layout(p, r, (int)M, S) + 1024;
    p.ok = p.smem <= kSmemMax;
    return p;
}

int max_clusters(int r, int64_t M, size_t smem, int cs);   // below, per instantiation

// Choose the split: whole tiles per CTA (CS = 1) or clusters of CS CTAs that
// share tiles, taking the one with the fewest items on the busiest CTA (a
// shared tile costs about one extra item of latency for its exchange).
Plan make_plan(int64_t M, int64_t N, int64_t K, int r) {
    const int64_t T = (N + 127) / 128, G = K / kGroup;
    const int sms = sm_count();
    Plan best{};
    double best_cost = 1e30;
    if (T * G * 8 >= ((int64_t)1 << 32) || T * (int64_t)sms >= ((int64_t)1 << 32)) return best;
    for (int cs = 1; cs <= 8; ++cs) {
        int64_t nc = sms / cs;
        if (nc > T) nc = T;
        if (nc < 1 || T / nc * G < cs) continue;
        Plan p{};
        for (int it = 0; it < 3; ++it) {
            p = plan_for(Work{T, G, (int)nc, cs}, M, r);
            if (!p.ok) break;
            const int mc = cs > 1 ? max_clusters(r, M, p.smem, cs) : sms;
            if (mc >= nc) break;
            if (mc < 1) { p.ok = false; break; }
            nc = mc;
        }
        if (!p.ok) continue;
        const double cost = p.L + (cs > 1 ? 1.0 : 0.0);
        if (cost < best_cost) { best_cost = cost; best = p; }
    }
    return best;
}

// cudaFuncSetAttribute once per (instantiation, device), safe from any host thread.
template <typename F>
cudaError_t ensure_smem_attr(F *fn, std::atomic<uint64_t> &done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemMax);
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

template <int R, int MT>
std::atomic<uint64_t> &attr_done() {
    static std::atomic<uint64_t> d{0};
    return d;
}

template <int R, int MT>
mq_status run(const uint16_t *X, const mq_weights *wt, int64_t M, uint16_t *Y, const Plan &p,
              cudaStream_t st) {
    cudaError_t e = ensure_smem_attr(nested_gemv_tc_kernel<R, MT>, attr_done<R, MT>());
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    Args a{};
    a.X = reinterpret_cast<const __nv_bfloat16 *>(X);
    a.planes = reinterpret_cast<const uint8_t *>(wt->planes);
    a.scales = reinterpret_cast<const uint8_t *>(wt->scales);
    a.Y = reinterpret_cast<__nv_bfloat16 *>(Y);
    a.w = p.w;
    a.N = wt->N;
    a.K = wt->K;
    a.G = wt->K / kGroup;
    a.plane_bytes = (int64_t)mq_plane_bytes(wt->N, wt->K, 1);
    a.M = (int)M;
    a.NB = p.NB;
    a.S = p.S;
    a.o_ring = p.o_ring; a.o_sring = p.o_sring; a.o_b = p.o_b; a.o_pair = p.o_pair;
    a.o_res = p.o_res; a.o_bar = p.o_bar; a.o_red = p.o_red; a.o_misc = p.o_misc;
    // programmatic dependent launch: this grid may start while the previous
    // kernel of the stream finishes; it waits for it before reading X
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.w.ctas());
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)p.w.CS;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.w.CS > 1 ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, nested_gemv_tc_kernel<R, MT>, a);
    if (e != cudaSuccess) return cuda_fail(e, "nested_gemv_tc_kernel launch");
    return MQ_OK;
}

// Clusters of cs CTAs (with `smem` bytes each) that can be resident at once.
template <int R, int MT>
int occ_clusters(size_t smem, int cs) {
    if (ensure_smem_attr(nested_gemv_tc_kernel<R, MT>, attr_done<R, MT>()) != cudaSuccess) return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cs);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at;
    at.id = cudaLaunchAttributeClusterDimension;
    at.val.clusterDim.x = (unsigned)cs;
    at.val.clusterDim.y = 1;
    at.val.clusterDim.z = 1;
    cfg.attrs = &at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, nested_gemv_tc_kernel<R, MT>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}
template <int R>
int occ_clusters_r(int64_t M, size_t smem, int cs) {
    if (M == 1) return occ_clusters<R, 1>(smem, cs);
    if (M == 2) return occ_clusters<R, 2>(smem, cs);
    if (M <= 4) return occ_clusters<R, 4>(smem, cs);
    return occ_clusters<R, 8>(smem, cs);
}

template <int R>
mq_status run_r(const uint16_t *X, const mq_weights *wt, int64_t M, uint16_t *Y, const Plan &p,
                cudaStream_t st) {
    if (M == 1) return run<R, 1>(X, wt, M, Y, p, st);
    if (M == 2) return run<R, 2>(X, wt, M, Y, p, st);
    if (M <= 4) return run<R, 4>(X, wt, M, Y, p, st);
    return run<R, 8>(X, wt, M, Y, p, st);
}

int max_clusters(int r, int64_t M, size_t smem, int cs) {
    switch (r) {
        case 1: return occ_clusters_r<1>(M, smem, cs);
        case 2: return occ_clusters_r<2>(M, smem, cs);
        case 3: return occ_clusters_r<3>(M, smem, cs);
        case 4: return occ_clusters_r<4>(M, smem, cs);
        case 5: return occ_clusters_r<5>(M, smem, cs);
        case 6: return occ_clusters_r<6>(M, smem, cs);
        case 7: return occ_clusters_r<7>(M, smem, cs);
        default: return occ_clusters_r<8>(M, smem, cs);
    }
}

// make_plan runs a search (and occupancy queries): keep the last plans.
Plan cached_plan(int64_t M, int64_t N, int64_t K, int r) {
    struct Entry { int64_t M, N, K; int r, dev; Plan p; };
    static std::mutex mu;
    static Entry tab[64];
    static int used = 0, next = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    {
        std::lock_guard<std::mutex> lk(mu);
        for (int i = 0; i < used; ++i)
            if (tab[i].M == M && tab[i].N == N && tab[i].K == K && tab[i].r == r && tab[i].dev == dev)
                return tab[i].p;
    }
    const Plan p = make_plan(M, N, K, r);
    std::lock_guard<std::mutex> lk(mu);
    tab[next] = Entry{M, N, K, r, dev, p};
    next = (next + 1) % 64;
    if (used < 64) ++used;
    return p;
}

}  // namespace

bool gemv_tc_take_timeout(bool *set) {
    unsigned v = 0, z = 0;
    if (cudaMemcpyFromSymbol(&v, g_gemv_timeout, sizeof(v)) != cudaSuccess) return false;
    if (v && cudaMemcpyToSymbol(g_gemv_timeout, &z, sizeof(z)) != cudaSuccess) return false;
    *set = v != 0;
    return true;
}

bool gemv_tc_supported(int64_t M, int64_t N, int64_t K, int r) {
    return M >= 1 && M <= kGemvMaxM && cached_plan(M, N, K, r).ok;
}

// The GEMV sums shared tiles inside clusters: it needs no workspace.
size_t gemv_tc_workspace_bytes(int64_t, int64_t, int64_t, int) { return 0; }

mq_status launch_gemv_tc(const uint16_t *X, const mq_weights *w, int64_t M, uint16_t *Y,
                         void *ws, size_t ws_bytes, cudaStream_t st) {
    (void)ws_bytes;
    const Plan p = cached_plan(M, w->N, w->K, w->r);
    if (!p.ok) return fail(MQ_ERR_UNSUPPORTED, "no tensor-core GEMV plan fits this shape");
    (void)ws;
    switch (w->r) {
        case 1: return run_r<1>(X, w, M, Y, p, st);
        case 2: return run_r<2>(X, w, M, Y, p, st);
        case 3: return run_r<3>(X, w, M, Y, p, st);
        case 4: return run_r<4>(X, w, M, Y, p, st);
        case 5: return run_r<5>(X, w, M, Y, p, st);
        case 6: return run_r<6>(X, w, M, Y, p, st);
        case 7: return run_r<7>(X, w, M, Y, p, st);
        default: return run_r<8>(X, w, M, Y, p, st);
    }
}

}  // namespace mq
