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
//   TMEM).  A thread of a decode warp owns one row: it reads the row's r
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
//   k = 32t + 4i + b holds slice j of z at column 32t + 8b + i.  A small
//   kernel builds the slices of every group once per call (x_prep_kernel);
//   each CTA then copies the tiles of its groups into shared memory.
// * D (128 x N, int32, TMEM) = exact per-group integer sums, read back with
//   tcgen05.ld and folded into fp32: y += s_g 2^(8-r) 2^(Eg-6) sum_j 2^(-7j) D_j
//   + s_g (2^(7-r) - 128) S_g.
//
// Work: the (128-row tile, group) items in tile order are cut into one
// contiguous range per CTA, row tiles being shared only by the CTAs of one
// thread-block cluster (shapes whose operands do not fit in shared memory
// are left to the GEMM).  The packed format stores the 2 KB block of one
// (tile, group) contiguously per plane, items in this order, so a run of
// items is one contiguous stream per plane.
//
// Roles (warp-specialised, every hand-off an mbarrier or a shared atomic,
// no CTA-wide barrier in the steady state):
//   producer warp   bulk copies of the planes and scales of batches of
//                   items into two rings of shared-memory stages;
//   8 decode warps  two quads; quad e decodes items e, e + 2, ...: warp q of
//                   a quad owns rows 32q .. 32q + 31 (its TMEM lane quarter)
//                   and stores the item's A into one of eight TMEM A slots;
//                   the last of the four warps to finish an item (a counter
//                   per A slot) issues the item's four K = 32 MMAs into one
//                   of the TMEM D slots and commits to the D slot's barrier
//                   (D full; the A slot is free again once it lands);
//   4 fold warps    one copies the X tiles of the CTA's groups (after the
//                   kernels before it in the stream have completed:
//                   programmatic dependent launch); all four then fold the D
//                   slots, several items per round, into fp32 rows and
//                   write Y (or send a shared tile's part to its owner).
// The producer and decode warps read only the weights, so with programmatic
// dependent launch they stream and decode while the kernels before it are
// still finishing.  Waiting warps back off between polls, leaving the issue
// slots to the warps doing the work.  Every wait is bounded (about a second);
// a wait that gives up sets a CTA abort flag that ends every other wait at
// once, and a device flag the host reads with mq_device_status.
#include <string.h>

#include <atomic>
#include <mutex>

#include "mq_common.cuh"
#include "mq_bits.cuh"
#include "mq_sm100.cuh"

namespace mq {
namespace {

using namespace sm100;

constexpr int kDecWarps = 8;                 // two quads of decode warps
constexpr int kFoldW0 = kDecWarps;           // fold warps kFoldW0 .. kFoldW0 + 3
constexpr int kProdWarp = kFoldW0 + 4;
constexpr int kThreads = (kProdWarp + 1) * 32;
constexpr int kB = 2;                        // items per ring batch (one per quad)
constexpr int kNA = 8;                       // A slots in TMEM (32 columns each)
constexpr uint32_t kTmemCols = 512;          // A slots in [0, 256), D slots in [256, 512)
constexpr uint32_t kDCol0 = 256;
constexpr int kSlices = 4;                   // int8 slices per x
constexpr size_t kSmemMax = 227 * 1024;      // shared memory of one CTA per SM
constexpr size_t kRingBytes = 144 * 1024;    // plane ring budget
constexpr uint32_t kPlaneBlk = 2048;         // one (tile, group) block of one plane
constexpr size_t kXOff = kTicketBytes;       // prepared X in the workspace (after the GEMM's tickets)

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

__device__ unsigned int g_gemv_timeout;     // set when a bounded wait gave up

// ------------------------------------------------------------- decomposition
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

// Batch class MT (M = 1, 2, <= 4, <= 8): MMA N and groups per B tile.  The
// slices of group g sit in B tile g / gpb at position g % gpb (rows
// 4 (pos M + m) + j), and fill D columns 4 (pos M + m) + j.
__host__ __device__ constexpr int class_nb(int MT) { return MT <= 4 ? 16 : 32; }
__host__ __device__ constexpr int class_gpb(int MT) { return MT == 1 ? 4 : MT == 2 ? 2 : 1; }
__host__ __device__ inline int batch_class(int64_t M) { return M == 1 ? 1 : M == 2 ? 2 : M <= 4 ? 4 : 8; }
// Items folded per round by a fold warp (D registers: 4 MT per item).
__host__ __device__ constexpr int fold_chunk(int MT) { return MT <= 2 ? 4 : MT == 4 ? 2 : 1; }

// The CTA's groups g0 .. g0 + nslot - 1 (mod G) as B tiles: the tiles of
// groups g0 .. min(gend, G - 1) first (na of them), then, when the range
// wraps past the last group, the tiles of groups 0 .. gend - G.
struct XSpan {
    int g0, nslot, ta0, na, nb;
    __host__ __device__ XSpan(int g0_, int nslot_, int G, int gpb) : g0(g0_), nslot(nslot_) {
        const int gend = g0 + nslot - 1;
        ta0 = g0 / gpb;
        na = (gend < G ? gend : G - 1) / gpb - ta0 + 1;
        nb = gend >= G ? (gend - G) / gpb + 1 : 0;
    }
    // shared-memory tile of group g (one of the CTA's groups)
    __host__ __device__ int tile_of(int g, int gpb) const { return g >= g0 ? g / gpb - ta0 : na + g / gpb; }
};

// Kernel arguments (one struct, passed as a grid constant).
struct Args {
    const uint8_t *planes;  // tiled planes (2 KB per (tile, group) block per plane)
    const uint8_t *scales;  // tiled fp16 scales (256 B per block)
    const uint8_t *xtiles;  // prepared X: B tiles of all groups (workspace)
    const float2 *xpairs;   // prepared X: {2^(8-r) 2^(Eg-6), S_g} per (group, m), 8 per group
    __nv_bfloat16 *Y;
    Work w;
    int64_t N, K, G;
    int64_t plane_bytes;    // bytes of one plane
    int M;                  // batch rows
    int nring, nss;         // batches in the plane ring / the scale ring
    // shared-memory offsets from the 1024-byte aligned base
    uint32_t o_ring, o_sring, o_b, o_pair, o_bar, o_red, o_misc;
};

// Shared-memory barriers of one CTA, in the order they are laid out.
struct Bars {
    uint64_t *full, *empty;     // [nring] plane ring
    uint64_t *sfull, *sempty;   // [nss] scale ring
    uint64_t *dfull, *dempty;   // [kND] TMEM D slots
    uint64_t *rbar;             // parts of the owned shared tile received
    uint64_t *xbar;             // the CTA's X tiles and pairs landed
};
__host__ __device__ inline int bar_count(int nring, int nss, int nd) {
    return 2 * nring + 2 * nss + 2 * nd + 2;
}

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

constexpr int kPrepWarps = 8;

// The B operand of every group, once per call: one warp per (group, batch
// row) task.  Writes B tile g / gpb (row 4 (pos M + m) + j, K-major with the
// 128-byte swizzle, ready to be copied into shared memory as is) and the
// pair {2^(8-r) 2^(Eg-6), S_g} at pairs[g * 8 + m].
template <int R, int MT>
__global__ void __launch_bounds__(kPrepWarps * 32)
x_prep_kernel(const uint16_t *__restrict__ X, int M, int64_t K, int G, uint8_t *__restrict__ tiles,
              float2 *__restrict__ pairs) {
    constexpr int NB = class_nb(MT), gpb = class_gpb(MT);
    pdl_launch_dependents();            // the GEMV may start streaming its weights
    pdl_wait();                         // X comes from the kernels before this one
    const int lane = threadIdx.x & 31;
    const int task = blockIdx.x * kPrepWarps + (threadIdx.x >> 5);
    if (task >= G * M) return;
    const int g = task / M, m = task - g * M;
    const int t = lane >> 3, wi = lane & 7;
    const int sh = field_shift<R>(wi);
    const uint16_t *xr = X + (int64_t)m * K + (int64_t)g * kGroup + 32 * t + wi;
    uint32_t hv[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) hv[b] = xr[8 * b];
    int emax = -1000;
    float sum = 0.f;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const int e8 = (int)((hv[b] >> 7) & 0xFFu);
        const int v = e8 ? e8 - sh : -1000;
        emax = v > emax ? v : emax;
        sum += __uint_as_float(hv[b] << 16);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const int other = __shfl_xor_sync(0xffffffffu, emax, o);
        emax = other > emax ? other : emax;
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
    }
    const int Eg = emax > -1000 ? emax - 127 : 0;
    int F[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) F[b] = fixed_point(hv[b], sh, Eg);
    uint32_t wd[kSlices];
    wd[0] = pack_bytes(F[0] >> 21, F[1] >> 21, F[2] >> 21, F[3] >> 21);
    wd[1] = pack_bytes(F[0] >> 14, F[1] >> 14, F[2] >> 14, F[3] >> 14) & 0x7F7F7F7Fu;
    wd[2] = pack_bytes(F[0] >> 7, F[1] >> 7, F[2] >> 7, F[3] >> 7) & 0x7F7F7F7Fu;
    wd[3] = pack_bytes(F[0], F[1], F[2], F[3]) & 0x7F7F7F7Fu;
    uint8_t *tile = tiles + (size_t)(g / gpb) * NB * 128;
    const int chunk = 2 * t + (wi >> 2);                 // 16-byte chunk of k = 32t + 4wi
#pragma unroll
    for (int j = 0; j < kSlices; ++j) {
        const int row = 4 * ((g % gpb) * M + m) + j;
        *reinterpret_cast<uint32_t *>(tile + sw128_offset(row, chunk) + 4 * (wi & 3)) = wd[j];
    }
    if (lane == 0) {
        // 2^(8-r) 2^(Eg-6), clamped to the normal fp32 range
        int ex = 2 - R + Eg;
        ex = ex < -126 ? -126 : (ex > 127 ? 127 : ex);
        pairs[(size_t)g * 8 + m] = make_float2(__int_as_float((ex + 127) << 23), sum);
    }
}

// ------------------------------------------------------------------ kernel
// D columns of one item (4 slices per batch row) into registers.
template <int MT>
__device__ __forceinline__ void read_d(uint32_t taddr, uint32_t *d) {
    if constexpr (MT == 1) tmem_ld4(taddr, d);
    else if constexpr (MT == 2) tmem_ld8(taddr, d);
    else if constexpr (MT == 4) tmem_ld16(taddr, d);
    else tmem_ld32(taddr, d);
}

// Shared-memory atomic add with acquire-release order (a counter that also
// hands over the tensor-memory stores of the warps that counted before).
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t *p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;"
                 : "=r"(old) : "r"(smem_u32(p)), "r"(v) : "memory");
    return old;
}

// MT: batch class (M = 1, M = 2, M <= 4, M <= 8), fixing the MMA N (16 or 32),
// the groups per B tile and the D columns read back per item.
template <int R, int MT>
__global__ void __launch_bounds__(kThreads, 1)
nested_gemv_tc_kernel(const __grid_constant__ Args a) {
    constexpr int NB = class_nb(MT), gpb = class_gpb(MT), CH = fold_chunk(MT);
    constexpr int kND = 256 / NB;                        // D slots in TMEM
    static_assert(kND >= kNA, "a decode warp waits on the D slot of the item kNA earlier");
    extern __shared__ uint8_t smem_raw[];
    // align the base by an offset so the compiler keeps the shared address space
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const Work &w = a.w;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Range rg = make_range(w, blockIdx.x);
    const int L = rg.L, M = a.M, G = (int)a.G;
    const int nring = a.nring, nss = a.nss;
    const int g0 = rg.u0 % G;
    const int nslot = L < G ? L : G;                     // distinct groups of the range
    const XSpan xs(g0, nslot, G, gpb);
    const int tf = rg.u0 / G, tl = (rg.u1 - 1) / G;      // first and last row tile

    Bars bar;
    bar.full = reinterpret_cast<uint64_t *>(smem + a.o_bar);
    bar.empty = bar.full + nring;
    bar.sfull = bar.empty + nring;
    bar.sempty = bar.sfull + nss;
    bar.dfull = bar.sempty + nss;
    bar.dempty = bar.dfull + kND;
    bar.rbar = bar.dempty + kND;
    bar.xbar = bar.rbar + 1;
    volatile int *flags = reinterpret_cast<volatile int *>(smem + a.o_misc);   // [0] abort [1] batches issued
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + a.o_misc + 8);
    uint32_t *acnt = reinterpret_cast<uint32_t *>(smem + a.o_misc + 16);      // [kNA] warps done per A slot
    uint32_t *icnt = acnt + kNA;                                               // [kND] commits per D slot
    float *red = reinterpret_cast<float *>(smem + a.o_red);    // [CS][M][128] parts of the owned tile

    // The CTA holding a tile's first item owns it; if its last tile continues
    // in later CTAs (of the same cluster), it waits for their parts.
    const bool owns_shared = tl * G >= rg.u0 && tl * G + G > rg.u1;
    const int own_nc = owns_shared ? (int)(w.cta_of((int64_t)tl * G + G - 1) - blockIdx.x + 1) : 0;

    {
        const int nb = bar_count(nring, nss, kND);
        for (int i = threadIdx.x; i < nb; i += kThreads) {
            uint32_t cnt;
            if (i < nring) cnt = 1;                                          // full
            else if (i < 2 * nring) cnt = 4 * kB;                            // empty: decode warps per item
            else if (i < 2 * nring + nss) cnt = 1;                           // sfull
            else if (i < 2 * nring + 2 * nss) cnt = 4;                       // sempty: fold warps
            else if (i < 2 * nring + 2 * nss + kND) cnt = 1;                 // dfull: commit
            else if (i < 2 * nring + 2 * nss + 2 * kND) cnt = 4;             // dempty: fold warps
            else if (i == 2 * nring + 2 * nss + 2 * kND)
                cnt = own_nc > 1 ? 128u * (uint32_t)(own_nc - 1) : 1u;       // rbar: sender threads
            else cnt = 1;                                                    // xbar
            mbar_init(bar.full + i, cnt);
        }
        if (threadIdx.x < kNA + kND) acnt[threadIdx.x] = 0;
        if (threadIdx.x == 0) { flags[0] = 0; flags[1] = 0; }
    }
    fence_mbar_init();
    __syncthreads();
    // every CTA of the cluster has initialised its barriers before any part is sent
    if (w.CS > 1) cluster_arrive();
    bool cluster_waited = false;

    if (warp == kProdWarp) {
        // ---------------------------------------------------------- producer
        // batch b = items [kB b, kB b + kB): one bulk copy per plane and one
        // for the scales (consecutive items are consecutive blocks), into
        // plane ring slot b % nring and scale ring slot b % nss
        if (lane == 0) {
            const int nbatch = (L + kB - 1) / kB;
            int s = 0, ks = 0, ss = 0, kss = 0;
            for (int b = 0; b < nbatch; ++b) {
                if (ks > 0 && !mbar_wait_backoff(bar.empty + s, (uint32_t)(ks - 1) & 1u, flags)) break;
                if (kss > 0 && !mbar_wait_backoff(bar.sempty + ss, (uint32_t)(kss - 1) & 1u, flags)) break;
                const int i0 = b * kB, n = (L - i0) < kB ? (L - i0) : kB;
                const int64_t u = rg.u0 + i0;
                mbar_expect_tx(bar.full + s, (uint32_t)n * kPlaneBlk * R);
#pragma unroll
                for (int p = 0; p < R; ++p)
                    bulk_g2s(smem + a.o_ring + ((size_t)s * R + p) * kB * kPlaneBlk,
                             a.planes + p * a.plane_bytes + u * kPlaneBlk, (uint32_t)n * kPlaneBlk,
                             bar.full + s);
                mbar_expect_tx(bar.sfull + ss, (uint32_t)n * 256);
                bulk_g2s(smem + a.o_sring + (size_t)ss * kB * 256, a.scales + u * 256, (uint32_t)n * 256,
                         bar.sfull + ss);
                flags[1] = b + 1;
                // the next kernel of the stream may start (it waits for this
                // one before it reads what this one writes)
                if (b == 0) pdl_launch_dependents();
                if (++s == nring) { s = 0; ++ks; }
                if (++ss == nss) { ss = 0; ++kss; }
            }
        }
    } else {
        // TMEM: eight A slots of 32 columns, then the D slots
        if (warp == 0) {
            tmem_alloc(tmem_slot, kTmemCols);
            tmem_relinquish();
        }
        tc_fence_before();
        named_sync(1, kProdWarp * 32);
        tc_fence_after();
        const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(tmem_slot);
        const int qq = warp & 3, row = qq * 32 + lane;
        const uint32_t lane_base = (uint32_t)(32 * qq) << 16;

        if (warp < kDecWarps) {
            // ---------------------------------------------------------- decode
            const int quad = warp >> 2;
            const uint32_t idesc = idesc_u8s8(NB);
            const uint32_t b0 = smem_u32(smem + a.o_b);
            int s = 0, k = 0;                            // ring slot of item i's batch, its fill
            int g = g0 + quad >= G ? g0 + quad - G : g0 + quad;   // group of item i
            bool xready = false;
            for (int i = quad; i < L; i += 2) {
                // (kB == 2: item i is element `quad` of batch i / 2)
                if (!mbar_wait_backoff(bar.full + s, (uint32_t)k & 1u, flags)) break;
                uint4 pw[R];
                const uint8_t *src = smem + a.o_ring + ((size_t)s * R * kB + quad) * kPlaneBlk + row * 16;
#pragma unroll
                for (int p = 0; p < R; ++p)
                    pw[p] = *reinterpret_cast<const uint4 *>(src + (size_t)p * kB * kPlaneBlk);
                __syncwarp();
                if (lane == 0) mbar_arrive(bar.empty + s);
                uint32_t A[32];
#pragma unroll
                for (int t4 = 0; t4 < 4; ++t4) {
                    uint32_t P[8];
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        const uint4 &v = pw[p < R ? p : 0];
                        P[p] = p < R ? (t4 == 0 ? v.x : t4 == 1 ? v.y : t4 == 2 ? v.z : v.w) : 0u;
                    }
                    field_operands<R>(P, A + 8 * t4);
                }
                // A slot i % kNA is free once the MMAs of item i - kNA are done:
                // their commit completes that item's D-slot barrier
                const int as = i & (kNA - 1);
                if (i >= kNA) {
                    const int j = i - kNA;
                    if (!mbar_wait_backoff(bar.dfull + j % kND, (uint32_t)(j / kND) & 1u, flags)) break;
                }
                tc_fence_after();
                tmem_st32(tmem + lane_base + (uint32_t)as * 32, A);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                uint32_t old = 0;
                if (lane == 0) old = atom_add_acq_rel(acnt + as, 1u);
                old = __shfl_sync(0xffffffffu, old, 0);
                if (old == 4u * (uint32_t)(i / kNA) + 3u && lane == 0) {
                    // the last warp of the quad for this item: issue its MMAs
                    bool ok = true;
                    if (!xready) {
                        ok = mbar_wait_backoff(bar.xbar, 0u, flags);
                        xready = ok;
                    }
                    const int ds = i % kND;
                    if (ok && i >= kND) ok = mbar_wait_backoff(bar.dempty + ds, (uint32_t)((i / kND) - 1) & 1u, flags);
                    if (ok) {
                        tc_fence_after();
                        const uint32_t baddr = b0 + (uint32_t)(xs.tile_of(g, gpb) * NB * 128);
                        const uint32_t dcol = tmem + kDCol0 + (uint32_t)(ds * NB);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_i8_ts(dcol, tmem + (uint32_t)(as * 32 + 8 * kk), smem_desc_sw128(baddr + 32 * kk),
                                      idesc, kk > 0 ? 1u : 0u);
                        mma_commit(bar.dfull + ds);
                        atomicAdd(icnt + ds, 1u);
                    }
                }
                if (flags[0]) break;
                if (++s == nring) { s = 0; ++k; }
                g += 2;                                   // (G may be 1)
                if (g >= G) g -= G;
                if (g >= G) g -= G;
            }
        } else {
            // ------------------------------------------------------------ fold
            const int fw = warp - kFoldW0;
            if (fw == 0 && lane == 0) {
                // the CTA's X tiles and pairs, once the X of this call is ready
                pdl_wait();
                const size_t tb = (size_t)NB * 128;
                const int na_groups = (xs.g0 + nslot - 1 < G ? nslot : G - xs.g0);
                const uint32_t bytes = (uint32_t)((xs.na + xs.nb) * tb + (size_t)nslot * 64);
                mbar_expect_tx(bar.xbar, bytes);
                bulk_g2s(smem + a.o_b, a.xtiles + xs.ta0 * tb, (uint32_t)(xs.na * tb), bar.xbar);
                if (xs.nb) bulk_g2s(smem + a.o_b + xs.na * tb, a.xtiles, (uint32_t)(xs.nb * tb), bar.xbar);
                bulk_g2s(smem + a.o_pair, a.xpairs + (size_t)xs.g0 * 8, (uint32_t)(na_groups * 64), bar.xbar);
                if (na_groups < nslot)
                    bulk_g2s(smem + a.o_pair + na_groups * 64, a.xpairs, (uint32_t)((nslot - na_groups) * 64),
                             bar.xbar);
            }
            const float2 *pairs = reinterpret_cast<const float2 *>(smem + a.o_pair);
            constexpr float kOffset = (float)(128 >> (R - 1)) * 0.5f - 128.0f;   // 2^(7-r) - 128
            float y[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) y[m] = 0.f;
            int t = tf, g = g0, cur = tf, slot = 0;
            bool ok = mbar_wait_backoff(bar.xbar, 0u, flags);
            const uint32_t red_base = smem_u32(red);
            // a finished tile: into Y, or (a tile that started in an earlier
            // CTA) into the owner's shared memory
            auto flush = [&](int tile) {
                const int64_t ra = (int64_t)tile * G, rb = ra + G;
                if (ra >= rg.u0 && rb <= rg.u1) {
                    const int64_t n = (int64_t)tile * 128 + row;
                    if (n < a.N) {
#pragma unroll
                        for (int m = 0; m < MT; ++m)
                            if (m < M) a.Y[(int64_t)m * a.N + n] = __float2bfloat16_rn(y[m]);
                    }
                } else if (ra < rg.u0) {
                    const int64_t owner = w.cta_of(ra);
                    const uint32_t orank = (uint32_t)(owner % w.CS);
                    const int j = (int)(blockIdx.x - owner);
                    if (!cluster_waited) { cluster_wait(); cluster_waited = true; }
#pragma unroll
                    for (int m = 0; m < MT; ++m)
                        if (m < M)
                            st_cluster_f32(cluster_map(red_base + (uint32_t)(((j * M + m) * 128 + row) * 4), orank),
                                           y[m]);
                    mbar_arrive_remote(cluster_map(smem_u32(bar.rbar), orank));
                }
                // else: the owned shared tile (the last one), kept in y
            };
            for (int i0 = 0; ok && i0 < L; i0 += CH) {
                const int n = L - i0 < CH ? L - i0 : CH;
                // wait for the items' D slots (and each new scale batch)
#pragma unroll
                for (int j = 0; j < CH; ++j) {
                    const int i = i0 + j;
                    if (j < n && ok) {
                        if ((i & (kB - 1)) == 0)
                            ok = mbar_wait_backoff(bar.sfull + (i / kB) % nss, (uint32_t)((i / kB) / nss) & 1u, flags);
                        if (ok) ok = mbar_wait_backoff(bar.dfull + i % kND, (uint32_t)(i / kND) & 1u, flags);
                    }
                }
                if (!ok) break;
                tc_fence_after();
                uint32_t d[CH][4 * MT];
#pragma unroll
                for (int j = 0; j < CH; ++j) {
                    if (j < n) {
                        const int i = i0 + j, gj = (g0 + slot + j) % G;
                        read_d<MT>(tmem + lane_base + kDCol0 + (uint32_t)((i % kND) * NB + 4 * M * (gj % gpb)), d[j]);
                    }
                }
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
#pragma unroll
                    for (int j = 0; j < CH; ++j)
                        if (j < n) mbar_arrive(bar.dempty + (i0 + j) % kND);
                }
#pragma unroll
                for (int j = 0; j < CH; ++j) {
                    if (j < n) {
                        const int i = i0 + j, e = i & (kB - 1), ss = (i / kB) % nss;
                        const float sc = __half2float(*reinterpret_cast<const __half *>(
                            smem + a.o_sring + ((size_t)ss * kB + e) * 256 + row * 2));
                        if (e == kB - 1 || i == L - 1) {
                            __syncwarp();
                            if (lane == 0) mbar_arrive(bar.sempty + ss);
                        }
                        if (t != cur) {
                            flush(cur);
#pragma unroll
                            for (int m = 0; m < MT; ++m) y[m] = 0.f;
                            cur = t;
                        }
#pragma unroll
                        for (int m = 0; m < MT; ++m) {
                            if (m < M) {
                                const float v = (float)(int)d[j][4 * m] + 0x1p-7f * (float)(int)d[j][4 * m + 1] +
                                                0x1p-14f * (float)(int)d[j][4 * m + 2] +
                                                0x1p-21f * (float)(int)d[j][4 * m + 3];
                                const float2 ge = pairs[slot * 8 + m];
                                y[m] = fmaf(sc * ge.x, v, fmaf(sc * kOffset, ge.y, y[m]));
                            }
                        }
                        if (++slot == G) slot = 0;
                        if (++g == G) { g = 0; ++t; }
                    }
                }
            }
            if (ok && !flags[0]) {
                flush(cur);
                if (own_nc > 1) {
                    // the owned last tile: wait for the other parts, sum in CTA order
                    const uint64_t t0 = global_ns();
                    bool got = true;
                    while (!mbar_try_wait_cluster(bar.rbar, 0u)) {
                        if (flags[0] || global_ns() - t0 > kWaitNs) { got = false; flags[0] = 1; break; }
                    }
                    if (got) {
                        const int64_t n = (int64_t)tl * 128 + row;
#pragma unroll
                        for (int m = 0; m < MT; ++m) {
                            if (m < M) {
                                float v = y[m];
                                for (int j = 1; j < own_nc; ++j) v += red[(j * M + m) * 128 + row];
                                if (n < a.N) a.Y[(int64_t)m * a.N + n] = __float2bfloat16_rn(v);
                            }
                        }
                    }
                }
            }
        }
    }

    // ---- end: after an abort, let the copies and MMAs already issued land;
    // then meet the cluster (no CTA leaves while another may still write into
    // its shared memory) and free TMEM
    __syncwarp();
    __syncthreads();
    if (flags[0] && threadIdx.x == 0) {
        const int issued = flags[1];
        for (int b = (issued > nring ? issued - nring : 0); b < issued; ++b)
            mbar_wait_bounded(bar.full + b % nring, (uint32_t)(b / nring) & 1u);
        for (int b = (issued > nss ? issued - nss : 0); b < issued; ++b)
            mbar_wait_bounded(bar.sfull + b % nss, (uint32_t)(b / nss) & 1u);
        for (int ds = 0; ds < kND; ++ds) {
            const uint32_t c = icnt[ds];
            if (c) mbar_wait_bounded(bar.dfull + ds, (c - 1) & 1u);
        }
        atomicOr(&g_gemv_timeout, 1u);
    }
    // (the X copy is waited for by the fold warps; on an abort before that
    // wait, let it land here)
    if (flags[0] && threadIdx.x == 32 * kFoldW0) mbar_wait_bounded(bar.xbar, 0u);
    tc_fence_before();
    __syncthreads();
    if (w.CS > 1) {
        if (!cluster_waited) cluster_wait();
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
    int nring, nss, nslot, nxt, L;
    uint32_t o_ring, o_sring, o_b, o_pair, o_bar, o_red, o_misc;
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

// Shared-memory layout for `nring` plane batches and `nss` scale batches;
// returns its size without the alignment slack.
size_t layout(Plan &p, int r, int M, int nring, int nss) {
    const int MT = batch_class(M), NB = class_nb(MT), nd = 256 / NB;
    size_t o = 0;
    p.o_ring = 0;
    o = (size_t)nring * kB * r * kPlaneBlk;
    p.o_sring = align_up(o, 128);
    o = p.o_sring + (size_t)nss * kB * 256;
    p.o_b = align_up(o, 1024);
    o = p.o_b + (size_t)p.nxt * NB * 128;
    p.o_pair = align_up(o, 16);
    o = p.o_pair + (size_t)p.nslot * 8 * 8;
    p.o_bar = align_up(o, 16);
    o = p.o_bar + (size_t)bar_count(nring, nss, nd) * 8;
    p.o_red = align_up(o, 16);
    o = p.o_red + (p.w.CS > 1 ? (size_t)p.w.CS * M * 128 * 4 : 0);
    p.o_misc = align_up(o, 16);
    o = p.o_misc + 16 + (size_t)(kNA + nd) * 4;            // flags, TMEM address, counters
    return o;
}

// Ranges, rings and shared memory for one (clusters, CTAs per cluster) split.
Plan plan_for(const Work &w, int64_t M, int r) {
    Plan p{};
    p.w = w;
    const int64_t G = w.KC;
    const int gpb = class_gpb(batch_class(M));
    int64_t L = 0;
    int nxt = 0;
    for (int64_t b = 0; b < w.ctas(); ++b) {
        const int64_t u0 = w.first(b), u1 = w.first(b + 1);
        if (u1 <= u0) return p;                            // an empty CTA: not a valid split
        L = u1 - u0 > L ? u1 - u0 : L;
        const int ns = (int)(u1 - u0 < G ? u1 - u0 : G);
        const XSpan xs((int)(u0 % G), ns, (int)G, gpb);
        nxt = xs.na + xs.nb > nxt ? xs.na + xs.nb : nxt;
    }
    p.L = (int)L;
    p.nslot = (int)(L < G ? L : G);
    p.nxt = nxt;
    const int nbatch = (int)((L + kB - 1) / kB);
    const size_t batch = (size_t)kB * r * kPlaneBlk;
    // the plane ring: up to kRingBytes, at least one batch (or the whole
    // range), within the shared memory left by the X operand
    int nring = (int)(kRingBytes / batch);
    if (nring < 2) nring = 2;
    if (nring > nbatch) nring = nbatch;
    auto total = [&](int nr) {
        const int ns = nbatch < nr + 8 ? nbatch : nr + 8;
        return layout(p, r, (int)M, nr, ns) + 1024;
    };
    while (nring > 1 && total(nring) > kSmemMax) --nring;
    if (total(nring) > kSmemMax) return p;
    p.nring = nring;
    p.nss = nbatch < nring + 8 ? nbatch : nring + 8;
    p.smem = layout(p, r, (int)M, p.nring, p.nss) + 1024;
    p.ok = p.smem <= kSmemMax;
    return p;
}

int max_clusters(int r, int64_t M, size_t smem, int cs);   // below, per instantiation

// Choose the split: whole tiles per CTA (CS = 1) or clusters of CS CTAs that
// share tiles, taking the one with the fewest items on the busiest CTA (a
// shared tile costs about one extra item of latency for its exchange).  At
// most one CTA per SM.
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

// Workspace of the prepared X: B tiles of all groups, then the pairs.
size_t xprep_tile_bytes(int64_t M, int64_t K) {
    const int MT = batch_class(M), gpb = class_gpb(MT);
    const int64_t G = K / kGroup;
    return (size_t)((G + gpb - 1) / gpb) * class_nb(MT) * 128;
}
size_t xprep_bytes(int64_t M, int64_t K) { return xprep_tile_bytes(M, K) + (size_t)(K / kGroup) * 64; }

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
              void *ws, cudaStream_t st) {
    cudaError_t e = ensure_smem_attr(nested_gemv_tc_kernel<R, MT>, attr_done<R, MT>());
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    uint8_t *xt = static_cast<uint8_t *>(ws) + kXOff;
    float2 *xp = reinterpret_cast<float2 *>(xt + xprep_tile_bytes(M, wt->K));
    const int G = (int)(wt->K / kGroup);
    // programmatic dependent launch for both kernels: each may start while
    // the kernel before it finishes, and waits for it before reading its output
    cudaLaunchAttribute pdl;
    pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl.val.programmaticStreamSerializationAllowed = 1;
    {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)((G * M + kPrepWarps - 1) / kPrepWarps));
        cfg.blockDim = dim3(kPrepWarps * 32);
        cfg.stream = st;
        cfg.attrs = &pdl;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, x_prep_kernel<R, MT>, X, (int)M, (int64_t)wt->K, G, xt, xp);
        if (e != cudaSuccess) return cuda_fail(e, "x_prep_kernel launch");
    }
    Args a{};
    a.planes = reinterpret_cast<const uint8_t *>(wt->planes);
    a.scales = reinterpret_cast<const uint8_t *>(wt->scales);
    a.xtiles = xt;
    a.xpairs = xp;
    a.Y = reinterpret_cast<__nv_bfloat16 *>(Y);
    a.w = p.w;
    a.N = wt->N;
    a.K = wt->K;
    a.G = G;
    a.plane_bytes = (int64_t)mq_plane_bytes(wt->N, wt->K, 1);
    a.M = (int)M;
    a.nring = p.nring;
    a.nss = p.nss;
    a.o_ring = p.o_ring; a.o_sring = p.o_sring; a.o_b = p.o_b; a.o_pair = p.o_pair;
    a.o_bar = p.o_bar; a.o_red = p.o_red; a.o_misc = p.o_misc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.w.ctas());
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0] = pdl;
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
    switch (batch_class(M)) {
        case 1: return occ_clusters<R, 1>(smem, cs);
        case 2: return occ_clusters<R, 2>(smem, cs);
        case 4: return occ_clusters<R, 4>(smem, cs);
        default: return occ_clusters<R, 8>(smem, cs);
    }
}

template <int R>
mq_status run_r(const uint16_t *X, const mq_weights *wt, int64_t M, uint16_t *Y, const Plan &p,
                void *ws, cudaStream_t st) {
    switch (batch_class(M)) {
        case 1: return run<R, 1>(X, wt, M, Y, p, ws, st);
        case 2: return run<R, 2>(X, wt, M, Y, p, ws, st);
        case 4: return run<R, 4>(X, wt, M, Y, p, ws, st);
        default: return run<R, 8>(X, wt, M, Y, p, ws, st);
    }
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

// The GEMV keeps the X operand of the call (built once per call) in the
// workspace, after the GEMM's ticket region (which it leaves untouched).
size_t gemv_tc_workspace_bytes(int64_t M, int64_t, int64_t K, int) { return kXOff + xprep_bytes(M, K); }

mq_status launch_gemv_tc(const uint16_t *X, const mq_weights *w, int64_t M, uint16_t *Y,
                         void *ws, size_t ws_bytes, cudaStream_t st) {
    const Plan p = cached_plan(M, w->N, w->K, w->r);
    if (!p.ok) return fail(MQ_ERR_UNSUPPORTED, "no tensor-core GEMV plan fits this shape");
    if (!ws || ws_bytes < gemv_tc_workspace_bytes(M, w->N, w->K, w->r))
        return fail(MQ_ERR_WORKSPACE, "GEMV workspace missing or too small");
    switch (w->r) {
        case 1: return run_r<1>(X, w, M, Y, p, ws, st);
        case 2: return run_r<2>(X, w, M, Y, p, ws, st);
        case 3: return run_r<3>(X, w, M, Y, p, ws, st);
        case 4: return run_r<4>(X, w, M, Y, p, ws, st);
        case 5: return run_r<5>(X, w, M, Y, p, ws, st);
        case 6: return run_r<6>(X, w, M, Y, p, ws, st);
        case 7: return run_r<7>(X, w, M, Y, p, ws, st);
        default: return run_r<8>(X, w, M, Y, p, ws, st);
    }
}

}  // namespace mq
