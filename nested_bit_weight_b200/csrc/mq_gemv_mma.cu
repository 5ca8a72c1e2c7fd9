// Batch M <= 8: the nested r-bit product on warp MMAs (u8 x s8 -> s32), one
// stream-K kernel per call.
//
// The r-bit model is the first r bit planes of the parent ("MatGPTQ:
// Efficient and Accurate Inference over Nested Quantized Models", abstract:
// an r-bit model reads exactly r bits); its level is
//     v_r(q) = 2^(8-r) q + 2^(7-r) - 128,   w = s_g v_r(q),
// so per 128-column group g and batch row m
//     sum_k x_k w_k = s_g ( 2^(8-r) sum_k x_k q_k + (2^(7-r) - 128) S_g ),
// with S_g = sum_k x_k.  The kernel computes sum_k x_k q_k on the tensor pipe:
//
// * Weights (MMA operand A).  A lane owns one 32-column word of a group for two
//   rows, reads r plane words per row, and rearranges them into 8 registers
//   whose 4 bytes each hold one field q << sh(i) (i = register, sh its bit
//   offset inside the byte): one AND per register, no shift.  Byte b of
//   register i is column 8b + i of the word.
// * X (operand B).  z_k = x_k 2^(-sh(k)) is cut into four int8 slices relative
//   to the group exponent Eg = max_k floor(log2 |z_k|):
//       z_k = 2^(Eg-27) (a_1 2^21 + a_2 2^14 + a_3 2^7 + a_4),
//   so sum_k A_k z_k = sum_k q_k x_k exactly for every x within 2^-14 of the
//   group's largest.  Slice j of batch row m is MMA column 4m + j.
// * Per group the four k32 MMAs give D_j exactly (|D| < 2^22); the MMA adds
//   the bits of 2^23 + 2^22 so D converts to fp32 with one subtraction.  The
//   fp16 scale times 2^(8-r) 2^(Eg-6) is applied per group in fp32, the
//   slice weights 2^(-7j) and the offset term once per 16 x 1024 item.
//
// Work: the (16-row tile, 1024-column chunk) items of the matrix, in tile
// order (K split into Q segments only when X's slices would not fit in shared
// memory), are cut into one contiguous range per CTA (one CTA per SM, equal
// item counts within one).  A producer warp streams the CTA's items into a
// ring of shared-memory stages with TMA (planes: one 3-D box per item, 128-byte
// swizzle; scales: one 2-D box); eight consumer warps take items round-robin.
// Partial sums of a tile are combined in a fixed order inside the CTA; a tile
// shared with another CTA (at most two per CTA when Q = 1, processed first) is
// combined through the workspace by whichever CTA arrives last, again in a
// fixed order, so results do not depend on timing.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <string.h>

#include "mq_common.cuh"
#include "mq_bits.cuh"

namespace mq {
namespace {

constexpr int kCW = 16;                      // consumer warps
constexpr int kThreads = (kCW + 2) * 32;     // + a producer warp and an epilogue warp
constexpr int kProd = kCW, kEpi = kCW + 1;   // their warp indices
constexpr int kCG = 8;                       // groups per chunk (one TMA box)
constexpr int kSlices = 4;                   // int8 slices per x
constexpr uint32_t kMagicBits = 0x4B400000u; // fp32 bits of 2^23 + 2^22
constexpr float kMagic = 12582912.0f;
// Per-CTA shared memory budget (one CTA per SM).
constexpr size_t kSmemBudget = 220 * 1024;
constexpr uint64_t kWaitNs = 1000000000ull;  // bound on any mbarrier wait (1 s)
constexpr int kHeadItems = 8;                // items streamed before X is requested
// X operand of one 1024-column chunk: per MMA column c = 4m + j a 1040-byte
// slice block (8 groups x 128 B; the 16-byte pad puts columns c and c + 1 in
// different bank quarters), then the pairs {2^(8-r) 2^(Eg-6), S} per (group, m).
constexpr int kColBytes = kCG * 128 + 16;
__host__ __device__ constexpr uint32_t x_block_bytes(int M) { return 4u * M * kColBytes + kCG * 8 * 8; }

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
__device__ __forceinline__ void field_operands(const uint32_t (&P)[8], uint32_t (&A)[8]) {
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
        byte_words<R>(P, A);
    }
}

// D = A(16x32 u8) * B(32x8 s8) + C, C given as one value for all four lanes.
__device__ __forceinline__ void mma_first(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1, uint32_t c) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(c));
}
__device__ __forceinline__ void mma_acc(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ------------------------------------------------------ barriers and copies
__device__ unsigned int g_gemv_timeout;     // set when a bounded wait gave up

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
__device__ __forceinline__ void bar_arrive(uint64_t *b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(b)) : "memory");
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ bool bar_try(uint64_t *b, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n .reg .pred p;\n"
                 " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 1000000;\n"
                 " selp.u32 %0, 1, 0, p;\n}"
                 : "=r"(ok) : "r"(smem_addr(b)), "r"(parity) : "memory");
    return ok != 0;
}
// Wait for the phase of parity `parity` to complete (the waiting thread is
// suspended, not spinning); gives up after about a second (returns false) so
// that a lost copy cannot hang the GPU.
__device__ __forceinline__ bool bar_wait(uint64_t *b, uint32_t parity) {
    if (bar_try(b, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!bar_try(b, parity))
        if (global_ns() - t0 > kWaitNs) return false;
    return true;
}
// Release/acquire on a shared-memory word (the producer's issue count).
__device__ __forceinline__ void st_release(int *p, int v) {
    asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(p)), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_addr(p)) : "memory");
    return v;
}
// One 3-D box (words x rows x planes) of the plane tensor.
__device__ __forceinline__ void tma_box3(void *dst, const CUtensorMap *map, int x, int y, int z,
                                         uint64_t *b) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(smem_addr(dst)), "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_addr(b)) : "memory");
}
// One 2-D box (elements x rows).
__device__ __forceinline__ void tma_box2(void *dst, const CUtensorMap *map, int x, int y,
                                         uint64_t *b) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_addr(dst)), "l"(map), "r"(x), "r"(y), "r"(smem_addr(b)) : "memory");
}
// 16-byte asynchronous global -> shared copy (L2 only).
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
// Arrival ticket: acquire-release add at GPU scope, returns the old value.
__device__ __forceinline__ unsigned ticket_add(unsigned *p) {
    unsigned old;
    asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
    return old;
}

// ------------------------------------------------------------ decomposition
// Items u = 0 .. W-1, W = T * KC (T 16-row tiles, KC 1024-column chunks).  The
// chunks are split into Q segments: segment ks holds chunks [cbeg(ks),
// cbeg(ks+1)) and items T cbeg(ks) .. T cbeg(ks+1) - 1 in (tile, chunk)
// order.  CTA b owns items [first(b), first(b+1)).  A "run" is the items of
// one tile inside one segment; its CTA-local part is summed inside the CTA.
struct Work {
    int64_t T, KC, W, C;
    int Q;
    __host__ __device__ int64_t cbeg(int64_t ks) const { return (ks * KC + Q - 1) / Q; }
    __host__ __device__ int64_t seg_of(int64_t u) const { return (u / T) * Q / KC; }
    __host__ __device__ int64_t first(int64_t b) const { return b * W / C; }
    __host__ __device__ int64_t cta_of(int64_t u) const { return ((u + 1) * C - 1) / W; }
};

struct Item {
    int64_t tile, kc, ks;
    int64_t run_a, run_b;   // the tile's items in this segment: [run_a, run_b)
};

__host__ __device__ __noinline__ Item item_at(const Work &w, int64_t u) {
    Item it;
    it.ks = w.seg_of(u);
    const int64_t c0 = w.cbeg(it.ks), kcs = w.cbeg(it.ks + 1) - c0, base = w.T * c0;
    const int64_t rel = u - base;
    it.tile = rel / kcs;
    it.kc = c0 + rel % kcs;
    it.run_a = base + it.tile * kcs;
    it.run_b = it.run_a + kcs;
    return it;
}

// Number of CTAs that hold items of `tile` (over all segments).
__host__ __device__ __noinline__ int64_t contributors(const Work &w, int64_t tile) {
    int64_t n = 0;
    for (int64_t ks = 0; ks < w.Q; ++ks) {
        const int64_t c0 = w.cbeg(ks), kcs = w.cbeg(ks + 1) - c0;
        if (kcs <= 0) continue;
        const int64_t a = w.T * c0 + tile * kcs;
        n += w.cta_of(a + kcs - 1) - w.cta_of(a) + 1;
    }
    return n;
}

// Index of u's run among the runs of the range starting at u0 (runs counted
// in item order): the number of run starts v with u0 < v <= u.
__host__ __device__ __noinline__ int64_t run_index(const Work &w, int64_t u0, int64_t u) {
    if (w.Q == 1) return u / w.KC - u0 / w.KC;
    int64_t n = 0;
    for (int64_t ks = w.seg_of(u0); ks <= w.seg_of(u); ++ks) {
        const int64_t c0 = w.cbeg(ks), kcs = w.cbeg(ks + 1) - c0, base = w.T * c0;
        if (kcs <= 0) continue;
        const int64_t lo = (u0 + 1 > base) ? u0 + 1 : base;
        const int64_t end = w.T * w.cbeg(ks + 1) - 1;
        const int64_t hi = u < end ? u : end;
        if (lo <= hi) n += (hi - base) / kcs - (lo - base + kcs - 1) / kcs + 1;
    }
    return n;
}

// One CTA's items [u0, u1) and their processing order.  With Q = 1 the
// range's last tile, when it is shared with the next CTA, is moved right
// after the first tile, so both shared tiles finish early.
struct Range {
    int u0, u1, L;
    int nf, nl;             // when reordered: items of the first / last tile
    bool reorder;
};
__host__ __device__ inline Range make_range(const Work &w, int64_t b) {
    Range r;
    r.u0 = (int)w.first(b);
    r.u1 = (int)w.first(b + 1);
    r.L = r.u1 - r.u0;
    r.nf = r.nl = 0;
    r.reorder = false;
    if (w.Q == 1 && r.L > 0) {
        const int KC = (int)w.KC;
        const int tf = r.u0 / KC, tl = (r.u1 - 1) / KC;
        if (tl != tf && r.u1 % KC != 0) {
            r.reorder = true;
            r.nf = (r.u0 % KC) ? (tf + 1) * KC - r.u0 : 0;
            r.nl = r.u1 - tl * KC;
        }
    }
    return r;
}
// Natural position (u - u0) of the i-th processed item.
__host__ __device__ inline int order_pos(const Range &r, int i) {
    if (!r.reorder || i < r.nf) return i;
    if (i < r.nf + r.nl) return (r.L - r.nl) + (i - r.nf);
    return r.nf + (i - r.nf - r.nl);
}
// Tile and chunk of item u (one 32-bit division when Q = 1).
__host__ __device__ inline void tile_chunk(const Work &w, int u, int &tile, int &kc) {
    if (w.Q == 1) {
        tile = u / (int)w.KC;
        kc = u - tile * (int)w.KC;
    } else {
        const Item it = item_at(w, u);
        tile = (int)it.tile;
        kc = (int)it.kc;
    }
}

// Chunk slots of a CTA: per segment it touches, a circular window of the
// segment's chunks starting at the chunk of its first item there.
struct SegWindow { int64_t c0, kcs, start, len; };
__host__ __device__ __noinline__ SegWindow seg_window(const Work &w, int64_t u0, int64_t u1, int64_t ks) {
    SegWindow s;
    s.c0 = w.cbeg(ks);
    s.kcs = w.cbeg(ks + 1) - s.c0;
    const int64_t base = w.T * s.c0, end = w.T * w.cbeg(ks + 1);
    const int64_t a = u0 > base ? u0 : base, b = u1 < end ? u1 : end;
    s.start = s.kcs > 0 ? (a - base) % s.kcs : 0;
    s.len = b > a ? (b - a < s.kcs ? b - a : s.kcs) : 0;
    return s;
}
__host__ __device__ __noinline__ int64_t chunk_slots(const Work &w, int64_t u0, int64_t u1) {
    if (w.Q == 1) return u1 - u0 < w.KC ? u1 - u0 : w.KC;
    int64_t n = 0;
    for (int64_t ks = w.seg_of(u0); ks <= w.seg_of(u1 - 1); ++ks) n += seg_window(w, u0, u1, ks).len;
    return n;
}
__host__ __device__ __noinline__ int64_t slot_of_chunk(const Work &w, int64_t u0, int64_t u1,
                                                 int64_t ks, int64_t kc) {
    int64_t base = 0;
    for (int64_t k2 = w.seg_of(u0); k2 < ks; ++k2) base += seg_window(w, u0, u1, k2).len;
    const SegWindow s = seg_window(w, u0, u1, ks);
    return base + (kc - s.c0 - s.start + s.kcs) % s.kcs;
}
__host__ __device__ __noinline__ int64_t chunk_of_slot(const Work &w, int64_t u0, int64_t u1, int64_t slot) {
    for (int64_t ks = w.seg_of(u0); ks <= w.seg_of(u1 - 1); ++ks) {
        const SegWindow s = seg_window(w, u0, u1, ks);
        if (slot < s.len) return s.c0 + (s.start + slot) % s.kcs;
        slot -= s.len;
    }
    return -1;
}

// What a consumer needs about one processed item (built once per CTA).
struct Entry {
    int tile, kc, slot, run;   // run: CTA-local index of the item's run
    int ps, pe;                // the run's natural positions [ps, pe)
    int kcf, nctb;             // chunk of the run's first item; CTAs sharing the tile
};

__host__ __device__ inline Entry make_entry(const Work &w, const Range &r, int i) {
    Entry e;
    const int p = order_pos(r, i), u = r.u0 + p;
    if (w.Q == 1) {
        const int KC = (int)w.KC;
        e.tile = u / KC;
        e.kc = u - e.tile * KC;
        const int ra = e.tile * KC, rb = ra + KC;
        e.ps = (ra > r.u0 ? ra : r.u0) - r.u0;
        e.pe = (rb < r.u1 ? rb : r.u1) - r.u0;
        e.run = e.tile - r.u0 / KC;
        const int ks0 = r.u0 - (r.u0 / KC) * KC;           // chunk of the first item
        e.slot = e.kc - ks0 < 0 ? e.kc - ks0 + KC : e.kc - ks0;
        e.kcf = (r.u0 + e.ps) - ra;
        e.nctb = (ra < r.u0 || rb > r.u1) ? (int)(w.cta_of(rb - 1) - w.cta_of(ra) + 1) : 1;
    } else {
        const Item it = item_at(w, u);
        e.tile = (int)it.tile;
        e.kc = (int)it.kc;
        e.ps = (int)((it.run_a > r.u0 ? it.run_a : r.u0) - r.u0);
        e.pe = (int)((it.run_b < r.u1 ? it.run_b : r.u1) - r.u0);
        e.run = (int)run_index(w, r.u0, u);
        e.slot = (int)slot_of_chunk(w, r.u0, r.u1, it.ks, it.kc);
        e.kcf = (int)item_at(w, r.u0 + e.ps).kc;
        e.nctb = (int)contributors(w, it.tile);
    }
    return e;
}
// Chunk held by slot `slot` of the CTA.
__host__ __device__ inline int slot_chunk(const Work &w, const Range &r, int slot) {
    if (w.Q == 1) {
        const int KC = (int)w.KC;
        const int c = r.u0 - (r.u0 / KC) * KC + slot;
        return c >= KC ? c - KC : c;
    }
    return (int)chunk_of_slot(w, r.u0, r.u1, slot);
}

// Kernel arguments (one struct, passed as a grid constant).
struct Args {
    const __nv_bfloat16 *X;
    const __half *scales;
    __nv_bfloat16 *Y;
    float *part;            // [T][KC][16 M] partial sums of shared tiles
    unsigned *tickets;      // [T] arrivals at shared tiles (zero between calls)
    Work w;
    int64_t N, K, G;
    int M, S, scales_tma, scales_cta;
    const uint8_t *xops;    // X operand blocks of every chunk (x_slices_kernel output)
    uint32_t xblk;          // x_block_bytes(M)
    // shared-memory offsets from the 1024-byte aligned base
    uint32_t o_ring, o_sring, o_xs, o_zero, o_res, o_cnt, o_bar, o_tab, o_rbar, o_run, o_sc;
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

// The X operand of a call, built once: one warp per (group g, batch row m).
// With the group exponent Eg = max floor(log2 |z|), z = x 2^(-sh), it writes
// into chunk g / 8's block (x_block_bytes(M) bytes): the int8 slices of z for
// column c = 4m + j at c*kColBytes + (g % 8)*128 + 32t + 4w (byte b of that
// word is column 32t + 8b + w of the group: the order in which the B
// fragments read it), and the pair {2^(8-r) 2^(Eg-6), S = sum of the group's
// x} at 4M*kColBytes + ((g % 8)*8 + m)*8.
template <int R>
__global__ void __launch_bounds__(256)
x_slices_kernel(const __nv_bfloat16 *__restrict__ X, int M, int64_t K, uint8_t *__restrict__ out) {
    // the product kernel may start streaming weights now
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // X comes from the previous kernel of the stream
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t G = K / kGroup;
    const int64_t task = (int64_t)blockIdx.x * 8 + warp;
    if (task >= G * M) return;
    const int64_t g = task / M;
    const int m = (int)(task - g * M);
    const int t = lane >> 3, wi = lane & 7;
    const int sh = field_shift<R>(wi);
    const uint16_t *xr = reinterpret_cast<const uint16_t *>(X) + (int64_t)m * K + g * kGroup + 32 * t + wi;
    uint32_t h[4];
    int emax = -1000;
    float sum = 0.f;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        h[b] = xr[8 * b];
        const int e8 = (int)((h[b] >> 7) & 0xFFu);
        const int v = e8 ? e8 - sh : -1000;
        emax = v > emax ? v : emax;
        sum += __uint_as_float(h[b] << 16);
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
    for (int b = 0; b < 4; ++b) F[b] = fixed_point(h[b], sh, Eg);
    uint32_t wd[kSlices];
    wd[0] = pack_bytes(F[0] >> 21, F[1] >> 21, F[2] >> 21, F[3] >> 21);
    wd[1] = pack_bytes(F[0] >> 14, F[1] >> 14, F[2] >> 14, F[3] >> 14) & 0x7F7F7F7Fu;
    wd[2] = pack_bytes(F[0] >> 7, F[1] >> 7, F[2] >> 7, F[3] >> 7) & 0x7F7F7F7Fu;
    wd[3] = pack_bytes(F[0], F[1], F[2], F[3]) & 0x7F7F7F7Fu;
    uint8_t *blk = out + (g / kCG) * (int64_t)x_block_bytes(M);
    const int grp = (int)(g % kCG);
    uint8_t *dst = blk + grp * 128 + 32 * t + 4 * wi;
#pragma unroll
    for (int j = 0; j < kSlices; ++j)
        *reinterpret_cast<uint32_t *>(dst + (size_t)(4 * m + j) * kColBytes) = wd[j];
    if (lane == 0) {
        // 2^(8-r) 2^(Eg-6), clamped to the normal fp32 range
        int ex = 2 - R + Eg;
        ex = ex < -126 ? -126 : (ex > 127 ? 127 : ex);
        *reinterpret_cast<float2 *>(blk + 4 * M * kColBytes + (grp * 8 + m) * 8) =
            make_float2(__int_as_float((ex + 127) << 23), sum);
    }
}

// ------------------------------------------------------------------ kernel
__device__ __forceinline__ float scale_of(const uint4 &v, int grp) {
    const uint32_t wv = grp < 2 ? v.x : grp < 4 ? v.y : grp < 6 ? v.z : v.w;
    return __half2float(__ushort_as_half((unsigned short)((wv >> (16 * (grp & 1))) & 0xFFFFu)));
}

template <int R, int NT>
__global__ void __launch_bounds__(kThreads, 1)
nested_gemv_kernel(const __grid_constant__ CUtensorMap pmap, const __grid_constant__ CUtensorMap smap,
                   const __grid_constant__ Args a) {
    constexpr uint32_t kStage = 2048u * R;              // planes of one item: R x 16 x 128 B
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const Work &w = a.w;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Range rg = make_range(w, blockIdx.x);
    const int L = rg.L, S = a.S;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + a.o_bar);
    uint64_t *empty = full + S;
    int *flags = reinterpret_cast<int *>(empty + S);     // [0] error, [1] items issued, [2] X requested
    uint64_t *rbar = reinterpret_cast<uint64_t *>(smem + a.o_rbar);   // per run: this CTA's part is out
    int2 *runinfo = reinterpret_cast<int2 *>(smem + a.o_run);        // per run: {tile, contributors}
    int *cnt = reinterpret_cast<int *>(smem + a.o_cnt);
    Entry *tab = reinterpret_cast<Entry *>(smem + a.o_tab);

    if (warp == kProd && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(&pmap) : "memory");
        if (a.scales_tma) asm volatile("prefetch.tensormap [%0];" ::"l"(&smap) : "memory");
    }
    if (threadIdx.x < 2 * S) {
        bar_init(full + threadIdx.x, 1);                 // full[0..S), then empty[0..S)
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (threadIdx.x == 0) {
        flags[0] = 0;
        flags[1] = 0;
        flags[2] = 0;
    }
    for (int i = threadIdx.x; i < 256; i += kThreads) reinterpret_cast<uint32_t *>(smem + a.o_zero)[i] = 0u;
    for (int i = threadIdx.x; i < L; i += kThreads) {
        cnt[i] = 0;
        bar_init(rbar + i, 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncthreads();

    // Producer warp: lane j issues item i0 + j of each batch of 32 (item i ->
    // stage i % S).  Planes by TMA (rows >= N and columns >= K arrive as
    // zeros); scales by TMA or, when the scale rows are not 16-byte aligned,
    // by the lane itself with plain loads.  After a batch, lane 0 publishes
    // how many items are issued (consumers wait for that before waiting on a
    // reused stage, whose barrier is tested by parity).
    // A batch holds at most S items, so every stage it reuses was filled by an
    // earlier, already published batch (no wait on an unpublished item).
    const int batch = S < 32 ? S : 32;
    auto produce = [&](int i0, int i1) {
        for (int base = i0; base < i1; base += batch) {
            const int i = base + lane;
            int ok = 1;
            if (lane < batch && i < i1) {
                const int st = i % S;
                if (i >= S) ok = (int)bar_wait(empty + st, (uint32_t)((i / S) - 1) & 1u);
                if (ok) {
                    int tile, kc;
                    tile_chunk(w, rg.u0 + order_pos(rg, i), tile, kc);
                    uint8_t *dst = smem + a.o_ring + (size_t)st * kStage;
                    uint8_t *sdst = smem + a.o_sring + (size_t)st * 256;
                    if (!a.scales_cta && !a.scales_tma) {
                        __half *sh = reinterpret_cast<__half *>(sdst);
                        for (int rr = 0; rr < 16; ++rr) {
                            const int64_t n = (int64_t)tile * 16 + rr;
                            for (int gq = 0; gq < kCG; ++gq) {
                                const int64_t gg = (int64_t)kc * kCG + gq;
                                sh[rr * 8 + gq] = (n < a.N && gg < a.G) ? a.scales[n * a.G + gg]
                                                                        : __float2half(0.f);
                            }
                        }
                    }
                    const bool stma = !a.scales_cta && a.scales_tma;
                    bar_expect(full + st, kStage + (stma ? 256u : 0u));
                    tma_box3(dst, &pmap, kc * 32, tile * 16, 0, full + st);
                    if (stma) tma_box2(sdst, &smap, kc * kCG, tile * 16, full + st);
                }
            }
            __syncwarp();
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) { st_release(&flags[0], 1); atomicOr(&g_gemv_timeout, 1u); }
                break;
            }
            if (lane == 0) st_release(&flags[1], base + batch < i1 ? base + batch : i1);
        }
    };
    // Per-CTA scales (Q = 1): the fp16 scales of every row of the CTA's tiles,
    // all groups, as [tile - tf][16][G]; loaded by the consumer threads.
    const bool cta_scales = a.scales_cta != 0;
    const int64_t tf = rg.u0 / w.KC;
    if (warp == kProd) {
        // A first few items now; the rest once the consumers have asked for X,
        // so that X does not queue behind the whole weight stream.
        const int first = L < S ? L : S;
        const int head = first < kHeadItems ? first : kHeadItems;
        produce(0, head);
        // the next call may start now: it only streams weights until it waits
        if (lane == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        int ok = 1;
        if (lane == 0 && ld_acquire(&flags[2]) == 0) {
            const uint64_t t0 = global_ns();
            while (ld_acquire(&flags[2]) == 0) {
                if (global_ns() - t0 > kWaitNs) { ok = 0; break; }
                __nanosleep(128);
            }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
            if (lane == 0) { st_release(&flags[0], 1); atomicOr(&g_gemv_timeout, 1u); }
        } else {
            produce(head, first);
            if (L > S) produce(S, L);
        }
    } else if (warp < kCW) {
        if (cta_scales) {
            const int64_t tl = (rg.u1 - 1) / w.KC;
            const int nrow = (int)(tl - tf + 1) * 16;
            __half *sc = reinterpret_cast<__half *>(smem + a.o_sc);
            if (a.G % 8 == 0) {
                const int per = (int)(a.G / 8);             // 16-byte pieces per row
                for (int c = threadIdx.x; c < nrow * per; c += kCW * 32) {
                    const int rr = c / per, o = c - rr * per;
                    const int64_t n = tf * 16 + rr;
                    if (n < a.N) cp_async16(sc + (size_t)rr * a.G + 8 * o, a.scales + n * a.G + 8 * o);
                    else *reinterpret_cast<uint4 *>(sc + (size_t)rr * a.G + 8 * o) = make_uint4(0u, 0u, 0u, 0u);
                }
                asm volatile("cp.async.commit_group;" ::: "memory");
            } else {
                for (int c = threadIdx.x; c < nrow * a.G; c += kCW * 32) {
                    const int rr = (int)(c / a.G);
                    const int64_t n = tf * 16 + rr;
                    sc[c] = n < a.N ? a.scales[n * a.G + (c - (int64_t)rr * a.G)] : __float2half(0.f);
                }
            }
        }
        // item table (no dependence on X)
        for (int i = threadIdx.x; i < L; i += kCW * 32) tab[i] = make_entry(w, rg, i);
        // X operand blocks of this CTA's chunks, built by the preceding
        // x_slices_kernel: read only after it has finished
        asm volatile("griddepcontrol.wait;" ::: "memory");
        // (16-byte asynchronous copies by the consumer threads: they do not
        // queue behind the producer's weight copies, which mostly start after
        // these are issued)
        {
            const int nslot = (int)chunk_slots(w, rg.u0, rg.u1);
            const int per = (int)(a.xblk / 16);
            for (int c = threadIdx.x; c < nslot * per; c += kCW * 32) {
                const int sl = c / per, o = c - sl * per;
                cp_async16(smem + a.o_xs + (size_t)sl * a.xblk + (size_t)o * 16,
                           a.xops + (size_t)slot_chunk(w, rg, sl) * a.xblk + (size_t)o * 16);
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
            asm volatile("bar.sync 1, %0;" ::"r"(kCW * 32) : "memory");
            if (threadIdx.x == 0) st_release(&flags[2], 1);        // X requested: stream the rest
            asm volatile("cp.async.wait_group 0;" ::: "memory");
            asm volatile("bar.sync 1, %0;" ::"r"(kCW * 32) : "memory");
        }
        const int g = lane >> 2, t = lane & 3;
        float *res = reinterpret_cast<float *>(smem + a.o_res);
        const int M = a.M;
        constexpr float kOffset = (float)(128 >> (R - 1)) * 0.5f - 128.0f;   // 2^(7-r) - 128
        for (int i = warp; i < L; i += kCW) {
            const int st = i % S;
            // A stage's full barrier is waited on by parity, so item i may be
            // waited for only once item i - S has landed: that holds as soon as
            // the producer has issued item i (it first waited for i - S to be
            // consumed).
            int issued_ok = 1;
            if (lane == 0 && ld_acquire(&flags[1]) <= i) {
                const uint64_t t0 = global_ns();
                while (ld_acquire(&flags[1]) <= i) {
                    if (ld_acquire(&flags[0]) || global_ns() - t0 > kWaitNs) { issued_ok = 0; break; }
                    __nanosleep(256);
                }
            }
            issued_ok = __shfl_sync(0xffffffffu, issued_ok, 0);
            if (!issued_ok || !__all_sync(0xffffffffu, bar_wait(full + st, (uint32_t)(i / S) & 1u))) {
                if (lane == 0) { st_release(&flags[0], 1); atomicOr(&g_gemv_timeout, 1u); }
                break;
            }
            const Entry e = tab[i];
            const int p = order_pos(rg, i);
            const int ng = (int)((a.G - (int64_t)e.kc * kCG) < kCG ? (a.G - (int64_t)e.kc * kCG) : kCG);
            const uint32_t *pl = reinterpret_cast<const uint32_t *>(smem + a.o_ring + (size_t)st * kStage);
            uint4 sc_lo, sc_hi;                  // the 8 groups' scales of rows g and g + 8
            if (!cta_scales) {
                const uint8_t *sc = smem + a.o_sring + (size_t)st * 256;
                sc_lo = *reinterpret_cast<const uint4 *>(sc + 16 * g);
                sc_hi = *reinterpret_cast<const uint4 *>(sc + 16 * (g + 8));
            } else {
                const __half *sc = reinterpret_cast<const __half *>(smem + a.o_sc) +
                                   ((size_t)(e.tile - tf) * 16 + g) * a.G + (size_t)e.kc * kCG;
                if (a.G % 8 == 0) {
                    sc_lo = *reinterpret_cast<const uint4 *>(sc);
                    sc_hi = *reinterpret_cast<const uint4 *>(sc + 8 * a.G);
                } else {
                    uint32_t lo[4], hi[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int g0 = 2 * q, g1 = 2 * q + 1;
                        const bool v0 = e.kc * kCG + g0 < a.G, v1 = e.kc * kCG + g1 < a.G;
                        lo[q] = (v0 ? __half_as_ushort(sc[g0]) : 0u) | ((v1 ? (uint32_t)__half_as_ushort(sc[g1]) : 0u) << 16);
                        hi[q] = (v0 ? __half_as_ushort(sc[8 * a.G + g0]) : 0u) |
                                ((v1 ? (uint32_t)__half_as_ushort(sc[8 * a.G + g1]) : 0u) << 16);
                    }
                    sc_lo = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                    sc_hi = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                }
            }
            const uint8_t *xs = smem + a.o_xs + (size_t)e.slot * a.xblk;
            const uint8_t *xb[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int c = 8 * nt + g;
                xb[nt] = (c < 4 * M ? xs + c * kColBytes : smem + a.o_zero) + 32 * t;
            }
            const float2 *gs = reinterpret_cast<const float2 *>(xs + 4 * M * kColBytes);
            float acc[NT][4], off[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
                off[nt][0] = off[nt][1] = 0.f;
            }
#pragma unroll
            for (int grp = 0; grp < kCG; ++grp) {
                if (grp < ng) {
                    uint32_t A0[8], A1[8];
                    {
                        uint32_t P[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            P[q] = q < R ? pl[(q * 16 + g) * 32 + ((grp ^ g) << 2) + t] : 0u;
                        field_operands<R>(P, A0);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            P[q] = q < R ? pl[(q * 16 + g + 8) * 32 + ((grp ^ g) << 2) + t] : 0u;
                        field_operands<R>(P, A1);
                    }
                    const float s_lo = scale_of(sc_lo, grp), s_hi = scale_of(sc_hi, grp);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        // lanes whose column is beyond 4M read a zero area laid out alike
                        const uint8_t *bp = xb[nt] + grp * 128;
                        const uint4 B0 = *reinterpret_cast<const uint4 *>(bp);
                        const uint4 B1 = *reinterpret_cast<const uint4 *>(bp + 16);
                        int d[4];
                        mma_first(d, A0[0], A1[0], A0[1], A1[1], B0.x, B0.y, kMagicBits);
                        mma_acc(d, A0[2], A1[2], A0[3], A1[3], B0.z, B0.w);
                        mma_acc(d, A0[4], A1[4], A0[5], A1[5], B1.x, B1.y);
                        mma_acc(d, A0[6], A1[6], A0[7], A1[7], B1.z, B1.w);
                        const int mm = 2 * nt + (t >> 1) < M ? 2 * nt + (t >> 1) : M - 1;
                        const float2 ge = gs[grp * 8 + mm];   // {2^(8-r) 2^(Eg-6), S}
                        const float se_lo = s_lo * ge.x, se_hi = s_hi * ge.x;
                        acc[nt][0] = fmaf(se_lo, __int_as_float(d[0]) - kMagic, acc[nt][0]);
                        acc[nt][1] = fmaf(se_lo, __int_as_float(d[1]) - kMagic, acc[nt][1]);
                        acc[nt][2] = fmaf(se_hi, __int_as_float(d[2]) - kMagic, acc[nt][2]);
                        acc[nt][3] = fmaf(se_hi, __int_as_float(d[3]) - kMagic, acc[nt][3]);
                        off[nt][0] = fmaf(s_lo, ge.y, off[nt][0]);
                        off[nt][1] = fmaf(s_hi, ge.y, off[nt][1]);
                    }
                }
            }
            // the stage is free once every lane has read it
            __syncwarp();
            if (lane == 0) bar_arrive(empty + st);

            // columns 4m .. 4m+3 -> batch row m: lanes t = 2(m % 2), +1 hold them
            float *out = res + p * 16 * M;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int m = 2 * nt + (t >> 1);
                // slices j = 2(t % 2) and j + 1 carry 2^(-7j)
                const float fx = (t & 1) ? 0x1p-14f : 1.0f, fy = (t & 1) ? 0x1p-21f : 0x1p-7f;
                float v_lo = fx * acc[nt][0] + fy * acc[nt][1];
                float v_hi = fx * acc[nt][2] + fy * acc[nt][3];
                v_lo += __shfl_xor_sync(0xffffffffu, v_lo, 1);
                v_hi += __shfl_xor_sync(0xffffffffu, v_hi, 1);
                if ((t & 1) == 0 && m < M) {
                    out[m * 16 + g] = fmaf(kOffset, off[nt][0], v_lo);
                    out[m * 16 + g + 8] = fmaf(kOffset, off[nt][1], v_hi);
                }
            }
            __syncwarp();
            int last = 0;
            if (lane == 0) {
                __threadfence_block();
                last = atomicAdd(&cnt[e.run], 1) == e.pe - e.ps - 1;
            }
            last = __shfl_sync(0xffffffffu, last, 0);
            if (!last) continue;
            __threadfence_block();
            // this CTA's part of the tile (idx = m * 16 + row), summed in chunk order
            for (int idx = lane; idx < 16 * M; idx += 32) {
                float v = 0.f;
                for (int q = e.ps; q < e.pe; ++q) v += res[q * 16 * M + idx];
                if (e.nctb == 1) {
                    const int64_t n = (int64_t)e.tile * 16 + (idx & 15);
                    if (n < a.N) a.Y[(int64_t)(idx >> 4) * a.N + n] = __float2bfloat16_rn(v);
                } else {
                    a.part[((int64_t)e.tile * w.KC + e.kcf) * 16 * M + idx] = v;
                }
            }
            // a tile shared with other CTAs goes to the epilogue warp
            __syncwarp();
            if (e.nctb != 1 && lane == 0) {
                runinfo[e.run] = make_int2(e.tile, e.nctb);
                bar_arrive(rbar + e.run);
            }
        }
    } else if (warp == kEpi) {
        // Tiles shared with other CTAs: after this CTA's part is in the
        // workspace, take an arrival ticket; the last CTA to arrive sums every
        // part in chunk order and writes Y.  (Off the consumers' path: they
        // never wait on these global round trips.)
        const int M = a.M;
        const int nruns = (int)run_index(w, rg.u0, rg.u1 - 1) + 1;
        for (int run = 0; run < nruns; ++run) {
            if (w.Q == 1) {
                // only the range's first and last tiles can extend past it
                const int64_t ra = (rg.u0 / w.KC + run) * w.KC;
                if (ra >= rg.u0 && ra + w.KC <= rg.u1) continue;
            }
            if (!__all_sync(0xffffffffu, bar_wait(rbar + run, 0u))) {
                if (lane == 0) { st_release(&flags[0], 1); atomicOr(&g_gemv_timeout, 1u); }
                break;
            }
            const int2 ri = runinfo[run];            // {tile, contributing CTAs}
            unsigned old = 0;
            if (lane == 0) old = ticket_add(&a.tickets[ri.x]);
            old = __shfl_sync(0xffffffffu, old, 0);
            if (old != (unsigned)(ri.y - 1)) continue;
            __threadfence();
            for (int idx = lane; idx < 16 * M; idx += 32) {
                float v = 0.f;
                for (int64_t ks = 0; ks < w.Q; ++ks) {
                    const int64_t c0 = w.cbeg(ks), kcs = w.cbeg(ks + 1) - c0;
                    if (kcs <= 0) continue;
                    const int64_t ra = w.T * c0 + (int64_t)ri.x * kcs;
                    for (int64_t c = w.cta_of(ra); c <= w.cta_of(ra + kcs - 1); ++c) {
                        const int64_t fa = w.first(c) > ra ? w.first(c) : ra;
                        v += __ldcg(a.part + ((int64_t)ri.x * w.KC + c0 + (fa - ra)) * 16 * M + idx);
                    }
                }
                const int64_t n = (int64_t)ri.x * 16 + (idx & 15);
                if (n < a.N) a.Y[(int64_t)(idx >> 4) * a.N + n] = __float2bfloat16_rn(v);
            }
            __syncwarp();
            if (lane == 0) a.tickets[ri.x] = 0u;
        }
    }

    // after a timed-out wait: let the copies already issued land before exit
    __syncthreads();
    if (flags[0] && threadIdx.x == 0) {
        const int issued = flags[1];
        for (int st = 0; st < S && st < issued; ++st) {
            const int last = st + ((issued - 1 - st) / S) * S;
            bar_wait(full + st, (uint32_t)(last / S) & 1u);
        }
    }
}

// ---------------------------------------------------------------- host side
struct Plan {
    Work w;
    int NT, S, nslot, L, nruns;
    uint32_t o_ring, o_sring, o_xs, o_zero, o_res, o_cnt, o_bar, o_tab, o_rbar, o_run, o_sc;
    int ntile;              // Q = 1: most tiles a CTA touches (per-CTA scale block rows / 16)
    int64_t G;
    size_t smem;            // dynamic shared memory per CTA (with alignment slack)
    size_t part_off, xops_off, ws_bytes;
    bool ok;
};

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

inline uint32_t align_up(size_t x, size_t a) { return (uint32_t)((x + a - 1) / a * a); }

// Lays out shared memory for S stages; returns the size without slack.
size_t layout(Plan &p, int r, int M, int S) {
    size_t o = 0;
    p.o_ring = 0;
    o = (size_t)S * 2048 * r;
    p.o_sring = align_up(o, 128);
    o = p.o_sring + (size_t)S * 256;
    p.o_xs = align_up(o, 128);
    o = p.o_xs + (size_t)p.nslot * x_block_bytes(M);
    p.o_zero = align_up(o, 128);
    o = p.o_zero + 1024;
    p.o_res = align_up(o, 16);
    o = p.o_res + (size_t)p.L * 16 * M * 4;
    p.o_cnt = align_up(o, 16);
    o = p.o_cnt + (size_t)(p.L > p.nruns ? p.L : p.nruns) * 4;
    p.o_tab = align_up(o, 16);
    o = p.o_tab + (size_t)p.L * sizeof(Entry);
    p.o_rbar = align_up(o, 16);
    o = p.o_rbar + (size_t)p.L * 8;
    p.o_run = align_up(o, 16);
    o = p.o_run + (size_t)p.L * 8;
    p.o_sc = align_up(o, 16);
    o = p.o_sc + (size_t)p.ntile * 16 * p.G * 2;
    p.o_bar = align_up(o, 16);
    o = p.o_bar + (size_t)(2 * S + 1) * 8 + 16;
    return o;
}

Plan make_plan(int64_t M, int64_t N, int64_t K, int r) {
    Plan p{};
    const int64_t T = (N + 15) / 16, G = K / kGroup, KC = (G + kCG - 1) / kCG;
    p.G = G;
    const int64_t W = T * KC;
    p.NT = (int)((4 * M + 7) / 8);
    const size_t stage = (size_t)2048 * r + 256;
    // one CTA per SM; more CTAs (in waves) only when a CTA's share of the
    // items does not fit in shared memory at any K split
    for (int64_t mult = 1; mult <= 16; mult *= 2) {
    const int64_t C = W < sm_count() * mult ? W : sm_count() * mult;
    for (int64_t Q = 1; Q <= KC; ++Q) {
        Work w{T, KC, W, C, (int)Q};
        int64_t L = 0, ns = 0, nr = 0, nt = 0;
        for (int64_t b = 0; b < C; ++b) {
            const int64_t u0 = w.first(b), u1 = w.first(b + 1);
            if (u1 <= u0) continue;
            L = u1 - u0 > L ? u1 - u0 : L;
            if (Q == 1) {
                const int64_t tt = (u1 - 1) / KC - u0 / KC + 1;
                nt = tt > nt ? tt : nt;
            }
            const int64_t c = chunk_slots(w, u0, u1);
            ns = c > ns ? c : ns;
            const int64_t rr = run_index(w, u0, u1 - 1) + 1;
            nr = rr > nr ? rr : nr;
        }
        p.w = w;
        p.L = (int)L;
        p.nslot = (int)ns;
        p.nruns = (int)nr;
        p.ntile = (int)nt;
        const size_t fixed = layout(p, r, (int)M, 0);
        if (fixed + 2 * stage + 1024 > kSmemBudget) continue;
        int S = (int)((kSmemBudget - 1024 - fixed) / stage);
        if (S > L) S = (int)L;
        // few stages hide little latency: prefer another K split while it helps
        if (S < 4 && S < L && Q < KC) continue;
        p.S = S < 2 ? 2 : S;
        p.smem = layout(p, r, (int)M, p.S) + 1024;
        p.part_off = kTicketBytes;
        p.xops_off = (p.part_off + (size_t)W * 16 * M * sizeof(float) + 255) & ~(size_t)255;
        p.ws_bytes = p.xops_off + (size_t)KC * x_block_bytes((int)M);
        p.ok = p.smem <= 227 * 1024;
        return p;
    }
    }
    p.ok = false;
    return p;
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

// The r planes as [r][N][K/32] words; box (32 words, 16 rows, r planes) with
// the 128-byte swizzle.  Cached per (buffer, shape, r).
mq_status plane_map(const mq_weights *w, CUtensorMap *out) {
    struct Slot { const void *p; int64_t N, K; int r; CUtensorMap map; };
    static thread_local Slot cache[32];
    static thread_local int next = 0;
    for (auto &c : cache)
        if (c.p == w->planes && c.N == w->N && c.K == w->K && c.r == w->r) { *out = c.map; return MQ_OK; }
    auto encode = encoder();
    if (!encode) return fail(MQ_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const cuuint64_t dims[3] = {(cuuint64_t)(w->K / 32), (cuuint64_t)w->N, (cuuint64_t)w->r};
    const cuuint64_t strides[2] = {(cuuint64_t)(w->K / 8), (cuuint64_t)(w->N * (w->K / 8))};
    const cuuint32_t box[3] = {32u, 16u, (cuuint32_t)w->r};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    CUtensorMap m;
    const CUresult res = encode(&m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t *>(w->planes),
                                dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (res != CUDA_SUCCESS) return fail(MQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the planes");
    cache[next] = Slot{w->planes, w->N, w->K, w->r, m};
    next = (next + 1) % 32;
    *out = m;
    return MQ_OK;
}

// The fp16 scales [N][G] with a (8 groups, 16 rows) box; needs G % 8 == 0
// (16-byte row pitch).  Otherwise *ok = false and the kernel copies scales
// with plain loads.
mq_status scale_map(const mq_weights *w, CUtensorMap *out, bool *ok) {
    const int64_t G = w->K / kGroup;
    *ok = (G % 8) == 0;
    memset(out, 0, sizeof(*out));
    if (!*ok) return MQ_OK;
    struct Slot { const void *p; int64_t N, K; CUtensorMap map; };
    static thread_local Slot cache[32];
    static thread_local int next = 0;
    for (auto &c : cache)
        if (c.p == w->scales && c.N == w->N && c.K == w->K) { *out = c.map; return MQ_OK; }
    auto encode = encoder();
    if (!encode) return fail(MQ_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
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

template <int R, int NT>
mq_status run(const uint16_t *X, const mq_weights *wt, int64_t M, uint16_t *Y, char *ws,
              const Plan &p, cudaStream_t st) {
    static bool attr_set = false;          // per instantiation
    static size_t attr_smem = 0;
    cudaError_t e;
    if (!attr_set || attr_smem < p.smem) {
        e = cudaFuncSetAttribute(nested_gemv_kernel<R, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(227 * 1024));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        e = cudaFuncSetAttribute(nested_gemv_kernel<R, NT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 100);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        // the same shared-memory carve-out for the prep kernel, so that the SMs
        // need no reconfiguration between the two kernels of a call
        e = cudaFuncSetAttribute(x_slices_kernel<R>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        attr_set = true;
        attr_smem = 227 * 1024;
    }
    CUtensorMap pmap, smap;
    bool stma = false;
    mq_status ms = plane_map(wt, &pmap);
    if (ms == MQ_OK) ms = scale_map(wt, &smap, &stma);
    if (ms != MQ_OK) return ms;
    Args a{};
    a.X = reinterpret_cast<const __nv_bfloat16 *>(X);
    a.scales = reinterpret_cast<const __half *>(wt->scales);
    a.Y = reinterpret_cast<__nv_bfloat16 *>(Y);
    a.part = reinterpret_cast<float *>(ws + p.part_off);
    a.tickets = reinterpret_cast<unsigned *>(ws);
    a.w = p.w;
    a.N = wt->N;
    a.K = wt->K;
    a.G = wt->K / kGroup;
    a.M = (int)M;
    a.S = p.S;
    a.scales_tma = stma ? 1 : 0;
    a.xops = reinterpret_cast<const uint8_t *>(ws + p.xops_off);
    a.xblk = x_block_bytes((int)M);
    a.o_ring = p.o_ring; a.o_sring = p.o_sring; a.o_xs = p.o_xs; a.o_zero = p.o_zero;
    a.o_res = p.o_res; a.o_cnt = p.o_cnt; a.o_bar = p.o_bar; a.o_tab = p.o_tab;
    a.o_rbar = p.o_rbar; a.o_run = p.o_run; a.o_sc = p.o_sc;
    a.scales_cta = p.w.Q == 1 ? 1 : 0;
    // Both kernels are programmatic dependent launches: each may start while
    // its predecessor in the stream finishes and waits for it before reading
    // what the predecessor wrote (X, then the X operand blocks).
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t pc = {};
    const int64_t tasks = (wt->K / kGroup) * M;
    pc.gridDim = dim3((unsigned)((tasks + 7) / 8));
    pc.blockDim = dim3(256);
    pc.stream = st;
    pc.attrs = pdl;
    pc.numAttrs = 1;
    e = cudaLaunchKernelEx(&pc, x_slices_kernel<R>, reinterpret_cast<const __nv_bfloat16 *>(X), (int)M,
                           wt->K, reinterpret_cast<uint8_t *>(ws + p.xops_off));
    if (e != cudaSuccess) return cuda_fail(e, "x_slices_kernel launch");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.w.C);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, nested_gemv_kernel<R, NT>, pmap, smap, a);
    if (e != cudaSuccess) return cuda_fail(e, "nested_gemv_kernel launch");
    return MQ_OK;
}

template <int R>
mq_status run_r(const uint16_t *X, const mq_weights *w, int64_t M, uint16_t *Y, char *ws,
                const Plan &p, cudaStream_t st) {
    switch (p.NT) {
        case 1: return run<R, 1>(X, w, M, Y, ws, p, st);
        case 2: return run<R, 2>(X, w, M, Y, ws, p, st);
        case 3: return run<R, 3>(X, w, M, Y, ws, p, st);
        default: return run<R, 4>(X, w, M, Y, ws, p, st);
    }
}

}  // namespace

size_t gemv_mma_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
    const Plan p = make_plan(M, N, K, r);
    return p.ok ? p.ws_bytes : 0;
}

mq_status launch_gemv_mma(const uint16_t *X, const mq_weights *w, int64_t M, uint16_t *Y,
                          void *ws, size_t ws_bytes, cudaStream_t st) {
    const Plan p = make_plan(M, w->N, w->K, w->r);
    if (!p.ok) return fail(MQ_ERR_UNSUPPORTED, "no GEMV plan fits in shared memory for this shape");
    if (p.ws_bytes > ws_bytes) return fail(MQ_ERR_WORKSPACE, "GEMV workspace too small");
    if (p.w.T > (int64_t)(kTicketBytes / sizeof(unsigned)))
        return fail(MQ_ERR_UNSUPPORTED, "too many row tiles for the arrival-ticket region");
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
