// Host-side check of the batched tensor-core GEMM (compiled with the kernel's
// own source; no GPU needed).
//   * decode: for r = 1..8 and random codes, the plane words of one 32-column
//     word -> word_pairs -> centring give, in TMEM column c, the levels v_r of
//     columns 2c and 2c + 1 exactly (v_r = 2^(8-r) q + 2^(7-r) - 128, q the
//     code's top r bits); the byte permute against its definition;
//   * work split: over many shapes and CTA counts, every (X block, tile, group)
//     item belongs to one CTA, cta_of agrees with the ranges, the CTAs of a
//     shared tile fit the partial-sum slots, the partial sums stay inside the
//     workspace, and the shared memory of every (r, BM) inside 227 KB.
// Prints "checked=<n> bad=<m>" and exits 1 if m > 0.
#include "../../nested_bit_weight_b200/csrc/mq_gemm_tc.cu"

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <cmath>
#include <vector>

namespace mq {
mq_status cuda_fail(cudaError_t, const char *) { return MQ_ERR_CUDA; }
void set_error(mq_status, const char *, ...) {}
}  // namespace mq

using namespace mq;

static float bf16_to_float(uint32_t h) {
    const uint32_t u = h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}
static float bits_to_float(uint32_t u) {
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static long checked = 0, bad = 0;

template <int R>
static void check_decode(unsigned seed) {
    srand(seed);
    for (int trial = 0; trial < 2000; ++trial) {
        uint8_t code[32];
        for (int j = 0; j < 32; ++j) code[j] = (uint8_t)(rand() & 255);
        if (trial == 0) memset(code, 0, 32);
        if (trial == 1) memset(code, 255, 32);
        uint32_t P[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int p = 0; p < R; ++p)
            for (int j = 0; j < 32; ++j) P[p] |= (uint32_t)((code[j] >> (7 - p)) & 1) << j;
        uint32_t v[16];
        word_pairs<R>(P, v);                                   // the kernel's own bit code
        for (int c = 0; c < 16; ++c) {                         // TMEM column c: k = 2c, 2c + 1
            float v0, v1;
            if (R <= 6) {
                // the kernel subtracts 384 - 2^(7-r) in bf16: exact, as both
                // operands and the result have <= 8 significant bits
                const float cc = 384.0f - (float)(1 << (7 - R));
                v0 = bf16_to_float(v[c] & 0xFFFFu) - cc;
                v1 = bf16_to_float(v[c] >> 16) - cc;
            } else {
                const float cc = 4194432.0f - (R == 8 ? 0.5f : 1.0f);
                v0 = bits_to_float(0x4A800000u | ((v[c] & 0xFFu) << 1)) - cc;
                v1 = bits_to_float(0x4A800000u | ((v[c] >> 8) << 1)) - cc;
            }
            const int k0 = 2 * c, k1 = k0 + 1;
            const float half = ldexpf(1.0f, 7 - R);            // 2^(7-r), 0.5 for r = 8
            const float w0 = ldexpf(1.0f, 8 - R) * (float)(code[k0] >> (8 - R)) + half - 128.0f;
            const float w1 = ldexpf(1.0f, 8 - R) * (float)(code[k1] >> (8 - R)) + half - 128.0f;
            ++checked;
            if (v0 != w0 || v1 != w1) {
                if (bad < 10) printf("decode r=%d column %d: %g %g, want %g %g\n", R, c, v0, v1, w0, w1);
                ++bad;
            }
        }
    }
}

// prmt against its definition on a few fixed cases (the host branch is what
// the decode check above runs; these pin the selector convention)
static void check_prmt() {
    const uint32_t a = 0x33221100u, b = 0x77665544u;
    const struct { uint32_t sel, want; } cases[] = {
        {0x3210u, 0x33221100u}, {0x7654u, 0x77665544u}, {0x0123u, 0x00112233u},
        {0x5140u, 0x55114400u}, {0x6622u, 0x66662222u}};
    for (const auto &c : cases) {
        ++checked;
        if (prmt(a, b, c.sel) != c.want) { ++bad; printf("prmt sel %04x: %08x\n", c.sel, prmt(a, b, c.sel)); }
    }
}

static void check_split(int64_t M, int64_t N, int64_t K, int sms) {
    const TcPlan p = tc_plan(M, N, K, sms);
    const int64_t W = (int64_t)p.MB * p.T * p.G;
    ++checked;
    if (p.P < 1 || p.P > sms || p.BM * p.MB < M ||
        (p.MB - 1) * p.BM >= M || p.T * 128 < N || p.G * 128 != K) {
        if (bad < 10) printf("plan M=%ld N=%ld K=%ld: P=%d BM=%d\n", (long)M, (long)N, (long)K, p.P, p.BM);
        ++bad;
        return;
    }
    // ranges partition the items, in order, each CTA at least one item
    int64_t prev = 0;
    for (int b = 0; b < p.P; ++b) {
        const int64_t f = range_first(b, W, p.P), l = range_first(b + 1, W, p.P);
        ++checked;
        if (f != prev || l <= f || cta_of(f, W, p.P) != b || cta_of(l - 1, W, p.P) != b) {
            if (bad < 10) printf("range b=%d [%ld, %ld) prev %ld\n", b, (long)f, (long)l, (long)prev);
            ++bad;
        }
        prev = l;
    }
    ++checked;
    if (prev != W) { ++bad; printf("ranges end at %ld, W=%ld\n", (long)prev, (long)W); }
    // the regions of the workspace: tickets, partial sums, sums of X
    ++checked;
    if (p.part_off < kTicketBytes || p.sumx_off < p.part_off || p.sumx_off % 16 ||
        p.sumx_off + (size_t)p.G * p.MB * p.BM * sizeof(float) > p.ws_bytes) {
        ++bad;
        printf("workspace regions M=%ld N=%ld K=%ld\n", (long)M, (long)N, (long)K);
    }
    // tiles shared between CTAs: slots, partial-sum bounds
    const size_t part_elems = (p.sumx_off - p.part_off) / sizeof(float);
    for (int64_t tu = 0; tu < (int64_t)p.MB * p.T; ++tu) {
        const int cf = cta_of(tu * p.G, W, p.P), cl = cta_of(tu * p.G + p.G - 1, W, p.P);
        const int cnt = cl - cf + 1;
        ++checked;
        if (cnt < 1 || cnt > p.maxc) { ++bad; printf("tile %ld spans %d CTAs, maxc %d\n", (long)tu, cnt, p.maxc); continue; }
        if (cnt > 1) {
            const size_t last = ((size_t)tu * p.maxc + (cnt - 1)) * p.BM * 128 + (size_t)(p.BM - 1) * 128 + 127;
            ++checked;
            if (last >= part_elems) { ++bad; printf("partials of tile %ld past the workspace\n", (long)tu); }
        }
    }
}

int main() {
    check_decode<1>(1); check_decode<2>(2); check_decode<3>(3); check_decode<4>(4);
    check_decode<5>(5); check_decode<6>(6); check_decode<7>(7); check_decode<8>(8);
    check_prmt();
    // shared memory of every (r, BM) within one CTA's 227 KB, >= 2 ring items per decode group
    for (int r = 1; r <= 8; ++r)
        for (int BM : {32, 64, 128}) {
            ++checked;
            const int groups = BM == 128 ? 1 : 2;              // decode groups sharing the ring
            if (tc_smem_bytes(r, BM) > 227 * 1024 || ring_items(r, BM) / groups < 2) {
                ++bad;
                printf("smem r=%d BM=%d: %zu bytes, ring %d\n", r, BM, tc_smem_bytes(r, BM), ring_items(r, BM));
            }
        }
    const long shapes[][2] = {{4096, 4096}, {1024, 4096}, {14336, 4096}, {4096, 14336}, {1, 128},
                              {37, 384},    {130, 256},   {300, 1408},   {28672, 8192}, {8192, 28672},
                              {12288, 4096}, {1, 128 * 200}, {1 << 17, 4096}, {640, 1280}};
    const long Ms[] = {1, 3, 8, 9, 16, 31, 32, 33, 64, 65, 100, 128, 129, 256, 300};
    const int sms[] = {1, 2, 7, 148};
    for (const auto &sh : shapes)
        for (long M : Ms)
            for (int s : sms) check_split(M, sh[0], sh[1], s);
    printf("checked=%ld bad=%ld\n", checked, bad);
    return bad ? 1 : 0;
}
