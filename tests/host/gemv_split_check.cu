// Host-side check of the M <= 8 GEMV's work split and shared-memory plans
// (compiled with the kernel's own source; no GPU needed).  For many shapes,
// batch classes, bit widths and (clusters, CTAs per cluster) splits:
//   * every (row tile, group) item belongs to exactly one CTA, and cta_of
//     agrees with the ranges;
//   * a row tile is shared only by CTAs of one cluster, and the CTA that
//     sends a tile's part finds the tile as its owner's last tile, in a
//     slot that exists;
//   * the shared-memory layout stays within 227 KB and its regions do not
//     overlap.
// Prints "checked=<n> bad=<m>" and exits 1 if m > 0.
#include "../../nested_bit_weight_b200/csrc/mq_gemv_tc.cu"

#include <cstdio>

extern "C" size_t mq_plane_bytes(int64_t, int64_t, int) { return 0; }
namespace mq {
mq_status cuda_fail(cudaError_t, const char *) { return MQ_ERR_CUDA; }
void set_error(mq_status, const char *, ...) {}
}  // namespace mq

using namespace mq;

int main() {
    const long shapes[][2] = {{4096, 4096}, {1024, 4096}, {14336, 4096}, {4096, 14336}, {1, 128},
                              {7, 384},     {130, 256},   {33, 1280},    {1000, 1024},  {8192, 8192},
                              {28672, 8192}, {8192, 28672}, {257, 2048}, {300, 128},    {640, 1280},
                              {2048, 14336}, {300, 28672}, {128, 128 * 200}};
    long bad = 0, checked = 0;
    for (const auto &sh : shapes)
        for (int M = 1; M <= 8; ++M)
            for (int r = 1; r <= 8; ++r)
                for (int cs = 1; cs <= 8; ++cs)
                    for (int shrink = 0; shrink < 3; ++shrink) {
                        const long N = sh[0], K = sh[1], T = (N + 127) / 128, G = K / 128;
                        long nc = 148 / cs - shrink * 5;
                        if (nc > T) nc = T;
                        if (nc < 1 || T / nc * G < cs) continue;
                        const Plan p = plan_for(Work{T, G, (int)nc, cs}, M, r);
                        if (!p.ok) continue;
                        ++checked;
                        const Work &w = p.w;
                        long covered = 0;
                        for (long b = 0; b < w.ctas(); ++b) {
                            const long u0 = w.first(b), u1 = w.first(b + 1), L = u1 - u0;
                            if (L <= 0 || L > p.L) ++bad;
                            covered += L;
                            if (w.cta_of(u0) != b || w.cta_of(u1 - 1) != b) ++bad;
                            const long tf = u0 / G, ntile = (u1 - 1) / G - tf + 1, tl = (u1 - 1) / G;
                            if (ntile > p.ntile) ++bad;
                            if (tl * G >= u0 && tl * G + G > u1) {            // owns a shared last tile
                                const long last = w.cta_of(tl * G + G - 1);
                                if (last / cs != b / cs || last - b + 1 > cs) ++bad;
                            }
                            if (tf * G < u0) {                                 // sends its first tile
                                const long owner = w.cta_of(tf * G);
                                const long olt = tf - w.first(owner) / G;
                                if (owner / cs != b / cs || b - owner < 1 || b - owner >= cs) ++bad;
                                if (olt < 0 || olt >= p.ntile) ++bad;
                                if ((w.first(owner + 1) - 1) / G != tf) ++bad;
                            }
                        }
                        if (covered != T * G) ++bad;
                        if (p.o_misc + 64 + 1024 != p.smem || p.smem > 227 * 1024) ++bad;
                        if (p.o_red < p.o_bar + (2 * (p.S / kBatch) + kTeams + p.ntile) * 8) ++bad;
                        if (cs > 1 && p.o_misc < p.o_red + (size_t)p.ntile * cs * M * 128 * 4) ++bad;
                        if (p.S % kBatch != 0 || p.S < 1) ++bad;
                    }
    std::printf("checked=%ld bad=%ld\n", checked, bad);
    return bad ? 1 : 0;
}
