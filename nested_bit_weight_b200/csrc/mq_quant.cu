// One-shot multi-precision quantizer (host): the parent codes and scales of
// the nested format from float weights and a layer's Hessian proxy
// ("MatGPTQ: Efficient and Accurate Inference over Nested Quantized Models",
// abstract: a multi-precision objective with bit-slicing and cross-bit error
// compensation; Tables 6-7: the lambda weighting of the bit widths), on
// GPTQ's column loop:
//   * U = the upper Cholesky factor of (H + damp * mean(diag H) * I)^-1
//     (mq_matgptq_prepare);
//   * per 128-column group, when its first column is reached, a row's scale
//     is s = alpha * max|w| / 127.5 over the group's current weights, alpha
//     taken from a grid for the least lambda-weighted error of the group;
//   * each weight's 8-bit code q minimises sum_r lambda_r (w - s v_r(q_r))^2
//     over the nested levels v_r of every width r (ties: the smallest code);
//   * the error carried to the later columns of the row is the
//     lambda-weighted mean of the slice errors e:  w_j -= e / U[k,k] * U[k,j]
//     (the update of the row's shared remainder that minimises the
//     lambda-weighted sum of the widths' quadratic losses).
// The asymmetric variant (mq_matgptq_quantize_asym; captions of Tables 5-7)
// takes the levels u_r = 2^(8-r) q_r + 2^(7-r) - z on a grid that spans each
// group's range, centred on it (asym_grid below); the rest is the same loop.
// Rows are independent given U, so threads take blocks of rows; every
// operation is fp64 in a fixed order, the same whatever the thread count.
#include <immintrin.h>
#include <math.h>
#include <stdlib.h>

#include <algorithm>
#include <cmath>
#include <atomic>
#include <memory>
#include <mutex>
#include <thread>
#include <vector>

#include "mq_common.cuh"

using namespace mq;

namespace {

// v_r of the top r bits of code q, exactly: 2^(8-r) q_r + 2^(7-r) - 128.
inline double level_of(int q, int r) {
    const double a = (double)(1u << (8 - r));
    const double b = r == 8 ? 0.5 : (double)(1u << (7 - r));
    return a * (double)(q >> (8 - r)) + b - 128.0;
}

struct Objective {
    const int32_t *rs;
    const double *lams;
    int nr;
    std::vector<double> levels;   // [r][256]

    Objective(const int32_t *rs_, const double *lams_, int nr_) : rs(rs_), lams(lams_), nr(nr_) {
        levels.resize((size_t)nr * 256);
        for (int i = 0; i < nr; ++i)
            for (int q = 0; q < 256; ++q) levels[(size_t)i * 256 + q] = level_of(q, rs[i]);
    }

    // (codes with s v_i(q) <= w, codes with s v_i(q) < w) for s > 0: the
    // count of width r's levels (blocks of 2^(8-r) equal codes) below w
    // estimated from w / s and then settled by exact comparisons with the
    // rounded products, so the counts are those a search over sv would give
    void counts(int i, const double *svi, double w, double inv_s, double off, int &le, int &lt) const {
        const int r = rs[i], step = 1 << (8 - r), nblk = 1 << r;
        const double x = (w * inv_s - (levels[(size_t)i * 256] + off)) / step + 1.0;
        int j = x > 0.0 ? (x < nblk ? (int)x : nblk) : 0;   // NaN -> 0
        while (j < nblk && svi[j * step] <= w) ++j;
        while (j > 0 && svi[(j - 1) * step] > w) --j;
        int k = j;
        while (k > 0 && svi[(k - 1) * step] >= w) --k;
        le = j * step;
        lt = k * step;
    }

    // sv[i][q] = s * (v_i(q) + off) for one scale s >= 0 and level offset
    // off = 128 - z (0 for the symmetric levels; v_i(q) + off is exact, so
    // each product is the level's one rounding), non-decreasing in q
    void products(double s, double off, double *sv) const {
        for (int i = 0; i < nr * 256; ++i) sv[i] = s * (levels[(size_t)i] + off);
    }

    // the objective at code q, its terms summed in the order of the widths
    double cost(double w, const double *sv, int q) const {
        double c = 0.0;
        for (int i = 0; i < nr; ++i) {
            const double d = w - sv[i * 256 + q];
            c += lams[i] * d * d;
        }
        return c;
    }

    // The first q in 0..255 of least cost(w, sv, q), found exactly without
    // evaluating every code.  Each term lambda (w - s v_i(q))^2, rounded, is
    // non-increasing in q up to A_i, the last code with s v_i(q) <= w, and
    // non-decreasing from B_i, the first code with s v_i(q) >= w (rounding is
    // monotone and keeps the sign of w - s v_i(q)); so is their rounded sum
    // (addition is monotone in each operand).  Hence the cost cannot fall
    // below its value on [min(a, b), max(a, b)], a = min A_i, b = max B_i,
    // outside it, and the first minimum lies inside it or, when the cost is
    // flat at the window's left end, further left by equal steps.
    // inv_s = 1 / s when s > 0 and off (as in products) are hints for
    // locating A_i and B_i; inv_s = 0 searches instead.
    int best_code(double w, const double *sv, double inv_s, double off) const {
        int a = 256, b = -1;
        for (int i = 0; i < nr; ++i) {
            if (!(lams[i] > 0.0)) continue;          // a zero term is flat everywhere
            const double *p = sv + i * 256;
            int le, lt;
            if (inv_s > 0.0) {
                counts(i, p, w, inv_s, off, le, lt);
            } else {
                le = (int)(std::upper_bound(p, p + 256, w) - p);
                lt = (int)(std::lower_bound(p, p + 256, w) - p);
            }
            a = std::min(a, le - 1);
            b = std::max(b, lt);
        }
        const int q0 = std::max(0, std::min(a, b)), q1 = std::min(255, std::max(a, b));
        int best = q0;
        double bc = cost(w, sv, q0);
        for (int q = q0 + 1; q <= q1; ++q) {
            const double c = cost(w, sv, q);
            if (c < bc) {
                best = q;
                bc = c;
            }
        }
        if (best == q0) {
            while (best > 0) {
                const double c = cost(w, sv, best - 1);
                if (!(c <= bc)) break;
                bc = c;
                --best;
            }
        }
        return best;
    }
};

// sum a[i] b[i], four interleaved partial sums
inline double dot(const double *a, const double *b, int64_t m) {
    double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
    int64_t i = 0;
    for (; i + 4 <= m; i += 4) {
        s0 += a[i] * b[i];
        s1 += a[i + 1] * b[i + 1];
        s2 += a[i + 2] * b[i + 2];
        s3 += a[i + 3] * b[i + 3];
    }
    for (; i < m; ++i) s0 += a[i] * b[i];
    return (s0 + s1) + (s2 + s3);
}

// f(i) for i in [i0, i1), spread over up to nt threads by a shared counter
// (rows of unequal cost balance themselves); an exception in any thread is
// rethrown here after all have joined
template <class F>
void parallel_rows(int64_t i0, int64_t i1, int nt, F &&f) {
    if (i1 <= i0) return;
    std::atomic<int64_t> next{i0};
    std::exception_ptr err;
    std::mutex mu;
    auto work = [&]() {
        try {
            for (int64_t i; (i = next.fetch_add(1)) < i1;) f(i);
        } catch (...) {                        // first failure wins; the others stop taking rows
            std::lock_guard<std::mutex> g(mu);
            if (!err) err = std::current_exception();
            next.store(i1);
        }
    };
    const int m = (int)std::min<int64_t>(nt, i1 - i0);
    std::vector<std::thread> pool;
    pool.reserve((size_t)m);
    for (int t = 1; t < m; ++t) {
        try {
            pool.emplace_back(work);
        } catch (...) {                        // fewer threads: the rest of the rows run here
            break;
        }
    }
    work();
    for (auto &th : pool) th.join();
    if (err) std::rethrow_exception(err);
}

// T[r][c] += sum_{p0 <= p < p1} A[r][p] B[p][c] for r < 4, c < 8 (rows of
// A, B and T at strides lda, ldb, ldt): the inner block of the triangular
// inverse
inline void gemm4x8(const double *A, int64_t lda, const double *B, int64_t ldb, int64_t p0, int64_t p1,
                    double *T, int64_t ldt) {
    double acc[4][8];
    for (int r = 0; r < 4; ++r)
        for (int c = 0; c < 8; ++c) acc[r][c] = T[r * ldt + c];
    for (int64_t p = p0; p < p1; ++p) {
        const double *bp = B + p * ldb;
        for (int r = 0; r < 4; ++r) {
            const double a = A[r * lda + p];
            for (int c = 0; c < 8; ++c) acc[r][c] += a * bp[c];
        }
    }
    for (int r = 0; r < 4; ++r)
        for (int c = 0; c < 8; ++c) T[r * ldt + c] = acc[r][c];
}

// The same kernels with AVX2 and FMA (and the tile product with AVX-512),
// used by the prepare step when the CPU has them (rounding differs from the
// portable loops within the prepare step's own error; the code search never
// uses them).  MQ_PORTABLE_HOST=1 in the environment selects the portable
// loops, MQ_NO_AVX512=1 stops at AVX2.
enum class Simd { portable, avx2, avx512 };

bool env_set(const char *name) {
    const char *v = getenv(name);
    return v && v[0] == '1';
}

Simd host_simd() {
    static const Simd s = [] {
        __builtin_cpu_init();
        if (env_set("MQ_PORTABLE_HOST") || !__builtin_cpu_supports("avx2") || !__builtin_cpu_supports("fma"))
            return Simd::portable;
        if (!env_set("MQ_NO_AVX512") && __builtin_cpu_supports("avx512f")) return Simd::avx512;
        return Simd::avx2;
    }();
    return s;
}

bool have_avx2_fma() { return host_simd() != Simd::portable; }

// rows of A (and of T) per call of the tile product: 8 with AVX-512, else 4
inline int64_t tile_rows(Simd s) { return s == Simd::avx512 ? 8 : 4; }

__attribute__((target("avx2,fma"))) inline double hsum(__m256d v) {
    alignas(32) double t[4];
    _mm256_store_pd(t, v);
    return (t[0] + t[1]) + (t[2] + t[3]);
}

__attribute__((target("avx2,fma"))) double dot_avx2(const double *a, const double *b, int64_t m) {
    __m256d s0 = _mm256_setzero_pd(), s1 = _mm256_setzero_pd();
    int64_t i = 0;
    for (; i + 8 <= m; i += 8) {
        s0 = _mm256_fmadd_pd(_mm256_loadu_pd(a + i), _mm256_loadu_pd(b + i), s0);
        s1 = _mm256_fmadd_pd(_mm256_loadu_pd(a + i + 4), _mm256_loadu_pd(b + i + 4), s1);
    }
    for (; i + 4 <= m; i += 4) s0 = _mm256_fmadd_pd(_mm256_loadu_pd(a + i), _mm256_loadu_pd(b + i), s0);
    double r = hsum(_mm256_add_pd(s0, s1));
    for (; i < m; ++i) r += a[i] * b[i];
    return r;
}

__attribute__((target("avx2,fma"))) void gemm4x8_avx2(const double *A, int64_t lda, const double *B,
                                                      int64_t ldb, int64_t p0, int64_t p1, double *T,
                                                      int64_t ldt) {
    const double *a0 = A, *a1 = A + lda, *a2 = A + 2 * lda, *a3 = A + 3 * lda;
    __m256d t00 = _mm256_loadu_pd(T), t01 = _mm256_loadu_pd(T + 4);
    __m256d t10 = _mm256_loadu_pd(T + ldt), t11 = _mm256_loadu_pd(T + ldt + 4);
    __m256d t20 = _mm256_loadu_pd(T + 2 * ldt), t21 = _mm256_loadu_pd(T + 2 * ldt + 4);
    __m256d t30 = _mm256_loadu_pd(T + 3 * ldt), t31 = _mm256_loadu_pd(T + 3 * ldt + 4);
    for (int64_t p = p0; p < p1; ++p) {
        const double *bp = B + p * ldb;
        const __m256d b0 = _mm256_loadu_pd(bp), b1 = _mm256_loadu_pd(bp + 4);
        __m256d a = _mm256_broadcast_sd(a0 + p);
        t00 = _mm256_fmadd_pd(a, b0, t00);
        t01 = _mm256_fmadd_pd(a, b1, t01);
        a = _mm256_broadcast_sd(a1 + p);
        t10 = _mm256_fmadd_pd(a, b0, t10);
        t11 = _mm256_fmadd_pd(a, b1, t11);
        a = _mm256_broadcast_sd(a2 + p);
        t20 = _mm256_fmadd_pd(a, b0, t20);
        t21 = _mm256_fmadd_pd(a, b1, t21);
        a = _mm256_broadcast_sd(a3 + p);
        t30 = _mm256_fmadd_pd(a, b0, t30);
        t31 = _mm256_fmadd_pd(a, b1, t31);
    }
    _mm256_storeu_pd(T, t00);
    _mm256_storeu_pd(T + 4, t01);
    _mm256_storeu_pd(T + ldt, t10);
    _mm256_storeu_pd(T + ldt + 4, t11);
    _mm256_storeu_pd(T + 2 * ldt, t20);
    _mm256_storeu_pd(T + 2 * ldt + 4, t21);
    _mm256_storeu_pd(T + 3 * ldt, t30);
    _mm256_storeu_pd(T + 3 * ldt + 4, t31);
}

__attribute__((target("avx512f"))) void gemm8x8_avx512(const double *A, int64_t lda, const double *B,
                                                       int64_t ldb, int64_t p0, int64_t p1, double *T,
                                                       int64_t ldt) {
    __m512d t0 = _mm512_loadu_pd(T), t1 = _mm512_loadu_pd(T + ldt), t2 = _mm512_loadu_pd(T + 2 * ldt),
            t3 = _mm512_loadu_pd(T + 3 * ldt), t4 = _mm512_loadu_pd(T + 4 * ldt),
            t5 = _mm512_loadu_pd(T + 5 * ldt), t6 = _mm512_loadu_pd(T + 6 * ldt),
            t7 = _mm512_loadu_pd(T + 7 * ldt);
    for (int64_t p = p0; p < p1; ++p) {
        const __m512d b = _mm512_loadu_pd(B + p * ldb);
        t0 = _mm512_fmadd_pd(_mm512_set1_pd(A[p]), b, t0);
        t1 = _mm512_fmadd_pd(_mm512_set1_pd(A[lda + p]), b, t1);
        t2 = _mm512_fmadd_pd(_mm512_set1_pd(A[2 * lda + p]), b, t2);
        t3 = _mm512_fmadd_pd(_mm512_set1_pd(A[3 * lda + p]), b, t3);
        t4 = _mm512_fmadd_pd(_mm512_set1_pd(A[4 * lda + p]), b, t4);
        t5 = _mm512_fmadd_pd(_mm512_set1_pd(A[5 * lda + p]), b, t5);
        t6 = _mm512_fmadd_pd(_mm512_set1_pd(A[6 * lda + p]), b, t6);
        t7 = _mm512_fmadd_pd(_mm512_set1_pd(A[7 * lda + p]), b, t7);
    }
    _mm512_storeu_pd(T, t0);
    _mm512_storeu_pd(T + ldt, t1);
    _mm512_storeu_pd(T + 2 * ldt, t2);
    _mm512_storeu_pd(T + 3 * ldt, t3);
    _mm512_storeu_pd(T + 4 * ldt, t4);
    _mm512_storeu_pd(T + 5 * ldt, t5);
    _mm512_storeu_pd(T + 6 * ldt, t6);
    _mm512_storeu_pd(T + 7 * ldt, t7);
}

// T[r][c] += sum_{p0 <= p < p1} A[r][p] B[p][c], r < tile_rows(s), c < 8
inline void gemm_tile(Simd s, const double *A, int64_t lda, const double *B, int64_t ldb, int64_t p0,
                      int64_t p1, double *T, int64_t ldt) {
    if (s == Simd::avx512) gemm8x8_avx512(A, lda, B, ldb, p0, p1, T, ldt);
    else if (s == Simd::avx2) gemm4x8_avx2(A, lda, B, ldb, p0, p1, T, ldt);
    else gemm4x8(A, lda, B, ldb, p0, p1, T, ldt);
}

// M = L^-1 (both n x n row-major, lower triangular; M zero on entry above
// the diagonal and written everywhere on and below it), by blocks of kRB
// rows, each after the ones above it:
//   M[I, J] = -L[I, I]^-1 (L[I, 0:i0] M[0:i0, J])  for the columns J < i0,
//   M[I, I] = L[I, I]^-1,
// the product taken kCW columns per task and kPB terms at a time so that
// its operands stay in cache.
void invert_lower(const double *L, int64_t n, double *M, int nt, Simd simd) {
    constexpr int64_t kRB = 128, kCW = 64, kPB = 256;
    const int64_t R = tile_rows(simd);
    for (int64_t i0 = 0; i0 < n; i0 += kRB) {
        const int64_t b = std::min(kRB, n - i0);
        parallel_rows(0, (i0 + kCW - 1) / kCW, nt, [&](int64_t task) {
            const int64_t j0 = task * kCW, w = std::min(kCW, i0 - j0);
            std::vector<double> T((size_t)(kRB * kCW), 0.0), Bp((size_t)(kPB * kCW), 0.0);
            // T = L[I, j0:i0] M[j0:i0, j0:j0+w]  (M[p][j] = 0 for p < j), each
            // kPB x kCW block of M first copied to a contiguous buffer
            for (int64_t pp = j0; pp < i0; pp += kPB) {
                const int64_t pe = std::min(i0, pp + kPB);
                for (int64_t p = pp; p < pe; ++p)
                    std::copy(M + p * n + j0, M + p * n + j0 + w, Bp.data() + (p - pp) * kCW);
                const double *B = Bp.data() - pp * kCW;   // row p of the block at B + p * kCW
                for (int64_t r0 = 0; r0 < b; r0 += R) {
                    const double *A = L + (i0 + r0) * n;
                    for (int64_t c0 = 0; c0 < w; c0 += 8) {
                        double *Tt = T.data() + r0 * kCW + c0;
                        if (r0 + R <= b && c0 + 8 <= w) {
                            gemm_tile(simd, A, n, B + c0, kCW, pp, pe, Tt, kCW);
                        } else {
                            for (int64_t r = 0; r < std::min<int64_t>(R, b - r0); ++r)
                                for (int64_t c = 0; c < std::min<int64_t>(8, w - c0); ++c) {
                                    double v = Tt[r * kCW + c];
                                    for (int64_t p = pp; p < pe; ++p) v += A[r * n + p] * B[p * kCW + c0 + c];
                                    Tt[r * kCW + c] = v;
                                }
                        }
                    }
                }
            }
            // M[I, j0:j0+w] = -L[I, I]^-1 T, down the block's rows
            double v[kCW];
            for (int64_t r = 0; r < b; ++r) {
                const double *li = L + (i0 + r) * n + i0;
                for (int64_t c = 0; c < w; ++c) v[c] = -T[(size_t)(r * kCW + c)];
                for (int64_t q = 0; q < r; ++q) {
                    const double lq = li[q];
                    const double *mq = M + (i0 + q) * n + j0;
                    for (int64_t c = 0; c < w; ++c) v[c] -= lq * mq[c];
                }
                double *mi = M + (i0 + r) * n + j0;
                for (int64_t c = 0; c < w; ++c) mi[c] = v[c] / li[r];
            }
        });
        // M[I, I] = L[I, I]^-1
        for (int64_t c = 0; c < b; ++c) {
            M[(i0 + c) * n + i0 + c] = 1.0 / L[(i0 + c) * n + i0 + c];
            for (int64_t r = c + 1; r < b; ++r) {
                double v = 0.0;
                for (int64_t q = c; q < r; ++q) v += L[(i0 + r) * n + i0 + q] * M[(i0 + q) * n + i0 + c];
                M[(i0 + r) * n + i0 + c] = -v / L[(i0 + r) * n + i0 + r];
            }
        }
    }
}

// Rows n0..n1-1 (at most kRowBlock), column by column together: each tile of
// U that the feedback reads then serves a block of rows rather than one row.
// Every row still takes exactly the operations, in the order, of quantizing
// it alone.
constexpr int64_t kRowBlock = 16;

// x (fp32) rounded to the nearest fp16 value, ties to even, as a double
// (infinite past the largest finite fp16, 65504): IEEE binary16 has 11
// significant bits down to 2^-14 and a fixed step of 2^-24 below
double fp16_value(float x) {
    const double v = x;
    if (!std::isfinite(v)) return v;
    const double a = fabs(v);
    int e;
    frexp(a, &e);                                  // a = m 2^e, 0.5 <= m < 1
    const double step = a < 0x1p-14 ? 0x1p-24 : ldexp(1.0, e - 11);
    const double r = nearbyint(v / step) * step;   // the default rounding: to nearest, ties to even
    return fabs(r) > 65504.0 ? copysign(INFINITY, v) : r;
}

// The asymmetric grid of one group for one multiplier: it spans alpha times
// the group's range [lo, hi] and is centred on it, s = alpha (hi - lo) / 255
// and z = 128 - (hi + lo) / (2 s), z as stored (fp32, then fp16); a group of
// zero range, or one whose z is no finite fp16, takes the symmetric grid
// (s = alpha max|w| / 127.5, z = 128).
void asym_grid(double lo, double hi, double alpha, double &s, double &z) {
    if (hi > lo) {
        s = alpha * (hi - lo) / 255.0;
        z = fp16_value((float)(128.0 - (hi + lo) / (2.0 * s)));
        if (std::isfinite(z)) return;
    }
    s = alpha * std::max(fabs(lo), fabs(hi)) / 127.5;
    z = 128.0;
}

// w[j] -= f u[j] for j0 <= j < j1: one rounded product and one rounded
// difference per element (no fused multiply-add), as the oracle computes it
inline void feedback(double *w, const double *u, double f, int64_t j0, int64_t j1) {
    for (int64_t j = j0; j < j1; ++j) w[j] -= f * u[j];
}

// the same, four lanes at a time (AVX2 without FMA: each lane rounds exactly
// as the scalar loop does)
__attribute__((target("avx2"))) void feedback_avx2(double *w, const double *u, double f, int64_t j0,
                                                  int64_t j1) {
    const __m256d fv = _mm256_set1_pd(f);
    int64_t j = j0;
    for (; j + 4 <= j1; j += 4)
        _mm256_storeu_pd(w + j, _mm256_sub_pd(_mm256_loadu_pd(w + j), _mm256_mul_pd(fv, _mm256_loadu_pd(u + j))));
    for (; j < j1; ++j) w[j] -= f * u[j];
}

// The feedback of one group's 128 columns (factors F[b][k], U's rows of the
// group from Ug, row stride K) to the columns j0..K-1 of nb rows of w:
// w[b][j] -= F[b][k] U[k][j] for k = 0..127 in order, each a rounded product
// and a rounded difference.  By tiles of 16 columns: the tile of U copied to
// a contiguous buffer (its 128 rows lie a row of U apart), then each row's
// 16 weights held in registers through the 128 updates.
constexpr int64_t kFbTile = 16;

inline void feedback_group(double *w, int64_t nb, int64_t K, const double *Ug, const double *F, int64_t j0) {
    for (int64_t jt = j0; jt < K; jt += kFbTile) {
        const int64_t je = std::min(K, jt + kFbTile);
        for (int64_t b = 0; b < nb; ++b) {
            double *wb = w + b * K;
            for (int64_t k = 0; k < 128; ++k) {
                const double fk = F[b * 128 + k];
                const double *u = Ug + k * K;
                for (int64_t j = jt; j < je; ++j) wb[j] -= fk * u[j];
            }
        }
    }
}

__attribute__((target("avx2"))) void feedback_group_avx2(double *w, int64_t nb, int64_t K, const double *Ug,
                                                        const double *F, int64_t j0) {
    static_assert(kFbTile == 16, "four vectors of four per row");
    alignas(32) double ut[128 * kFbTile];     // the tile of U, contiguous (one page walk per row of U)
    int64_t jt = j0;
    for (; jt + kFbTile <= K; jt += kFbTile) {
        for (int64_t k = 0; k < 128; ++k)
            for (int64_t c = 0; c < kFbTile; ++c) ut[k * kFbTile + c] = Ug[k * K + jt + c];
        int64_t b = 0;
        for (; b + 2 <= nb; b += 2) {                 // two rows: eight independent chains
            double *wa = w + b * K + jt, *wc = wa + K;
            __m256d a0 = _mm256_loadu_pd(wa), a1 = _mm256_loadu_pd(wa + 4), a2 = _mm256_loadu_pd(wa + 8),
                    a3 = _mm256_loadu_pd(wa + 12);
            __m256d c0 = _mm256_loadu_pd(wc), c1 = _mm256_loadu_pd(wc + 4), c2 = _mm256_loadu_pd(wc + 8),
                    c3 = _mm256_loadu_pd(wc + 12);
            const double *Fa = F + b * 128, *Fc = Fa + 128;
            for (int64_t k = 0; k < 128; ++k) {
                const __m256d fa = _mm256_set1_pd(Fa[k]), fc = _mm256_set1_pd(Fc[k]);
                const double *u = ut + k * kFbTile;
                const __m256d u0 = _mm256_load_pd(u), u1 = _mm256_load_pd(u + 4), u2 = _mm256_load_pd(u + 8),
                              u3 = _mm256_load_pd(u + 12);
                a0 = _mm256_sub_pd(a0, _mm256_mul_pd(fa, u0));
                c0 = _mm256_sub_pd(c0, _mm256_mul_pd(fc, u0));
                a1 = _mm256_sub_pd(a1, _mm256_mul_pd(fa, u1));
                c1 = _mm256_sub_pd(c1, _mm256_mul_pd(fc, u1));
                a2 = _mm256_sub_pd(a2, _mm256_mul_pd(fa, u2));
                c2 = _mm256_sub_pd(c2, _mm256_mul_pd(fc, u2));
                a3 = _mm256_sub_pd(a3, _mm256_mul_pd(fa, u3));
                c3 = _mm256_sub_pd(c3, _mm256_mul_pd(fc, u3));
            }
            _mm256_storeu_pd(wa, a0);
            _mm256_storeu_pd(wa + 4, a1);
            _mm256_storeu_pd(wa + 8, a2);
            _mm256_storeu_pd(wa + 12, a3);
            _mm256_storeu_pd(wc, c0);
            _mm256_storeu_pd(wc + 4, c1);
            _mm256_storeu_pd(wc + 8, c2);
            _mm256_storeu_pd(wc + 12, c3);
        }
        for (; b < nb; ++b) {
            double *wb = w + b * K + jt;
            __m256d w0 = _mm256_loadu_pd(wb), w1 = _mm256_loadu_pd(wb + 4), w2 = _mm256_loadu_pd(wb + 8),
                    w3 = _mm256_loadu_pd(wb + 12);
            const double *Fb = F + b * 128;
            for (int64_t k = 0; k < 128; ++k) {
                const __m256d fk = _mm256_set1_pd(Fb[k]);
                const double *u = ut + k * kFbTile;
                w0 = _mm256_sub_pd(w0, _mm256_mul_pd(fk, _mm256_loadu_pd(u)));
                w1 = _mm256_sub_pd(w1, _mm256_mul_pd(fk, _mm256_loadu_pd(u + 4)));
                w2 = _mm256_sub_pd(w2, _mm256_mul_pd(fk, _mm256_loadu_pd(u + 8)));
                w3 = _mm256_sub_pd(w3, _mm256_mul_pd(fk, _mm256_loadu_pd(u + 12)));
            }
            _mm256_storeu_pd(wb, w0);
            _mm256_storeu_pd(wb + 4, w1);
            _mm256_storeu_pd(wb + 8, w2);
            _mm256_storeu_pd(wb + 12, w3);
        }
    }
    if (jt < K) {
        for (int64_t b = 0; b < nb; ++b)
            for (int64_t k = 0; k < 128; ++k) {
                const double fk = F[b * 128 + k];
                const double *u = Ug + k * K;
                for (int64_t j = jt; j < K; ++j) w[b * K + j] -= fk * u[j];
            }
    }
}

void quantize_rows(const float *W, int64_t K, const double *U, const Objective &obj, const double *alphas,
                   int na, double lsum, int64_t n0, int64_t n1, uint8_t *codes, float *scales, float *zeros) {
    const bool avx = have_avx2_fma();
    const int64_t G = K / 128, nb = n1 - n0;
    const size_t nsv = (size_t)obj.nr * 256;
    std::vector<double> w((size_t)(nb * K)), sv(nsv * (size_t)nb), f((size_t)(nb * 128)), inv_s((size_t)nb),
        off((size_t)nb, 0.0);
    for (int64_t b = 0; b < nb; ++b)
        for (int64_t k = 0; k < K; ++k) w[(size_t)(b * K + k)] = (double)W[(n0 + b) * K + k];
    for (int64_t g = 0; g < G; ++g) {
        // each row's scale (and zero point), from its group's current weights
        for (int64_t b = 0; b < nb; ++b) {
            const double *wb = w.data() + b * K;
            double *svb = sv.data() + nsv * (size_t)b;
            double mx = 0.0, lo = wb[128 * g], hi = wb[128 * g];
            for (int64_t k = 128 * g; k < 128 * g + 128; ++k) {
                mx = std::max(mx, fabs(wb[k]));
                lo = std::min(lo, wb[k]);
                hi = std::max(hi, wb[k]);
            }
            const double base = mx / 127.5;
            double best_s = 0.0, best_z = 128.0, best_t = 0.0;
            for (int ia = 0; ia < na; ++ia) {
                double st = base * alphas[ia], zt = 128.0;
                if (zeros) asym_grid(lo, hi, alphas[ia], st, zt);
                const double inv = st > 0.0 ? 1.0 / st : 0.0;
                obj.products(st, 128.0 - zt, svb);
                double t = 0.0;
                for (int64_t k = 128 * g; k < 128 * g + 128; ++k) {
                    const double x = wb[k];
                    const int q = obj.best_code(x, svb, inv, 128.0 - zt);
                    for (int i = 0; i < obj.nr; ++i) {
                        const double d = x - svb[(size_t)i * 256 + q];
                        t += obj.lams[i] * d * d;
                    }
                }
                if (ia == 0 || t < best_t) {
                    best_s = st;
                    best_z = zt;
                    best_t = t;
                }
            }
            scales[(n0 + b) * G + g] = (float)best_s;
            if (zeros) zeros[(n0 + b) * G + g] = (float)best_z;
            off[(size_t)b] = 128.0 - best_z;
            obj.products(best_s, off[(size_t)b], svb);
            inv_s[(size_t)b] = best_s > 0.0 ? 1.0 / best_s : 0.0;
        }
        // the group's columns in order; each column's feedback reaches the
        // rest of the group at once and the later groups' columns after the
        // group (below): every weight still takes the updates of all earlier
        // columns one at a time in column order, before anything reads it
        const int64_t ge = 128 * g + 128;
        for (int64_t k = 128 * g; k < ge; ++k) {
            for (int64_t b = 0; b < nb; ++b) {
                const double *svb = sv.data() + nsv * (size_t)b;
                const double x = w[(size_t)(b * K + k)];
                const int q = obj.best_code(x, svb, inv_s[(size_t)b], off[(size_t)b]);
                codes[(n0 + b) * K + k] = (uint8_t)q;
                double e = 0.0;
                for (int i = 0; i < obj.nr; ++i) e += obj.lams[i] * (x - svb[(size_t)i * 256 + q]);
                e /= lsum;
                f[(size_t)(b * 128 + (k - 128 * g))] = e / U[k * K + k];
            }
            const double *urow = U + k * K;
            for (int64_t b = 0; b < nb; ++b) {
                const double fb = f[(size_t)(b * 128 + (k - 128 * g))];
                if (avx) feedback_avx2(w.data() + b * K, urow, fb, k + 1, ge);
                else feedback(w.data() + b * K, urow, fb, k + 1, ge);
            }
        }
        if (ge < K) {
            if (avx) feedback_group_avx2(w.data(), nb, K, U + 128 * g * K, f.data(), ge);
            else feedback_group(w.data(), nb, K, U + 128 * g * K, f.data(), ge);
        }
    }
}

}  // namespace

extern "C" mq_status mq_matgptq_prepare(const double *H, int64_t K, double damp, double *U_out) {
    return host_guarded([&]() -> mq_status {
        if (!H || !U_out) return fail(MQ_ERR_INVALID_ARG, "NULL argument to mq_matgptq_prepare");
        if (K < 1 || K > 65536) return fail(MQ_ERR_INVALID_ARG, "need 1 <= K <= 65536");
        if (!(damp >= 0.0)) return fail(MQ_ERR_INVALID_ARG, "damp must be >= 0");
        // A = H + damp * mean(diag H) * I and J the reversal (J A J reverses
        // rows and columns).  With J A J = L L^T (lower Cholesky), A = R R^T for
        // the upper R = J L J, so A^-1 = R^-T R^-1 and U = R^-1 = J L^-1 J is the
        // upper factor with U^T U = A^-1 (unique for a positive diagonal).
        const int64_t n = K;
        double mean = 0.0;
        for (int64_t i = 0; i < n; ++i) mean += H[i * n + i];
        mean /= (double)K;
        const double add = damp * mean;
        auto P = [&](int64_t i, int64_t j) {
            return H[(n - 1 - i) * n + (n - 1 - j)] + (i == j ? add : 0.0);
        };
        const int nt = std::max(1, std::min<int>(64, (int)std::thread::hardware_concurrency()));
        // L starts as the lower triangle of J A J and is factorised in place;
        // its upper triangle is never read, so the buffer is not initialised
        // (its pages are first touched by the threads that copy the rows)
        std::unique_ptr<double[]> L(new double[(size_t)n * n]);
        double *Lp = L.get();
        parallel_rows(0, n, nt, [&](int64_t i) {
            for (int64_t j = 0; j <= i; ++j) Lp[i * n + j] = P(i, j);
        });
        const Simd simd = host_simd();
        const bool avx = simd != Simd::portable;
        const int64_t R = tile_rows(simd);
        auto dotv = [avx](const double *a, const double *b, int64_t m) {
            return avx ? dot_avx2(a, b, m) : dot(a, b, m);
        };
        // Right-looking blocked Cholesky, kNB columns per panel: factor the
        // panel's diagonal block, solve the rows below it against that block,
        // then subtract the panel's product from the trailing lower triangle
        // (4 x 8 tiles by the same kernel as the inverse, against the panel
        // transposed and negated, kGR rows per task so that each 8-column tile
        // of it is reused from cache).
        constexpr int64_t kNB = 128, kGR = 32;
        std::vector<double> Pt;
        for (int64_t j0 = 0; j0 < n; j0 += kNB) {
            const int64_t j1 = std::min(n, j0 + kNB), nb = j1 - j0;
            for (int64_t i = j0; i < j1; ++i)
                for (int64_t j = j0; j <= i; ++j) {
                    const double v = Lp[i * n + j] - dotv(Lp + i * n + j0, Lp + j * n + j0, j - j0);
                    if (i == j) {
                        if (!(v > 0.0) || !isfinite(v))
                            return fail(MQ_ERR_UNSUPPORTED, "the damped Hessian is not positive definite");
                        Lp[i * n + i] = sqrt(v);
                    } else {
                        Lp[i * n + j] = v / Lp[j * n + j];
                    }
                }
            const int64_t m = n - j1;
            if (m == 0) break;
            parallel_rows(j1, n, nt, [&](int64_t i) {
                double *li = Lp + i * n;
                for (int64_t j = j0; j < j1; ++j)
                    li[j] = (li[j] - dotv(li + j0, Lp + j * n + j0, j - j0)) / Lp[j * n + j];
            });
            // Pt: the panel's rows below j1, negated and transposed, in tiles of 8
            // columns each contiguous (tile t, term p, column c at (t nb + p) 8 + c;
            // the last tile padded with zeros)
            const int64_t m8 = (m + 7) / 8 * 8;
            Pt.resize((size_t)(nb * m8));
            parallel_rows(0, m8, nt, [&](int64_t jj) {
                double *dst = Pt.data() + (jj / 8) * nb * 8 + jj % 8;
                if (jj >= m) {
                    for (int64_t p = 0; p < nb; ++p) dst[p * 8] = 0.0;
                    return;
                }
                const double *lj = Lp + (j1 + jj) * n + j0;
                for (int64_t p = 0; p < nb; ++p) dst[p * 8] = -lj[p];
            });
            const int64_t ng = (m + kGR - 1) / kGR;
            parallel_rows(0, ng, nt, [&](int64_t t) {
                const int64_t g0 = j1 + (ng - 1 - t) * kGR;          // largest groups first
                const int64_t g1 = std::min(n, g0 + kGR);
                // chunks of kCC columns (their panel tiles stay in cache), each
                // row tile of the group running along the chunk
                constexpr int64_t kCC = 64;
                for (int64_t jc = j1; jc < g1; jc += kCC)
                for (int64_t i = g0; i < g1; i += R) {
                    for (int64_t jt = jc; jt < std::min(g1, jc + kCC); jt += 8) {
                        if (jt > i + R - 1) break;                    // the rest lies above the diagonal
                        const double *B = Pt.data() + (jt - j1) * nb;    // tile (jt - j1) / 8
                        if (i + R <= g1 && jt + 8 <= n) {
                            // writes of the tile's entries above the diagonal
                            // land in L's unread upper triangle
                            gemm_tile(simd, Lp + i * n + j0, n, B, 8, 0, nb, Lp + i * n + jt, n);
                        } else {
                            for (int64_t r = i; r < std::min(i + R, g1); ++r)
                                for (int64_t c = jt; c < std::min(jt + 8, r + 1); ++c) {
                                    double v = 0.0;
                                    for (int64_t p = 0; p < nb; ++p) v += Lp[r * n + j0 + p] * B[p * 8 + (c - jt)];
                                    Lp[r * n + c] += v;
                                }
                        }
                    }
                }
            });
        }
        // M = L^-1 into U_out, then U = J M J: the 180-degree rotation of the
        // matrix, i.e. the flat array reversed
        parallel_rows(0, n, nt, [&](int64_t i) { std::fill(U_out + i * n, U_out + (i + 1) * n, 0.0); });
        invert_lower(Lp, n, U_out, nt, simd);
        std::reverse(U_out, U_out + (size_t)n * n);
        for (int64_t i = 0; i < n; ++i)
            if (!(U_out[i * n + i] > 0.0) || !isfinite(U_out[i * n + i])) return fail(MQ_ERR_UNSUPPORTED, "the damped Hessian is too ill-conditioned to invert");
        return MQ_OK;
    });
}

static mq_status quantize_common(const float *W, int64_t N, int64_t K, const double *U, const int32_t *rs,
                                 const double *lambdas, int n_r, const double *alphas, int n_alpha,
                                 int threads, uint8_t *codes_out, float *scales_out, float *zeros_out) {
    return host_guarded([&]() -> mq_status {
        if (!W || !U || !rs || !lambdas || !alphas || !codes_out || !scales_out)
            return fail(MQ_ERR_INVALID_ARG, "NULL argument to mq_matgptq_quantize");
        if (N < 1 || K < kGroup || K % kGroup) return fail(MQ_ERR_INVALID_ARG, "need N >= 1 and K a positive multiple of 128");
        if (n_r < 1 || n_r > 8 || n_alpha < 1) return fail(MQ_ERR_INVALID_ARG, "need 1 <= n_r <= 8 and n_alpha >= 1");
        double lsum = 0.0;
        for (int i = 0; i < n_r; ++i) {
            if (rs[i] < 1 || rs[i] > 8) return fail(MQ_ERR_INVALID_ARG, "bit widths must be in 1..8");
            if (!(lambdas[i] >= 0.0) || !isfinite(lambdas[i])) return fail(MQ_ERR_INVALID_ARG, "lambdas must be finite and >= 0");
            lsum += lambdas[i];
        }
        if (!(lsum > 0.0)) return fail(MQ_ERR_INVALID_ARG, "the lambdas must not all be zero");
        for (int i = 0; i < n_alpha; ++i)
            if (!(alphas[i] > 0.0) || !isfinite(alphas[i])) return fail(MQ_ERR_INVALID_ARG, "alphas must be finite and > 0");
        for (int64_t k = 0; k < K; ++k)
            if (!(U[k * K + k] != 0.0)) return fail(MQ_ERR_INVALID_ARG, "U has a zero on its diagonal");
        for (int64_t i = 0; i < N * K; ++i)
            if (!isfinite(W[i])) return fail(MQ_ERR_INVALID_ARG, "W holds a non-finite value");
        const Objective obj(rs, lambdas, n_r);
        const int nt = threads > 0 ? threads : (int)std::max(1u, std::thread::hardware_concurrency());
        const int64_t nblocks = (N + kRowBlock - 1) / kRowBlock;
        parallel_rows(0, nblocks, nt, [&](int64_t blk) {
            quantize_rows(W, K, U, obj, alphas, n_alpha, lsum, blk * kRowBlock,
                          std::min<int64_t>(N, (blk + 1) * kRowBlock), codes_out, scales_out, zeros_out);
        });
        return MQ_OK;
    });
}

extern "C" mq_status mq_matgptq_quantize(const float *W, int64_t N, int64_t K, const double *U,
                                         const int32_t *rs, const double *lambdas, int n_r,
                                         const double *alphas, int n_alpha, int threads,
                                         uint8_t *codes_out, float *scales_out) {
    return quantize_common(W, N, K, U, rs, lambdas, n_r, alphas, n_alpha, threads, codes_out, scales_out,
                           nullptr);
}

extern "C" mq_status mq_matgptq_quantize_asym(const float *W, int64_t N, int64_t K, const double *U,
                                              const int32_t *rs, const double *lambdas, int n_r,
                                              const double *alphas, int n_alpha, int threads,
                                              uint8_t *codes_out, float *scales_out, float *zeros_out) {
    if (!zeros_out) return fail(MQ_ERR_INVALID_ARG, "NULL zeros_out");
    return quantize_common(W, N, K, U, rs, lambdas, n_r, alphas, n_alpha, threads, codes_out, scales_out,
                           zeros_out);
}
