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
// Rows are independent given U, so threads take blocks of rows; every
// operation is fp64 in a fixed order, the same whatever the thread count.
#include <immintrin.h>
#include <math.h>
#include <stdlib.h>

#include <algorithm>
#include <atomic>
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

    // sv[i][q] = s * v_i(q) for one scale s (non-decreasing in q for s >= 0)
    void products(double s, double *sv) const {
        for (int i = 0; i < nr * 256; ++i) sv[i] = s * levels[(size_t)i];
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
    int best_code(double w, const double *sv) const {
        int a = 256, b = -1;
        for (int i = 0; i < nr; ++i) {
            if (!(lams[i] > 0.0)) continue;          // a zero term is flat everywhere
            const double *p = sv + i * 256;
            a = std::min(a, (int)(std::upper_bound(p, p + 256, w) - p) - 1);
            b = std::max(b, (int)(std::lower_bound(p, p + 256, w) - p));
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

// out[r] = sum_p a[r * lda + p] b[p] for r < 4, p < m: four rows against one
inline void dot4(const double *a, int64_t lda, const double *b, int64_t m, double *out) {
    const double *a0 = a, *a1 = a + lda, *a2 = a + 2 * lda, *a3 = a + 3 * lda;
    double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0, t0 = 0.0, t1 = 0.0, t2 = 0.0, t3 = 0.0;
    int64_t p = 0;
    for (; p + 2 <= m; p += 2) {
        const double b0 = b[p], b1 = b[p + 1];
        s0 += a0[p] * b0;
        t0 += a0[p + 1] * b1;
        s1 += a1[p] * b0;
        t1 += a1[p + 1] * b1;
        s2 += a2[p] * b0;
        t2 += a2[p + 1] * b1;
        s3 += a3[p] * b0;
        t3 += a3[p + 1] * b1;
    }
    if (p < m) {
        s0 += a0[p] * b[p];
        s1 += a1[p] * b[p];
        s2 += a2[p] * b[p];
        s3 += a3[p] * b[p];
    }
    out[0] = s0 + t0;
    out[1] = s1 + t1;
    out[2] = s2 + t2;
    out[3] = s3 + t3;
}

// f(i) for i in [i0, i1), spread over up to nt threads by a shared counter
// (rows of unequal cost balance themselves)
template <class F>
void parallel_rows(int64_t i0, int64_t i1, int nt, F &&f) {
    if (i1 <= i0) return;
    std::atomic<int64_t> next{i0};
    auto work = [&]() {
        for (int64_t i; (i = next.fetch_add(1)) < i1;) f(i);
    };
    const int m = (int)std::min<int64_t>(nt, i1 - i0);
    std::vector<std::thread> pool;
    for (int t = 1; t < m; ++t) pool.emplace_back(work);
    work();
    for (auto &th : pool) th.join();
}

// acc[4 r + t] = sum_{p0 <= p < p1} L[i0 + r][p] x[p - p0][t], r, t < 4 (x
// holds rows of four)
inline void acc4x4(const double *L, int64_t n, int64_t i0, int64_t p0, int64_t p1, const double *x,
                   double *acc) {
    for (int r = 0; r < 16; ++r) acc[r] = 0.0;
    for (int64_t p = p0; p < p1; ++p) {
        const double *xp = x + (p - p0) * 4;
        for (int r = 0; r < 4; ++r) {
            const double l = L[(i0 + r) * n + p];
            for (int t = 0; t < 4; ++t) acc[4 * r + t] += l * xp[t];
        }
    }
}

// The same three kernels with AVX2 and FMA, used by the prepare step when
// the CPU has both (rounding differs from the portable loops within the
// prepare step's own error; the code search never uses them).
// (MQ_PORTABLE_HOST=1 in the environment selects the portable loops.)
bool have_avx2_fma() {
    static const bool ok = (__builtin_cpu_init(), __builtin_cpu_supports("avx2")) && __builtin_cpu_supports("fma") &&
                           !(getenv("MQ_PORTABLE_HOST") && getenv("MQ_PORTABLE_HOST")[0] == '1');
    return ok;
}

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

__attribute__((target("avx2,fma"))) void dot4_avx2(const double *a, int64_t lda, const double *b, int64_t m,
                                                   double *out) {
    const double *a0 = a, *a1 = a + lda, *a2 = a + 2 * lda, *a3 = a + 3 * lda;
    __m256d s0 = _mm256_setzero_pd(), s1 = _mm256_setzero_pd(), s2 = _mm256_setzero_pd(),
            s3 = _mm256_setzero_pd();
    int64_t p = 0;
    for (; p + 4 <= m; p += 4) {
        const __m256d bv = _mm256_loadu_pd(b + p);
        s0 = _mm256_fmadd_pd(_mm256_loadu_pd(a0 + p), bv, s0);
        s1 = _mm256_fmadd_pd(_mm256_loadu_pd(a1 + p), bv, s1);
        s2 = _mm256_fmadd_pd(_mm256_loadu_pd(a2 + p), bv, s2);
        s3 = _mm256_fmadd_pd(_mm256_loadu_pd(a3 + p), bv, s3);
    }
    out[0] = hsum(s0);
    out[1] = hsum(s1);
    out[2] = hsum(s2);
    out[3] = hsum(s3);
    for (; p < m; ++p) {
        out[0] += a0[p] * b[p];
        out[1] += a1[p] * b[p];
        out[2] += a2[p] * b[p];
        out[3] += a3[p] * b[p];
    }
}

__attribute__((target("avx2,fma"))) void acc4x4_avx2(const double *L, int64_t n, int64_t i0, int64_t p0,
                                                     int64_t p1, const double *x, double *acc) {
    const double *l0 = L + i0 * n, *l1 = l0 + n, *l2 = l1 + n, *l3 = l2 + n;
    __m256d a0 = _mm256_setzero_pd(), a1 = _mm256_setzero_pd(), a2 = _mm256_setzero_pd(),
            a3 = _mm256_setzero_pd();
    for (int64_t p = p0; p < p1; ++p) {
        const __m256d xv = _mm256_loadu_pd(x + (p - p0) * 4);
        a0 = _mm256_fmadd_pd(_mm256_broadcast_sd(l0 + p), xv, a0);
        a1 = _mm256_fmadd_pd(_mm256_broadcast_sd(l1 + p), xv, a1);
        a2 = _mm256_fmadd_pd(_mm256_broadcast_sd(l2 + p), xv, a2);
        a3 = _mm256_fmadd_pd(_mm256_broadcast_sd(l3 + p), xv, a3);
    }
    _mm256_storeu_pd(acc, a0);
    _mm256_storeu_pd(acc + 4, a1);
    _mm256_storeu_pd(acc + 8, a2);
    _mm256_storeu_pd(acc + 12, a3);
}

// Rows n0..n1-1 (at most kRowBlock), column by column together: each row of
// U is then read once per block of rows rather than once per row (the
// feedback streams U's upper triangle for every column).  Every row still
// takes exactly the operations, in the order, of quantizing it alone.
constexpr int64_t kRowBlock = 16;

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

void quantize_rows(const float *W, int64_t K, const double *U, const Objective &obj, const double *alphas,
                   int na, double lsum, int64_t n0, int64_t n1, uint8_t *codes, float *scales) {
    const bool avx = have_avx2_fma();
    const int64_t G = K / 128, nb = n1 - n0;
    const size_t nsv = (size_t)obj.nr * 256;
    std::vector<double> w((size_t)(nb * K)), sv(nsv * (size_t)nb), f((size_t)nb);
    for (int64_t b = 0; b < nb; ++b)
        for (int64_t k = 0; k < K; ++k) w[(size_t)(b * K + k)] = (double)W[(n0 + b) * K + k];
    for (int64_t g = 0; g < G; ++g) {
        // each row's scale, from its group's current weights
        for (int64_t b = 0; b < nb; ++b) {
            const double *wb = w.data() + b * K;
            double *svb = sv.data() + nsv * (size_t)b;
            double mx = 0.0;
            for (int64_t k = 128 * g; k < 128 * g + 128; ++k) mx = std::max(mx, fabs(wb[k]));
            const double base = mx / 127.5;
            double best_a = 0.0, best_t = 0.0;
            for (int ia = 0; ia < na; ++ia) {
                obj.products(base * alphas[ia], svb);
                double t = 0.0;
                for (int64_t k = 128 * g; k < 128 * g + 128; ++k) {
                    const double x = wb[k];
                    const int q = obj.best_code(x, svb);
                    for (int i = 0; i < obj.nr; ++i) {
                        const double d = x - svb[(size_t)i * 256 + q];
                        t += obj.lams[i] * d * d;
                    }
                }
                if (ia == 0 || t < best_t) {
                    best_a = alphas[ia];
                    best_t = t;
                }
            }
            const double s = base * best_a;
            scales[(n0 + b) * G + g] = (float)s;
            obj.products(s, svb);
        }
        for (int64_t k = 128 * g; k < 128 * g + 128; ++k) {
            for (int64_t b = 0; b < nb; ++b) {
                const double *svb = sv.data() + nsv * (size_t)b;
                const double x = w[(size_t)(b * K + k)];
                const int q = obj.best_code(x, svb);
                codes[(n0 + b) * K + k] = (uint8_t)q;
                double e = 0.0;
                for (int i = 0; i < obj.nr; ++i) e += obj.lams[i] * (x - svb[(size_t)i * 256 + q]);
                e /= lsum;
                f[(size_t)b] = e / U[k * K + k];
            }
            const double *urow = U + k * K;
            for (int64_t b = 0; b < nb; ++b) {
                if (avx) feedback_avx2(w.data() + b * K, urow, f[(size_t)b], k + 1, K);
                else feedback(w.data() + b * K, urow, f[(size_t)b], k + 1, K);
            }
        }
    }
}

}  // namespace

extern "C" mq_status mq_matgptq_prepare(const double *H, int64_t K, double damp, double *U_out) {
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
    std::vector<double> L((size_t)n * n, 0.0);
    double *Lp = L.data();
    // Cholesky by panels of kPanel columns: the panel's diagonal rows in
    // order, then every row below it (independent of one another) in threads
    constexpr int64_t kPanel = 64;
    const bool avx = have_avx2_fma();
    auto dotv = [avx](const double *a, const double *b, int64_t m) {
        return avx ? dot_avx2(a, b, m) : dot(a, b, m);
    };
    for (int64_t j0 = 0; j0 < n; j0 += kPanel) {
        const int64_t j1 = std::min(n, j0 + kPanel);
        for (int64_t i = j0; i < j1; ++i)
            for (int64_t j = j0; j <= i; ++j) {
                const double v = P(i, j) - dotv(Lp + i * n, Lp + j * n, j);
                if (i == j) {
                    if (!(v > 0.0) || !isfinite(v))
                        return fail(MQ_ERR_UNSUPPORTED, "the damped Hessian is not positive definite");
                    Lp[i * n + i] = sqrt(v);
                } else {
                    Lp[i * n + j] = v / Lp[j * n + j];
                }
            }
        // rows below the panel, four at a time (each panel row read once for four)
        parallel_rows(0, (n - j1 + 3) / 4, nt, [&](int64_t t) {
            const int64_t i0 = j1 + 4 * t;
            const int m = (int)std::min<int64_t>(4, n - i0);
            for (int64_t j = j0; j < j1; ++j) {
                double acc[4];
                if (m == 4) {
                    if (avx) dot4_avx2(Lp + i0 * n, n, Lp + j * n, j, acc);
                    else dot4(Lp + i0 * n, n, Lp + j * n, j, acc);
                } else {
                    for (int r = 0; r < m; ++r) acc[r] = dotv(Lp + (i0 + r) * n, Lp + j * n, j);
                }
                for (int r = 0; r < m; ++r) Lp[(i0 + r) * n + j] = (P(i0 + r, j) - acc[r]) / Lp[j * n + j];
            }
        });
    }
    // columns c0..c0+3 of L^-1 together by forward substitution, rows four
    // at a time (each row of L read once for four columns; x_t[p] = 0 above
    // the diagonal), written reversed into U: U[n-1-i][n-1-c] = (L^-1)[i][c]
    std::fill(U_out, U_out + (size_t)n * n, 0.0);
    parallel_rows(0, (n + 3) / 4, nt, [&](int64_t blk) {
        const int64_t c0 = blk * 4;
        const int mc = (int)std::min<int64_t>(4, n - c0);
        std::vector<double> x((size_t)(n - c0) * 4, 0.0);
        double acc[16];
        for (int64_t i0 = c0; i0 < n; i0 += 4) {
            const int m = (int)std::min<int64_t>(4, n - i0);
            if (m == 4) {
                if (avx) acc4x4_avx2(Lp, n, i0, c0, i0, x.data(), acc);
                else acc4x4(Lp, n, i0, c0, i0, x.data(), acc);
            } else {
                for (int r = 0; r < 16; ++r) acc[r] = 0.0;
                for (int r = 0; r < m; ++r)
                    for (int64_t p = c0; p < i0; ++p)
                        for (int t = 0; t < 4; ++t) acc[4 * r + t] += Lp[(i0 + r) * n + p] * x[(size_t)((p - c0) * 4 + t)];
            }
            for (int r = 0; r < m; ++r) {
                const int64_t i = i0 + r;
                const double *li = Lp + i * n;
                double *a = acc + 4 * r;
                for (int64_t p = i0; p < i; ++p)
                    for (int t = 0; t < 4; ++t) a[t] += li[p] * x[(size_t)((p - c0) * 4 + t)];
                double *xi = x.data() + (i - c0) * 4;
                for (int t = 0; t < mc; ++t) {
                    const int64_t c = c0 + t;
                    xi[t] = i < c ? 0.0 : i == c ? 1.0 / li[i] : -a[t] / li[i];
                }
            }
        }
        for (int t = 0; t < mc; ++t) {
            const int64_t c = c0 + t;
            for (int64_t i = c; i < n; ++i) U_out[(n - 1 - i) * n + (n - 1 - c)] = x[(size_t)((i - c0) * 4 + t)];
        }
    });
    for (int64_t i = 0; i < n; ++i)
        if (!(U_out[i * n + i] > 0.0) || !isfinite(U_out[i * n + i])) return fail(MQ_ERR_UNSUPPORTED, "the damped Hessian is too ill-conditioned to invert");
    return MQ_OK;
}

extern "C" mq_status mq_matgptq_quantize(const float *W, int64_t N, int64_t K, const double *U,
                                         const int32_t *rs, const double *lambdas, int n_r,
                                         const double *alphas, int n_alpha, int threads,
                                         uint8_t *codes_out, float *scales_out) {
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
                      std::min<int64_t>(N, (blk + 1) * kRowBlock), codes_out, scales_out);
    });
    return MQ_OK;
}
