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
//     lambda-weighted mean of the slice errors e:  w_j -= e / U[k,k] * U[k,j].
// Rows are independent given U, so threads take rows; every operation is
// fp64 in a fixed order.
#include <math.h>

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
    // argmin over q of sum_r lambda_r (w - s v_r(q))^2, the first minimum;
    // each cost sums its terms in the order of the widths (the loop over q
    // is the vectorised one, which leaves every cost's own sum unchanged)
    int best_code(double w, double s) const {
        alignas(64) double c[256];
        for (int q = 0; q < 256; ++q) c[q] = 0.0;
        for (int i = 0; i < nr; ++i) {
            const double lam = lams[i];
            const double *lv = levels.data() + (size_t)i * 256;
            for (int q = 0; q < 256; ++q) {
                const double d = w - s * lv[q];
                c[q] += lam * d * d;
            }
        }
        int best = 0;
        for (int q = 1; q < 256; ++q)
            if (c[q] < c[best]) best = q;
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

void quantize_rows(const float *W, int64_t K, const double *U, const Objective &obj, const double *alphas,
                   int na, double lsum, int64_t n0, int64_t n1, uint8_t *codes, float *scales) {
    const int64_t G = K / 128;
    std::vector<double> w((size_t)K);
    for (int64_t n = n0; n < n1; ++n) {
        for (int64_t k = 0; k < K; ++k) w[(size_t)k] = (double)W[n * K + k];
        for (int64_t g = 0; g < G; ++g) {
            double mx = 0.0;
            for (int64_t k = 128 * g; k < 128 * g + 128; ++k) mx = std::max(mx, fabs(w[(size_t)k]));
            const double base = mx / 127.5;
            double best_a = 0.0, best_t = 0.0;
            for (int ia = 0; ia < na; ++ia) {
                const double s = base * alphas[ia];
                double t = 0.0;
                for (int64_t k = 128 * g; k < 128 * g + 128; ++k) {
                    const int q = obj.best_code(w[(size_t)k], s);
                    for (int i = 0; i < obj.nr; ++i) {
                        const double d = w[(size_t)k] - s * obj.levels[(size_t)i * 256 + q];
                        t += obj.lams[i] * d * d;
                    }
                }
                if (ia == 0 || t < best_t) {
                    best_a = alphas[ia];
                    best_t = t;
                }
            }
            const double s = base * best_a;
            scales[n * G + g] = (float)s;
            for (int64_t k = 128 * g; k < 128 * g + 128; ++k) {
                const int q = obj.best_code(w[(size_t)k], s);
                codes[n * K + k] = (uint8_t)q;
                double e = 0.0;
                for (int i = 0; i < obj.nr; ++i) e += obj.lams[i] * (w[(size_t)k] - s * obj.levels[(size_t)i * 256 + q]);
                e /= lsum;
                const double f = e / U[k * K + k];
                const double *urow = U + k * K;
                for (int64_t j = k + 1; j < K; ++j) w[(size_t)j] -= f * urow[j];
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
    for (int64_t j0 = 0; j0 < n; j0 += kPanel) {
        const int64_t j1 = std::min(n, j0 + kPanel);
        for (int64_t i = j0; i < j1; ++i)
            for (int64_t j = j0; j <= i; ++j) {
                const double v = P(i, j) - dot(Lp + i * n, Lp + j * n, j);
                if (i == j) {
                    if (!(v > 0.0) || !isfinite(v))
                        return fail(MQ_ERR_UNSUPPORTED, "the damped Hessian is not positive definite");
                    Lp[i * n + i] = sqrt(v);
                } else {
                    Lp[i * n + j] = v / Lp[j * n + j];
                }
            }
        parallel_rows(j1, n, nt, [&](int64_t i) {
            for (int64_t j = j0; j < j1; ++j)
                Lp[i * n + j] = (P(i, j) - dot(Lp + i * n, Lp + j * n, j)) / Lp[j * n + j];
        });
    }
    // column c of L^-1 by forward substitution (columns independent), written
    // reversed into U: U[n-1-i][n-1-c] = (L^-1)[i][c]
    std::fill(U_out, U_out + (size_t)n * n, 0.0);
    parallel_rows(0, n, nt, [&](int64_t c) {
        std::vector<double> x((size_t)(n - c));
        x[0] = 1.0 / Lp[c * n + c];
        for (int64_t i = c + 1; i < n; ++i)
            x[(size_t)(i - c)] = -dot(Lp + i * n + c, x.data(), i - c) / Lp[i * n + i];
        for (int64_t i = c; i < n; ++i) U_out[(n - 1 - i) * n + (n - 1 - c)] = x[(size_t)(i - c)];
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
    const Objective obj(rs, lambdas, n_r);
    int nt = threads > 0 ? threads : (int)std::max(1u, std::thread::hardware_concurrency());
    nt = (int)std::min<int64_t>(nt, N);
    std::vector<std::thread> pool;
    const int64_t per = (N + nt - 1) / nt;
    for (int t = 0; t < nt; ++t) {
        const int64_t n0 = t * per, n1 = std::min<int64_t>(N, n0 + per);
        if (n0 >= n1) break;
        pool.emplace_back(quantize_rows, W, K, U, std::cref(obj), alphas, n_alpha, lsum, n0, n1, codes_out, scales_out);
    }
    for (auto &th : pool) th.join();
    return MQ_OK;
}
