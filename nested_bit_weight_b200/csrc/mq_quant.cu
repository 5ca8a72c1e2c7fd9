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
    // argmin over q of sum_r lambda_r (w - s v_r(q))^2, the first minimum
    int best_code(double w, double s) const {
        int best = 0;
        double best_c = 0.0;
        for (int q = 0; q < 256; ++q) {
            double c = 0.0;
            for (int i = 0; i < nr; ++i) {
                const double d = w - s * levels[(size_t)i * 256 + q];
                c += lams[i] * d * d;
            }
            if (q == 0 || c < best_c) {
                best = q;
                best_c = c;
            }
        }
        return best;
    }
};

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
    const size_t n = (size_t)K;
    double mean = 0.0;
    for (size_t i = 0; i < n; ++i) mean += H[i * n + i];
    mean /= (double)K;
    // L L^T = H + damp * mean * I (lower Cholesky)
    std::vector<double> L(n * n, 0.0);
    for (size_t j = 0; j < n; ++j) {
        double d = H[j * n + j] + damp * mean;
        for (size_t p = 0; p < j; ++p) d -= L[j * n + p] * L[j * n + p];
        if (!(d > 0.0)) return fail(MQ_ERR_UNSUPPORTED, "the damped Hessian is not positive definite");
        const double ljj = sqrt(d);
        L[j * n + j] = ljj;
        for (size_t i = j + 1; i < n; ++i) {
            double v = H[i * n + j];
            for (size_t p = 0; p < j; ++p) v -= L[i * n + p] * L[j * n + p];
            L[i * n + j] = v / ljj;
        }
    }
    // M = L^-1 (lower), then Hinv = M^T M
    std::vector<double> Mi(n * n, 0.0);
    for (size_t j = 0; j < n; ++j) {
        Mi[j * n + j] = 1.0 / L[j * n + j];
        for (size_t i = j + 1; i < n; ++i) {
            double v = 0.0;
            for (size_t p = j; p < i; ++p) v -= L[i * n + p] * Mi[p * n + j];
            Mi[i * n + j] = v / L[i * n + i];
        }
    }
    std::vector<double> Hinv(n * n, 0.0);
    for (size_t i = 0; i < n; ++i)
        for (size_t j = 0; j <= i; ++j) {
            double v = 0.0;
            for (size_t p = i; p < n; ++p) v += Mi[p * n + i] * Mi[p * n + j];
            Hinv[i * n + j] = v;
            Hinv[j * n + i] = v;
        }
    // U upper with U^T U = Hinv: U = R^T, R R^T = Hinv the lower Cholesky
    std::fill(U_out, U_out + n * n, 0.0);
    std::vector<double> R(n * n, 0.0);
    for (size_t j = 0; j < n; ++j) {
        double d = Hinv[j * n + j];
        for (size_t p = 0; p < j; ++p) d -= R[j * n + p] * R[j * n + p];
        if (!(d > 0.0)) return fail(MQ_ERR_UNSUPPORTED, "the inverse Hessian is not positive definite");
        const double rjj = sqrt(d);
        R[j * n + j] = rjj;
        for (size_t i = j + 1; i < n; ++i) {
            double v = Hinv[i * n + j];
            for (size_t p = 0; p < j; ++p) v -= R[i * n + p] * R[j * n + p];
            R[i * n + j] = v / rjj;
        }
    }
    for (size_t i = 0; i < n; ++i)
        for (size_t j = i; j < n; ++j) U_out[i * n + j] = R[j * n + i];
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
