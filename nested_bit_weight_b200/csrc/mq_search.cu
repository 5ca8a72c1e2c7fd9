// Budget-aware per-layer bit-width search (host only): a multiple-choice
// knapsack solved exactly by dynamic programming ("MatGPTQ: Accurate and
// Efficient Post-Training Matryoshka Quantization", author-page abstract:
// budget-aware search for heterogeneous per-layer bit-widths; the r chosen
// per layer feeds mq_gemm_chain).
//
// best[b] over the layers seen so far = the least (error, bytes) pair whose
// bytes use at most b units, a unit being the greatest common divisor of all
// candidate byte counts (so the program is exact); a per-(layer, b) choice
// table rebuilds the assignment from b = budget / unit.
#include <math.h>

#include <limits>
#include <vector>

#include "mq_common.cuh"

using namespace mq;

namespace {

uint64_t gcd_u64(uint64_t a, uint64_t b) {
    while (b) {
        const uint64_t t = a % b;
        a = b;
        b = t;
    }
    return a;
}

}  // namespace

extern "C" mq_status mq_bitwidth_search(const mq_choice *choices, int n_layers, int n_choices,
                                        uint64_t budget_bytes, int *choice_out, double *error_out) {
    return host_guarded([&]() -> mq_status {
        if (!choices || !choice_out) return fail(MQ_ERR_INVALID_ARG, "NULL argument to mq_bitwidth_search");
        if (n_layers < 1 || n_choices < 1 || n_choices > 32767)
            return fail(MQ_ERR_INVALID_ARG, "need n_layers >= 1 and 1 <= n_choices <= 32767");
        const size_t total = (size_t)n_layers * n_choices;
        uint64_t unit = 0, min_bytes = 0;
        for (int l = 0; l < n_layers; ++l) {
            uint64_t lmin = std::numeric_limits<uint64_t>::max();
            for (int j = 0; j < n_choices; ++j) {
                const mq_choice &c = choices[(size_t)l * n_choices + j];
                if (!(c.error >= 0.0) || !isfinite(c.error))
                    return fail(MQ_ERR_INVALID_ARG, "every candidate error must be finite and >= 0");
                unit = gcd_u64(unit, c.bytes);
                if (c.bytes < lmin) lmin = c.bytes;
            }
            if (min_bytes > std::numeric_limits<uint64_t>::max() - lmin)
                return fail(MQ_ERR_UNSUPPORTED, "candidate bytes overflow");
            min_bytes += lmin;
        }
        (void)total;
        if (min_bytes > budget_bytes) return fail(MQ_ERR_UNSUPPORTED, "no choice fits the budget");
        if (unit == 0) unit = 1;                               // every candidate costs 0 bytes
        const uint64_t B = budget_bytes / unit;
        if ((double)n_layers * ((double)B + 1.0) > (double)(1u << 26))
            return fail(MQ_ERR_UNSUPPORTED, "the dynamic program would exceed 2^26 cells");

        const size_t W = (size_t)B + 1;
        const double inf = std::numeric_limits<double>::infinity();
        std::vector<double> err_prev(W, 0.0), err_cur(W);
        std::vector<uint64_t> units_prev(W, 0), units_cur(W);
        std::vector<int16_t> pick((size_t)n_layers * W, -1);
        for (int l = 0; l < n_layers; ++l) {
            for (size_t b = 0; b < W; ++b) {
                double best_e = inf;
                uint64_t best_u = 0;
                int best_j = -1;
                for (int j = 0; j < n_choices; ++j) {
                    const mq_choice &c = choices[(size_t)l * n_choices + j];
                    const uint64_t cu = c.bytes / unit;
                    if (cu > b || err_prev[b - cu] == inf) continue;
                    const double e = err_prev[b - cu] + c.error;
                    const uint64_t u = units_prev[b - cu] + cu;
                    if (e < best_e || (e == best_e && u < best_u)) {   // strict: the lowest index wins ties
                        best_e = e;
                        best_u = u;
                        best_j = j;
                    }
                }
                err_cur[b] = best_e;
                units_cur[b] = best_u;
                pick[(size_t)l * W + b] = (int16_t)best_j;
            }
            err_prev.swap(err_cur);
            units_prev.swap(units_cur);
        }
        if (err_prev[B] == inf) return fail(MQ_ERR_UNSUPPORTED, "no choice fits the budget");
        uint64_t b = B;
        for (int l = n_layers - 1; l >= 0; --l) {
            const int j = pick[(size_t)l * W + b];
            choice_out[l] = j;
            b -= choices[(size_t)l * n_choices + j].bytes / unit;
        }
        if (error_out) *error_out = err_prev[B];
        return MQ_OK;
    });
}
