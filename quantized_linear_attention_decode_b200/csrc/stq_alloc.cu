// stq_alloc.cu -- lifetime-aware mixed-precision bit allocation (host code).
//
// Method: "STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent
// State Quantization" (paper.rainbus.top/paper/2609.38169), "core
// innovation" (first point) and "method steps", offline calibration steps
// (1)-(3):
//   - an old error's square decays by the retention rate, about
//     exp(2 j l_u) after j steps, so a unit u with mean log retention l_u
//     carries the lifetime weight L_u = sum_{j=0}^{H-1} exp(2 j l_u);
//   - the widths b_u minimise sum_u L_u d_u(b_u) subject to
//     sum_u n_u b_u <= b_bar sum_u n_u (Eq. 8), by a multiple-choice dynamic
//     programme (GDN: one unit per head) or a Lagrangian allocation (KDA: one
//     unit per key row);
//   - the units of highest remaining risk are then kept as FP16 pivots.
// Readings where the page is silent: the horizon H is an argument; a pivot's
// remaining risk is L_u d_u(b_u) under the allocated width (its FP16 error is
// taken as zero), and pivots sit outside the nominal budget (the page's
// effective widths, 6.36 bits at a 6-bit budget, exceed the budget).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <numeric>
#include <vector>

#include "stq_internal.h"

namespace {

constexpr double kMaxDpCells = 4e8;  // units x budget steps the exact programme may use

// L_u for one unit: the sum itself (H terms) for short horizons, the
// geometric-series closed form otherwise.
double lifetime_weight(double ell, int horizon)
{
    if (horizon <= 4096) {
        double s = 0.0;
        for (int j = 0; j < horizon; ++j) s += std::exp(2.0 * j * ell);
        return s;
    }
    const double q = std::exp(2.0 * ell);
    if (std::fabs(1.0 - q) < 1e-12) return static_cast<double>(horizon);
    return std::expm1(2.0 * horizon * ell) / std::expm1(2.0 * ell);
}

struct Problem {
    int U, C;
    const double *n;       // [U] values per unit
    const uint8_t *width;  // [C] candidate widths, strictly increasing
    const double *d;       // [U][C] distortion
    const double *w;       // [U] lifetime weight
    double budget;         // total bits allowed
};

double objective(const Problem &P, const std::vector<int> &pick)
{
    double f = 0.0;
    for (int u = 0; u < P.U; ++u) f += P.w[u] * P.d[(size_t)u * P.C + pick[u]];
    return f;
}

double cost(const Problem &P, const std::vector<int> &pick)
{
    double c = 0.0;
    for (int u = 0; u < P.U; ++u) c += P.n[u] * P.width[pick[u]];
    return c;
}

// Exact multiple-choice knapsack over integer costs n_u b (divided by their
// common divisor).  Returns STQ_ERR_UNSUPPORTED when the table would be too
// large or the costs are not integers.
stq_status solve_dp(const Problem &P, std::vector<int> &pick, char *why, size_t why_len)
{
    std::vector<long long> ni(P.U);
    long long g = 0;
    for (int u = 0; u < P.U; ++u) {
        const double r = std::nearbyint(P.n[u]);
        if (r != P.n[u] || r <= 0 || r > 1e12) {
            std::snprintf(why, why_len, "unit_values[%d] = %g is not a positive integer", u, P.n[u]);
            return STQ_ERR_UNSUPPORTED;
        }
        ni[u] = static_cast<long long>(r);
        for (int k = 0; k < P.C; ++k) g = std::gcd(g, ni[u] * P.width[k]);
    }
    const long long B = static_cast<long long>(std::floor(P.budget / static_cast<double>(g) + 1e-9));
    if ((double)P.U * (double)(B + 1) > kMaxDpCells) {
        std::snprintf(why, why_len, "dynamic programme too large (%d units x %lld budget steps); use the "
                      "Lagrangian method", P.U, B + 1);
        return STQ_ERR_UNSUPPORTED;
    }
    const double inf = HUGE_VAL;
    std::vector<double> best(B + 1, inf), next(B + 1);
    std::vector<uint8_t> choice((size_t)P.U * (B + 1), 0xFF);
    best[0] = 0.0;
    for (int u = 0; u < P.U; ++u) {
        std::fill(next.begin(), next.end(), inf);
        uint8_t *ch = &choice[(size_t)u * (B + 1)];
        for (int k = 0; k < P.C; ++k) {
            const long long c = ni[u] * P.width[k] / g;
            const double f = P.w[u] * P.d[(size_t)u * P.C + k];
            for (long long j = c; j <= B; ++j) {
                if (best[j - c] == inf) continue;
                const double v = best[j - c] + f;
                if (v < next[j]) {  // strict: the smallest width wins ties
                    next[j] = v;
                    ch[j] = static_cast<uint8_t>(k);
                }
            }
        }
        best.swap(next);
    }
    long long j = -1;
    double f = inf;
    for (long long b = 0; b <= B; ++b)
        if (best[b] < f) {  // the cheapest of the optimal assignments
            f = best[b];
            j = b;
        }
    if (j < 0) {
        std::snprintf(why, why_len, "no assignment fits the budget");
        return STQ_ERR_ARG;
    }
    for (int u = P.U - 1; u >= 0; --u) {
        const int k = choice[(size_t)u * (B + 1) + j];
        pick[u] = k;
        j -= ni[u] * P.width[k] / g;
    }
    return STQ_OK;
}

// Each unit's minimiser of w d + lambda n b (the smallest width on ties).
void lagrange_pick(const Problem &P, double lambda, std::vector<int> &pick)
{
    for (int u = 0; u < P.U; ++u) {
        int bk = 0;
        double bv = HUGE_VAL;
        for (int k = 0; k < P.C; ++k) {
            const double v = P.w[u] * P.d[(size_t)u * P.C + k] + lambda * P.n[u] * P.width[k];
            if (v < bv) {
                bv = v;
                bk = k;
            }
        }
        pick[u] = bk;
    }
}

// Smallest multiplier (bisection, 200 halvings) whose per-unit minimisers
// fit the budget.  The result minimises sum w d over every assignment that
// costs no more than it does.
stq_status solve_lagrange(const Problem &P, std::vector<int> &pick, char *why, size_t why_len)
{
    lagrange_pick(P, 0.0, pick);
    if (cost(P, pick) <= P.budget) return STQ_OK;
    double hi = 1.0;
    for (int it = 0; it < 400; ++it) {
        lagrange_pick(P, hi, pick);
        if (cost(P, pick) <= P.budget) break;
        hi *= 4.0;
        if (it == 399 || !std::isfinite(hi)) {
            std::snprintf(why, why_len, "no assignment fits the budget");
            return STQ_ERR_ARG;
        }
    }
    double lo = 0.0;
    for (int it = 0; it < 200; ++it) {
        const double mid = 0.5 * (lo + hi);
        if (mid <= lo || mid >= hi) break;
        lagrange_pick(P, mid, pick);
        if (cost(P, pick) <= P.budget) hi = mid;
        else lo = mid;
    }
    lagrange_pick(P, hi, pick);
    return STQ_OK;
}

}  // namespace

extern "C" {

stq_status stq_lifetime_weight(int32_t num_units, const double *log_retention, int32_t horizon,
                               double *weight_out)
{
    if (num_units < 0 || horizon < 1 || (num_units > 0 && (!log_retention || !weight_out)))
        return stq::fail_status(STQ_ERR_ARG, "bad argument to stq_lifetime_weight");
    for (int u = 0; u < num_units; ++u) {
        const double l = log_retention[u];
        if (!(l <= 0.0) || !std::isfinite(l))
            return stq::fail_status(STQ_ERR_ARG, "log_retention[%d] = %g (must be finite and <= 0)", u, l);
        weight_out[u] = lifetime_weight(l, horizon);
    }
    return STQ_OK;
}

stq_status stq_allocate_bits(int32_t num_units, const double *unit_values, int32_t num_choices,
                             const uint8_t *choices, const double *distortion, const double *weight,
                             double mean_bits, int32_t method, int32_t num_pivots, uint8_t pivot_bits,
                             uint8_t *bits_out, double *objective_out)
{
    if (num_units < 1 || num_choices < 1 || num_choices > 16 || !unit_values || !choices || !distortion ||
        !weight || !bits_out)
        return stq::fail_status(STQ_ERR_ARG, "bad argument to stq_allocate_bits");
    if (method != STQ_ALLOC_DP && method != STQ_ALLOC_LAGRANGE)
        return stq::fail_status(STQ_ERR_ARG, "method %d", method);
    if (num_pivots < 0 || num_pivots > num_units)
        return stq::fail_status(STQ_ERR_ARG, "num_pivots = %d of %d units", num_pivots, num_units);
    for (int k = 0; k < num_choices; ++k)
        if (choices[k] == 0 || (k > 0 && choices[k] <= choices[k - 1]))
            return stq::fail_status(STQ_ERR_ARG, "choices must be positive and strictly increasing");
    double total = 0.0;
    for (int u = 0; u < num_units; ++u) {
        if (!(unit_values[u] > 0.0) || !std::isfinite(unit_values[u]) || !(weight[u] >= 0.0) ||
            !std::isfinite(weight[u]))
            return stq::fail_status(STQ_ERR_ARG, "unit %d: values %g, weight %g", u, unit_values[u], weight[u]);
        for (int k = 0; k < num_choices; ++k) {
            const double d = distortion[(size_t)u * num_choices + k];
            if (!(d >= 0.0) || !std::isfinite(d))
                return stq::fail_status(STQ_ERR_ARG, "distortion[%d][%d] = %g", u, k, d);
        }
        total += unit_values[u];
    }
    if (!(mean_bits > 0.0) || !std::isfinite(mean_bits))
        return stq::fail_status(STQ_ERR_ARG, "mean_bits = %g", mean_bits);
    Problem P{num_units, num_choices, unit_values, choices, distortion, weight, mean_bits * total};
    if (P.budget + 1e-9 * P.budget < total * choices[0])
        return stq::fail_status(STQ_ERR_ARG, "budget %g bits per value is below the smallest width %d",
                                mean_bits, choices[0]);
    std::vector<int> pick(num_units, 0);
    char why[256] = {0};
    const stq_status st = method == STQ_ALLOC_DP ? solve_dp(P, pick, why, sizeof why)
                                                 : solve_lagrange(P, pick, why, sizeof why);
    if (st != STQ_OK) return stq::fail_status(st, "%s", why);
    if (objective_out) *objective_out = objective(P, pick);
    for (int u = 0; u < num_units; ++u) bits_out[u] = choices[pick[u]];
    // pivots: the num_pivots units of largest remaining risk w d(b) (lowest index first on ties)
    if (num_pivots > 0) {
        std::vector<int> order(num_units);
        std::iota(order.begin(), order.end(), 0);
        auto risk = [&](int u) { return P.w[u] * P.d[(size_t)u * P.C + pick[u]]; };
        std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return risk(a) > risk(b); });
        for (int i = 0; i < num_pivots; ++i) bits_out[order[i]] = pivot_bits;
    }
    return STQ_OK;
}

}  // extern "C"
