// Host-side window math: per-pair RoPE frequencies, the per-pair distance
// window and the closed-form count of kept query-key terms.
//
// Source: "ATFlash — Per-RoPE-Wavelength Attention Windows" README, section
// "The idea" (w_r = k * lambda_r; the reduction is input-independent with a
// closed form) and the arXiv 2608.02947 abstract.  Everything here is fp64 or
// integer and runs once per call; the kernels receive the integer table.
#include <math.h>
#include <stdint.h>

#include "internal.h"

namespace atf {

static const double kTwoPi = 6.283185307179586476925286766559;

void theta_table(int D, double base, double *theta) {
    for (int r = 0; r < D / 2; ++r) theta[r] = pow(base, -2.0 * (double)r / (double)D);
}

// A caller's frequency table (scaled RoPE): finite, in (0, pi], non-increasing
// in r, so that the windows w_r do not decrease and the pairs kept at any
// distance are a suffix r >= r*(d), which the kernels rely on.
bool theta_valid(int D, const double *theta) {
    if (!theta || D < 2 || D > 2 * kMaxPairs || (D & 1)) return false;
    for (int r = 0; r < D / 2; ++r) {
        const double t = theta[r];
        if (!(t > 0.0) || !(t <= kTwoPi / 2)) return false;  // rejects NaN too
        if (r > 0 && t > theta[r - 1]) return false;
    }
    return true;
}

int window_table_theta(int D, const double *theta, double k, int64_t N, int64_t *w) {
    if (!theta_valid(D, theta) || isnan(k) || k < 0.0 || N < 1 || !w) return ATFLASH_ERR_INVALID_ARG;
    for (int r = 0; r < D / 2; ++r) {
        double lambda = kTwoPi / theta[r];
        double x = floor(k * lambda);  // +inf when k = +inf
        w[r] = (x >= (double)(N - 1)) ? (N - 1) : (int64_t)x;
    }
    return ATFLASH_OK;
}

int window_table(int D, double base, double k, int64_t N, int64_t *w) {
    if (D < 2 || D > 2 * kMaxPairs || (D & 1) || !(base > 1.0) || isnan(k) || k < 0.0 || N < 1 || !w)
        return ATFLASH_ERR_INVALID_ARG;
    double theta[kMaxPairs];
    theta_table(D, base, theta);
    return window_table_theta(D, theta, k, N, w);
}

// Pair r is kept on the causal cells at distance d <= W_r = min(w_r, N-1);
// distance d occurs N - d times, so kept_r = (W_r + 1)(2N - W_r)/2.
static int terms_from_windows(int64_t N, int D, const int64_t *w, atflash_terms *out);

int pruned_terms(int64_t N, int D, double base, double k, atflash_terms *out) {
    if (!out) return ATFLASH_ERR_INVALID_ARG;
    int64_t w[kMaxPairs];
    int rc = window_table(D, base, k, N, w);
    if (rc != ATFLASH_OK) return rc;
    return terms_from_windows(N, D, w, out);
}

int pruned_terms_theta(int64_t N, int D, const double *theta, double k, atflash_terms *out) {
    if (!out) return ATFLASH_ERR_INVALID_ARG;
    int64_t w[kMaxPairs];
    int rc = window_table_theta(D, theta, k, N, w);
    if (rc != ATFLASH_OK) return rc;
    return terms_from_windows(N, D, w, out);
}

static int terms_from_windows(int64_t N, int D, const int64_t *w, atflash_terms *out) {
    typedef unsigned __int128 u128;
    u128 n = (u128)N, kept = 0;
    for (int r = 0; r < D / 2; ++r) {
        u128 W = (u128)w[r];
        kept += (W + 1) * (2 * n - W) / 2;
    }
    u128 total = (u128)(D / 2) * n * (n + 1) / 2;
    if (2 * total > (u128)UINT64_MAX) return ATFLASH_ERR_INVALID_ARG;  // counts must fit in uint64
    out->total = (uint64_t)total;
    out->kept = (uint64_t)kept;
    out->pruned = (uint64_t)(total - kept);
    out->total_dims = (uint64_t)(2 * total);
    out->kept_dims = (uint64_t)(2 * kept);
    return ATFLASH_OK;
}

}  // namespace atf
