/*
 * Plain fp64 CPU oracle for per-RoPE-wavelength windowed causal attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * includes this file; only the tests, the package's smoke check and the CPU
 * baseline leg of bench.py load it.  It shares no code, header, table or
 * constant generator with the CUDA path.
 *
 * What it computes (source: "ATFlash — Per-RoPE-Wavelength Attention
 * Windows", gh.bsm-lab.com/ATFlash/ATFlash-Kernel, sections "The idea" and
 * "Porting to something else"; arXiv 2608.02947 abstract):
 *
 *   theta_r  = base^(-2r/D),  lambda_r = 2*pi / theta_r,  r = 0 .. D/2-1
 *   w_r      = floor(k * lambda_r)                 (the per-pair distance window)
 *   pair r   = dims (r, r + D/2)                   (rotate-half RoPE layout)
 *   x~_r     = x_r cos(p theta_r) - x_{r+H} sin(p theta_r)
 *   x~_{r+H} = x_{r+H} cos(p theta_r) + x_r sin(p theta_r)
 *   t_r(n,m) = q~_{n,r} k~_{m,r} + q~_{n,r+H} k~_{m,r+H}
 *   s(n,m)   = (1/sqrt(D)) * sum over r with (n-m) <= w_r of t_r(n,m),  m <= n
 *   o_n      = sum_m softmax_m(s(n,.)) v_m      (two passes: max, then sums)
 *
 * Scaled RoPE: orc_set_theta installs a caller's table theta_r (D/2 values)
 * that replaces base^(-2r/D) in both the window (lambda_r = 2*pi/theta_r) and
 * the rotation, until it is cleared; the definitions above are otherwise
 * unchanged.  (The pages derive the window table from the model's RoPE
 * configuration, "rope_scaling" included.)
 *
 * Token-level selection under the window (the abstract: token-level sparse
 * methods such as MInference are orthogonal to the frequency-level window, which
 * can be applied on top of them): orc_prefill_rows_sparse takes a block mask
 * over (query tile, key tile) pairs of `tile` positions each.  Key m is visible
 * to query n iff m <= n and (m and n lie in the same tile, or the mask entry of
 * their tiles is nonzero); the diagonal tile is always visible, so no row is
 * empty.  Invisible keys take no part in the softmax; the window applies to the
 * visible ones unchanged.
 *
 * k = +inf keeps every pair (plain causal RoPE attention).  A cell whose every
 * pair is pruned scores 0 (the empty sum), not -inf: the pages keep "the sum
 * over the rest" and drop no token.
 *
 * Every floating-point step is fp64; inputs arrive as float (they hold fp32
 * values or bf16 values widened exactly) and are widened on use.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_TWO_PI (2.0 * 3.14159265358979323846)
#define ORC_MAX_PAIRS 128

/* Installed frequency table (scaled RoPE); orc_theta_n == 0: none. */
static double orc_theta_tab[ORC_MAX_PAIRS];
static int orc_theta_n = 0;

/* Install theta[0..n-1] as the RoPE frequencies (n = 0 clears the table). */
int orc_set_theta(const double *theta, int n) {
    if (n < 0 || n > ORC_MAX_PAIRS || (n > 0 && !theta)) return -1;
    for (int r = 0; r < n; ++r) orc_theta_tab[r] = theta[r];
    orc_theta_n = n;
    return 0;
}

/* theta_r: the installed table, else base^(-2r/D). */
static double orc_theta(int r, int D, double base) {
    if (orc_theta_n > 0 && r < orc_theta_n) return orc_theta_tab[r];
    return pow(base, -2.0 * (double)r / (double)D);
}

/* Per-pair window limit floor(k * lambda_r) as a double (may be +inf).  The
 * pages' "w_r = k * lambda_r" with the floor of the integer-distance reading:
 * a pair is kept while the distance d satisfies d <= w_r. */
static double orc_limit(int r, int D, double base, double kwin) {
    double theta = orc_theta(r, D, base);
    double lambda = ORC_TWO_PI / theta;
    return floor(kwin * lambda);
}

int orc_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* w_r for r < D/2, as doubles (+inf when k = +inf). */
void orc_window_limits(int D, double base, double kwin, double *lim) {
    for (int r = 0; r < D / 2; ++r) lim[r] = orc_limit(r, D, base, kwin);
}

/* Brute-force term count over one (sequence, head): every causal cell (n, m),
 * m <= n < N, and every pair r; counts pair-terms with n - m <= w_r. */
void orc_count_bruteforce(int64_t N, int D, double base, double kwin,
                          uint64_t *kept, uint64_t *total) {
    int H = D / 2;
    double *lim = (double *)malloc(sizeof(double) * (size_t)H);
    orc_window_limits(D, base, kwin, lim);
    uint64_t kp = 0, tt = 0;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t m = 0; m <= n; ++m)
            for (int r = 0; r < H; ++r) {
                tt += 1;
                if ((double)(n - m) <= lim[r]) kp += 1;
            }
    free(lim);
    *kept = kp;
    *total = tt;
}

/* Closed form of the same count (the pages: "input-independent, with a closed
 * form").  Pair r is kept on the cells with distance d <= W_r = min(w_r, N-1);
 * distance d occurs N - d times in the causal triangle, so
 *   kept_r = sum_{d=0}^{W_r} (N - d) = (W_r + 1)(2N - W_r) / 2. */
void orc_count_closed(int64_t N, int D, double base, double kwin,
                      uint64_t *kept, uint64_t *total) {
    int H = D / 2;
    uint64_t kp = 0;
    for (int r = 0; r < H; ++r) {
        double l = orc_limit(r, D, base, kwin);
        uint64_t W = (l >= (double)(N - 1)) ? (uint64_t)(N - 1) : (uint64_t)l;
        kp += (W + 1) * (2 * (uint64_t)N - W) / 2;
    }
    *kept = kp;
    *total = (uint64_t)H * (uint64_t)N * (uint64_t)(N + 1) / 2;
}

/* Smallest number of kept pairs over all causal cells, by brute force (the
 * pages' "every key stays reachable through the low-frequency pairs"). */
int64_t orc_min_kept_pairs(int64_t N, int D, double base, double kwin) {
    int H = D / 2;
    double *lim = (double *)malloc(sizeof(double) * (size_t)H);
    orc_window_limits(D, base, kwin, lim);
    int64_t mn = H;
    for (int64_t d = 0; d < N; ++d) {
        int64_t c = 0;
        for (int r = 0; r < H; ++r) c += ((double)d <= lim[r]) ? 1 : 0;
        if (c < mn) mn = c;
    }
    free(lim);
    return mn;
}

/* Rotate-half RoPE of one D-vector at position pos, fp64. */
static void orc_rope(const float *x, int D, double base, int64_t pos, double *y) {
    int H = D / 2;
    for (int r = 0; r < H; ++r) {
        double theta = orc_theta(r, D, base);
        double phi = (double)pos * theta;
        double c = cos(phi), s = sin(phi);
        double a = (double)x[r], b = (double)x[r + H];
        y[r] = a * c - b * s;
        y[r + H] = b * c + a * s;
    }
}

static void orc_copy_widen(const float *x, int D, double *y) {
    for (int i = 0; i < D; ++i) y[i] = (double)x[i];
}

/* Windowed score of one (query, key) cell at distance d, from rotated vectors. */
static double orc_score(const double *qt, const double *kt, int D, const double *lim, int64_t d) {
    int H = D / 2;
    double acc = 0.0;
    for (int r = 0; r < H; ++r) {
        if ((double)d <= lim[r]) acc += qt[r] * kt[r] + qt[r + H] * kt[r + H];
    }
    return acc / sqrt((double)D);
}

/* Is key m visible to query n under the block mask row of n's tile (NULL: all
 * keys 0..n are)? */
static int orc_visible(const unsigned char *mask_row, int64_t tile, int64_t n, int64_t m) {
    if (!mask_row) return 1;
    return m / tile == n / tile || mask_row[m / tile] != 0;
}

/* Attention output of one query row over the visible keys among 0..n (rotated
 * keys kt[m*D..]), two-pass softmax.  out[D]; *lse = natural log-sum-exp of the
 * scores. */
static void orc_row(const double *qt, const double *kt, const float *v, int64_t v_stride,
                    int64_t n, int D, const double *lim, const unsigned char *mask_row, int64_t tile,
                    double *scores, double *out, double *lse) {
    double mx = -INFINITY;
    for (int64_t m = 0; m <= n; ++m) {
        if (!orc_visible(mask_row, tile, n, m)) continue;
        scores[m] = orc_score(qt, kt + (size_t)m * D, D, lim, n - m);
        if (scores[m] > mx) mx = scores[m];
    }
    double den = 0.0;
    for (int i = 0; i < D; ++i) out[i] = 0.0;
    for (int64_t m = 0; m <= n; ++m) {
        if (!orc_visible(mask_row, tile, n, m)) continue;
        double p = exp(scores[m] - mx);
        den += p;
        const float *vm = v + (size_t)m * (size_t)v_stride;
        for (int i = 0; i < D; ++i) out[i] += p * (double)vm[i];
    }
    for (int i = 0; i < D; ++i) out[i] /= den;
    if (lse) *lse = mx + log(den);
}

/* Rotate (or just widen) keys 0..nk-1 of one KV head.  k points at key 0 of the
 * head; consecutive keys are k_stride floats apart. */
static double *orc_rotated_keys(const float *k, int64_t k_stride, int64_t nk, int D,
                                double base, int krot) {
    double *kt = (double *)malloc(sizeof(double) * (size_t)nk * (size_t)D);
    if (!kt) return NULL;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < nk; ++m) {
        if (krot) orc_copy_widen(k + (size_t)m * k_stride, D, kt + (size_t)m * D);
        else orc_rope(k + (size_t)m * k_stride, D, base, m, kt + (size_t)m * D);
    }
    return kt;
}

/*
 * Prefill output for selected query rows of one sequence.
 *   q_rows [nrows][Hq][D]  (un-rotated query vectors of the selected rows)
 *   rows   [nrows]         (their positions n, 0 <= n < N)
 *   k, v   [N][Hkv][D]     (un-rotated keys, values of the sequence)
 *   out    [nrows][Hq][D], lse [nrows][Hq] (lse may be NULL)
 * Query head h reads KV head h / (Hq / Hkv).  Returns 0, or -1 on bad input.
 */
static int orc_prefill_rows_masked(const float *q_rows, const int64_t *rows, int64_t nrows,
                                   const float *k, const float *v, int Hq, int Hkv, int64_t N, int D,
                                   double base, double kwin, const unsigned char *block_mask, int64_t tile,
                                   double *out, double *lse) {
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv || D <= 0 || D % 2 || N <= 0) return -1;
    if (block_mask && tile <= 0) return -1;
    int64_t ntiles = block_mask ? (N + tile - 1) / tile : 0;
    int G = Hq / Hkv;
    int H = D / 2;
    int64_t nmax = 0;
    for (int64_t i = 0; i < nrows; ++i) {
        if (rows[i] < 0 || rows[i] >= N) return -1;
        if (rows[i] > nmax) nmax = rows[i];
    }
    double *lim = (double *)malloc(sizeof(double) * (size_t)H);
    orc_window_limits(D, base, kwin, lim);
    int rc = 0;
    for (int g = 0; g < Hkv && rc == 0; ++g) {
        double *kt = orc_rotated_keys(k + (size_t)g * D, (int64_t)Hkv * D, nmax + 1, D, base, 0);
        if (!kt) { rc = -1; break; }
        const float *vg = v + (size_t)g * D;
        int64_t ntask = nrows * G;
#pragma omp parallel
        {
            double *scores = (double *)malloc(sizeof(double) * (size_t)(nmax + 1));
            double *qt = (double *)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 1)
            for (int64_t t = 0; t < ntask; ++t) {
                int64_t i = t / G;
                int h = g * G + (int)(t % G);
                int64_t n = rows[i];
                const unsigned char *mrow =
                    block_mask ? block_mask + ((size_t)g * ntiles + (size_t)(n / tile)) * (size_t)ntiles : NULL;
                orc_rope(q_rows + ((size_t)i * Hq + h) * D, D, base, n, qt);
                orc_row(qt, kt, vg, (int64_t)Hkv * D, n, D, lim, mrow, tile, scores,
                        out + ((size_t)i * Hq + h) * D,
                        lse ? lse + (size_t)i * Hq + h : NULL);
            }
            free(scores);
            free(qt);
        }
        free(kt);
    }
    free(lim);
    return rc;
}

int orc_prefill_rows(const float *q_rows, const int64_t *rows, int64_t nrows,
                     const float *k, const float *v, int Hq, int Hkv, int64_t N, int D,
                     double base, double kwin, double *out, double *lse) {
    return orc_prefill_rows_masked(q_rows, rows, nrows, k, v, Hq, Hkv, N, D, base, kwin, NULL, 0, out, lse);
}

/*
 * The same under a token-level block selection: block_mask [Hkv][T][T] with
 * T = ceil(N / tile); entry (g, i, j) != 0 makes key tile j visible to query
 * tile i for the query heads of KV head g (entries j > i only ever cover keys
 * past the query and so change nothing; the diagonal entry is ignored: the
 * diagonal tile is always visible).
 */
int orc_prefill_rows_sparse(const float *q_rows, const int64_t *rows, int64_t nrows,
                            const float *k, const float *v, int Hq, int Hkv, int64_t N, int D,
                            double base, double kwin, const unsigned char *block_mask, int64_t tile,
                            double *out, double *lse) {
    if (!block_mask) return -1;
    return orc_prefill_rows_masked(q_rows, rows, nrows, k, v, Hq, Hkv, N, D, base, kwin, block_mask, tile, out,
                                   lse);
}

/*
 * Decode: one query token per sequence b at position L_b - 1 = seqlens[b] - 1,
 * attending keys 0 .. L_b - 1 of a contiguous cache.
 *   q [B][Hq][D] (un-rotated), kcache, vcache [B][Hkv][Nmax][D],
 *   krot = 1 if kcache already holds rotated keys (then it is used as is).
 *   out [B][Hq][D], lse [B][Hq] (may be NULL).
 */
int orc_decode(const float *q, const float *kcache, const float *vcache, const int32_t *seqlens,
               int B, int Hq, int Hkv, int64_t Nmax, int D, double base, double kwin, int krot,
               double *out, double *lse) {
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv || D <= 0 || D % 2 || Nmax <= 0 || B <= 0) return -1;
    int G = Hq / Hkv;
    int H = D / 2;
    double *lim = (double *)malloc(sizeof(double) * (size_t)H);
    orc_window_limits(D, base, kwin, lim);
    int rc = 0;
    for (int b = 0; b < B && rc == 0; ++b) {
        int64_t L = seqlens[b];
        if (L <= 0 || L > Nmax) { rc = -1; break; }
        for (int g = 0; g < Hkv && rc == 0; ++g) {
            size_t base_off = ((size_t)b * Hkv + g) * (size_t)Nmax * D;
            double *kt = orc_rotated_keys(kcache + base_off, D, L, D, base, krot);
            if (!kt) { rc = -1; break; }
            double *scores = (double *)malloc(sizeof(double) * (size_t)L);
            double *qt = (double *)malloc(sizeof(double) * (size_t)D);
            for (int j = 0; j < G; ++j) {
                int h = g * G + j;
                orc_rope(q + ((size_t)b * Hq + h) * D, D, base, L - 1, qt);
                orc_row(qt, kt, vcache + base_off, D, L - 1, D, lim, NULL, 0, scores,
                        out + ((size_t)b * Hq + h) * D, lse ? lse + (size_t)b * Hq + h : NULL);
            }
            free(scores);
            free(qt);
            free(kt);
        }
    }
    free(lim);
    return rc;
}

/* Rotate-half RoPE of rows of D-vectors at the given positions (exposed so the
 * tests can pin the rotation against the relative-angle identity). */
void orc_rope_rows(const float *x, const int64_t *pos, int64_t nrows, int D, double base, double *y) {
    for (int64_t i = 0; i < nrows; ++i) orc_rope(x + (size_t)i * D, D, base, pos[i], y + (size_t)i * D);
}

/* Windowed score matrix of one head, all causal cells (small N only):
 * s[n][m] for m <= n, 0 above the diagonal.  Exposed for pinning. */
void orc_scores(const float *q, const float *k, int64_t N, int D, double base, double kwin, double *s) {
    int H = D / 2;
    double *lim = (double *)malloc(sizeof(double) * (size_t)H);
    orc_window_limits(D, base, kwin, lim);
    double *qt = (double *)malloc(sizeof(double) * (size_t)N * D);
    double *kt = (double *)malloc(sizeof(double) * (size_t)N * D);
    for (int64_t n = 0; n < N; ++n) {
        orc_rope(q + (size_t)n * D, D, base, n, qt + (size_t)n * D);
        orc_rope(k + (size_t)n * D, D, base, n, kt + (size_t)n * D);
    }
    for (int64_t n = 0; n < N; ++n)
        for (int64_t m = 0; m < N; ++m)
            s[(size_t)n * N + m] = (m <= n) ? orc_score(qt + (size_t)n * D, kt + (size_t)m * D, D, lim, n - m) : 0.0;
    free(qt);
    free(kt);
    free(lim);
}
