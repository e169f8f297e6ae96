/*
 * QuEST oracle: a plain, slow, deliberately literal CPU implementation of the
 * QuEST quantizer, trust-mask backward and integer linear layer, in fp64 / int64.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test-suite, the package smoke check and
 * the benchmark's CPU-baseline leg may load this library. The product (the CUDA
 * library) shares no code with it and never calls it.
 *
 * What it follows (method source: "QuEST: Stable Training of LLMs with 1-Bit
 * Weights and Activations", Panferov et al., arXiv 2502.05003):
 *   - pith.science review, "What carries the argument": a Hadamard transform of
 *     weights and activations, projection onto a uniform grid whose scale
 *     minimises the L2 error against a standard Gaussian, and a backward pass
 *     that multiplies the gradient *in the Hadamard domain* by a binary mask
 *     zeroing entries whose quantization error exceeds half an interval.
 *   - atlas.scime.ai summary, "Approach": Hadamard transform with RMS
 *     normalisation, MSE-optimal clipping fitted to a Gaussian, trust threshold.
 *   - pith.science review, "Assumptions & free parameters": after RMS
 *     normalisation the data is treated as N(0,1) plus tails; alpha* comes from
 *     a fixed N(0,1) target; Hadamard matrices are orthogonal, so a transform
 *     applied to both matmul operands leaves the product unchanged.
 *   - pith.science review, Figure 2 caption: two Hadamard transforms on the
 *     forward pass, two inverse transforms on the backward pass.
 *
 * Readings where the pages are silent (each is listed with its reason in the
 * design notes of the repository):
 *   - Hadamard matrix: Sylvester order, H[i][j] = (-1)^popcount(i & j),
 *     normalised by 1/sqrt(n); the inverse is the same matrix (symmetric,
 *     orthogonal).
 *   - RMS is taken over the transformed values y of an "rms group" (a multiple
 *     of the Hadamard block that divides the row).
 *   - Grid: symmetric midrise, 2^b levels at (i + 1/2) * Delta,
 *     i = -2^(b-1) .. 2^(b-1)-1, Delta = alpha_b * r / 2^(b-1).
 *   - alpha_b = 2^(b-1) * Delta*, Delta* the step minimising the Gaussian MSE.
 *   - Code q = clamp(floor(y / Delta)); mask m = [ |t - (q + 1/2)| <= T/2 ].
 *   - A group with r == 0 gives Delta = 0, q = 0, dequant 0, m = 1.
 *   - No gradient flows through r.
 *   - GEMM operand form c = 2q + 1, Y = acc * Delta_x * Delta_w / 4.
 *
 * Every computation is the definition written out: an explicit n x n Hadamard
 * matrix and an O(n^2) matrix-vector product per block, a golden-section
 * minimisation of the closed-form Gaussian MSE, and a triple-loop integer GEMM.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL -1

/* ------------------------------------------------------------------------- */
/* Hadamard matrix (Sylvester construction, natural order).                   */
/* ------------------------------------------------------------------------- */

static int popcount_int(unsigned v) {
    int c = 0;
    while (v) {
        c += (int)(v & 1u);
        v >>= 1;
    }
    return c;
}

static int is_pow2(int64_t n) { return n > 0 && (n & (n - 1)) == 0; }

/* Fills H (n x n, row-major) with the UNNORMALISED entries (-1)^popcount(i&j). */
int oracle_hadamard(int n, double* H) {
    if (!is_pow2(n) || n > 4096) return ORACLE_EINVAL;
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j)
            H[(int64_t)i * n + j] = (popcount_int((unsigned)(i & j)) & 1) ? -1.0 : 1.0;
    return ORACLE_OK;
}

/* y = (1/sqrt(n)) * H * x for one block; H is the unnormalised matrix. */
static void hadamard_block(const double* H, int n, const double* x, double* y) {
    const double norm = 1.0 / sqrt((double)n);
    for (int i = 0; i < n; ++i) {
        double acc = 0.0;
        for (int j = 0; j < n; ++j) acc += H[(int64_t)i * n + j] * x[j];
        y[i] = acc * norm;
    }
}

/* ------------------------------------------------------------------------- */
/* Gaussian MSE of the midrise uniform quantizer and its minimiser.           */
/* ------------------------------------------------------------------------- */

static double phi(double x) { return exp(-0.5 * x * x) / sqrt(2.0 * M_PI); }

/* P(a <= X < b) for X ~ N(0,1); b may be +INFINITY. */
static double gauss_mass(double a, double b) {
    double ub = isinf(b) ? 0.0 : erfc(b / sqrt(2.0));
    return 0.5 * (erfc(a / sqrt(2.0)) - ub);
}

/* Integral over [a, b) of (x - c)^2 phi(x) dx, using
 *   int x^2 phi = [Phi] + a phi(a) - b phi(b),   int x phi = phi(a) - phi(b). */
static double cell_sq_error(double a, double b, double c) {
    double mass = gauss_mass(a, b);
    double pa = phi(a);
    double pb = isinf(b) ? 0.0 : phi(b);
    double bpb = isinf(b) ? 0.0 : b * pb;
    double m2 = mass + a * pa - bpb;
    double m1 = pa - pb;
    return m2 - 2.0 * c * m1 + c * c * mass;
}

/* E[(X - Q(X))^2], X ~ N(0,1), Q the 2^bits-level midrise quantizer of step
 * delta: levels (i + 1/2) delta, decision thresholds at integer multiples of
 * delta, outermost cells open to +-infinity. Uses the symmetry X -> -X. */
double oracle_gauss_mse(int bits, double delta) {
    if (bits < 1 || bits > 16 || !(delta > 0.0)) return NAN;
    const int half = 1 << (bits - 1);
    double total = 0.0;
    for (int i = 0; i < half; ++i) {
        double a = i * delta;
        double b = (i == half - 1) ? INFINITY : (i + 1) * delta;
        double c = (i + 0.5) * delta;
        total += cell_sq_error(a, b, c);
    }
    return 2.0 * total;
}

/* Golden-section minimisation of oracle_gauss_mse over delta in [lo, hi]. */
static double golden_min(int bits, double lo, double hi, double tol) {
    const double g = (sqrt(5.0) - 1.0) / 2.0;
    double a = lo, b = hi;
    double c = b - g * (b - a), d = a + g * (b - a);
    double fc = oracle_gauss_mse(bits, c), fd = oracle_gauss_mse(bits, d);
    while (b - a > tol) {
        if (fc < fd) {
            b = d; d = c; fd = fc;
            c = b - g * (b - a); fc = oracle_gauss_mse(bits, c);
        } else {
            a = c; c = d; fc = fd;
            d = a + g * (b - a); fd = oracle_gauss_mse(bits, d);
        }
    }
    return 0.5 * (a + b);
}

/* alpha_b = 2^(b-1) * argmin_delta MSE(delta): the clip edge of the grid.
 * Also returns the optimal step and the minimal Gaussian MSE. */
int oracle_alpha(int bits, double* alpha, double* delta_opt, double* mse_opt) {
    if (bits < 1 || bits > 16) return ORACLE_EINVAL;
    double d = golden_min(bits, 1e-4, 4.0, 1e-13);
    if (alpha) *alpha = ldexp(d, bits - 1);
    if (delta_opt) *delta_opt = d;
    if (mse_opt) *mse_opt = oracle_gauss_mse(bits, d);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* Forward quantizer.                                                         */
/* ------------------------------------------------------------------------- */

/* Distance from t to the nearest point where the mask value changes, given
 * the code cell q(t). Flip points are c +- T/2 (c = q + 1/2) that lie inside
 * the t-range of their own cell; the element's own cell and both neighbours are
 * searched. */
static double mask_flip_distance(double t, int q, int lo, int hi, double trust) {
    double best = INFINITY;
    for (int k = q - 1; k <= q + 1; ++k) {
        if (k < lo || k > hi) continue;
        double cell_lo = (k == lo) ? -INFINITY : (double)k;
        double cell_hi = (k == hi) ? INFINITY : (double)(k + 1);
        double c = k + 0.5;
        double f[2] = {c - 0.5 * trust, c + 0.5 * trust};
        for (int s = 0; s < 2; ++s)
            if (f[s] > cell_lo && f[s] < cell_hi) {
                double dd = fabs(t - f[s]);
                if (dd < best) best = dd;
            }
    }
    return best;
}

/*
 * Quantizes x [rows, cols] (row stride ld, fp64 values) block by block.
 *   had       Hadamard block size (power of two), divides cols.
 *   rms_group RMS group length (multiple of had, divides cols).
 *   bits      1..8; trust T > 0; alpha the grid clip for this bit-width.
 * Outputs (all dense, row-major, may be NULL unless stated):
 *   y      [rows, cols]   transformed values (Hadamard domain)
 *   t      [rows, cols]   pre-round value y / Delta (0 where Delta == 0)
 *   q      [rows, cols]   integer code                        (required)
 *   yhat   [rows, cols]   dequantised value (q + 1/2) Delta, Hadamard domain
 *   mask   [rows, cols]   1 = gradient kept, 0 = zeroed
 *   scale  [rows, cols / rms_group]   Delta per group
 *   d_round [rows, cols]  distance of t to the nearest code decision boundary
 *   d_mask  [rows, cols]  distance of t to the nearest mask flip point
 */
int oracle_quantize(const double* x, int64_t rows, int64_t cols, int64_t ld, int had,
                    int64_t rms_group, int bits, double trust, double alpha, double* y_out,
                    double* t_out, int32_t* q, double* yhat, uint8_t* mask, double* scale,
                    double* d_round, double* d_mask) {
    if (rows < 0 || cols <= 0 || ld < cols || !is_pow2(had) || cols % had != 0) return ORACLE_EINVAL;
    if (rms_group <= 0 || rms_group % had != 0 || cols % rms_group != 0) return ORACLE_EINVAL;
    if (bits < 1 || bits > 8 || !(trust > 0.0) || !(alpha > 0.0) || q == NULL) return ORACLE_EINVAL;

    const int lo = -(1 << (bits - 1)), hi = (1 << (bits - 1)) - 1;
    const double levels_half = ldexp(1.0, bits - 1);
    double* H = (double*)malloc(sizeof(double) * had * had);
    double* y = (double*)malloc(sizeof(double) * cols);
    if (!H || !y) { free(H); free(y); return ORACLE_EINVAL; }
    oracle_hadamard(had, H);

    for (int64_t r = 0; r < rows; ++r) {
        const double* xr = x + r * ld;
        /* Step 1: blockwise Hadamard transform of the row. */
        for (int64_t b0 = 0; b0 < cols; b0 += had) hadamard_block(H, had, xr + b0, y + b0);

        for (int64_t g0 = 0; g0 < cols; g0 += rms_group) {
            /* Step 2: RMS of the transformed values of the group. */
            double ss = 0.0;
            for (int64_t j = 0; j < rms_group; ++j) ss += y[g0 + j] * y[g0 + j];
            double rms = sqrt(ss / (double)rms_group);
            /* Step 3: Gaussian-fitted step. */
            double delta = alpha * rms / levels_half;
            if (scale) scale[r * (cols / rms_group) + g0 / rms_group] = delta;
            /* Step 4: project onto the grid; step 5: trust mask. */
            for (int64_t j = 0; j < rms_group; ++j) {
                int64_t idx = r * cols + g0 + j;
                double yv = y[g0 + j];
                double tv, dr, dm;
                int qv;
                uint8_t mv;
                if (delta == 0.0) {
                    tv = 0.0; qv = 0; mv = 1; dr = INFINITY; dm = INFINITY;
                } else {
                    tv = yv / delta;
                    double fl = floor(tv);
                    if (fl < lo) fl = lo;
                    if (fl > hi) fl = hi;
                    qv = (int)fl;
                    double err = fabs(tv - (qv + 0.5));
                    mv = (err <= 0.5 * trust) ? 1 : 0;
                    /* nearest interior code boundary: integers lo+1 .. hi */
                    double k = nearbyint(tv);
                    if (k < lo + 1) k = lo + 1;
                    if (k > hi) k = hi;
                    dr = (hi > lo) ? fabs(tv - k) : INFINITY;
                    dm = mask_flip_distance(tv, qv, lo, hi, trust);
                }
                if (y_out) y_out[idx] = yv;
                if (t_out) t_out[idx] = tv;
                q[idx] = qv;
                if (yhat) yhat[idx] = (qv + 0.5) * delta;
                if (mask) mask[idx] = mv;
                if (d_round) d_round[idx] = dr;
                if (d_mask) d_mask[idx] = dm;
            }
        }
    }
    free(H);
    free(y);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* 2:4-sparse INT4 variant.                                                   */
/*                                                                           */
/* The pages evaluate QuEST on 2:4-sparse INT4 (atlas.scime.ai summary,        */
/* ablation table: adding 2:4 sparsity to QuEST INT4 hurts accuracy;           */
/* pith.science review, results list and Figure 4a: INT, FP and INT+sparse     */
/* formats at 4 bits) without spelling the format out. Reading: the same       */
/* Hadamard transform and RMS (over every value of the rms group); then, in    */
/* each run of four consecutive transformed values along the row, the two of   */
/* largest magnitude are kept (on equal magnitudes the lower index wins) and   */
/* the other two become zero; kept values go onto the b-bit midrise grid whose */
/* step minimises the MSE of the KEPT values when the input is N(0,1) (the     */
/* Gaussian fit of this format); the trust mask applies the half-interval rule */
/* to each value's total error, so a pruned value (rebuilt as 0) keeps its     */
/* gradient iff |t| <= T/2.                                                   */
/* ------------------------------------------------------------------------- */

/* Density of the magnitude a of a kept value: four iid N(0,1) values, the two
 * largest magnitudes kept. With F(a) = erf(a / sqrt 2) the half-normal CDF and
 * f(a) = 2 phi(a) its density, the k-th smallest of four magnitudes has density
 * 4!/((k-1)!(4-k)!) F^(k-1) (1-F)^(4-k) f; a kept value is the 3rd or the 4th
 * with probability 1/2 each: (12 F^2 (1-F) + 4 F^3) f / 2 = (6 F^2 - 4 F^3) f. */
static double kept_density(double a) {
    double F = erf(a / sqrt(2.0));
    return (6.0 * F * F - 4.0 * F * F * F) * 2.0 * phi(a);
}

/* Integral over [a, b] of (x - c)^2 kept_density(x) dx, composite Simpson. */
static double kept_cell_sq_error(double a, double b, double c) {
    const int n = 2000;                       /* even */
    const double h = (b - a) / n;
    double acc = 0.0;
    for (int i = 0; i <= n; ++i) {
        double x = a + i * h;
        double w = (i == 0 || i == n) ? 1.0 : ((i & 1) ? 4.0 : 2.0);
        acc += w * (x - c) * (x - c) * kept_density(x);
    }
    return acc * h / 3.0;
}

/* E[(X - Q(X))^2 | X kept], Q the 2^bits-level midrise quantizer of step delta
 * (levels (i + 1/2) delta, thresholds at multiples of delta, outer cells open).
 * The grid and the kept-value law are both symmetric, so the integral runs over
 * magnitudes; the open outer cell is cut 40 beyond its start (the density there
 * is below 1e-300). */
double oracle_sparse24_mse(int bits, double delta) {
    if (bits < 1 || bits > 8 || !(delta > 0.0)) return NAN;
    const int half = 1 << (bits - 1);
    double total = 0.0;
    for (int i = 0; i < half; ++i) {
        double a = i * delta;
        double b = (i == half - 1) ? a + 40.0 : (i + 1) * delta;
        total += kept_cell_sq_error(a, b, (i + 0.5) * delta);
    }
    return total;
}

/* alpha_b of the 2:4-sparse format: 2^(b-1) times the step minimising
 * oracle_sparse24_mse (golden section). */
int oracle_sparse24_alpha(int bits, double* alpha, double* delta_opt, double* mse_opt) {
    if (bits < 1 || bits > 8) return ORACLE_EINVAL;
    const double g = (sqrt(5.0) - 1.0) / 2.0;
    double a = 1e-3, b = 6.0;
    double c = b - g * (b - a), d = a + g * (b - a);
    double fc = oracle_sparse24_mse(bits, c), fd = oracle_sparse24_mse(bits, d);
    while (b - a > 1e-11) {
        if (fc < fd) {
            b = d; d = c; fd = fc;
            c = b - g * (b - a); fc = oracle_sparse24_mse(bits, c);
        } else {
            a = c; c = d; fc = fd;
            d = a + g * (b - a); fd = oracle_sparse24_mse(bits, d);
        }
    }
    double dopt = 0.5 * (a + b);
    if (alpha) *alpha = ldexp(dopt, bits - 1);
    if (delta_opt) *delta_opt = dopt;
    if (mse_opt) *mse_opt = oracle_sparse24_mse(bits, dopt);
    return ORACLE_OK;
}

/*
 * 2:4-sparse quantizer of x [rows, cols] (row stride ld), cols a multiple of 4.
 * Outputs as oracle_quantize, plus:
 *   kept    [rows, cols]  1 where the value survives the pruning  (required)
 *   q       [rows, cols]  the code of a kept value, 0 for a pruned one (required)
 *   yhat    [rows, cols]  (q + 1/2) Delta for kept values, 0 for pruned ones
 *   d_round [rows, cols]  kept: distance of t to the nearest code boundary; pruned: inf
 *   d_mask  [rows, cols]  distance of t to the nearest flip point of its mask rule
 *   d_prune [rows, cols]  for every value of a run of four: the gap between the
 *                         2nd and 3rd largest |t| of the run (where the choice of
 *                         kept values would change)
 */
int oracle_quantize_sparse24(const double* x, int64_t rows, int64_t cols, int64_t ld, int had,
                             int64_t rms_group, int bits, double trust, double alpha, double* y_out,
                             double* t_out, int32_t* q, uint8_t* kept, double* yhat, uint8_t* mask,
                             double* scale, double* d_round, double* d_mask, double* d_prune) {
    if (rows < 0 || cols <= 0 || ld < cols || !is_pow2(had) || had < 4 || cols % had != 0) return ORACLE_EINVAL;
    if (rms_group <= 0 || rms_group % had != 0 || cols % rms_group != 0) return ORACLE_EINVAL;
    if (bits < 1 || bits > 8 || !(trust > 0.0) || !(alpha > 0.0) || q == NULL || kept == NULL)
        return ORACLE_EINVAL;

    const int lo = -(1 << (bits - 1)), hi = (1 << (bits - 1)) - 1;
    const double levels_half = ldexp(1.0, bits - 1);
    double* H = (double*)malloc(sizeof(double) * had * had);
    double* y = (double*)malloc(sizeof(double) * cols);
    if (!H || !y) { free(H); free(y); return ORACLE_EINVAL; }
    oracle_hadamard(had, H);

    for (int64_t r = 0; r < rows; ++r) {
        const double* xr = x + r * ld;
        /* Step 1: blockwise Hadamard transform of the row. */
        for (int64_t b0 = 0; b0 < cols; b0 += had) hadamard_block(H, had, xr + b0, y + b0);
        for (int64_t g0 = 0; g0 < cols; g0 += rms_group) {
            /* Step 2: RMS over every transformed value of the group. */
            double ss = 0.0;
            for (int64_t j = 0; j < rms_group; ++j) ss += y[g0 + j] * y[g0 + j];
            double rms = sqrt(ss / (double)rms_group);
            /* Step 3: the step fitted to the kept values of a Gaussian input. */
            double delta = alpha * rms / levels_half;
            if (scale) scale[r * (cols / rms_group) + g0 / rms_group] = delta;
            for (int64_t j0 = 0; j0 < rms_group; j0 += 4) {
                /* Step 4: in the run of four, keep the two largest magnitudes. An
                 * element is kept when fewer than two others beat it (a larger
                 * magnitude, or an equal one at a lower index). */
                double mag[4];
                for (int i = 0; i < 4; ++i) mag[i] = fabs(y[g0 + j0 + i]);
                int keep[4];
                for (int i = 0; i < 4; ++i) {
                    int beaten = 0;
                    for (int k = 0; k < 4; ++k)
                        if (k != i && (mag[k] > mag[i] || (mag[k] == mag[i] && k < i))) ++beaten;
                    keep[i] = beaten < 2;
                }
                /* the 2nd and 3rd largest magnitudes, for the exemption distance */
                double srt[4];
                for (int i = 0; i < 4; ++i) srt[i] = mag[i];
                for (int i = 0; i < 4; ++i)
                    for (int k = i + 1; k < 4; ++k)
                        if (srt[k] > srt[i]) { double tmp = srt[i]; srt[i] = srt[k]; srt[k] = tmp; }
                double gap = (delta == 0.0) ? INFINITY : (srt[1] - srt[2]) / delta;
                /* Step 5: project the kept values onto the grid; step 6: trust mask. */
                for (int i = 0; i < 4; ++i) {
                    int64_t idx = r * cols + g0 + j0 + i;
                    double yv = y[g0 + j0 + i];
                    double tv = 0.0, dr = INFINITY, dm = INFINITY, yh = 0.0;
                    int qv = 0;
                    uint8_t mv = 1;
                    if (delta != 0.0) {
                        tv = yv / delta;
                        if (keep[i]) {
                            double fl = floor(tv);
                            if (fl < lo) fl = lo;
                            if (fl > hi) fl = hi;
                            qv = (int)fl;
                            mv = (fabs(tv - (qv + 0.5)) <= 0.5 * trust) ? 1 : 0;
                            double k = nearbyint(tv);
                            if (k < lo + 1) k = lo + 1;
                            if (k > hi) k = hi;
                            dr = (hi > lo) ? fabs(tv - k) : INFINITY;
                            dm = mask_flip_distance(tv, qv, lo, hi, trust);
                            yh = (qv + 0.5) * delta;
                        } else {
                            mv = (fabs(tv) <= 0.5 * trust) ? 1 : 0;
                            dm = fabs(fabs(tv) - 0.5 * trust);
                        }
                    }
                    if (y_out) y_out[idx] = yv;
                    if (t_out) t_out[idx] = tv;
                    q[idx] = qv;
                    kept[idx] = (uint8_t)keep[i];
                    if (yhat) yhat[idx] = yh;
                    if (mask) mask[idx] = mv;
                    if (d_round) d_round[idx] = dr;
                    if (d_mask) d_mask[idx] = dm;
                    if (d_prune) d_prune[idx] = gap;
                }
            }
        }
    }
    free(H);
    free(y);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* FP4 (E2M1) grid variant.                                                   */
/*                                                                           */
/* The pages evaluate QuEST on an FP4 grid as well as the INT4 one (pith.science */
/* review, "What carries the argument" and its results list) without spelling */
/* the variant out. Reading: the same Hadamard transform and RMS, the grid is   */
/* the 15 signed E2M1 values scaled by Delta = s* r, s* minimising the Gaussian */
/* MSE of round-to-nearest onto that grid, and the trust mask keeps an element  */
/* whose error is at most T/2 of the grid interval that holds it (the last one, */
/* [4, 6], beyond the grid).                                                  */
/* ------------------------------------------------------------------------- */

/* Value of a 4-bit E2M1 code: bit 3 sign, bits 2..1 exponent (bias 1), bit 0
 * mantissa; exponent 0 is subnormal (0 or 0.5). No infinities or NaNs. */
double oracle_e2m1_value(int code) {
    int sign = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return sign ? -mag : mag;
}

/* The 8 non-negative grid magnitudes in increasing order (codes 0..7). */
static void e2m1_magnitudes(double v[8]) {
    for (int c = 0; c < 8; ++c) v[c] = oracle_e2m1_value(c);
}

/* E[(X - s Q(X / s))^2] for X ~ N(0,1), Q round-to-nearest onto the E2M1 grid
 * (saturating at +-6): cell k of the positive side runs from the midpoint
 * below level k to the midpoint above it, the last cell is open. */
double oracle_fp4_gauss_mse(double s) {
    if (!(s > 0.0)) return NAN;
    double v[8];
    e2m1_magnitudes(v);
    double total = 0.0;
    for (int k = 0; k < 8; ++k) {
        double a = (k == 0) ? 0.0 : 0.5 * (v[k - 1] + v[k]) * s;
        double b = (k == 7) ? INFINITY : 0.5 * (v[k] + v[k + 1]) * s;
        total += cell_sq_error(a, b, v[k] * s);
    }
    return 2.0 * total;
}

/* s* = argmin_s oracle_fp4_gauss_mse(s), golden section over [lo, hi]. */
int oracle_fp4_scale(double* s_opt, double* mse_opt) {
    const double g = (sqrt(5.0) - 1.0) / 2.0;
    double a = 0.01, b = 2.0;
    double c = b - g * (b - a), d = a + g * (b - a);
    double fc = oracle_fp4_gauss_mse(c), fd = oracle_fp4_gauss_mse(d);
    while (b - a > 1e-13) {
        if (fc < fd) {
            b = d; d = c; fd = fc;
            c = b - g * (b - a); fc = oracle_fp4_gauss_mse(c);
        } else {
            a = c; c = d; fc = fd;
            d = a + g * (b - a); fd = oracle_fp4_gauss_mse(d);
        }
    }
    double sv = 0.5 * (a + b);
    if (s_opt) *s_opt = sv;
    if (mse_opt) *mse_opt = oracle_fp4_gauss_mse(sv);
    return ORACLE_OK;
}

/* Round-to-nearest of t onto the E2M1 grid by search over all 16 codes; a tie
 * goes to the code with mantissa bit 0 (nearest-even). The sign bit is the sign
 * bit of t, so small negative t gives the code of -0. */
int oracle_e2m1_round(double t) {
    int best = -1;
    double bd = INFINITY;
    for (int c = 0; c < 8; ++c) {
        double d = fabs(fabs(t) - oracle_e2m1_value(c));
        if (d < bd || (d == bd && (c & 1) == 0)) { bd = d; best = c; }
    }
    return best | (signbit(t) ? 8 : 0);
}

/* Width of the grid interval that holds |t| (the last interval beyond 6). */
static double e2m1_interval(double t) {
    double v[8], a = fabs(t);
    e2m1_magnitudes(v);
    for (int k = 0; k < 7; ++k)
        if (a < v[k + 1]) return v[k + 1] - v[k];
    return v[7] - v[6];
}

/*
 * FP4-grid quantizer, same argument conventions as oracle_quantize; `s_opt` is
 * the Gaussian-optimal scale of the grid (Delta = s_opt * rms). Outputs:
 *   code  [rows, cols]  4-bit E2M1 code (required)
 *   value [rows, cols]  Q(t), the grid value of the code
 *   yhat = value * Delta; mask; scale = Delta; t; y;
 *   d_round  distance of t to the nearest decision point (a midpoint between
 *            neighbouring grid values, or 0 where the sign bit flips)
 *   d_mask   distance of t to the nearest point where the mask changes
 */
int oracle_quantize_fp4(const double* x, int64_t rows, int64_t cols, int64_t ld, int had,
                        int64_t rms_group, double trust, double s_opt, double* y_out, double* t_out,
                        uint8_t* code, double* value, double* yhat, uint8_t* mask, double* scale,
                        double* d_round, double* d_mask) {
    if (rows < 0 || cols <= 0 || ld < cols || !is_pow2(had) || cols % had != 0) return ORACLE_EINVAL;
    if (rms_group <= 0 || rms_group % had != 0 || cols % rms_group != 0) return ORACLE_EINVAL;
    if (!(trust > 0.0) || !(s_opt > 0.0) || code == NULL) return ORACLE_EINVAL;

    double v[8];
    e2m1_magnitudes(v);
    double* H = (double*)malloc(sizeof(double) * had * had);
    double* y = (double*)malloc(sizeof(double) * cols);
    if (!H || !y) { free(H); free(y); return ORACLE_EINVAL; }
    oracle_hadamard(had, H);

    for (int64_t r = 0; r < rows; ++r) {
        const double* xr = x + r * ld;
        for (int64_t b0 = 0; b0 < cols; b0 += had) hadamard_block(H, had, xr + b0, y + b0);
        for (int64_t g0 = 0; g0 < cols; g0 += rms_group) {
            double ss = 0.0;
            for (int64_t j = 0; j < rms_group; ++j) ss += y[g0 + j] * y[g0 + j];
            double delta = s_opt * sqrt(ss / (double)rms_group);
            if (scale) scale[r * (cols / rms_group) + g0 / rms_group] = delta;
            for (int64_t j = 0; j < rms_group; ++j) {
                int64_t idx = r * cols + g0 + j;
                double yv = y[g0 + j], tv, qv, dr, dm;
                int cv;
                uint8_t mv;
                if (delta == 0.0) {
                    tv = 0.0; cv = 0; qv = 0.0; mv = 1; dr = INFINITY; dm = INFINITY;
                } else {
                    tv = yv / delta;
                    cv = oracle_e2m1_round(tv);
                    qv = oracle_e2m1_value(cv);
                    mv = (fabs(tv - qv) <= 0.5 * trust * e2m1_interval(tv)) ? 1 : 0;
                    /* decision points: 0 and the midpoints between neighbours */
                    double a = fabs(tv);
                    dr = a;
                    for (int k = 0; k < 7; ++k) {
                        double d = fabs(a - 0.5 * (v[k] + v[k + 1]));
                        if (d < dr) dr = d;
                    }
                    /* mask flips: 6 + T beyond the grid; for T < 1 also
                     * v_k + (T/2) w_k and v_(k+1) - (T/2) w_k in each interval */
                    dm = fabs(a - (v[7] + 0.5 * trust * (v[7] - v[6])));
                    if (trust < 1.0)
                        for (int k = 0; k < 7; ++k) {
                            double w = v[k + 1] - v[k];
                            double f0 = v[k] + 0.5 * trust * w, f1 = v[k + 1] - 0.5 * trust * w;
                            if (fabs(a - f0) < dm) dm = fabs(a - f0);
                            if (fabs(a - f1) < dm) dm = fabs(a - f1);
                        }
                }
                if (y_out) y_out[idx] = yv;
                if (t_out) t_out[idx] = tv;
                code[idx] = (uint8_t)cv;
                if (value) value[idx] = qv;
                if (yhat) yhat[idx] = qv * delta;
                if (mask) mask[idx] = mv;
                if (d_round) d_round[idx] = dr;
                if (d_mask) d_mask[idx] = dm;
            }
        }
    }
    free(H);
    free(y);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* Trust backward: g_x = H^T (m . g) / sqrt(n) per Hadamard block.            */
/* ------------------------------------------------------------------------- */

int oracle_trust_bwd(const double* g, const uint8_t* mask, int64_t rows, int64_t cols, int had,
                     double* gx) {
    if (rows < 0 || cols <= 0 || !is_pow2(had) || cols % had != 0) return ORACLE_EINVAL;
    double* H = (double*)malloc(sizeof(double) * had * had);
    double* mg = (double*)malloc(sizeof(double) * had);
    if (!H || !mg) { free(H); free(mg); return ORACLE_EINVAL; }
    oracle_hadamard(had, H);
    const double norm = 1.0 / sqrt((double)had);
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b0 = 0; b0 < cols; b0 += had) {
            const int64_t base = r * cols + b0;
            for (int j = 0; j < had; ++j) mg[j] = mask[base + j] ? g[base + j] : 0.0;
            /* transpose product: out[i] = sum_j H[j][i] * mg[j] */
            for (int i = 0; i < had; ++i) {
                double acc = 0.0;
                for (int j = 0; j < had; ++j) acc += H[(int64_t)j * had + i] * mg[j];
                gx[base + i] = acc * norm;
            }
        }
    free(H);
    free(mg);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* Integer linear layer.                                                      */
/* ------------------------------------------------------------------------- */

/* acc[m][n] = sum_k A[m][k] * B[n][k]  (A: [M,K], B: [N,K], both K-contiguous). */
int oracle_gemm_i8(const int8_t* A, const int8_t* B, int64_t M, int64_t N, int64_t K,
                   int64_t* acc) {
    if (M < 0 || N < 0 || K < 0) return ORACLE_EINVAL;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k) s += (int64_t)A[m * K + k] * (int64_t)B[n * K + k];
            acc[m * N + n] = s;
        }
    return ORACLE_OK;
}

/* Y[m][n] = acc[m][n] * (Delta_a[m] / 2) * (Delta_b[n] / 2): the c = 2q+1 codes
 * carry a factor 2 each relative to (q + 1/2). */
int oracle_dequant_linear(const int64_t* acc, const double* delta_a, const double* delta_b,
                          int64_t M, int64_t N, double* y) {
    if (M < 0 || N < 0) return ORACLE_EINVAL;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            y[m * N + n] = (double)acc[m * N + n] * (delta_a[m] * 0.5) * (delta_b[n] * 0.5);
    return ORACLE_OK;
}

/* Linear layer with one scale per (row, group of `group` consecutive K
 * indices) on both operands:
 *   Y[m][n] = sum_g (Delta_a[m][g] / 2) * (Delta_b[n][g] / 2) * acc_g[m][n],
 *   acc_g[m][n] = sum over k in group g of A[m][k] * B[n][k]   (int64).
 * `mag` (nullable) receives sum_g |term_g|, the scale of the rounding error
 * of any finite-precision sum of the G terms. */
int oracle_linear_grouped(const int8_t* A, const int8_t* B, const double* delta_a,
                          const double* delta_b, int64_t M, int64_t N, int64_t K, int64_t group,
                          double* y, double* mag) {
    if (M < 0 || N < 0 || K < 0 || group <= 0 || K % group != 0) return ORACLE_EINVAL;
    const int64_t G = K / group;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double sum = 0.0, abs_sum = 0.0;
            for (int64_t g = 0; g < G; ++g) {
                int64_t acc = 0;
                for (int64_t k = g * group; k < (g + 1) * group; ++k)
                    acc += (int64_t)A[m * K + k] * (int64_t)B[n * K + k];
                const double term = (double)acc * (delta_a[m * G + g] * 0.5) * (delta_b[n * G + g] * 0.5);
                sum += term;
                abs_sum += fabs(term);
            }
            y[m * N + n] = sum;
            if (mag) mag[m * N + n] = abs_sum;
        }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* Rounding of an fp64 value to bfloat16, round-to-nearest-even, one rounding. */
/* ------------------------------------------------------------------------- */

uint16_t oracle_bf16_rne(double v) {
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isinf(a)) return sign | 0x7F80;
    if (a == 0.0) return sign;
    /* quantum of the bf16 grid at this magnitude: 8 significant bits for
     * normals (|a| >= 2^-126), fixed 2^-133 for subnormals. */
    int e;
    frexp(a, &e); /* a = f * 2^e, f in [0.5, 1) */
    double quantum = (a >= ldexp(1.0, -126)) ? ldexp(1.0, e - 8) : ldexp(1.0, -133);
    double k = a / quantum;              /* exact: quantum is a power of two */
    double kr = nearbyint(k);            /* default mode: ties to even */
    double rv = kr * quantum;
    if (rv >= ldexp(1.0, 128)) return sign | 0x7F80;
    float f = (float)rv;                 /* exact: rv has <= 8 significant bits */
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    return (uint16_t)(sign | (uint16_t)((bits >> 16) & 0x7FFF));
}

void oracle_bf16_rne_array(const double* v, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_rne(v[i]);
}
