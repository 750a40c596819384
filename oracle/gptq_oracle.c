/*
 * Float64 CPU oracle of the GPTQ layer quantizer -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline / reference
 * arm load this file's library.  It shares no code with the CUDA library and
 * is deliberately plain: every step below is the algorithm as the GPTQ pages
 * state it, one column at a time, with no blocking or reordering beyond what
 * the pages' own pseudo-code does.
 *
 * Sources (page titles; the text is the pages' restatement of OBQ/GPTQ):
 *  - "GPTQ (GPT Quantization)", section "Fondation theorique : OBQ":
 *      quantize column i, e_i = w_i - q_i,
 *      W_F <- W_F - e_i / (H^-1)_ii * (H^-1)_{i,F}.
 *  - same page, "Algorithme complet (pseudo-code)": H = 2 X^T X, H += lambda I,
 *    H^-1 through Cholesky, columns walked in batches with a lazy update of the
 *    remaining columns after each batch.
 *  - "Optimization Gptq" (AutoGPTQ guide), "Quantizacao group-wise": every
 *    group of consecutive weights has its own scale and zero-point.
 *
 * Readings where the pages are silent or garbled (each is restated beside the
 * code that depends on it):
 *  - (H^-1)_{i,F} is the inverse of the Hessian restricted to the columns not
 *    yet quantized: after column i is quantized it is eliminated from H^-1 by
 *    one Gaussian-elimination step (the OBQ derivation).
 *  - group parameters are taken at the group's first column from the current
 *    (already error-compensated) weights; the range always contains 0; an
 *    all-equal range becomes [-1, 1]; rounding is round-half-to-even.
 *  - the pseudo-code's lazy update divides by diag(H^-1) after the product; the
 *    shapes only fit with the division applied per column of Err before it,
 *    and the in-batch feedback of the OBQ step is kept.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Asymmetric min-max quantizer parameters of one group (AutoGPTQ guide,
 * "Quantizacao group-wise": own scale and zero point per group).
 *
 * Default (pure == 0): the range is widened to contain 0, so the integer zero
 * point lies in [0, 2^b - 1] and 0 is exactly representable.
 * pure != 0: the range is the group's own [min, max]; the zero point may lie
 * outside [0, 2^b - 1] (every code still does).  Two groups fall back to the
 * widened range: a constant group (its own range is empty) and one whose real
 * zero point lies more than 2^20 levels away (a range that narrow next to its
 * offset from zero is below the resolution of fp32 arithmetic on w / s). */
void orc_quant_params(const double *x, int64_t n, int bits, int pure, double *scale,
                      double *zero_real, int32_t *zero)
{
    double maxq = (double)((1 << bits) - 1);
    double xmin = 0.0, xmax = 0.0; /* widened: the range always contains 0 */
    if (pure && n > 0) {
        xmin = x[0];
        xmax = x[0];
    }
    for (int64_t k = 0; k < n; ++k) {
        if (x[k] < xmin) xmin = x[k];
        if (x[k] > xmax) xmax = x[k];
    }
    if (pure) {
        int widen = (xmax == xmin);
        if (!widen) widen = fabs(xmin / ((xmax - xmin) / maxq)) > 1048576.0;
        if (widen) {
            if (xmin > 0.0) xmin = 0.0;
            if (xmax < 0.0) xmax = 0.0;
        }
    }
    if (xmax == xmin) {
        /* all-zero group: the range becomes [-1, 1], so s = 2 / (2^b - 1) and
         * -xmin / s = (2^b - 1) / 2 exactly, a tie that rounds half to even
         * to 2^(b-1).  Taken exactly so that it does not depend on how the
         * division rounds; every code is then z and the group dequantizes
         * to exactly 0. */
        *scale = 2.0 / maxq;
        *zero_real = 0.5 * maxq;
        *zero = (int32_t)1 << (bits - 1);
        return;
    }
    double s = (xmax - xmin) / maxq;
    double zr = -xmin / s;
    *scale = s;
    *zero_real = zr;
    *zero = (int32_t)nearbyint(zr);
}

/* Code of one weight: clamp(rint(w / s) + z, 0, 2^bits - 1). */
int32_t orc_quantize(double w, double s, int32_t z, int bits)
{
    double maxq = (double)((1 << bits) - 1);
    double q = nearbyint(w / s) + (double)z;
    if (q < 0.0) q = 0.0;
    if (q > maxq) q = maxq;
    return (int32_t)q;
}

/* Validity of a candidate code c for the real level y = w / s + z: the oracle's
 * own rounding, or a neighbouring level whose rounding boundary lies within
 * tol of y (several codes are correct when w sits on a tie within tol). */
static int code_is_valid(int32_t c, int32_t q, double y, double tol, int bits)
{
    int32_t maxq = (1 << bits) - 1;
    if (c == q) return 1;
    if (c < 0 || c > maxq) return 0;
    return fabs((double)c - y) <= 0.5 + tol;
}

/*
 * The OBQ / GPTQ column loop, unbatched, with explicit per-column Gaussian
 * elimination of M = H^-1 ("GPTQ (GPT Quantization)", section
 * "Fondation theorique : OBQ").
 *
 *   W       r x d row-major.  In: the weights (dead columns zeroed, columns in
 *           quantization order).  Out: W[:, i] holds column i as it was when it
 *           was quantized (after the feedback of every earlier column).
 *   M       d x d row-major, in: inverse of the damped Hessian (only the upper
 *           triangle, j >= i, is read).  Destroyed.
 *   g       group size (1 <= g; a caller maps "-1" to d).
 *   pure    the group range rule of orc_quant_params (0: widened to 0).
 *   codes   r x d uint8; scales / zeros  [ceil(d/g)][r].
 *   U       optional d x d row-major (NULL to skip): row i receives the
 *           eliminated row of M scaled by 1/sqrt(M_ii), for columns >= i.
 *   fcodes, fzeros, fwpre, fscales  optional (NULL): another
 *           implementation's codes, zero points, pre-quantization weights and
 *           scales.  When given, the loop checks each code and zero point for
 *           validity and then continues with them (teacher forcing), so a
 *           legitimate tie decided the other way does not desynchronise the
 *           rest of the row.  The validity window of a code widens by the
 *           other side's own deviation in the decision's inputs:
 *           |w' - w| / s + |y - z| min(|s' - s| / s, stol) levels.
 *   tau     slack (in quantization levels) added to every validity window.
 *   stol    largest relative scale deviation accepted (a scale further off
 *           counts as invalid and widens no window beyond stol).
 *   stats   out [7]: code ties taken the other way, invalid codes, zero-point
 *           ties taken the other way, invalid zero points, elements compared,
 *           groups compared, invalid scales.
 *   max_dev out: max |fwpre - w| / s over all elements (0 without fwpre).
 *   first_tie  optional out [r]: per row, the first column whose code or
 *           (group-opening) zero point differs from the loop's own decision,
 *           d if none.  Until that column the forced run is the free run.
 */
int orc_gptq_columns(double *W, int64_t r, int64_t d, double *M, int bits,
                     int64_t g, int pure, uint8_t *codes, double *scales, int32_t *zeros,
                     double *U, const uint8_t *fcodes, const int32_t *fzeros,
                     const double *fwpre, const double *fscales, double tau, double stol,
                     int64_t *stats, double *max_dev, int64_t *first_tie)
{
    int64_t s_code_tie = 0, s_code_bad = 0, s_zero_tie = 0, s_zero_bad = 0;
    int64_t s_elems = 0, s_groups = 0, s_scale_bad = 0;
    double dev = 0.0;
    double *cur_s = (double *)malloc(sizeof(double) * (size_t)r);
    int32_t *cur_z = (int32_t *)malloc(sizeof(int32_t) * (size_t)r);
    double *coef = (double *)malloc(sizeof(double) * (size_t)r);
    /* a zero point that differs from the oracle's is judged at the end of its
     * group, against the drift the other side showed on that group's weights */
    double *zwin = (double *)calloc((size_t)r, sizeof(double));
    double *gdev = (double *)calloc((size_t)r, sizeof(double));
    double *sdev = (double *)calloc((size_t)r, sizeof(double));
    if (!cur_s || !cur_z || !coef || !zwin || !gdev || !sdev) {
        free(cur_s); free(cur_z); free(coef); free(zwin); free(gdev); free(sdev);
        return -1;
    }
    if (first_tie)
        for (int64_t row = 0; row < r; ++row) first_tie[row] = d;

    for (int64_t i = 0; i < d; ++i) {
        const double piv = M[i * d + i];
        if (!(piv > 0.0)) {
            free(cur_s); free(cur_z); free(coef); free(zwin); free(gdev); free(sdev);
            return -2;
        }
        const int64_t grp = i / g;
        const int new_group = (i % g) == 0;
        const int64_t gend = (grp * g + g < d) ? grp * g + g : d; /* end of i's group */

#pragma omp parallel for reduction(+:s_code_tie,s_code_bad,s_zero_tie,s_zero_bad,s_elems,s_groups,s_scale_bad) reduction(max:dev) schedule(static)
        for (int64_t row = 0; row < r; ++row) {
            double *w = W + row * d;
            if (new_group) {
                /* group parameters from the current weights of columns
                 * [i, i+g) of this row */
                double s, zr;
                int32_t z;
                orc_quant_params(w + i, gend - i, bits, pure, &s, &zr, &z);
                if (fscales) {
                    const double ds = fabs(fscales[grp * r + row] - s) / s;
                    if (ds > stol) ++s_scale_bad;
                    sdev[row] = ds < stol ? ds : stol;
                }
                if (fzeros) {
                    int32_t zf = fzeros[grp * r + row];
                    /* distance past the rounding window, judged at group end */
                    zwin[row] = (zf != z) ? fabs((double)zf - zr) - 0.5 - tau : -1.0;
                    if (zf != z) {
                        zwin[row] -= fabs(zr) * sdev[row];
                        if (first_tie && first_tie[row] > i) first_tie[row] = i;
                    }
                    gdev[row] = 0.0;
                    z = zf;
                    ++s_groups;
                }
                cur_s[row] = s;
                cur_z[row] = z;
                scales[grp * r + row] = s;
                zeros[grp * r + row] = z;
            }
            const double s = cur_s[row];
            const int32_t z = cur_z[row];
            const double wi = w[i];
            int32_t q = orc_quantize(wi, s, z, bits);
            if (fcodes) {
                const double y = wi / s + (double)z;
                double tol = tau;
                if (fwpre) {
                    double dv = fabs(fwpre[row * d + i] - wi) / s;
                    if (dv > dev) dev = dv;
                    if (dv > gdev[row]) gdev[row] = dv;
                    tol += dv;
                }
                tol += fabs(y - (double)z) * sdev[row];
                int32_t c = (int32_t)fcodes[row * d + i];
                if (c != q) {
                    if (code_is_valid(c, q, y, tol, bits)) ++s_code_tie;
                    else ++s_code_bad;
                    if (first_tie && first_tie[row] > i) first_tie[row] = i;
                }
                q = c;
                ++s_elems;
            }
            codes[row * d + i] = (uint8_t)q;
            if (fzeros && (i + 1 == gend) && zwin[row] >= 0.0) {
                if (zwin[row] <= gdev[row]) ++s_zero_tie;
                else ++s_zero_bad;
            }
            const double what = s * (double)(q - z);
            /* OBQ step: W_F <- W_F - e / M_ii * M_{i,F} */
            coef[row] = (wi - what) / piv;
        }

        /* feedback into the columns not yet quantized */
#pragma omp parallel for schedule(static)
        for (int64_t row = 0; row < r; ++row) {
            double *w = W + row * d;
            const double c = coef[row];
            const double *mi = M + i * d;
            for (int64_t f = i + 1; f < d; ++f) w[f] -= c * mi[f];
        }

        if (U) {
            const double inv_sqrt = 1.0 / sqrt(piv);
            for (int64_t f = 0; f < i; ++f) U[i * d + f] = 0.0;
            for (int64_t f = i; f < d; ++f) U[i * d + f] = M[i * d + f] * inv_sqrt;
        }

        /* eliminate column i from M: M_FF <- M_FF - M_Fi M_iF / M_ii.  Only
         * the upper triangle is stored; the update term is symmetric in
         * (a, b), so the matrix stays exactly symmetric. */
        const double inv_piv = 1.0 / piv;
#pragma omp parallel for schedule(dynamic, 16)
        for (int64_t a = i + 1; a < d; ++a) {
            const double mia = M[i * d + a];
            double *ma = M + a * d;
            const double *mi = M + i * d;
            for (int64_t b = a; b < d; ++b) ma[b] -= (mia * mi[b]) * inv_piv;
        }
    }
    if (stats) {
        stats[0] = s_code_tie; stats[1] = s_code_bad;
        stats[2] = s_zero_tie; stats[3] = s_zero_bad;
        stats[4] = s_elems; stats[5] = s_groups; stats[6] = s_scale_bad;
    }
    if (max_dev) *max_dev = dev;
    free(cur_s); free(cur_z); free(coef); free(zwin); free(gdev); free(sdev);
    return 0;
}

/*
 * The same column loop driven by the rows of U instead of an elimination of
 * M: with U upper and U^T U = H^-1, row i of the reduced inverse is
 * U_ii * U[i, i:], so the OBQ step is W_F <- W_F - (e / U_ii) U_{i,F}
 * (identical to orc_gptq_columns up to rounding; pinned against it).  For
 * large d, where the explicit elimination is too slow, U comes from a
 * library Cholesky factor of the library inverse.  Arguments as in
 * orc_gptq_columns, with U (d x d, row-major, upper) in place of M.
 */
int orc_gptq_columns_u(double *W, int64_t r, int64_t d, const double *U, int bits, int64_t g,
                       int pure, uint8_t *codes, double *scales, int32_t *zeros,
                       const uint8_t *fcodes, const int32_t *fzeros, const double *fwpre,
                       const double *fscales, double tau, double stol, int64_t *stats,
                       double *max_dev, int64_t *first_tie)
{
    int64_t s_code_tie = 0, s_code_bad = 0, s_zero_tie = 0, s_zero_bad = 0;
    int64_t s_elems = 0, s_groups = 0, s_scale_bad = 0;
    double dev = 0.0;
    int rc = 0;
#pragma omp parallel for reduction(+:s_code_tie,s_code_bad,s_zero_tie,s_zero_bad,s_elems,s_groups,s_scale_bad) reduction(max:dev) schedule(dynamic, 1)
    for (int64_t row = 0; row < r; ++row) {
        double *w = W + row * d;
        double s = 1.0;
        int32_t z = 0;
        double zwin = -1.0, gdv = 0.0; /* pending zero-point check, group drift */
        double sdv = 0.0;              /* the group's scale deviation, capped at stol */
        if (first_tie) first_tie[row] = d;
        for (int64_t i = 0; i < d; ++i) {
            const double uii = U[i * d + i];
            if (!(uii > 0.0)) { rc = -2; break; }
            if (i % g == 0) {
                const int64_t gend = (i + g < d) ? i + g : d;
                double zr;
                orc_quant_params(w + i, gend - i, bits, pure, &s, &zr, &z);
                if (fscales) {
                    const double ds = fabs(fscales[(i / g) * r + row] - s) / s;
                    if (ds > stol) ++s_scale_bad;
                    sdv = ds < stol ? ds : stol;
                }
                if (fzeros) {
                    int32_t zf = fzeros[(i / g) * r + row];
                    zwin = (zf != z) ? fabs((double)zf - zr) - 0.5 - tau : -1.0;
                    if (zf != z) {
                        zwin -= fabs(zr) * sdv;
                        if (first_tie && first_tie[row] > i) first_tie[row] = i;
                    }
                    gdv = 0.0;
                    z = zf;
                    ++s_groups;
                }
                scales[(i / g) * r + row] = s;
                zeros[(i / g) * r + row] = z;
            }
            const double wi = w[i];
            int32_t q = orc_quantize(wi, s, z, bits);
            if (fcodes) {
                const double y = wi / s + (double)z;
                double tol = tau;
                if (fwpre) {
                    double dv = fabs(fwpre[row * d + i] - wi) / s;
                    if (dv > dev) dev = dv;
                    if (dv > gdv) gdv = dv;
                    tol += dv;
                }
                tol += fabs(y - (double)z) * sdv;
                int32_t c = (int32_t)fcodes[row * d + i];
                if (c != q) {
                    if (code_is_valid(c, q, y, tol, bits)) ++s_code_tie;
                    else ++s_code_bad;
                    if (first_tie && first_tie[row] > i) first_tie[row] = i;
                }
                q = c;
                ++s_elems;
            }
            codes[row * d + i] = (uint8_t)q;
            if (fzeros && ((i + 1) % g == 0 || i + 1 == d) && zwin >= 0.0) {
                if (zwin <= gdv) ++s_zero_tie;
                else ++s_zero_bad;
                zwin = -1.0;
            }
            const double e = (wi - s * (double)(q - z)) / uii;
            const double *ui = U + i * d;
            for (int64_t f = i + 1; f < d; ++f) w[f] -= e * ui[f];
        }
    }
    if (stats) {
        stats[0] = s_code_tie; stats[1] = s_code_bad;
        stats[2] = s_zero_tie; stats[3] = s_zero_bad;
        stats[4] = s_elems; stats[5] = s_groups; stats[6] = s_scale_bad;
    }
    if (max_dev) *max_dev = dev;
    return rc;
}

/*
 * Per-column Gaussian elimination of M alone: after step k the trailing block
 * M[k:, k:] is the inverse of H[k:, k:].  Row i of U is the eliminated row i
 * scaled by 1/sqrt(M_ii) (so U^T U = H^-1, U upper).  Stops after `steps`
 * eliminations (steps = d for the full U).
 */
int orc_eliminate(double *M, int64_t d, int64_t steps, double *U)
{
    for (int64_t i = 0; i < steps; ++i) {
        const double piv = M[i * d + i];
        if (!(piv > 0.0)) return -2;
        if (U) {
            const double inv_sqrt = 1.0 / sqrt(piv);
            for (int64_t f = 0; f < i; ++f) U[i * d + f] = 0.0;
            for (int64_t f = i; f < d; ++f) U[i * d + f] = M[i * d + f] * inv_sqrt;
        }
        const double inv_piv = 1.0 / piv;
#pragma omp parallel for schedule(dynamic, 16)
        for (int64_t a = i + 1; a < d; ++a) {
            const double mia = M[i * d + a];
            double *ma = M + a * d;
            const double *mi = M + i * d;
            for (int64_t b = a; b < d; ++b) ma[b] -= (mia * mi[b]) * inv_piv;
        }
    }
    return 0;
}

/*
 * The pages' batched form ("Algorithme complet (pseudo-code)"): columns are
 * walked in batches of B; inside a batch each column is quantized and its
 * error fed forward to the batch's later columns only; after the batch the
 * remaining columns receive all of the batch's errors in one product
 * W[:, i1:] -= Err U[i0:i1, i1:] ("lazy update").  U is the upper factor of
 * H^-1 (row i = eliminated row i / sqrt(M_ii)), so e / M_ii * M_{i,F} equals
 * (e / U_ii) * U_{i,F}; Err holds e_j / U_jj.
 */
int orc_gptq_blocked(double *W, int64_t r, int64_t d, const double *U, int bits,
                     int64_t g, int pure, int64_t B, uint8_t *codes, double *scales,
                     int32_t *zeros)
{
    double *err = (double *)malloc(sizeof(double) * (size_t)(r * B));
    double *cur_s = (double *)malloc(sizeof(double) * (size_t)r);
    int32_t *cur_z = (int32_t *)malloc(sizeof(int32_t) * (size_t)r);
    if (!err || !cur_s || !cur_z) { free(err); free(cur_s); free(cur_z); return -1; }
    for (int64_t i0 = 0; i0 < d; i0 += B) {
        const int64_t i1 = (i0 + B < d) ? i0 + B : d;
#pragma omp parallel for schedule(static)
        for (int64_t row = 0; row < r; ++row) {
            double *w = W + row * d;
            for (int64_t j = i0; j < i1; ++j) {
                if (j % g == 0) {
                    const int64_t gend = (j + g < d) ? j + g : d;
                    double s, zr;
                    int32_t z;
                    orc_quant_params(w + j, gend - j, bits, pure, &s, &zr, &z);
                    cur_s[row] = s;
                    cur_z[row] = z;
                    scales[(j / g) * r + row] = s;
                    zeros[(j / g) * r + row] = z;
                }
                const double s = cur_s[row];
                const int32_t z = cur_z[row];
                const int32_t q = orc_quantize(w[j], s, z, bits);
                codes[row * d + j] = (uint8_t)q;
                const double e = (w[j] - s * (double)(q - z)) / U[j * d + j];
                err[row * B + (j - i0)] = e;
                for (int64_t f = j + 1; f < i1; ++f) w[f] -= e * U[j * d + f];
            }
            /* lazy update of the remaining columns */
            for (int64_t j = i0; j < i1; ++j) {
                const double e = err[row * B + (j - i0)];
                const double *uj = U + j * d;
                for (int64_t f = i1; f < d; ++f) w[f] -= e * uj[f];
            }
        }
    }
    free(err); free(cur_s); free(cur_z);
    return 0;
}

/* Round-to-nearest baseline: the same group quantizer with no error feedback. */
void orc_rtn(const double *W, int64_t r, int64_t d, int bits, int64_t g, int pure,
             uint8_t *codes, double *scales, int32_t *zeros)
{
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < r; ++row) {
        const double *w = W + row * d;
        double s = 1.0;
        int32_t z = 0;
        for (int64_t j = 0; j < d; ++j) {
            if (j % g == 0) {
                const int64_t gend = (j + g < d) ? j + g : d;
                double zr;
                orc_quant_params(w + j, gend - j, bits, pure, &s, &zr, &z);
                scales[(j / g) * r + row] = s;
                zeros[(j / g) * r + row] = z;
            }
            codes[row * d + j] = (uint8_t)orc_quantize(w[j], s, z, bits);
        }
    }
}
