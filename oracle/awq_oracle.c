/*
 * awq_oracle.c -- plain, slow CPU oracle for the AWQ INT4 hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this code.  It shares no
 * source, header, table or helper with the CUDA library, and the CUDA library
 * never calls it.
 *
 * What it computes (sources, by page and section):
 *   [P1] "From-Scratch AWQ INT4 Quantization on Qwen3-8B", sections
 *        "AWQ scaling", "Group-wise symmetric INT4",
 *        "AutoAWQ / HF-AWQ GEMM on-disk format" and exporter step 4.
 *   [P3] "AWQ architecture, in depth: ...", sections "The scale search as
 *        code" and "Quantization, storage and packing".
 *   [P4] "Weight-Only Quantization: GPTQ and AWQ", section 4 "Tiny example"
 *        and sections 6-9 "Under the hood: the packed format".
 *   Asymmetric INT4: [P3] "Quantization, storage and packing" (a 16-bit
 *        scale and a 4-bit zero point per group and output channel) and
 *        "The scale search as code" (the worked example: values up to 0.5
 *        in magnitude give a step of about 1/15 and a worst rounding error
 *        of about 0.033).  The pages give no formula; the reading here is the
 *        min-max grid: range = max(max ws - min ws, 1e-5), q_scale =
 *        fp16(range / 15), zero = clamp(rint(-min ws / q_scale), 0, 15),
 *        q = clamp(rint(ws / q_scale) + zero, 0, 15) (orc_fake_quant_group_asym).
 *   Duo scaling: [P3] "The scale search as code" (with duo scaling the
 *        candidate is also divided by the mean normalised weight magnitude
 *        raised to 1 - r).
 *   Norm-group scales: [P1] "AutoAWQ / HF-AWQ GEMM on-disk format",
 *        exporter steps 1-2 (one shared scale per norm group: the geometric
 *        mean of the member linears' scales, then re-quantisation with it).
 *   Clip search: [P3] "The pipeline end to end", step 5 (an optional search
 *        of a clipping range per output channel that shrinks the
 *        quantisation range); [P5] "AWQ, Reproduced" (the paper also clips
 *        the weight range).  The pages give no formula; the reading here:
 *        ratios c_i = RN((20 - i) / 20), the group's largest |ws| scaled by
 *        c_i before the fp16 scale is formed, the same weighted error, and
 *        the first minimum per (row, group) (orc_clip_search).
 *
 * Precision (readings of the pages where they leave it open):
 *   - every decision that produces an integer (a code, the group scale, the
 *     chosen grid index) is taken in fp32 with IEEE round-to-nearest-even,
 *     the group scale then rounded to fp16 (round-to-nearest-even);
 *   - the activation mean is the exact real mean, rounded once to fp64 and
 *     then to fp32;
 *   - the scale table is computed in fp64 and rounded once to fp32;
 *   - error sums are the exact weighted squared error of those fp32
 *     decisions, evaluated in fp64.
 * Build with -O2 -ffp-contract=off and without -ffast-math.
 *
 * Parity pins: every function here is pinned by tests/test_oracle_pins.py
 * (worked example, closed forms, special cases, brute force); none is
 * "parity unpinned" except the claim that the packed words load in the
 * third-party AutoAWQ runtime, which is not present here.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_SCALE_FP32 1   /* flag: keep the group scale unrounded (fp32) */
#define ORC_DUO 2          /* flag: duo scaling candidates (see orc_scale_table_duo) */
#define ORC_ASYM 4         /* flag: asymmetric INT4 (see orc_fake_quant_group_asym) */

/* ---------------------------------------------------------------- fp16 -- */

static float h2f(uint16_t h)
{
    _Float16 v;
    memcpy(&v, &h, sizeof v);
    return (float)v;
}

static uint16_t f2h(float f)
{
    _Float16 v = (_Float16)f;          /* IEEE round-to-nearest-even */
    uint16_t h;
    memcpy(&h, &v, sizeof h);
    return h;
}

/* ------------------------------------------------------ activation stats --
 * x[j] = mean over tokens of |X[t, j]|        ([P1] "AWQ scaling";
 * [P3] "The scale search as code": x.abs().float().mean(dim=0)).
 *
 * Every |fp16| value is an integer multiple of 2^-24 below 2^16, so the sum
 * is accumulated exactly as an integer count of 2^-24 units.  A column that
 * holds an infinity gets +inf; one that holds a NaN gets NaN.
 */
void orc_act_stats(const uint16_t *X, int64_t T, int64_t d_in, int64_t ld,
                   float *x)
{
    for (int64_t j = 0; j < d_in; ++j) {
        int64_t units = 0;          /* sum of |X[t,j]| in units of 2^-24 */
        int saw_inf = 0, saw_nan = 0;
        for (int64_t t = 0; t < T; ++t) {
            float v = fabsf(h2f(X[t * ld + j]));
            if (isnan(v)) { saw_nan = 1; continue; }
            if (isinf(v)) { saw_inf = 1; continue; }
            units += (int64_t)ldexp((double)v, 24);   /* exact integer */
        }
        if (saw_nan)
            x[j] = NAN;
        else if (saw_inf)
            x[j] = INFINITY;
        else
            x[j] = (float)(ldexp((double)units, -24) / (double)T);
    }
}

/* ----------------------------------------------------------- scale table --
 * For grid index i (alpha = i / n_grid, [P3] "The scale search as code"):
 *   s_i[j] = max(x[j], 1e-4) ^ alpha
 *   s_i    = s_i / sqrt(max_j s_i[j] * min_j s_i[j])
 * The clamp sits on x before the power (the stated method); the power and the
 * normalisation are done in fp64 and rounded once to fp32.
 */
void orc_scale_table(const float *x, int64_t d_in, int n_grid, float *S)
{
    double *sd = (double *)malloc((size_t)d_in * sizeof(double));
    for (int i = 0; i < n_grid; ++i) {
        double alpha = (double)i / (double)n_grid;
        double mx = -INFINITY, mn = INFINITY;
        for (int64_t j = 0; j < d_in; ++j) {
            float xc = fmaxf(x[j], 1e-4f);
            sd[j] = pow((double)xc, alpha);
            if (sd[j] > mx) mx = sd[j];
            if (sd[j] < mn) mn = sd[j];
        }
        double norm = sqrt(mx * mn);
        for (int64_t j = 0; j < d_in; ++j)
            S[(int64_t)i * d_in + j] = (float)(sd[j] / norm);
    }
    free(sd);
}

/* ----------------------------------------------- group fake-quantisation --
 * One group of n consecutive input channels of one output row
 * ([P1] "Group-wise symmetric INT4"):
 *   ws[j]   = w[j] * s[j]                         (fp32)
 *   q_scale = max_j |ws[j]| / 7                   (fp32, then fp16 RNE
 *                                                  unless ORC_SCALE_FP32)
 *   q[j]    = clamp(rint(ws[j] / q_scale), -7, 7) (rint = half to even)
 * An all-zero group has q_scale = 0 and all codes 0.  A q_scale that
 * overflows fp16 is held at the largest finite fp16 value, 65504.
 * Returns 0, or 1 when the group holds a non-finite value (codes then 0 and
 * q_scale NaN).
 */
int orc_fake_quant_group(const float *w, const float *s, int64_t n, int flags,
                         int8_t *q, float *q_scale)
{
    float m = 0.0f;
    int nonfinite = 0;
    for (int64_t j = 0; j < n; ++j) {
        float ws = w[j] * s[j];
        if (!isfinite(ws)) nonfinite = 1;
        float a = fabsf(ws);
        if (a > m) m = a;
    }
    if (nonfinite) {
        for (int64_t j = 0; j < n; ++j) q[j] = 0;
        *q_scale = NAN;
        return 1;
    }
    float qs = m / 7.0f;
    if (!(flags & ORC_SCALE_FP32)) {
        qs = h2f(f2h(qs));
        if (isinf(qs)) qs = 65504.0f;
    }
    for (int64_t j = 0; j < n; ++j) {
        if (qs == 0.0f) { q[j] = 0; continue; }
        float ws = w[j] * s[j];
        float r = rintf(ws / qs);
        if (r > 7.0f) r = 7.0f;
        if (r < -7.0f) r = -7.0f;
        q[j] = (int8_t)r;
    }
    *q_scale = qs;
    return 0;
}

/* ---------------------------------------------------------- duo scaling --
 * [P3] "The scale search as code", duo scaling: per input channel the mean,
 * over every row of the concatenated member linears, of |w| divided by its
 * row's largest |w|:
 *     w_mean[j] = (1 / R) sum_r |W[r, j]| / max_k |W[r, k]|
 * each quotient correctly rounded in fp64 (an all-zero row contributes 0),
 * summed in fp64 in segment and row order.
 */
void orc_weight_mean(int n_seg, const uint16_t *const *W, const int64_t *d_out, int64_t d_in,
                     double *w_mean)
{
    int64_t rows = 0;
    for (int64_t j = 0; j < d_in; ++j) w_mean[j] = 0.0;
    for (int k = 0; k < n_seg; ++k) {
        for (int64_t r = 0; r < d_out[k]; ++r) {
            const uint16_t *row = W[k] + r * d_in;
            double mx = 0.0;
            for (int64_t j = 0; j < d_in; ++j) {
                double a = fabs((double)h2f(row[j]));
                if (a > mx) mx = a;
            }
            for (int64_t j = 0; j < d_in; ++j)
                w_mean[j] += mx > 0.0 ? fabs((double)h2f(row[j])) / mx : 0.0;
        }
        rows += d_out[k];
    }
    for (int64_t j = 0; j < d_in; ++j) w_mean[j] /= (double)rows;
}

/* Duo scale table ([P3] "The scale search as code"): for r = i / n_grid
 *     s[j] = x[j]^r / (w_mean[j]^(1 - r) + 1e-4),  then max(s, 1e-4),
 *     S[i][j] = s[j] / sqrt(max_j s * min_j s)
 * in fp64 (x as given, the clamp on s as the page writes it), rounded once
 * to fp32. */
void orc_scale_table_duo(const float *x, const double *w_mean, int64_t d_in, int n_grid,
                         float *S)
{
    double *sd = (double *)malloc((size_t)d_in * sizeof(double));
    for (int i = 0; i < n_grid; ++i) {
        double r = (double)i / (double)n_grid;
        double mx = -INFINITY, mn = INFINITY;
        for (int64_t j = 0; j < d_in; ++j) {
            double v = pow((double)x[j], r) / (pow(w_mean[j], 1.0 - r) + 1e-4);
            if (v < 1e-4) v = 1e-4;
            sd[j] = v;
            if (v > mx) mx = v;
            if (v < mn) mn = v;
        }
        double norm = sqrt(mx * mn);
        for (int64_t j = 0; j < d_in; ++j)
            S[(int64_t)i * d_in + j] = (float)(sd[j] / norm);
    }
    free(sd);
}

/* ------------------------------------------------------- asymmetric INT4 --
 * 16 levels 0..15 with a per-group zero point (min-max grid):
 *   ws = fl32(w s);  range = max(fl32(max ws - min ws), 1e-5)
 *   q_scale = fp16_rne(fl32(range / 15))        (unrounded with ORC_SCALE_FP32)
 *   zero    = clamp(rint(fl32(-min ws / q_scale)), 0, 15)
 *   q       = clamp(rint(fl32(ws / q_scale)) + zero, 0, 15)
 *   w_hat   = (q - zero) q_scale / s
 * A non-finite group gives q_scale NaN, zero 8 and codes 8 (return 1).
 */
int orc_fake_quant_group_asym(const float *w, const float *s, int64_t n, int flags,
                              uint8_t *q, float *q_scale, int *zero)
{
    float mx = -INFINITY, mn = INFINITY;
    int nonfinite = 0;
    for (int64_t j = 0; j < n; ++j) {
        float ws = w[j] * s[j];
        if (!isfinite(ws)) nonfinite = 1;
        if (ws > mx) mx = ws;
        if (ws < mn) mn = ws;
    }
    if (nonfinite) {
        for (int64_t j = 0; j < n; ++j) q[j] = 8;
        *q_scale = NAN;
        *zero = 8;
        return 1;
    }
    float range = mx - mn;
    if (range < 1e-5f) range = 1e-5f;
    float qs = range / 15.0f;
    if (!(flags & ORC_SCALE_FP32)) {
        qs = h2f(f2h(qs));
        if (isinf(qs)) qs = 65504.0f;
    }
    float z = rintf(-mn / qs);
    if (z < 0.0f) z = 0.0f;
    if (z > 15.0f) z = 15.0f;
    for (int64_t j = 0; j < n; ++j) {
        float ws = w[j] * s[j];
        float r = rintf(ws / qs) + z;
        if (r < 0.0f) r = 0.0f;
        if (r > 15.0f) r = 15.0f;
        q[j] = (uint8_t)r;
    }
    *q_scale = qs;
    *zero = (int)z;
    return 0;
}

/* ------------------------------------------------- weight-space scoring --
 * Activation-weighted reconstruction error of one candidate scale vector s
 * over one weight matrix W[d_out, d_in] (fp16, row-major)
 * ([P1] "AWQ scaling"):
 *     sum_{r,j} ( (W[r,j] - q[r,j] * q_scale[r,g(j)] / s[j]) * x[j] )^2
 * evaluated in fp64 from the fp32 decisions.  Returns NaN when any group is
 * non-finite.
 */
double orc_weighted_error(const uint16_t *W, int64_t d_out, int64_t d_in,
                          const float *x, const float *s, int64_t g, int flags)
{
    /* one partial per row, summed afterwards in row order, so the result
     * does not depend on how many threads ran the rows */
    double *row_err = (double *)malloc((size_t)d_out * sizeof(double));
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < d_out; ++r) {
        float w[g];
        int8_t q[g];
        uint8_t u[g];
        double acc = 0.0;
        for (int64_t k = 0; k < d_in / g; ++k) {
            const uint16_t *row = W + r * d_in + k * g;
            for (int64_t j = 0; j < g; ++j) w[j] = h2f(row[j]);
            float qs;
            int z = 0;
            int bad = (flags & ORC_ASYM)
                          ? orc_fake_quant_group_asym(w, s + k * g, g, flags, u, &qs, &z)
                          : orc_fake_quant_group(w, s + k * g, g, flags, q, &qs);
            if (bad) {
                acc = NAN;
                continue;
            }
            for (int64_t j = 0; j < g; ++j) {
                double level = (flags & ORC_ASYM) ? (double)((int)u[j] - z) : (double)q[j];
                double what = level * (double)qs / (double)s[k * g + j];
                double e = ((double)w[j] - what) * (double)x[k * g + j];
                acc += e * e;
            }
        }
        row_err[r] = acc;
    }
    double total = 0.0;
    for (int64_t r = 0; r < d_out; ++r) total += row_err[r];
    free(row_err);
    return total;
}

/* ---------------------------------------------------- norm-group scales --
 * [P1] exporter step 1: the linears that follow one norm (q/k/v; gate/up)
 * each get their own searched scale s_m; the norm can absorb only one, so
 * they share the per-channel geometric mean
 *     s_shared[j] = (prod_m s_m[j])^(1/n)
 * evaluated as the fp64 product in member order, then sqrt for n = 2 and
 * pow(., 1/n) otherwise, rounded once to fp32 (n = 1 copies s_0).
 */
void orc_geomean_scales(int n, const float *const *s, int64_t d_in, float *out)
{
    for (int64_t j = 0; j < d_in; ++j) {
        if (n == 1) {
            out[j] = s[0][j];
            continue;
        }
        double p = 1.0;
        for (int m = 0; m < n; ++m) p *= (double)s[m][j];
        double r = (n == 2) ? sqrt(p) : pow(p, 1.0 / (double)n);
        out[j] = (float)r;
    }
}

/* ------------------------------------------------------------- clipping --
 * Clip ratio i of the grid: c_i = (20 - i) / 20 rounded to fp32, so c_0 = 1
 * (no clipping) and each step shrinks the range by 5% of the group maximum.
 */
#define ORC_CLIP_DEN 20

float orc_clip_ratio(int i)
{
    return (float)((double)(ORC_CLIP_DEN - i) / (double)ORC_CLIP_DEN);
}

/* The group fake-quantisation with the range shrunk to c * max|w s|:
 *   m_c = fl32(c * max|ws|),  q_scale = fp16_rne(fl32(m_c / 7)),
 *   q = clamp(rint(ws / q_scale), -7, 7)
 * (values beyond the shrunk range saturate at +-7).  With c = 1 every
 * operation is the one of orc_fake_quant_group. */
int orc_fake_quant_group_clip(const float *w, const float *s, int64_t n, int flags,
                              float c, int8_t *q, float *q_scale)
{
    float m = 0.0f;
    int nonfinite = 0;
    for (int64_t j = 0; j < n; ++j) {
        float ws = w[j] * s[j];
        if (!isfinite(ws)) nonfinite = 1;
        float a = fabsf(ws);
        if (a > m) m = a;
    }
    if (nonfinite) {
        for (int64_t j = 0; j < n; ++j) q[j] = 0;
        *q_scale = NAN;
        return 1;
    }
    float mc = m * c;
    float qs = mc / 7.0f;
    if (!(flags & ORC_SCALE_FP32)) {
        qs = h2f(f2h(qs));
        if (isinf(qs)) qs = 65504.0f;
    }
    for (int64_t j = 0; j < n; ++j) {
        if (qs == 0.0f) { q[j] = 0; continue; }
        float ws = w[j] * s[j];
        float r = rintf(ws / qs);
        if (r > 7.0f) r = 7.0f;
        if (r < -7.0f) r = -7.0f;
        q[j] = (int8_t)r;
    }
    *q_scale = qs;
    return 0;
}

/* Weighted error of one group (n weights) at clip ratio c, in fp64:
 * sum_j ((w_j - q_j q_scale / s_j) x_j)^2; NaN for a non-finite group. */
double orc_clip_group_error(const float *w, const float *s, const float *x, int64_t n,
                            int flags, float c)
{
    int8_t q[n];
    float qs;
    if (orc_fake_quant_group_clip(w, s, n, flags, c, q, &qs)) return NAN;
    double acc = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        double what = (double)q[j] * (double)qs / (double)s[j];
        double e = ((double)w[j] - what) * (double)x[j];
        acc += e * e;
    }
    return acc;
}

/* Clip search at a fixed scale s (normally the scale search's s_best):
 * for every row r and group k, the first ratio index i < n_clip with the
 * smallest weighted error of that group wins (strict '<').
 *   clip_idx[r * G + k]  the chosen index (0 for a non-finite group)
 *   err[0]               total error with no clipping (index 0 everywhere)
 *   err[1]               total error with the chosen indices
 * Totals are summed per row, then over rows in order.  s == NULL: s = 1. */
void orc_clip_search(const uint16_t *W, int64_t d_out, int64_t d_in, const float *x,
                     const float *s, int64_t g, int n_clip, int flags,
                     uint8_t *clip_idx, double *err)
{
    int64_t G = d_in / g;
    double *row0 = (double *)malloc((size_t)d_out * sizeof(double));
    double *row1 = (double *)malloc((size_t)d_out * sizeof(double));
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < d_out; ++r) {
        float w[g], ones[g];
        for (int64_t j = 0; j < g; ++j) ones[j] = 1.0f;
        double a0 = 0.0, a1 = 0.0;
        for (int64_t k = 0; k < G; ++k) {
            for (int64_t j = 0; j < g; ++j) w[j] = h2f(W[r * d_in + k * g + j]);
            const float *sk = s ? s + k * g : ones;
            double best = orc_clip_group_error(w, sk, x + k * g, g, flags, orc_clip_ratio(0));
            double e0 = best;
            int b = 0;
            for (int i = 1; i < n_clip; ++i) {
                double e = orc_clip_group_error(w, sk, x + k * g, g, flags, orc_clip_ratio(i));
                if (e < best) {
                    best = e;
                    b = i;
                }
            }
            clip_idx[r * G + k] = (uint8_t)b;
            a0 += e0;
            a1 += best;
        }
        row0[r] = a0;
        row1[r] = a1;
    }
    double t0 = 0.0, t1 = 0.0;
    for (int64_t r = 0; r < d_out; ++r) {
        t0 += row0[r];
        t1 += row1[r];
    }
    err[0] = t0;
    err[1] = t1;
    free(row0);
    free(row1);
}

/* Output-space clip search at a fixed scale s ([P3] "The pipeline end to
 * end", step 5, with the candidates scored on the output as in [P3] "The
 * scale search as code", restricted to one group so that every (row, group)
 * choice is independent): for every row r, group k and ratio index i <
 * n_clip,
 *     e[r,k,i] = sum_t ( sum_{j in k} X[t,j] (W[r,j] - W_hat_i[r,j]) )^2
 * with W_hat_i the clipped fake-quantisation of orc_fake_quant_group_clip,
 * in fp64; clip_idx[r * G + k] = the first i with the smallest e.  err[0] is
 * the sum over rows and groups of e[., ., 0] (no clipping), err[1] of the
 * chosen e; summed per row, then over rows in order.  s == NULL: s = 1.  A
 * non-finite group keeps index 0 and makes the totals NaN. */
void orc_clip_search_output(const uint16_t *X, int64_t T, const uint16_t *W, int64_t d_out,
                            int64_t d_in, const float *s, int64_t g, int n_clip, int flags,
                            uint8_t *clip_idx, double *err)
{
    int64_t G = d_in / g;
    double *Xd = (double *)malloc((size_t)T * (size_t)d_in * sizeof(double));
    double *row0 = (double *)malloc((size_t)d_out * sizeof(double));
    double *row1 = (double *)malloc((size_t)d_out * sizeof(double));
    for (int64_t t = 0; t < T * d_in; ++t) Xd[t] = (double)h2f(X[t]);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < d_out; ++r) {
        float w[g], ones[g];
        int8_t q[g];
        double dw[g];
        for (int64_t j = 0; j < g; ++j) ones[j] = 1.0f;
        double a0 = 0.0, a1 = 0.0;
        for (int64_t k = 0; k < G; ++k) {
            for (int64_t j = 0; j < g; ++j) w[j] = h2f(W[r * d_in + k * g + j]);
            const float *sk = s ? s + k * g : ones;
            double best = 0.0, e0 = 0.0;
            int b = 0, bad = 0;
            for (int i = 0; i < n_clip; ++i) {
                float qs;
                if (orc_fake_quant_group_clip(w, sk, g, flags, orc_clip_ratio(i), q, &qs)) {
                    bad = 1;
                    break;
                }
                for (int64_t j = 0; j < g; ++j)
                    dw[j] = (double)w[j] - (double)q[j] * (double)qs / (double)sk[j];
                double e = 0.0;
                for (int64_t t = 0; t < T; ++t) {
                    double y = 0.0;
                    for (int64_t j = 0; j < g; ++j) y += Xd[t * d_in + k * g + j] * dw[j];
                    e += y * y;
                }
                if (i == 0) {
                    e0 = e;
                    best = e;
                } else if (e < best) {
                    best = e;
                    b = i;
                }
            }
            clip_idx[r * G + k] = (uint8_t)(bad ? 0 : b);
            a0 += bad ? NAN : e0;
            a1 += bad ? NAN : best;
        }
        row0[r] = a0;
        row1[r] = a1;
    }
    double t0 = 0.0, t1 = 0.0;
    for (int64_t r = 0; r < d_out; ++r) {
        t0 += row0[r];
        t1 += row1[r];
    }
    err[0] = t0;
    err[1] = t1;
    free(Xd);
    free(row0);
    free(row1);
}

/* ---------------------------------------------------------- scale search --
 * [P3] "The scale search as code" + [P1] "AWQ scaling": for every grid
 * index i the error of every weight segment that shares the input x is
 * summed; the first index with the smallest error wins (strict '<', so the
 * smallest alpha wins a tie).  s_best receives that row of the scale table
 * (the duo table with ORC_DUO in flags).  best = -1 (and s_best NaN) when
 * any error is not finite.
 */
void orc_scale_search(int n_seg, const uint16_t *const *W, const int64_t *d_out,
                      int64_t d_in, const float *x, int64_t g, int n_grid,
                      int flags, double *err, int32_t *best, float *s_best)
{
    float *S = (float *)malloc((size_t)n_grid * (size_t)d_in * sizeof(float));
    if (flags & ORC_DUO) {
        double *wm = (double *)malloc((size_t)d_in * sizeof(double));
        orc_weight_mean(n_seg, W, d_out, d_in, wm);
        orc_scale_table_duo(x, wm, d_in, n_grid, S);
        free(wm);
    } else {
        orc_scale_table(x, d_in, n_grid, S);
    }
    for (int i = 0; i < n_grid; ++i) {
        double e = 0.0;
        for (int k = 0; k < n_seg; ++k)
            e += orc_weighted_error(W[k], d_out[k], d_in, x,
                                    S + (int64_t)i * d_in, g, flags);
        err[i] = e;
    }
    int b = 0;
    int finite = 1;
    for (int i = 0; i < n_grid; ++i) {
        if (!isfinite(err[i])) finite = 0;
        if (err[i] < err[b]) b = i;
    }
    if (!finite) {
        *best = -1;
        for (int64_t j = 0; j < d_in; ++j) s_best[j] = NAN;
    } else {
        *best = b;
        memcpy(s_best, S + (int64_t)b * d_in, (size_t)d_in * sizeof(float));
    }
    free(S);
}

/* ----------------------------------------------------- quantise and pack --
 * AutoAWQ GEMM layout ([P1] "AutoAWQ / HF-AWQ GEMM on-disk format" and
 * exporter step 4; [P3] "Quantization, storage and packing"):
 *   u[r,j]          = q[r,j] + zero_point      (unsigned code)
 *   qweight[j, c]   = int32 whose nibble p (bits 4p..4p+3) holds
 *                     u[8c + order[p], j],  order = {0,2,4,6,1,3,5,7}
 *   scales[k, r]    = fp16 group scale of row r, group k
 *   qzeros[k, c]    = zero_point in all eight nibbles
 * s == NULL means s = 1 (plain round-to-nearest).  clip_idx (or NULL for
 * none) gives each (row, group) a clip ratio index as in orc_clip_search.
 * zero_point = -1 selects the asymmetric grid: codes 0..15 from
 * orc_fake_quant_group_asym and qzeros holding each (group, row)'s zero
 * point in the same nibble order (clip_idx is ignored then).
 * A non-finite group stores code zero_point and scale NaN.
 */
static const int kOrder[8] = {0, 2, 4, 6, 1, 3, 5, 7};

void orc_quantize_pack(const uint16_t *W, int64_t d_out, int64_t d_in,
                       const float *s, const uint8_t *clip_idx, int64_t g,
                       int zero_point, int32_t *qweight, uint16_t *scales,
                       int32_t *qzeros)
{
    int64_t G = d_in / g, C = d_out / 8;
    uint8_t *u = (uint8_t *)malloc((size_t)d_out * (size_t)d_in);
    float *w = (float *)malloc((size_t)g * sizeof(float));
    float *ones = (float *)malloc((size_t)g * sizeof(float));
    int8_t *q = (int8_t *)malloc((size_t)g);
    uint8_t *ua = (uint8_t *)malloc((size_t)g);
    uint8_t *zeros = (uint8_t *)malloc((size_t)d_out * (size_t)G);
    for (int64_t j = 0; j < g; ++j) ones[j] = 1.0f;

    for (int64_t r = 0; r < d_out; ++r) {
        for (int64_t k = 0; k < G; ++k) {
            for (int64_t j = 0; j < g; ++j) w[j] = h2f(W[r * d_in + k * g + j]);
            float qs;
            if (zero_point < 0) {
                int z;
                orc_fake_quant_group_asym(w, s ? s + k * g : ones, g, 0, ua, &qs, &z);
                zeros[r * G + k] = (uint8_t)z;
                for (int64_t j = 0; j < g; ++j) u[r * d_in + k * g + j] = ua[j];
                scales[k * d_out + r] = isnan(qs) ? (uint16_t)0x7E00 : f2h(qs);
                continue;
            }
            if (clip_idx)
                orc_fake_quant_group_clip(w, s ? s + k * g : ones, g, 0,
                                          orc_clip_ratio(clip_idx[r * G + k]), q, &qs);
            else
                orc_fake_quant_group(w, s ? s + k * g : ones, g, 0, q, &qs);
            scales[k * d_out + r] = isnan(qs) ? (uint16_t)0x7E00 : f2h(qs);
            for (int64_t j = 0; j < g; ++j)
                u[r * d_in + k * g + j] = (uint8_t)(q[j] + zero_point);
        }
    }
    for (int64_t j = 0; j < d_in; ++j) {
        for (int64_t c = 0; c < C; ++c) {
            uint32_t word = 0;
            for (int p = 0; p < 8; ++p)
                word |= (uint32_t)(u[(8 * c + kOrder[p]) * d_in + j] & 0xF)
                        << (4 * p);
            qweight[j * C + c] = (int32_t)word;
        }
    }
    if (zero_point < 0) {
        /* per (group, row) zero points, packed like the codes along rows */
        for (int64_t k = 0; k < G; ++k)
            for (int64_t c = 0; c < C; ++c) {
                uint32_t word = 0;
                for (int p = 0; p < 8; ++p)
                    word |= (uint32_t)(zeros[(8 * c + kOrder[p]) * G + k] & 0xF) << (4 * p);
                qzeros[k * C + c] = (int32_t)word;
            }
    } else {
        uint32_t zword = 0;
        for (int p = 0; p < 8; ++p) zword |= (uint32_t)(zero_point & 0xF) << (4 * p);
        for (int64_t k = 0; k < G; ++k)
            for (int64_t c = 0; c < C; ++c) qzeros[k * C + c] = (int32_t)zword;
    }
    free(ua);
    free(zeros);
    free(u);
    free(w);
    free(ones);
    free(q);
}

/* Inverse of the packing above: codes u[r, j] (unsigned, 0..15). */
void orc_unpack(const int32_t *qweight, int64_t d_out, int64_t d_in,
                uint8_t *u)
{
    int64_t C = d_out / 8;
    for (int64_t j = 0; j < d_in; ++j)
        for (int64_t c = 0; c < C; ++c) {
            uint32_t word = (uint32_t)qweight[j * C + c];
            for (int p = 0; p < 8; ++p)
                u[(8 * c + kOrder[p]) * d_in + j] = (uint8_t)((word >> (4 * p)) & 0xF);
        }
}

/* ------------------------------------------------ output-space scoring --
 * Optional scoring mode ([P3] "The scale search as code": the group output
 * compared with the full-precision output; [P4] section 2: the output error
 * is X (W - W_hat)):
 *     err[i] = || X (W - W_hat_i)^T ||_F^2
 * with W_hat_i = Q(W * s_i) / s_i from the same group fake-quantisation
 * (the asymmetric grid of orc_fake_quant_group_asym with ORC_ASYM in flags:
 * W_hat = (q - zero) q_scale / s), in fp64.  X is fp16 [T, d_in] row-major,
 * W fp16 [d_out, d_in].
 */
void orc_output_error(const uint16_t *X, int64_t T, const uint16_t *W,
                      int64_t d_out, int64_t d_in, const float *x, int64_t g,
                      int n_grid, int flags, double *err)
{
    float *S = (float *)malloc((size_t)n_grid * (size_t)d_in * sizeof(float));
    double *dW = (double *)malloc((size_t)d_out * (size_t)d_in * sizeof(double));
    double *Xd = (double *)malloc((size_t)T * (size_t)d_in * sizeof(double));
    double *tok = (double *)malloc((size_t)T * sizeof(double));
    int *bad_row = (int *)malloc((size_t)d_out * sizeof(int));
    orc_scale_table(x, d_in, n_grid, S);
    for (int64_t t = 0; t < T * d_in; ++t) Xd[t] = (double)h2f(X[t]);

    for (int i = 0; i < n_grid; ++i) {
        const float *s = S + (int64_t)i * d_in;
        /* W - W_hat_i, exactly (fp64) from the fp32 decisions */
#pragma omp parallel for schedule(static)
        for (int64_t r = 0; r < d_out; ++r) {
            float w[g];
            int8_t q[g];
            uint8_t u[g];
            bad_row[r] = 0;
            for (int64_t k = 0; k < d_in / g; ++k) {
                for (int64_t j = 0; j < g; ++j) w[j] = h2f(W[r * d_in + k * g + j]);
                float qs;
                int z = 0;
                int bad = (flags & ORC_ASYM)
                              ? orc_fake_quant_group_asym(w, s + k * g, g, flags, u, &qs, &z)
                              : orc_fake_quant_group(w, s + k * g, g, flags, q, &qs);
                if (bad) bad_row[r] = 1;
                for (int64_t j = 0; j < g; ++j) {
                    double level = (flags & ORC_ASYM) ? (double)((int)u[j] - z) : (double)q[j];
                    dW[r * d_in + k * g + j] =
                        (double)w[j] - level * (double)qs / (double)s[k * g + j];
                }
            }
        }
        /* ||X dW^T||^2: one partial per token, summed in token order */
#pragma omp parallel for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            double acc = 0.0;
            for (int64_t r = 0; r < d_out; ++r) {
                double y = 0.0;
                for (int64_t j = 0; j < d_in; ++j)
                    y += Xd[t * d_in + j] * dW[r * d_in + j];
                acc += y * y;
            }
            tok[t] = acc;
        }
        double total = 0.0;
        int bad = 0;
        for (int64_t t = 0; t < T; ++t) total += tok[t];
        for (int64_t r = 0; r < d_out; ++r) bad |= bad_row[r];
        err[i] = bad ? NAN : total;
    }
    free(S);
    free(dW);
    free(Xd);
    free(tok);
    free(bad_row);
}
