/*
 * ln_oracle.c -- CPU oracle for LayerNorm forward and its analytical backward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or load
 * this file: only the test suite, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or constant with the CUDA
 * library, and it never reads a value produced by the CUDA library.
 *
 * What it computes.  The pages this project follows name the operation but do
 * not print its equations:
 *   - "llm.c's Origin and the Future of LLM Compilers" (CUDA MODE talk page),
 *     chapter "Deconstructing PyTorch Abstractions and Setting Reference
 *     Baselines": LayerNorm forward and backward written over bare float
 *     arrays, no tensor wrapper;
 *   - "llm.c: Large Language Model Training in Pure C/CUDA Without
 *     Dependencies", features "Tensor Memory Layout" (flat row-major arrays,
 *     explicit stride arithmetic) and "Exact Analytical Backward Pass"
 *     (hand-derived gradients for LayerNorm).
 * The arithmetic below is therefore the textbook definition, written out in
 * the plainest order, every value in double:
 *
 *   mean_r = (1/C) sum_c x[r,c]
 *   var_r  = (1/C) sum_c (x[r,c] - mean_r)^2          (biased divisor C)
 *   rstd_r = 1 / sqrt(var_r + eps)                    (eps inside the root)
 *   xhat   = (x - mean_r) * rstd_r
 *   out    = xhat * w[c] + b[c]
 *
 * and, for the loss L = sum out * dout, the analytical gradient
 *
 *   g       = dout * w[c]
 *   dinp    = rstd_r * ( g - (1/C) sum_j g_j - xhat * (1/C) sum_j g_j xhat_j )
 *   dweight = sum_r dout * xhat      (column sum over all N rows)
 *   dbias   = sum_r dout             (column sum over all N rows)
 *
 * The dinp line follows from d xhat_j / d x_i = rstd (delta_ij - 1/C -
 * xhat_i xhat_j / C), which keeps the dependence of rstd on x through var_r.
 *
 * Layout: every array is flat and row-major; row r starts at offset r*C.
 * Outputs are overwritten, never accumulated into, except by the accumulating
 * backward variant below, which says so.
 *
 * Variants (after the two plain passes):
 *   - oracle_round_format: rounding of a real value to a binary floating-point
 *     format, to nearest with ties to even (IEEE 754 roundTiesToEven);
 *   - oracle_ln_forward_residual: the forward of x = round(resid + branch), the
 *     residual add that precedes LayerNorm in a GPT-2 block, fused the way
 *     "llm.c: Large Language Model Training in Pure C/CUDA Without
 *     Dependencies" credits its custom fused kernels for its speed;
 *   - oracle_ln_backward_ex: the backward with the gradients added to what the
 *     output arrays already hold (that page's multi-GPU question: gradients are
 *     accumulated locally), and/or with mean and rstd recomputed from inp by
 *     the forward instead of being passed in.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#define ORACLE_OK 0
#define ORACLE_BAD_SHAPE 2

/* Forward pass over N rows of C columns.  mean and rstd receive one value per
 * row.  Returns ORACLE_BAD_SHAPE for N < 0 or C <= 0, ORACLE_OK otherwise. */
int oracle_ln_forward(double *out, double *mean, double *rstd,
                      const double *inp, const double *weight, const double *bias,
                      int64_t N, int64_t C, double eps)
{
    if (N < 0 || C <= 0) return ORACLE_BAD_SHAPE;
    for (int64_t r = 0; r < N; r++) {
        const double *x = inp + r * C;

        double sum = 0.0;
        for (int64_t c = 0; c < C; c++) sum += x[c];
        double m = sum / (double)C;

        double sq = 0.0;
        for (int64_t c = 0; c < C; c++) {
            double dev = x[c] - m;
            sq += dev * dev;
        }
        double var = sq / (double)C;
        double s = 1.0 / sqrt(var + eps);

        double *o = out + r * C;
        for (int64_t c = 0; c < C; c++) {
            double xhat = (x[c] - m) * s;
            o[c] = xhat * weight[c] + bias[c];
        }
        mean[r] = m;
        rstd[r] = s;
    }
    return ORACLE_OK;
}

/* Backward pass.  mean and rstd are the per-row statistics the forward pass
 * saved; the backward is a function of exactly the arguments it is given and
 * does not recompute them.  dweight and dbias hold C values each and are
 * overwritten with the column sums over all N rows (zero when N == 0). */
int oracle_ln_backward(double *dinp, double *dweight, double *dbias,
                       const double *dout, const double *inp, const double *weight,
                       const double *mean, const double *rstd,
                       int64_t N, int64_t C)
{
    if (N < 0 || C <= 0) return ORACLE_BAD_SHAPE;
    for (int64_t c = 0; c < C; c++) {
        dweight[c] = 0.0;
        dbias[c] = 0.0;
    }
    for (int64_t r = 0; r < N; r++) {
        const double *x = inp + r * C;
        const double *dy = dout + r * C;
        double m = mean[r];
        double s = rstd[r];

        double sum_g = 0.0;
        double sum_gxhat = 0.0;
        for (int64_t c = 0; c < C; c++) {
            double xhat = (x[c] - m) * s;
            double g = dy[c] * weight[c];
            sum_g += g;
            sum_gxhat += g * xhat;
        }
        double mean_g = sum_g / (double)C;
        double mean_gxhat = sum_gxhat / (double)C;

        double *dx = dinp + r * C;
        for (int64_t c = 0; c < C; c++) {
            double xhat = (x[c] - m) * s;
            double g = dy[c] * weight[c];
            dx[c] = s * (g - mean_g - xhat * mean_gxhat);
            dweight[c] += dy[c] * xhat;
            dbias[c] += dy[c];
        }
    }
    return ORACLE_OK;
}

/* Round every in[i] to the nearest value of a binary floating-point format,
 * ties to the value whose last significand bit is 0.  The format has p
 * significant bits, its smallest normal magnitude is 2^emin, below that the
 * spacing stays 2^(emin - p + 1) (gradual underflow), and a result whose
 * magnitude exceeds max_finite is infinite (so values at or above
 * max_finite + half a spacing overflow, as round-to-nearest requires).
 *   fp32:      p = 24, emin = -126, max_finite = (2 - 2^-23) * 2^127
 *   bfloat16:  p =  8, emin = -126, max_finite = (2 - 2^-7)  * 2^127
 *   fp16:      p = 11, emin =  -14, max_finite = 65504
 * Zeros, infinities and NaNs pass through. */
int oracle_round_format(double *out, const double *in, int64_t n, int p, int emin,
                        double max_finite)
{
    if (n < 0 || p < 2 || p > 53) return ORACLE_BAD_SHAPE;
    for (int64_t i = 0; i < n; i++) {
        double v = in[i];
        if (v == 0.0 || !isfinite(v)) {
            out[i] = v;
            continue;
        }
        int e;
        frexp(v, &e);                      /* 2^(e-1) <= |v| < 2^e */
        int q = e - p;                     /* spacing of p-bit values there: 2^q */
        if (q < emin - p + 1) q = emin - p + 1;
        double r = ldexp(nearbyint(ldexp(v, -q)), q);   /* nearest, ties even */
        out[i] = fabs(r) > max_finite ? copysign(INFINITY, v) : r;
    }
    return ORACLE_OK;
}

/* Residual forward: x = round(resid + branch) elementwise (the sum of two
 * format values, exact in double or rounded far from any tie of the format,
 * then rounded once to the format), then the plain forward of x.  x receives
 * the rounded sums (the new residual stream). */
int oracle_ln_forward_residual(double *x, double *out, double *mean, double *rstd,
                               const double *resid, const double *branch,
                               const double *weight, const double *bias,
                               int64_t N, int64_t C, double eps,
                               int p, int emin, double max_finite)
{
    if (N < 0 || C <= 0) return ORACLE_BAD_SHAPE;
    for (int64_t i = 0; i < N * C; i++) x[i] = resid[i] + branch[i];
    int rc = oracle_round_format(x, x, N * C, p, emin, max_finite);
    if (rc != ORACLE_OK) return rc;
    return oracle_ln_forward(out, mean, rstd, x, weight, bias, N, C, eps);
}

/* Backward variants.
 *   recompute != 0: mean and rstd are those oracle_ln_forward computes from
 *     inp with eps (the mean and rstd arguments are not read);
 *   accumulate_dinp != 0: dinp holds a previous gradient on entry and the
 *     new one is added to it;
 *   accumulate_params != 0: likewise for dweight and dbias.
 * Returns ORACLE_BAD_SHAPE for a bad shape, 3 when memory runs out. */
int oracle_ln_backward_ex(double *dinp, double *dweight, double *dbias,
                          const double *dout, const double *inp, const double *weight,
                          const double *mean, const double *rstd,
                          int64_t N, int64_t C, double eps,
                          int accumulate_dinp, int accumulate_params, int recompute)
{
    if (N < 0 || C <= 0) return ORACLE_BAD_SHAPE;
    size_t nc = (size_t)(N * C), n = (size_t)N, c = (size_t)C;
    double *g_in = malloc((nc ? nc : 1) * sizeof(double));
    double *g_w = malloc(c * sizeof(double));
    double *g_b = malloc(c * sizeof(double));
    double *st_m = malloc((n ? n : 1) * sizeof(double));
    double *st_s = malloc((n ? n : 1) * sizeof(double));
    double *scratch = malloc((nc ? nc : 1) * sizeof(double));
    double *zeros = calloc(c, sizeof(double));
    int rc = 3;
    if (g_in && g_w && g_b && st_m && st_s && scratch && zeros) {
        const double *m = mean, *s = rstd;
        rc = ORACLE_OK;
        if (recompute) {
            rc = oracle_ln_forward(scratch, st_m, st_s, inp, weight, zeros, N, C, eps);
            m = st_m;
            s = st_s;
        }
        if (rc == ORACLE_OK)
            rc = oracle_ln_backward(g_in, g_w, g_b, dout, inp, weight, m, s, N, C);
        if (rc == ORACLE_OK) {
            for (size_t i = 0; i < nc; i++)
                dinp[i] = accumulate_dinp ? dinp[i] + g_in[i] : g_in[i];
            for (size_t j = 0; j < c; j++) {
                dweight[j] = accumulate_params ? dweight[j] + g_w[j] : g_w[j];
                dbias[j] = accumulate_params ? dbias[j] + g_b[j] : g_b[j];
            }
        }
    }
    free(g_in);
    free(g_w);
    free(g_b);
    free(st_m);
    free(st_s);
    free(scratch);
    free(zeros);
    return rc;
}
