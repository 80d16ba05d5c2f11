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
 * Outputs are overwritten, never accumulated into.
 */
#include <math.h>
#include <stdint.h>

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
