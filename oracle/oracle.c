/*
 * fp64 CPU oracle for the W4 + per-token-gated low-rank Error Compensator
 * (EC) linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check
 * and the benchmark's CPU-baseline leg load this code.  The CUDA library
 * never calls it, and it shares no code, header, table or helper with it.
 *
 * What it computes is the plain definition of the layer, written out loop by
 * loop, with no blocking, fusion or reordering beyond the definition:
 *
 *   What-the-pages-say: SPEAR, "A System for Post-Quantization Error-Adaptive
 *   Recovery Enabling Efficient Low-Bit LLM Serving", Abstract: weights are
 *   quantised to 4 bits per output channel ("per-channel quantization
 *   settings"), a lightweight Error Compensator corrects the layer's output,
 *   its strength is set by a per-token gate, and the correction is fused
 *   into the low-bit GEMM.  The pages give no equation; the readings below
 *   (additive rank-r EC, sigmoid-of-linear gate, round-to-nearest symmetric
 *   int4 with a stored per-channel zero point) are this library's.
 *
 *   pack     s[n] = fp32(max_k |W[n,k]|) / 7        (fp32 quotient)
 *            c    = round_half_even(fp32(W[n,k] / s[n]))
 *            q    = clamp(c, -8, 7) + 8,  z[n] = 8
 *            an all-zero row has s = 0 and every code 8
 *            code of k = 8j+i sits in bits [4i, 4i+3] of word j of row n
 *   pack_asym (the same abstract's "state-of-the-art 4-bit quantizers"
 *            commonly store a per-channel zero point; this is the plain
 *            min-max form of such a quantiser, with 0 kept in the range)
 *            lo = min(0, min_k W[n,k]),  hi = max(0, max_k W[n,k])
 *            s[n] = fp32( fp32(hi - lo) / 15 )
 *            z[n] = clamp(round_half_even(fp32(-lo / s[n])), 0, 15)
 *            q    = clamp(round_half_even(fp32(W[n,k] / s[n])) + z[n], 0, 15)
 *            an all-zero row has s = 0, z = 8 and every code 8
 *   forward  w^[n,k]  = s[n] * (q[n,k] - z[n])
 *            main     = sum_k x[t,k] * w^[n,k]
 *            logit_t  = sum_k x[t,k] * w_g[k] + b_g
 *            g_t      = 1 / (1 + exp(-logit_t))
 *            u[t,j]   = sum_k x[t,k] * A[k,j]
 *            corr     = g_t * sum_j u[t,j] * B[j,n]
 *            y[t,n]   = main + corr          (kept in fp64, no rounding)
 *
 * The code decision of pack is taken in fp32, the precision the kernels use:
 * the quotient of a bf16 by an fp32 scale is formed in fp64 and rounded to
 * fp32, which equals the correctly rounded fp32 quotient because fp64 carries
 * more than 2*24+2 bits (double rounding of a quotient is then innocuous).
 *
 * Build: gcc -O2 -fopenmp -fPIC -shared -fno-fast-math -ffp-contract=off.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Per-output-channel round-to-nearest int4 quantisation of one bf16 matrix
 * W [N][K] into codes [N][K/8] (uint32), s [N] (fp32) and z [N] (uint8). */
int oracle_pack(const uint16_t *W, int64_t N, int64_t K,
                uint32_t *codes, float *s, uint8_t *z)
{
    if (N < 0 || K < 0 || K % 8 != 0)
        return -1;
    const int64_t words = K / 8;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const uint16_t *row = W + n * K;
        double amax = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double a = fabs(bf16_to_f64(row[k]));
            if (a > amax)
                amax = a;
        }
        float sn = (float)(amax / 7.0);
        s[n] = sn;
        z[n] = 8;
        for (int64_t j = 0; j < words; ++j) {
            uint32_t word = 0;
            for (int i = 0; i < 8; ++i) {
                int q;
                if (sn == 0.0f) {
                    q = 8;
                } else {
                    float quot = (float)(bf16_to_f64(row[8 * j + i]) / (double)sn);
                    double c = nearbyint((double)quot); /* ties to even */
                    if (c < -8.0)
                        c = -8.0;
                    if (c > 7.0)
                        c = 7.0;
                    q = (int)c + 8;
                }
                word |= (uint32_t)q << (4 * i);
            }
            codes[n * words + j] = word;
        }
    }
    return 0;
}

/* Asymmetric (min-max) per-output-channel round-to-nearest int4 of W [N][K]
 * into codes [N][K/8], s [N] and a stored zero point z [N] (see the header
 * comment).  Every fp32 operation is formed in fp64 and rounded once to fp32,
 * which equals the correctly rounded fp32 operation (fp64 carries more than
 * 2*24+2 bits, so double rounding of a sum or quotient is innocuous). */
int oracle_pack_asym(const uint16_t *W, int64_t N, int64_t K,
                     uint32_t *codes, float *s, uint8_t *z)
{
    if (N < 0 || K < 0 || K % 8 != 0)
        return -1;
    const int64_t words = K / 8;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const uint16_t *row = W + n * K;
        double lo = 0.0, hi = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double w = bf16_to_f64(row[k]);
            if (w < lo)
                lo = w;
            if (w > hi)
                hi = w;
        }
        float range = (float)(hi - lo);
        float sa = (float)((double)range / 15.0);
        int zn = 8;
        if (sa != 0.0f) {
            double c = nearbyint((double)(float)(-lo / (double)sa));
            if (c < 0.0)
                c = 0.0;
            if (c > 15.0)
                c = 15.0;
            zn = (int)c;
        }
        s[n] = sa;
        z[n] = (uint8_t)zn;
        for (int64_t j = 0; j < words; ++j) {
            uint32_t word = 0;
            for (int i = 0; i < 8; ++i) {
                int q = zn;
                if (sa != 0.0f) {
                    float qt = (float)(bf16_to_f64(row[8 * j + i]) / (double)sa);
                    double c = nearbyint((double)qt) + (double)zn; /* ties to even */
                    if (c < 0.0)
                        c = 0.0;
                    if (c > 15.0)
                        c = 15.0;
                    q = (int)c;
                }
                word |= (uint32_t)q << (4 * i);
            }
            codes[n * words + j] = word;
        }
    }
    return 0;
}

static int code_at(const uint32_t *codes, int64_t K, int64_t n, int64_t k)
{
    uint32_t word = codes[n * (K / 8) + k / 8];
    return (int)((word >> (4 * (k % 8))) & 0xFu);
}

/* Gate and EC down-projection of the tokens listed in t_list:
 * g[i] = sigmoid(x[t].w_g + b_g), u[i][j] = x[t].A[:,j]. */
static void gate_and_u(const uint16_t *x, int64_t K, int32_t r,
                       const uint16_t *A, const uint16_t *wg, double b_g,
                       const int64_t *t_list, int64_t count, double *g, double *u)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        const uint16_t *xt = x + t_list[i] * K;
        double logit = 0.0;
        for (int64_t k = 0; k < K; ++k)
            logit += bf16_to_f64(xt[k]) * bf16_to_f64(wg[k]);
        logit += b_g;
        g[i] = 1.0 / (1.0 + exp(-logit));
        for (int32_t j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += bf16_to_f64(xt[k]) * bf16_to_f64(A[k * r + j]);
            u[i * (int64_t)r + j] = acc;
        }
    }
}

/* g[t] for every token t < M. */
int oracle_gate(const uint16_t *x, int64_t M, int64_t K, const uint16_t *wg,
                double b_g, double *g)
{
    if (M < 0 || K < 0)
        return -1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < M; ++t) {
        double logit = 0.0;
        for (int64_t k = 0; k < K; ++k)
            logit += bf16_to_f64(x[t * K + k]) * bf16_to_f64(wg[k]);
        logit += b_g;
        g[t] = 1.0 / (1.0 + exp(-logit));
    }
    return 0;
}

/* Full forward: y [M][N] (fp64).  ec_on = 0 drops the correction term.
 * g_out [M] and corr_out [M][N] may be NULL. */
int oracle_forward(const uint16_t *x, int64_t M, int64_t K, int64_t N, int32_t r,
                   const uint32_t *codes, const float *s, const uint8_t *z,
                   const uint16_t *A, const uint16_t *B, const uint16_t *wg,
                   double b_g, int32_t ec_on,
                   double *y, double *g_out, double *corr_out)
{
    if (M < 0 || K < 0 || N < 0 || r < 0 || K % 8 != 0)
        return -1;
    int64_t *t_list = malloc(sizeof(int64_t) * (size_t)(M > 0 ? M : 1));
    double *g = malloc(sizeof(double) * (size_t)(M > 0 ? M : 1));
    double *u = malloc(sizeof(double) * (size_t)(M * (r > 0 ? r : 1) + 1));
    if (!t_list || !g || !u) {
        free(t_list); free(g); free(u);
        return -2;
    }
    for (int64_t t = 0; t < M; ++t)
        t_list[t] = t;
    gate_and_u(x, K, r, A, wg, b_g, t_list, M, g, u);

#pragma omp parallel
    {
        double *w_hat = malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
#pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            for (int64_t k = 0; k < K; ++k)
                w_hat[k] = (double)s[n] * (double)(code_at(codes, K, n, k) - (int)z[n]);
            for (int64_t t = 0; t < M; ++t) {
                const uint16_t *xt = x + t * K;
                double main_part = 0.0;
                for (int64_t k = 0; k < K; ++k)
                    main_part += bf16_to_f64(xt[k]) * w_hat[k];
                double corr = 0.0;
                if (ec_on && r > 0) {
                    double ub = 0.0;
                    for (int32_t j = 0; j < r; ++j)
                        ub += u[t * r + j] * bf16_to_f64(B[(int64_t)j * N + n]);
                    corr = g[t] * ub;
                }
                y[t * N + n] = main_part + corr;
                if (corr_out)
                    corr_out[t * N + n] = corr;
            }
        }
        free(w_hat);
    }
    if (g_out)
        for (int64_t t = 0; t < M; ++t)
            g_out[t] = g[t];
    free(t_list); free(g); free(u);
    return 0;
}

/* The same definition evaluated only at the listed outputs (t_idx[i], n_idx[i]);
 * used to check full-size launches output by output. */
int oracle_forward_sampled(const uint16_t *x, int64_t M, int64_t K, int64_t N, int32_t r,
                           const uint32_t *codes, const float *s, const uint8_t *z,
                           const uint16_t *A, const uint16_t *B, const uint16_t *wg,
                           double b_g, int32_t ec_on,
                           const int64_t *t_idx, const int64_t *n_idx, int64_t count,
                           double *y_out)
{
    if (M < 0 || K < 0 || N < 0 || r < 0 || K % 8 != 0 || count < 0)
        return -1;
    for (int64_t i = 0; i < count; ++i)
        if (t_idx[i] < 0 || t_idx[i] >= M || n_idx[i] < 0 || n_idx[i] >= N)
            return -1;
    double *g = malloc(sizeof(double) * (size_t)(count > 0 ? count : 1));
    double *u = malloc(sizeof(double) * (size_t)(count * (r > 0 ? r : 1) + 1));
    if (!g || !u) {
        free(g); free(u);
        return -2;
    }
    gate_and_u(x, K, r, A, wg, b_g, t_idx, count, g, u);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        int64_t t = t_idx[i], n = n_idx[i];
        double main_part = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double w_hat = (double)s[n] * (double)(code_at(codes, K, n, k) - (int)z[n]);
            main_part += bf16_to_f64(x[t * K + k]) * w_hat;
        }
        double corr = 0.0;
        if (ec_on && r > 0) {
            double ub = 0.0;
            for (int32_t j = 0; j < r; ++j)
                ub += u[i * r + j] * bf16_to_f64(B[(int64_t)j * N + n]);
            corr = g[i] * ub;
        }
        y_out[i] = main_part + corr;
    }
    free(g); free(u);
    return 0;
}
