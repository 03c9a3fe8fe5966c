/*
 * rb_oracle.c -- plain, slow fp64 CPU oracle for residual binarization.
 *
 * TEST INFRASTRUCTURE ONLY. The tests, the package's smoke check and the
 * bench's CPU-baseline leg call this code to produce expected values; the
 * product path never links or calls it, and it shares no code with the CUDA
 * kernels.
 *
 * What it computes (one function per step, each written out directly):
 *
 *  rbo_pack   -- residual path derivation. RaBiT (arXiv 2602.05367), section
 *               4.2 "Coupled Training" and appendix G "RaBiT training": every
 *               path is taken from one shared full-precision weight; path k
 *               binarizes the residual left by paths 1..k-1 and the residual is
 *               updated after each path (appendix A: R1 = W_FP - W^_1,
 *               B2 = sign(R1)). The per-path scale is the closed-form
 *               least-squares scale for fixed signs, mean |R| over the row or
 *               over a group of 128 columns, which is the "cascaded analytical
 *               residual" initialisation of QBB (atlas.scime.ai summary of
 *               "QBB: Quantization with Binary Bases for LLMs", Approach). The
 *               pages do not print the formula; this is the plainest reading.
 *               sign(0) = +1, including -0.0.
 *
 *  rbo_matvec -- the layer output y = sum_k alpha_k (.) (B_k x), RaBiT
 *               section 4.1 (binary cores with per-channel scales, evaluated
 *               with additions and subtractions): evaluated here as a direct
 *               fp64 sum of +x_j / -x_j, with no masked-sum identity, so it is
 *               independent of the way the kernels evaluate it.
 *
 *  rbo_pack_fixed -- the same sequential derivation with scales the caller
 *               gives instead of mean |R|: RaBiT section 4.1 ("dual-scale"
 *               binary cores with per-channel output and input scaling
 *               vectors, W^_k = diag(h_k) B_k diag(g_k)) and section 4.2
 *               (paths derived in turn from the shared weight, scales
 *               learned). Signs only: B_k = sign(R_{k-1}),
 *               R_k[i][j] = R_{k-1}[i][j] - h_k[i] g_k[j] B_k[i][j].
 *
 *  rbo_dual_matvec -- the dual-scale block's output
 *               y = sum_k h_k (.) (B_k (g_k (.) x)), RaBiT section 4.1, with
 *               g_k (.) x taken as an fp16 activation (A16): each product is
 *               rounded to the nearest fp16 before the binary core sees it
 *               (a reading; the pages do not say in which precision the
 *               input vector is applied). Direct fp64 sum of +-x, as in
 *               rbo_matvec.
 *
 * Bit layout (a reading; RaBiT appendix D only says 32 columns go into one
 * uint32): bit j of word w of a row holds column 32*w + j, and a set bit
 * means +1. Planes are stored [N][M][K/32].
 *
 * Everything is fp64; sums of |R| use Neumaier-compensated long double.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

/* Compensated sum of |r[0..n)| in long double, rounded to double at the end. */
static long double abs_sum(const double* r, int64_t n) {
    long double s = 0.0L, c = 0.0L;
    for (int64_t j = 0; j < n; ++j) {
        long double v = fabsl((long double)r[j]);
        long double t = s + v;
        if (fabsl(s) >= fabsl(v)) c += (s - t) + v;
        else                      c += (v - t) + s;
        s = t;
    }
    return s + c;
}

/*
 * W      : M x K weights as doubles, row-major (exact copies of fp16/fp32).
 * N      : number of binary paths (>= 1).
 * G      : columns per scale group (K for one scale per row; must divide K).
 * planes : out, N*M*(K/32) words (K must be a multiple of 32).
 * alpha  : out, N*M*(K/G) scales.
 * rabs   : out (nullable), N*M*K values |R_{k-1}[i][j]|, the magnitude each
 *          sign decision was taken on (used to recognise near-zero ties).
 * Returns 0, or -1 on a bad shape.
 */
int rbo_pack(const double* W, int64_t M, int64_t K, int32_t N, int64_t G,
             uint32_t* planes, double* alpha, double* rabs) {
    if (M < 0 || K <= 0 || N < 1 || G <= 0 || K % G != 0 || K % 32 != 0) return -1;
    const int64_t words = K / 32, groups = K / G;
    memset(planes, 0, sizeof(uint32_t) * (size_t)(N * M * words));
#pragma omp parallel
    {
        double* R = (double*)malloc(sizeof(double) * (size_t)G);
#pragma omp for schedule(dynamic, 4)
        for (int64_t i = 0; i < M; ++i) {
            for (int64_t g = 0; g < groups; ++g) {
                const int64_t j0 = g * G;
                for (int64_t j = 0; j < G; ++j) R[j] = W[i * K + j0 + j];   /* R_0 = W */
                for (int32_t k = 0; k < N; ++k) {
                    /* alpha_k = mean |R_{k-1}| over the group */
                    const double a = (double)(abs_sum(R, G) / (long double)G);
                    alpha[((int64_t)k * M + i) * groups + g] = a;
                    for (int64_t j = 0; j < G; ++j) {
                        const int64_t col = j0 + j;
                        if (rabs) rabs[((int64_t)k * M + i) * K + col] = fabs(R[j]);
                        /* B_k = sign(R_{k-1}), with sign(0) = +1 (also for -0.0) */
                        const double b = (R[j] >= 0.0) ? 1.0 : -1.0;
                        if (b > 0.0)
                            planes[((int64_t)k * M + i) * words + col / 32] |= (uint32_t)1u << (col % 32);
                        /* R_k = R_{k-1} - alpha_k * B_k */
                        R[j] = R[j] - a * b;
                    }
                }
            }
        }
        free(R);
    }
    return 0;
}

/*
 * planes : N*M*(K/32) words in the layout above.
 * alpha  : N*M*(K/G) scales (as doubles; pass exact copies of whatever the
 *          caller stores, e.g. fp16 values widened to double).
 * x      : T x K activations as doubles.
 * y      : out, T x M outputs.
 * denom  : out (nullable), T x M values sum_k sum_j |alpha_k[i,g(j)] * x_t[j]|,
 *          the scale the output tolerance is measured against.
 */
int rbo_matvec(const uint32_t* planes, const double* alpha, int64_t M, int64_t K,
               int32_t N, int64_t G, const double* x, int64_t T,
               double* y, double* denom) {
    if (M < 0 || K <= 0 || N < 1 || G <= 0 || K % G != 0 || K % 32 != 0 || T < 0) return -1;
    const int64_t words = K / 32, groups = K / G;
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t i = 0; i < M; ++i) {
            double acc = 0.0, den = 0.0;
            for (int32_t k = 0; k < N; ++k) {
                const uint32_t* row = planes + ((int64_t)k * M + i) * words;
                const double* arow = alpha + ((int64_t)k * M + i) * groups;
                for (int64_t j = 0; j < K; ++j) {
                    const double a = arow[j / G];
                    const double xv = x[t * K + j];
                    const int bit = (int)((row[j / 32] >> (j % 32)) & 1u);
                    acc += bit ? a * xv : -(a * xv);
                    den += fabs(a * xv);
                }
            }
            y[t * M + i] = acc;
            if (denom) denom[t * M + i] = den;
        }
    }
    return 0;
}

/*
 * W      : M x K weights as doubles, row-major.
 * h      : N x M output-channel scales (h_k[i] >= 0).
 * g      : N x K input-channel scales, or NULL for all ones.
 * planes : out, N*M*(K/32) words.
 * rabs   : out (nullable), N*M*K values |R_{k-1}[i][j]|.
 */
int rbo_pack_fixed(const double* W, int64_t M, int64_t K, int32_t N, const double* h, const double* g,
                   uint32_t* planes, double* rabs) {
    if (M < 0 || K <= 0 || N < 1 || K % 32 != 0) return -1;
    const int64_t words = K / 32;
    memset(planes, 0, sizeof(uint32_t) * (size_t)(N * M * words));
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t i = 0; i < M; ++i) {
        for (int64_t j = 0; j < K; ++j) {
            double r = W[i * K + j];   /* R_0 = W */
            for (int32_t k = 0; k < N; ++k) {
                const double scale = h[(int64_t)k * M + i] * (g ? g[(int64_t)k * K + j] : 1.0);
                if (rabs) rabs[((int64_t)k * M + i) * K + j] = fabs(r);
                /* B_k = sign(R_{k-1}), sign(0) = +1 */
                const double b = (r >= 0.0) ? 1.0 : -1.0;
                if (b > 0.0) planes[((int64_t)k * M + i) * words + j / 32] |= (uint32_t)1u << (j % 32);
                /* R_k = R_{k-1} - h_k[i] g_k[j] B_k */
                r = r - scale * b;
            }
        }
    }
    return 0;
}

/*
 * planes : N*M*(K/32) words.   h : N x M.   g : N x K (NULL: all ones).
 * xk     : N x T x K, the fp16-rounded products g_k[j] * x_t[j] (the caller
 *          rounds them; see the header comment), as doubles.
 * y      : out, T x M.  denom : out (nullable), T x M values
 *          sum_k sum_j |h_k[i] * xk[k][t][j]|, the tolerance scale.
 */
int rbo_dual_matvec(const uint32_t* planes, const double* h, int64_t M, int64_t K, int32_t N,
                    const double* xk, int64_t T, double* y, double* denom) {
    if (M < 0 || K <= 0 || N < 1 || K % 32 != 0 || T < 0) return -1;
    const int64_t words = K / 32;
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t i = 0; i < M; ++i) {
            double acc = 0.0, den = 0.0;
            for (int32_t k = 0; k < N; ++k) {
                const uint32_t* row = planes + ((int64_t)k * M + i) * words;
                const double hk = h[(int64_t)k * M + i];
                const double* xr = xk + ((int64_t)k * T + t) * K;
                for (int64_t j = 0; j < K; ++j) {
                    const int bit = (int)((row[j / 32] >> (j % 32)) & 1u);
                    acc += bit ? hk * xr[j] : -(hk * xr[j]);
                    den += fabs(hk * xr[j]);
                }
            }
            y[t * M + i] = acc;
            if (denom) denom[t * M + i] = den;
        }
    }
    return 0;
}
