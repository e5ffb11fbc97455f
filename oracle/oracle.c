/*
 * oracle.c -- plain fp64 CPU reference for Stable Diffusion UNet attention.
 *
 * TEST INFRASTRUCTURE ONLY.  The tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may call this; the product path never does.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes follows the plain definition of exact attention,
 * O = softmax(scale * Q K^T) V, which both forms described in
 * "Speed Is All You Need: On-Device Acceleration of Large Diffusion Models
 * via GPU-Aware Optimizations" (news summary, section on the three
 * optimisations, "partially fused softmax" and "FlashAttention" paragraphs)
 * must reach: FlashAttention is called exact attention there, and the
 * partially fused form only regroups the same softmax around per-row
 * statistics L and S (an N x 2 tensor).
 *
 * Readings of what the page leaves open (stated again in the design notes):
 *   - A = scale * Q K^T, scale taken from the caller (1/sqrt(d) in the study);
 *   - L_i = max_j A_ij, S_i = sum_j exp(A_ij - L_i), natural base;
 *   - the normalisation divides once per output: o_ic = (sum_j e_ij v_jc) / S_i;
 *   - no mask.
 *
 * Layouts (row-major, contiguous): Q [B][H][N][d], K and V [B][H][M][d],
 * O [B][H][N][d], LS [B][H][N][2] (L at 0, S at 1), A [B][H][N][M].
 * Inputs are the exact values the GPU receives, widened to double.
 *
 * Every step runs in fp64 in plain index order; rows are spread over OpenMP
 * threads, which changes no arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Returns 0 on success, 1 on an allocation failure or bad sizes. */
int oracle_attention(int64_t B, int64_t H, int64_t N, int64_t M, int64_t d,
                     double scale,
                     const double *Q, const double *K, const double *V,
                     double *O, double *LS, double *A)
{
    if (B < 1 || H < 1 || N < 0 || M < 1 || d < 1) return 1;
    const int64_t rows = B * H * N;
    int failed = 0;

#pragma omp parallel
    {
        double *a = (double *)malloc((size_t)M * sizeof(double));
        double *e = (double *)malloc((size_t)M * sizeof(double));
        if (!a || !e) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < rows; ++r) {
            if (!a || !e) continue;
            const int64_t bh = r / N;
            const double *q = Q + r * d;
            const double *Kh = K + bh * M * d;
            const double *Vh = V + bh * M * d;

            /* step 1: scores a_ij = scale * sum_k q_ik k_jk */
            for (int64_t j = 0; j < M; ++j) {
                double dot = 0.0;
                for (int64_t k = 0; k < d; ++k) dot += q[k] * Kh[j * d + k];
                a[j] = scale * dot;
            }
            /* step 2: L_i = max_j a_ij */
            double L = a[0];
            for (int64_t j = 1; j < M; ++j)
                if (a[j] > L) L = a[j];
            /* step 3: e_ij = exp(a_ij - L_i), S_i = sum_j e_ij */
            double S = 0.0;
            for (int64_t j = 0; j < M; ++j) {
                e[j] = exp(a[j] - L);
                S += e[j];
            }
            /* step 4: o_ic = (sum_j e_ij v_jc) / S_i */
            double *o = O + r * d;
            for (int64_t c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int64_t j = 0; j < M; ++j) acc += e[j] * Vh[j * d + c];
                o[c] = acc / S;
            }
            LS[2 * r + 0] = L;
            LS[2 * r + 1] = S;
            if (A) {
                double *arow = A + r * M;
                for (int64_t j = 0; j < M; ++j) arow[j] = a[j];
            }
        }
        free(a);
        free(e);
    }
    return failed;
}
