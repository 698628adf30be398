/*
 * bsl_oracle.c -- plain fp64 CPU oracle for the block-sparse linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library
 * and its Python binding) may link, load or call this file; only the tests,
 * the package's smoke check and the benchmark's CPU-baseline leg do.  It
 * shares no code, header or table with the CUDA sources.
 *
 * What it computes.  Hugging Face pytorch_block_sparse release note,
 * "Block-Sparse Implementation and Usage": BlockSparseLinear is a drop-in
 * nn.Linear whose weight keeps only its nonzero b x b blocks.  torchao
 * sparsity README, introduction: the backend receives the pruned weight as
 * an ordinary dense tensor holding zeros at the pruned positions, and the
 * sparse product must equal the dense product with that tensor.  So the
 * oracle is the dense product, zeros included:
 *
 *   Wt[n][k]  = W[n][k] if mask[n/b][k/b] != 0, else 0      (dense with zeros)
 *   Y[m][n]   = sum_k X[m][k]  * Wt[n][k]                   (forward, Y = X Wt^T)
 *   dX[m][k]  = sum_n dY[m][n] * Wt[n][k]                   (input gradient, dX = dY Wt)
 *   dW[n][k]  = sum_m dY[m][n] * X[m][k], kept only where the mask is set
 *               (torchao README, "Pruning Criteria", out-of-place updates:
 *               dW' = dW (.) Mask)
 *
 * Every input is a bf16 bit pattern; it is widened exactly to double and all
 * sums run in double, in index order, over the full dense range (the zeros of
 * Wt included).  Each routine also returns sum |term| over the same index,
 * which the tests use to scale their tolerance.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC bsl_oracle.c -o liboracle.so
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_to_double(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Wt = W with zeros outside the mask, as a dense N x K double matrix. */
void bsl_oracle_dense_weight(int64_t N, int64_t K, int64_t b,
                             const uint16_t *W, const uint8_t *mask,
                             double *Wt)
{
    const int64_t C = K / b;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            Wt[n * K + k] = mask[(n / b) * C + (k / b)] ? bf16_to_double(W[n * K + k]) : 0.0;
}

/* bf16 matrix -> double matrix (exact). */
void bsl_oracle_widen(int64_t count, const uint16_t *src, double *dst)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i)
        dst[i] = bf16_to_double(src[i]);
}

/* Forward on the listed token rows: Y[i][n] = sum_k X[rows[i]][k] * Wt[n][k]. */
void bsl_oracle_forward_rows(int64_t M, int64_t N, int64_t K,
                             const double *X, const double *Wt,
                             const int64_t *rows, int64_t nrows,
                             double *Y, double *Yabs)
{
    (void)M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        const double *x = X + rows[i] * K;
        for (int64_t n = 0; n < N; ++n) {
            const double *w = Wt + n * K;
            double s = 0.0, a = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double t = x[k] * w[k];
                s += t;
                a += fabs(t);
            }
            Y[i * N + n] = s;
            Yabs[i * N + n] = a;
        }
    }
}

/* The same forward with the masked-out blocks skipped instead of multiplied
 * as zeros: for output n, only the k inside kept blocks of block row n / b
 * are visited, still in increasing k.  A skipped term is +-0, which never
 * changes a double sum that starts at +0, so the result is bit-identical to
 * bsl_oracle_forward_rows; it is timed beside it as the CPU baseline that
 * does only the stored blocks' work (the layer computes only the nonzero
 * blocks: Hugging Face pytorch_block_sparse release note, "Block-Sparse
 * Implementation and Usage"). */
void bsl_oracle_forward_rows_blockskip(int64_t M, int64_t N, int64_t K, int64_t b,
                                       const double *X, const double *Wt, const uint8_t *mask,
                                       const int64_t *rows, int64_t nrows,
                                       double *Y, double *Yabs)
{
    (void)M;
    const int64_t C = K / b;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        const double *x = X + rows[i] * K;
        for (int64_t n = 0; n < N; ++n) {
            const double *w = Wt + n * K;
            const uint8_t *mrow = mask + (n / b) * C;
            double s = 0.0, a = 0.0;
            for (int64_t c = 0; c < C; ++c) {
                if (!mrow[c]) continue;
                for (int64_t k = c * b; k < (c + 1) * b; ++k) {
                    double t = x[k] * w[k];
                    s += t;
                    a += fabs(t);
                }
            }
            Y[i * N + n] = s;
            Yabs[i * N + n] = a;
        }
    }
}

/* Input gradient on the listed token rows: dX[i][k] = sum_n dY[rows[i]][n] * Wt[n][k].
 * For each output element the terms are added in increasing n. */
void bsl_oracle_backward_input_rows(int64_t M, int64_t N, int64_t K,
                                    const double *dY, const double *Wt,
                                    const int64_t *rows, int64_t nrows,
                                    double *dX, double *dXabs)
{
    (void)M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        const double *dy = dY + rows[i] * N;
        double *s = dX + i * K;
        double *a = dXabs + i * K;
        for (int64_t k = 0; k < K; ++k) {
            s[k] = 0.0;
            a[k] = 0.0;
        }
        for (int64_t n = 0; n < N; ++n) {
            const double *w = Wt + n * K;
            for (int64_t k = 0; k < K; ++k) {
                double t = dy[n] * w[k];
                s[k] += t;
                a[k] += fabs(t);
            }
        }
    }
}

/* Weight gradient at listed blocks (block row br[i], block column bc[i]):
 *   dWb[i][u][v] = sum_m dY[m][br*b+u] * X[m][bc*b+v],  u, v in [0, b).
 * These are the entries of dW = dY^T X that the mask keeps. */
void bsl_oracle_backward_weight_blocks(int64_t M, int64_t N, int64_t K, int64_t b,
                                       const double *dY, const double *X,
                                       const int64_t *br, const int64_t *bc,
                                       int64_t nblocks,
                                       double *dWb, double *dWabs)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nblocks; ++i) {
        for (int64_t u = 0; u < b; ++u) {
            const int64_t n = br[i] * b + u;
            for (int64_t v = 0; v < b; ++v) {
                const int64_t k = bc[i] * b + v;
                double s = 0.0, a = 0.0;
                for (int64_t m = 0; m < M; ++m) {
                    double t = dY[m * N + n] * X[m * K + k];
                    s += t;
                    a += fabs(t);
                }
                dWb[(i * b + u) * b + v] = s;
                dWabs[(i * b + u) * b + v] = a;
            }
        }
    }
}

int bsl_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
