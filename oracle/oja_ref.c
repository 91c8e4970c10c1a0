/* Float64 sequential Oja subspace rule, one stream per OpenMP task.
 *
 * TEST INFRASTRUCTURE ONLY: part of the CPU oracle.  It is compiled by
 * oracle/build_oracle.py and called from oracle/lrkv_oracle.py; the product
 * library never links or loads it.
 *
 * Rule (OjaKV page, online subspace adaptation with Oja's algorithm for
 * online PCA): for each token x in order, y = P^T x and
 * P <- P + eta (x - P y) y^T.  After every qr_every-th token (counted from
 * the start of the stream, tokens_seen tokens before this call) P is
 * replaced by the Q factor of its QR decomposition with diag(R) > 0, done
 * here by Gram-Schmidt with one re-orthogonalisation pass per column, which
 * yields that unique Q for a full-rank P.
 *
 * P: [S][128][r] row-major, updated in place.  X: [S][n][128] float32.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define D 128

static void qr_positive(double *P, int r, double *col) {
  for (int j = 0; j < r; ++j) {
    for (int i = 0; i < D; ++i) col[i] = P[i * r + j];
    for (int pass = 0; pass < 2; ++pass) {
      for (int k = 0; k < j; ++k) {
        double h = 0.0;
        for (int i = 0; i < D; ++i) h += P[i * r + k] * col[i];
        for (int i = 0; i < D; ++i) col[i] -= h * P[i * r + k];
      }
    }
    double nrm = 0.0;
    for (int i = 0; i < D; ++i) nrm += col[i] * col[i];
    nrm = sqrt(nrm);
    for (int i = 0; i < D; ++i) P[i * r + j] = col[i] / nrm;
  }
}

static void oja_stream(double *P, const float *X, int r, int n, double eta,
                       int qr_every, long tokens_seen) {
  double *y = (double *)malloc(sizeof(double) * (size_t)r);
  double *x = (double *)malloc(sizeof(double) * D);
  double *z = (double *)malloc(sizeof(double) * D);
  for (int t = 0; t < n; ++t) {
    for (int i = 0; i < D; ++i) x[i] = (double)X[(size_t)t * D + i];
    for (int j = 0; j < r; ++j) y[j] = 0.0;
    for (int i = 0; i < D; ++i)
      for (int j = 0; j < r; ++j) y[j] += P[i * r + j] * x[i];
    for (int i = 0; i < D; ++i) {
      double py = 0.0;
      for (int j = 0; j < r; ++j) py += P[i * r + j] * y[j];
      z[i] = x[i] - py;
    }
    for (int i = 0; i < D; ++i)
      for (int j = 0; j < r; ++j) P[i * r + j] += eta * z[i] * y[j];
    if (qr_every > 0 && (tokens_seen + t + 1) % qr_every == 0)
      qr_positive(P, r, z);
  }
  free(y);
  free(x);
  free(z);
}

void oja_ref_f64(double *P, const float *X, int S, int r, int n, double eta,
                 int qr_every, long tokens_seen) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int s = 0; s < S; ++s)
    oja_stream(P + (size_t)s * D * r, X + (size_t)s * n * D, r, n, eta,
               qr_every, tokens_seen);
}

int oja_ref_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
