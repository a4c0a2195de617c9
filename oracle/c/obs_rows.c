/*
 * The oracle's unblocked column-wise OBS loop in plain C: test
 * infrastructure, never linked into the product library.
 *
 * Same definition, same operations and same order per row as obs_quantize
 * in oracle/quantizer.py (KronQ summary (hyper.ai), "Method", Prop. 1: rows
 * of W are independent given the inverse Cholesky factor U of the damped
 * H_X; KronQ review (pith.science), appendix, Algorithm 2: quantize column
 * j, e = (w_j - w_hat_j) / U[j, j], w_k -= e U[j, k] for every later column
 * k).  Integer decisions (grid, code) in fp32, the rest in fp64.  Build with
 * -ffp-contract=off so that no product and sum are fused: every operation
 * rounds exactly as numpy's does.  Rows are independent, so they are split
 * over threads; a group of rows shares the pass over each row of U.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ROW_GROUP 16

/* Asymmetric grid of the fp32 values w32[0..len): lo = min(0, min w),
 * hi = max(0, max w), scale = (hi - lo) / maxq, zero = clamp(rint(-lo / scale)). */
static void grid(const double* w, int64_t len, float maxq, float* scale, float* zero) {
  float lo = 0.f, hi = 0.f;
  for (int64_t k = 0; k < len; ++k) {
    const float v = (float)w[k];
    if (v < lo) lo = v;
    if (v > hi) hi = v;
  }
  if (lo == 0.f && hi == 0.f) {
    *scale = 1.f;
    *zero = 0.f;
    return;
  }
  const float span = hi - lo;
  const float s = span / maxq;
  float z = rintf((-lo) / s);
  if (z < 0.f) z = 0.f;
  if (z > maxq) z = maxq;
  *scale = s;
  *zero = z;
}

/*
 * W: rows x n fp64, row-major, overwritten (the loop's working copy).
 * U: n x n fp64 row-major (upper triangle read).
 * codes rows x n, W_hat rows x n; scales / zeros rows x ng (ng = 1 or n / group).
 * Returns 0, or -1 for invalid arguments.
 */
int kronq_oracle_obs_rows(double* W, int64_t rows, int64_t n, const double* U, int bits,
                          int group, uint8_t* codes, float* scales, uint8_t* zeros,
                          double* W_hat, int threads) {
  if (rows < 0 || n <= 0 || !W || !U || !codes || !scales || !zeros || !W_hat) return -1;
  if (bits < 1 || bits > 8) return -1;
  if (group != -1 && (group <= 0 || n % group)) return -1;
  const int64_t ng = group == -1 ? 1 : n / group;
  const float maxq = (float)((1 << bits) - 1);
  const int64_t nblocks = (rows + ROW_GROUP - 1) / ROW_GROUP;
  if (threads > 0) {
#ifdef _OPENMP
    omp_set_num_threads(threads);
#endif
  }
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t b = 0; b < nblocks; ++b) {
    const int64_t r0 = b * ROW_GROUP;
    const int64_t r1 = r0 + ROW_GROUP < rows ? r0 + ROW_GROUP : rows;
    float sc[ROW_GROUP], zr[ROW_GROUP];
    double e[ROW_GROUP];
    if (group == -1) {
      for (int64_t r = r0; r < r1; ++r) {
        grid(W + r * n, n, maxq, &sc[r - r0], &zr[r - r0]);
        scales[r] = sc[r - r0];
        zeros[r] = (uint8_t)zr[r - r0];
      }
    }
    for (int64_t j = 0; j < n; ++j) {
      const double* Uj = U + j * n;
      for (int64_t r = r0; r < r1; ++r) {
        double* w = W + r * n;
        const int64_t i = r - r0;
        if (group != -1 && j % group == 0) {
          grid(w + j, group, maxq, &sc[i], &zr[i]);
          scales[r * ng + j / group] = sc[i];
          zeros[r * ng + j / group] = (uint8_t)zr[i];
        }
        const float w32 = (float)w[j];
        const int64_t zi = (int64_t)zr[i];
        int64_t q = (int64_t)rintf(w32 / sc[i]) + zi;
        if (q < 0) q = 0;
        if (q > (int64_t)maxq) q = (int64_t)maxq;
        const double wh = (double)sc[i] * (double)(q - zi);
        e[i] = (w[j] - wh) / Uj[j];
        codes[r * n + j] = (uint8_t)q;
        W_hat[r * n + j] = wh;
      }
      for (int64_t r = r0; r < r1; ++r) {
        double* w = W + r * n;
        const double ei = e[r - r0];
        for (int64_t k = j + 1; k < n; ++k) w[k] = w[k] - ei * Uj[k];
      }
    }
  }
  return 0;
}
