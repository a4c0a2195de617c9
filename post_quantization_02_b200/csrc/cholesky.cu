// Damping and the inverse Cholesky factor U_c (H_d^-1 = U_c^T U_c, U_c upper).
//
// KronQ review (pith.science), appendix, Algorithm 2, steps 1-2:
// H_X <- H_X + lambda mean(diag H_X) I, then the inverse Cholesky factor.
//
// Route (fp32): with J the index reversal, R = J H_d J = L L^T (lower
// Cholesky), and U_c = J L^-1 J: then U_c^T U_c = J L^-T L^-1 J = (J R J)^-1
// = H_d^-1 and U_c is upper triangular.  So: reverse-copy and damp, blocked
// right-looking Cholesky (64-wide panels: one CTA factors and inverts the
// diagonal block in shared memory, the panel below is multiplied by that
// inverse, the trailing lower triangle gets a rank-64 update), blocked
// forward substitution for L^-1 (block row by block row), reverse-copy out.
#include "common.cuh"
#include "gemm_simt.cuh"

namespace {

constexpr int NB = 64;

__global__ void diag_sum_kernel(const float* __restrict__ H, int n, double* out) {
  __shared__ double red[256];
  double s = 0.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) s += (double)H[(int64_t)i * n + i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = red[0];
}

// R[a][b] = H[n-1-a][n-1-b] + delta [a == b], delta = damp_rel * mean(diag H)
__global__ void reverse_damp_kernel(const float* __restrict__ H, int n, float* __restrict__ R,
                                    float damp_rel, const double* __restrict__ diag_sum) {
  const float delta = (float)((double)damp_rel * (*diag_sum / (double)n));
  const int64_t total = (int64_t)n * n;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int a = (int)(e / n), b = (int)(e % n);
    float v = H[(int64_t)(n - 1 - a) * n + (n - 1 - b)];
    if (a == b) v += delta;
    R[e] = v;
  }
}

// Factor the diagonal block R[k:k+nb, k:k+nb] = L L^T in place (lower part,
// upper part zeroed) and write L^-1 to Linv (nb x nb, leading dim NB).
__global__ void __launch_bounds__(256) potrf_diag_kernel(float* __restrict__ R, int n, int k,
                                                         float* __restrict__ Linv, int32_t* info) {
  __shared__ float A[NB][NB + 1];
  __shared__ float X[NB][NB + 1];
  __shared__ int bad;
  const int nb = min(NB, n - k);
  const int tid = threadIdx.x;
  if (tid == 0) bad = 0;
  for (int e = tid; e < NB * NB; e += blockDim.x) {
    const int i = e / NB, j = e % NB;
    A[i][j] = (i < nb && j <= i) ? R[(int64_t)(k + i) * n + (k + j)] : 0.f;
  }
  __syncthreads();
  for (int j = 0; j < nb; ++j) {
    if (tid == 0) {
      const float d = A[j][j];
      if (!(d > 0.f) || !isfinite(d)) {
        bad = 1;
        A[j][j] = 1.f;  // keep going with a placeholder; the result is flagged
      } else {
        A[j][j] = sqrtf(d);
      }
    }
    __syncthreads();
    const float piv = A[j][j];
    for (int i = j + 1 + tid; i < nb; i += blockDim.x) A[i][j] = A[i][j] / piv;
    __syncthreads();
    const int rem = nb - j - 1;
    for (int e = tid; e < rem * rem; e += blockDim.x) {
      const int i = j + 1 + e / rem, c = j + 1 + e % rem;
      if (c <= i) A[i][c] = fmaf(-A[i][j], A[c][j], A[i][c]);
    }
    __syncthreads();
  }
  // X = L^-1, one column per thread by forward substitution
  if (tid < NB) {
    const int c = tid;
    for (int i = 0; i < NB; ++i) {
      float v = 0.f;
      if (i < nb && c < nb && i >= c) {
        v = (i == c) ? 1.f : 0.f;
        for (int p = c; p < i; ++p) v = fmaf(-A[i][p], X[p][c], v);
        v = v / A[i][i];
      }
      X[i][c] = v;
    }
  }
  __syncthreads();
  for (int e = tid; e < NB * NB; e += blockDim.x) {
    const int i = e / NB, j = e % NB;
    if (i < nb && j < nb) {
      R[(int64_t)(k + i) * n + (k + j)] = (j <= i) ? A[i][j] : 0.f;
      Linv[i * NB + j] = X[i][j];
    }
  }
  if (tid == 0 && bad) kq::record_error(info, KRONQ_ERR_NOT_PD);
}

// Panel below the diagonal block: P <- P L_kk^-T (in place, one 64-column tile).
__global__ void __launch_bounds__(256) trsm_panel_kernel(float* R, int n, int k,
                                                         const float* __restrict__ Linv) {
  const int nb = min(NB, n - k);
  const int r0 = k + nb;
  float* P = R + (int64_t)r0 * n + k;
  kq::gemm_tile64<false, true>(P, n, Linv, NB, P, n, n - r0, nb, nb, 1.f, 0.f, blockIdx.x, 0);
}

// Trailing lower triangle: T <- T - P P^T.
__global__ void __launch_bounds__(256) syrk_lower_kernel(float* R, int n, int k) {
  const int tm = blockIdx.y, tn = blockIdx.x;
  if (tn > tm) return;
  const int nb = min(NB, n - k);
  const int r0 = k + nb;
  const float* P = R + (int64_t)r0 * n + k;
  float* T = R + (int64_t)r0 * n + r0;
  kq::gemm_tile64<false, true>(P, n, P, n, T, n, n - r0, n - r0, nb, -1.f, 1.f, tm, tn);
}

// Block row i of X = L^-1, step 1: S_j = L[i, j:i] X[j:i, j] for every block j < i.
__global__ void __launch_bounds__(256) trtri_gemm_kernel(const float* __restrict__ L,
                                                         const float* __restrict__ X, int n, int i,
                                                         float* __restrict__ S) {
  const int j = blockIdx.x;
  const int r0 = i * NB, c0 = j * NB;
  const int rows = min(NB, n - r0);
  const int K = r0 - c0;
  kq::gemm_tile64<false, false>(L + (int64_t)r0 * n + c0, n, X + (int64_t)c0 * n + c0, n,
                                S + c0, n, rows, NB, K, 1.f, 0.f, 0, 0);
}

// Step 2: X[i, j] = -L_ii^-1 S_j for j < i (one GEMM over all of them), X_ii = L_ii^-1.
__global__ void __launch_bounds__(256) trtri_scale_kernel(float* __restrict__ X, int n, int i,
                                                          const float* __restrict__ S,
                                                          const float* __restrict__ Linv_ii) {
  const int r0 = i * NB;
  const int rows = min(NB, n - r0);
  if ((int)blockIdx.x == i) {
    for (int e = threadIdx.x; e < rows * rows; e += blockDim.x) {
      const int a = e / rows, b = e % rows;
      X[(int64_t)(r0 + a) * n + r0 + b] = Linv_ii[a * NB + b];
    }
    return;
  }
  kq::gemm_tile64<false, false>(Linv_ii, NB, S, n, X + (int64_t)r0 * n, n, rows, r0, rows, -1.f,
                                0.f, 0, blockIdx.x);
}

// U[a][b] = X[n-1-a][n-1-b] for a <= b, 0 below the diagonal.
__global__ void reverse_out_kernel(const float* __restrict__ X, int n, float* __restrict__ U) {
  const int64_t total = (int64_t)n * n;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int a = (int)(e / n), b = (int)(e % n);
    U[e] = (a <= b) ? X[(int64_t)(n - 1 - a) * n + (n - 1 - b)] : 0.f;
  }
}

size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

}  // namespace

size_t kq_cholesky_ws(int64_t n) {
  const int64_t nblk = (n + NB - 1) / NB;
  return align256(sizeof(double)) + 2 * align256((size_t)n * n * sizeof(float)) +
         align256((size_t)nblk * NB * NB * sizeof(float)) + align256((size_t)NB * n * sizeof(float));
}

int kq_cholesky_inv(const float* H, int64_t n64, float damp_rel, float* U, int32_t* info, void* ws,
                    size_t ws_bytes, cudaStream_t st) {
  if (n64 < 0 || !(damp_rel >= 0.f)) return KRONQ_ERR_INVALID_ARG;
  if (n64 == 0) return KRONQ_OK;
  if (!H || !U || H == U) return KRONQ_ERR_INVALID_ARG;
  if (n64 > 65536) return KRONQ_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < kq_cholesky_ws(n64) || !kqh::aligned(ws, 256)) return KRONQ_ERR_WORKSPACE;
  const int n = (int)n64;
  uint8_t* w = static_cast<uint8_t*>(ws);
  double* dsum = reinterpret_cast<double*>(w);
  w += align256(sizeof(double));
  float* R = reinterpret_cast<float*>(w);
  w += align256((size_t)n * n * sizeof(float));
  float* X = reinterpret_cast<float*>(w);
  w += align256((size_t)n * n * sizeof(float));
  float* Ld = reinterpret_cast<float*>(w);
  w += align256((size_t)((n + NB - 1) / NB) * NB * NB * sizeof(float));
  float* S = reinterpret_cast<float*>(w);

  const int sms = kqh::num_sms();
  diag_sum_kernel<<<1, 256, 0, st>>>(H, n, dsum);
  KQ_CHECK_LAUNCH();
  reverse_damp_kernel<<<4 * sms, 256, 0, st>>>(H, n, R, damp_rel, dsum);
  KQ_CHECK_LAUNCH();
  const int nblk = (n + NB - 1) / NB;
  for (int b = 0; b < nblk; ++b) {
    const int k = b * NB;
    potrf_diag_kernel<<<1, 256, 0, st>>>(R, n, k, Ld + (size_t)b * NB * NB, info);
    KQ_CHECK_LAUNCH();
    const int rest = n - k - NB;
    if (rest > 0) {
      const int tiles = (rest + kq::GT - 1) / kq::GT;
      trsm_panel_kernel<<<tiles, 256, 0, st>>>(R, n, k, Ld + (size_t)b * NB * NB);
      KQ_CHECK_LAUNCH();
      syrk_lower_kernel<<<dim3(tiles, tiles), 256, 0, st>>>(R, n, k);
      KQ_CHECK_LAUNCH();
    }
  }
  for (int i = 0; i < nblk; ++i) {
    if (i > 0) {
      trtri_gemm_kernel<<<i, 256, 0, st>>>(R, X, n, i, S);
      KQ_CHECK_LAUNCH();
    }
    trtri_scale_kernel<<<i + 1, 256, 0, st>>>(X, n, i, S, Ld + (size_t)i * NB * NB);
    KQ_CHECK_LAUNCH();
  }
  reverse_out_kernel<<<4 * sms, 256, 0, st>>>(X, n, U);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}
