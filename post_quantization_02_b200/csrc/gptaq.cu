// GPTAQ asymmetric calibration: the drift covariance and the correction
// matrix P of the column loop.
//
// KronQ review (pith.science), appendix, Algorithm 2, step 3:
// P = alpha (Delta X X^T L) (.) M_U L^T, L <- InverseCholesky(H_X), M_U the
// upper-triangular mask; KronQ summary (hyper.ai), "Method": the asymmetric
// objective (the quantized layer sees the drifted input X~, its target is
// the full-precision W X).  With U_c the upper factor the solver reads
// (H_d^-1 = U_c^T U_c), L = U_c^T, so
//   T = A U_c^T,   P = alpha triu(T) U_c,
// two n x n x n products on the tensor cores (tf32, three-term split: the
// fp32-accurate GEMM the solver and the inverse Cholesky use).
//
// The drift covariance A = (1/N) sum_t (x_t - x~_t) x~_t^T comes from one
// covariance of the two inputs side by side, [X~ | X] (N x 2n): its leading
// block is H~ = X~^T X~ / N, its lower-left block X^T X~ / N, and
// A = X^T X~ / N - H~.
#include "common.cuh"
#include "gemm_tc.cuh"
#include "tf32x3.cuh"

int kq_covariance(const uint16_t* A, int64_t N, int64_t d, int64_t lda, float* H, int64_t ldh,
                  float alpha, float beta, int32_t* info, cudaStream_t st);

namespace {

size_t a256(size_t b) { return (b + 255) & ~(size_t)255; }

// H[i][j] = C[i][j], A[i][j] = C[n + i][j] - C[i][j] for i, j < n (C: 2n x 2n).
__global__ void drift_extract_kernel(const float* __restrict__ C, int n, float* __restrict__ H,
                                     float* __restrict__ A) {
  const int64_t total = (int64_t)n * n;
  const int64_t ldc = 2 * (int64_t)n;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = e / n, j = e % n;
    const float h = C[i * ldc + j];
    H[e] = h;
    A[e] = C[(n + i) * ldc + j] - h;
  }
}

// hi / lo planes of a row-major n x n matrix S (ld n), or of its transpose,
// or of its upper triangle (entries below the diagonal written as 0); one
// 32 x 32 tile per CTA through shared memory (coalesced on both sides).
enum SplitMode { kSplitPlain = 0, kSplitTranspose = 1, kSplitUpper = 2 };

__global__ void __launch_bounds__(256) split_kernel(const float* __restrict__ S, int n, int mode,
                                                    float* __restrict__ Dh, float* __restrict__ Dl) {
  __shared__ float t[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;     // destination tile origin
  if (mode == kSplitTranspose) {
    // D[r][c] = S[c][r]: read the source tile (c0.., r0..) row by row
    for (int y = ty; y < 32; y += 8) {
      const int sr = c0 + y, sc = r0 + tx;
      t[y][tx] = (sr < n && sc < n) ? S[(int64_t)sr * n + sc] : 0.f;
    }
    __syncthreads();
    for (int y = ty; y < 32; y += 8) {
      const int r = r0 + y, c = c0 + tx;
      if (r < n && c < n) {
        const float v = t[tx][y];
        const float h = kq::tf32x3::hi(v);
        Dh[(int64_t)r * n + c] = h;
        Dl[(int64_t)r * n + c] = v - h;
      }
    }
    return;
  }
  for (int y = ty; y < 32; y += 8) {
    const int r = r0 + y, c = c0 + tx;
    if (r < n && c < n) {
      float v = S[(int64_t)r * n + c];
      if (mode == kSplitUpper && c < r) v = 0.f;
      const float h = kq::tf32x3::hi(v);
      Dh[(int64_t)r * n + c] = h;
      Dl[(int64_t)r * n + c] = v - h;
    }
  }
}

}  // namespace

size_t kq_drift_ws(int64_t n) { return a256((size_t)4 * n * n * sizeof(float)); }

size_t kq_correction_ws(int64_t n) {
  return 4 * a256((size_t)n * n * sizeof(float)) + a256((size_t)n * n * sizeof(float));
}

int kq_drift_covariance(const uint16_t* XqX, int64_t N, int64_t n, int64_t ld, float* H, float* A,
                        int32_t* info, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!H || !A || H == A || n <= 0 || N < 0 || ld < 2 * n) return KRONQ_ERR_INVALID_ARG;
  if (N > 0 && !XqX) return KRONQ_ERR_INVALID_ARG;
  if (n > 32768) return KRONQ_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < kq_drift_ws(n) || !kqh::aligned(ws, 256)) return KRONQ_ERR_WORKSPACE;
  float* C = static_cast<float*>(ws);
  const int s = kq_covariance(XqX, N, 2 * n, ld, C, 2 * n, N > 0 ? 1.f / (float)N : 0.f, 0.f,
                              info, st);
  if (s != KRONQ_OK) return s;
  drift_extract_kernel<<<4 * kqh::num_sms(), 256, 0, st>>>(C, (int)n, H, A);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

int kq_gptaq_correction(const float* A, const float* U, int64_t n64, float alpha, float* P,
                        int32_t* info, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!A || !U || !P || P == A || P == U || n64 <= 0) return KRONQ_ERR_INVALID_ARG;
  if (!(alpha == alpha)) return KRONQ_ERR_INVALID_ARG;
  if (n64 > 32768) return KRONQ_ERR_UNSUPPORTED;
  if (n64 % 4) return KRONQ_ERR_INVALID_ARG;               // 16-byte rows for the tensor maps
  if (!kqh::aligned(A, 16) || !kqh::aligned(U, 16) || !kqh::aligned(P, 16))
    return KRONQ_ERR_INVALID_ARG;
  if (!ws || ws_bytes < kq_correction_ws(n64) || !kqh::aligned(ws, 256)) return KRONQ_ERR_WORKSPACE;
  const int n = (int)n64;
  const size_t plane = a256((size_t)n * n * sizeof(float));
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* Ah = reinterpret_cast<float*>(w);
  float* Al = reinterpret_cast<float*>(w + plane);
  float* Bh = reinterpret_cast<float*>(w + 2 * plane);
  float* Bl = reinterpret_cast<float*>(w + 3 * plane);
  float* T = reinterpret_cast<float*>(w + 4 * plane);
  const dim3 g((n + 31) / 32, (n + 31) / 32);
  // T = A U_c^T  (both operands row-major: K-major for the NT product)
  split_kernel<<<g, 256, 0, st>>>(A, n, kSplitPlain, Ah, Al);
  KQ_CHECK_LAUNCH();
  split_kernel<<<g, 256, 0, st>>>(U, n, kSplitPlain, Bh, Bl);
  KQ_CHECK_LAUNCH();
  if (cudaMemsetAsync(T, 0, (size_t)n * n * sizeof(float), st) != cudaSuccess) return KRONQ_ERR_CUDA;
  {
    const kq::GemmNT p = {Ah, Al, n, Bh, Bl, n, T, n, n, n, n, 1.f, 0};
    const int s = kq_gemm_nt_tc(&p, 1, info, st);
    if (s != KRONQ_OK) return s;
  }
  // P = alpha triu(T) U_c: B rows = rows of U_c^T
  split_kernel<<<g, 256, 0, st>>>(T, n, kSplitUpper, Ah, Al);
  KQ_CHECK_LAUNCH();
  split_kernel<<<g, 256, 0, st>>>(U, n, kSplitTranspose, Bh, Bl);
  KQ_CHECK_LAUNCH();
  if (cudaMemsetAsync(P, 0, (size_t)n * n * sizeof(float), st) != cudaSuccess) return KRONQ_ERR_CUDA;
  const kq::GemmNT p = {Ah, Al, n, Bh, Bl, n, P, n, n, n, n, alpha, 0};
  return kq_gemm_nt_tc(&p, 1, info, st);
}
