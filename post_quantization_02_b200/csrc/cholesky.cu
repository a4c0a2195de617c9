// Damping and the inverse Cholesky factor U_c (H_d^-1 = U_c^T U_c, U_c upper).
//
// KronQ review (pith.science), appendix, Algorithm 2, steps 1-2:
// H_X <- H_X + lambda mean(diag H_X) I, then the inverse Cholesky factor.
//
// Route (fp32 throughout): with J the index reversal, R = J H_d J = L L^T
// (lower Cholesky) and U_c = J L^-1 J; then U_c^T U_c = J (L L^T)^-1 J =
// H_d^-1 and U_c is upper triangular.
//
// One right-looking sweep over 128-wide panels computes L and Y = L^-1
// together (block forward substitution of L Y = I carried along with the
// factorisation).  Step p (rows k = 128 p ...):
//   panel kernel   every CTA factors the 128 x 128 diagonal block
//                  R_pp = L_pp L_pp^T and inverts L_pp in shared memory, then
//                  either turns 128 rows of the panel into L_ip = R_ip L_pp^-T,
//                  or finishes 128 columns of block row p of Y:
//                  Y_pj = L_pp^-1 A_pj  (A_pj = -sum_{q<p} L_pq Y_qj), Y_pp = L_pp^-1.
//   update kernel  for every block row i > p: the trailing lower triangle
//                  R_ij -= L_ip L_jp^T and the accumulators A_ij -= L_ip Y_pj
//                  (j <= p), as 128 x 128 fp32 GEMM tiles with K = 128.
// Then U_c[a][b] = Y[n-1-a][n-1-b] (a <= b).
#include "common.cuh"
#include "gemm_simt.cuh"

namespace {

constexpr int NB = 128;
constexpr int LDD = NB + 1;   // padded leading dimension of the diagonal block in smem

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

// R[a][b] = H[n-1-a][n-1-b] + delta [a == b], delta = damp_rel * mean(diag H); Y = 0.
__global__ void reverse_damp_kernel(const float* __restrict__ H, int n, float* __restrict__ R,
                                    float* __restrict__ Y, float damp_rel,
                                    const double* __restrict__ diag_sum) {
  const float delta = (float)((double)damp_rel * (*diag_sum / (double)n));
  const int64_t total = (int64_t)n * n;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int a = (int)(e / n), b = (int)(e % n);
    float v = H[(int64_t)(n - 1 - a) * n + (n - 1 - b)];
    if (a == b) v += delta;
    R[e] = v;
    Y[e] = 0.f;
  }
}

// X = L^-1 for the lower Cholesky factor L of the 128 x 128 block in D
// (fp32; rows/columns kb .. NB-1 are padded with the identity by the caller;
// D is overwritten with scratch).
//
// One sweep of 128 column steps does the factorisation and the inverse
// together: at step j the pivot column of the Schur complement and the
// accumulated row j of L^-1 are both final, so with r = 1/sqrt(d_j):
//   L[i][j] = S[i][j] r,   Y[j][:] = A[j][:] r,
//   S[i][c] -= L[i][j] L[c][j]      (the trailing Schur complement)
//   A[i][:] -= L[i][j] Y[j][:]      (i > j, the rows of L^-1 still open).
// Thread (ty, tx) keeps the 8 x 8 tiles of S and A at rows 8ty.., columns
// 8tx.. in registers; warp w owns the column tiles tx = 2w, 2w+1 (ty = lane
// mod 16), so at step j a warp's choice is uniform: tiles with columns > j
// need the S update, tiles with columns <= j the A update (only the tile
// holding column j needs both).  Entries that are already final or never
// used absorb harmless updates.  After its last update, column j+1 of S and
// row j+1 of A are published to shared memory; one barrier per step.
__device__ void factor_and_invert(float* D, float* X, int kb, int* bad) {
  __shared__ __align__(16) float colbuf[2][NB];
  __shared__ __align__(16) float rowbuf[2][NB];
  const int tid = threadIdx.x;
  const int ty = tid & 15, tx = ((tid >> 5) << 1) | ((tid >> 4) & 1);
  float a[8][8], y[8][8];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      a[r][c] = D[(8 * ty + r) * LDD + 8 * tx + c];
      y[r][c] = (8 * ty + r == 8 * tx + c) ? 1.f : 0.f;
    }
  if (tid < NB) {
    colbuf[0][tid] = D[tid * LDD];          // column 0 of S
    rowbuf[0][tid] = (tid == 0) ? 1.f : 0.f;  // row 0 of A (identity)
  }
  __syncthreads();
  for (int jb = 0; jb < NB / 8; ++jb) {
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int j = 8 * jb + jj;
      const int b = jj & 1;                 // j & 1 (8 * jb is even)
      float d = colbuf[b][j];
      if (!(d > 0.f) || !isfinite(d)) {
        if (tid == 0 && j < kb) *bad = 1;
        d = 1.f;
      }
      const float rs = rsqrtf(d);
      if (tid < NB) X[j * LDD + tid] = rowbuf[b][tid] * rs;   // row j of L^-1, final
      const bool do_s = 8 * tx + 7 > j, do_a = 8 * tx <= j;
      {
        float li[8], lc[8], yj[8];
        {
          const float4 p0 = *reinterpret_cast<const float4*>(&colbuf[b][8 * ty]);
          const float4 p1 = *reinterpret_cast<const float4*>(&colbuf[b][8 * ty + 4]);
          const float4 q0 = *reinterpret_cast<const float4*>(&colbuf[b][8 * tx]);
          const float4 q1 = *reinterpret_cast<const float4*>(&colbuf[b][8 * tx + 4]);
          const float4 y0 = *reinterpret_cast<const float4*>(&rowbuf[b][8 * tx]);
          const float4 y1 = *reinterpret_cast<const float4*>(&rowbuf[b][8 * tx + 4]);
          li[0] = p0.x; li[1] = p0.y; li[2] = p0.z; li[3] = p0.w;
          li[4] = p1.x; li[5] = p1.y; li[6] = p1.z; li[7] = p1.w;
          lc[0] = q0.x; lc[1] = q0.y; lc[2] = q0.z; lc[3] = q0.w;
          lc[4] = q1.x; lc[5] = q1.y; lc[6] = q1.z; lc[7] = q1.w;
          yj[0] = y0.x; yj[1] = y0.y; yj[2] = y0.z; yj[3] = y0.w;
          yj[4] = y1.x; yj[5] = y1.y; yj[6] = y1.z; yj[7] = y1.w;
        }
        // published values are raw: scale L[.][j] by r, and Y[j][.] by r
#pragma unroll
        for (int r = 0; r < 8; ++r) li[r] *= rs;
        const float rs2 = rs * rs;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          lc[c] *= rs;
          yj[c] *= rs;
        }
        (void)rs2;
        if (do_s) {
#pragma unroll
          for (int r = 0; r < 8; ++r)
#pragma unroll
            for (int c = 0; c < 8; ++c) a[r][c] = fmaf(-li[r], lc[c], a[r][c]);
        }
        if (do_a) {
#pragma unroll
          for (int r = 0; r < 8; ++r)
#pragma unroll
            for (int c = 0; c < 8; ++c) y[r][c] = fmaf(-li[r], yj[c], y[r][c]);
        }
      }
      // publish column j+1 of S and row j+1 of A (their last update was just now)
      const int jn = j + 1;
      if (jn < NB) {
        if (tx == (jn >> 3)) {
          const int cl = (jj + 1) & 7;        // compile-time after unrolling
#pragma unroll
          for (int r = 0; r < 8; ++r) colbuf[b ^ 1][8 * ty + r] = (8 * ty + r >= jn) ? a[r][cl] : 0.f;
        }
        if (ty == (jn >> 3)) {
          const int rl = (jj + 1) & 7;
#pragma unroll
          for (int c = 0; c < 8; ++c) rowbuf[b ^ 1][8 * tx + c] = (8 * tx + c <= jn) ? y[rl][c] : 0.f;
        }
      }
      __syncthreads();
    }
  }
}

__global__ void __launch_bounds__(256, 1) panel_kernel(float* R, float* Y, int n, int k, int p,
                                                    int tiles_L, int32_t* info) {
  extern __shared__ float sm[];
  float* D = sm;                       // [NB][LDD]
  float* X = sm + NB * LDD;            // [NB][LDD]
  kq::Gemm128Smem& gs = *reinterpret_cast<kq::Gemm128Smem*>(sm + 2 * NB * LDD);
  __shared__ int bad;
  const int kb = min(NB, n - k);
  if (threadIdx.x == 0) bad = 0;
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
    const int i = e / NB, j = e % NB;
    float v = 0.f;
    if (i < kb && j <= i) v = R[(int64_t)(k + i) * n + (k + j)];
    else if (i == j) v = 1.f;
    D[i * LDD + j] = v;
  }
  __syncthreads();
  factor_and_invert(D, X, kb, &bad);
  if (blockIdx.x == 0 && threadIdx.x == 0 && bad) kq::record_error(info, KRONQ_ERR_NOT_PD);

  if ((int)blockIdx.x < tiles_L) {
    // 128 rows of the panel: L_ip = R_ip L_pp^-T (in place)
    const int r0 = k + kb + NB * blockIdx.x;
    float* P = R + (int64_t)r0 * n + k;
    kq::gemm128<true>(gs, P, n, X, LDD, P, n, n - r0 < NB ? n - r0 : NB, kb, kb, 1.f, 0.f);
  } else {
    const int j = blockIdx.x - tiles_L;  // column block of Y's block row p
    if (j < p) {
      float* B = Y + (int64_t)k * n + NB * j;
      kq::gemm128<false>(gs, X, LDD, B, n, B, n, kb, NB, kb, 1.f, 0.f);
    } else {
      for (int e = threadIdx.x; e < kb * kb; e += blockDim.x) {
        const int a = e / kb, b = e % kb;
        Y[(int64_t)(k + a) * n + k + b] = X[a * LDD + b];
      }
    }
  }
}

// Trailing updates after panel p.  blockIdx.y: block row below the panel;
// blockIdx.x < p+1: Y accumulator column block; else: trailing R column block.
__global__ void __launch_bounds__(256) update_kernel(float* R, float* Y, int n, int k, int p) {
  __shared__ kq::Gemm128Smem gs;
  const int kb = min(NB, n - k);
  const int ti = blockIdx.y, tj = blockIdx.x;
  const int r0 = k + kb + NB * ti;
  const int M = min(NB, n - r0);
  const float* L = R + (int64_t)r0 * n + k;
  if (tj <= p) {
    float* C = Y + (int64_t)r0 * n + NB * tj;
    kq::gemm128<false>(gs, L, n, Y + (int64_t)k * n + NB * tj, n, C, n, M, NB, kb, -1.f, 1.f);
  } else {
    const int sj = tj - (p + 1);
    if (sj > ti) return;
    const int c0 = k + kb + NB * sj;
    float* C = R + (int64_t)r0 * n + c0;
    kq::gemm128<true>(gs, L, n, R + (int64_t)c0 * n + k, n, C, n, M, min(NB, n - c0), kb, -1.f, 1.f);
  }
}

// U[a][b] = Y[n-1-a][n-1-b] for a <= b, 0 below the diagonal.
__global__ void reverse_out_kernel(const float* __restrict__ Y, int n, float* __restrict__ U) {
  const int64_t total = (int64_t)n * n;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int a = (int)(e / n), b = (int)(e % n);
    U[e] = (a <= b) ? Y[(int64_t)(n - 1 - a) * n + (n - 1 - b)] : 0.f;
  }
}

size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

constexpr size_t kPanelSmem = (size_t)2 * NB * LDD * sizeof(float) + sizeof(kq::Gemm128Smem);

}  // namespace

size_t kq_cholesky_ws(int64_t n) {
  return align256(sizeof(double)) + 2 * align256((size_t)n * n * sizeof(float));
}

int kq_cholesky_inv(const float* H, int64_t n64, float damp_rel, float* U, int32_t* info, void* ws,
                    size_t ws_bytes, cudaStream_t st) {
  if (n64 < 0 || !(damp_rel >= 0.f)) return KRONQ_ERR_INVALID_ARG;
  if (n64 == 0) return KRONQ_OK;
  if (!H || !U || H == U) return KRONQ_ERR_INVALID_ARG;
  if (n64 > 65536) return KRONQ_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < kq_cholesky_ws(n64) || !kqh::aligned(ws, 256)) return KRONQ_ERR_WORKSPACE;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(panel_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kPanelSmem) != cudaSuccess)
      return KRONQ_ERR_CUDA;
    attr = true;
  }
  const int n = (int)n64;
  uint8_t* w = static_cast<uint8_t*>(ws);
  double* dsum = reinterpret_cast<double*>(w);
  w += align256(sizeof(double));
  float* R = reinterpret_cast<float*>(w);
  w += align256((size_t)n * n * sizeof(float));
  float* Y = reinterpret_cast<float*>(w);

  const int sms = kqh::num_sms();
  diag_sum_kernel<<<1, 256, 0, st>>>(H, n, dsum);
  KQ_CHECK_LAUNCH();
  reverse_damp_kernel<<<4 * sms, 256, 0, st>>>(H, n, R, Y, damp_rel, dsum);
  KQ_CHECK_LAUNCH();
  const int nblk = (n + NB - 1) / NB;
  for (int p = 0; p < nblk; ++p) {
    const int k = p * NB;
    const int kb = n - k < NB ? n - k : NB;
    const int rest = n - k - kb;
    const int tiles_L = (rest + NB - 1) / NB;
    panel_kernel<<<tiles_L + p + 1, 256, kPanelSmem, st>>>(R, Y, n, k, p, tiles_L, info);
    KQ_CHECK_LAUNCH();
    if (rest > 0) {
      update_kernel<<<dim3(p + 1 + tiles_L, tiles_L), 256, 0, st>>>(R, Y, n, k, p);
      KQ_CHECK_LAUNCH();
    }
  }
  reverse_out_kernel<<<4 * sms, 256, 0, st>>>(Y, n, U);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}
