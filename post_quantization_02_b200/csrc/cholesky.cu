// Damping and the inverse Cholesky factor U_c (H_d^-1 = U_c^T U_c, U_c upper).
//
// KronQ review (pith.science), appendix, Algorithm 2, steps 1-2:
// H_X <- H_X + lambda mean(diag H_X) I, then the inverse Cholesky factor.
//
// Route (fp32 throughout): with J the index reversal, R = J H_d J = L L^T
// (lower Cholesky) and U_c = J L^-1 J; then U_c^T U_c = J (L L^T)^-1 J =
// H_d^-1 and U_c is upper triangular.
//
// The matrix is padded with the identity to np = a multiple of 128 (which
// leaves the leading blocks of L and L^-1 unchanged).  One right-looking
// sweep over 128-wide panels computes L and Z = L^-T together (block
// forward substitution of L Y = I carried along with the factorisation,
// stored transposed so that every product has both operands K-major).
// Step p (rows k = 128 p ...):
//   panel kernel   every CTA factors the 128 x 128 diagonal block
//                  R_pp = L_pp L_pp^T and inverts L_pp in shared memory, then
//                  either turns 128 rows of the panel into L_ip = R_ip L_pp^-T,
//                  or finishes 128 rows of block column p of Z:
//                  Z_jp = B_jp L_pp^-T (B_jp = -sum_{q<p} Z_jq L_pq^T), Z_pp = L_pp^-T.
//   update         one tensor-core launch (tf32, three-term split) for
//                  R[k+128:, k+128:] -= L L^T (lower triangle) and
//                  Z[:k+128, k+128:] -= Z[:k+128, k:k+128] L^T, L = the panel rows.
// Then U_c[a][b] = Z[n-1-b][n-1-a] (a <= b).
#include "common.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"

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

// R[a][b] = H[n-1-a][n-1-b] + delta [a == b] for a, b < n, the identity on
// the padding up to np (a multiple of 128), delta = damp_rel * mean(diag H);
// Z = 0.  Padding with the identity leaves the leading n x n blocks of the
// factor and of its inverse unchanged.
__global__ void reverse_damp_kernel(const float* __restrict__ H, int n, int np,
                                    float* __restrict__ R, float* __restrict__ Z, float damp_rel,
                                    const double* __restrict__ diag_sum) {
  const float delta = (float)((double)damp_rel * (*diag_sum / (double)n));
  const int64_t total = (int64_t)np * np;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int a = (int)(e / np), b = (int)(e % np);
    float v;
    if (a < n && b < n) {
      v = H[(int64_t)(n - 1 - a) * n + (n - 1 - b)];
      if (a == b) v += delta;
    } else {
      v = (a == b) ? 1.f : 0.f;
    }
    R[e] = v;
    Z[e] = 0.f;
  }
}

// One warp factors the 32 x 32 diagonal block at offset o of D (lower part
// valid, already updated) and inverts the factor: on return D holds L_oo
// and X holds L_oo^-1 (both lower).  Lane i keeps row i of the block in
// registers; pivot step j needs no barrier: the pivot comes from lane j,
// the column L[:, j] and the row j of L^-1 travel by shuffles.
//   L[i][j] = a_i[j] r,  r = 1 / sqrt(a_j[j])
//   a_i[c] -= L[i][j] L[c][j]            (c > j, the Schur complement)
//   Y[j][:] = y_j[:] r,  y_i[:] -= L[i][j] Y[j][:]   (i > j, rows of L^-1)
__device__ __forceinline__ void warp_leaf32(float* D, float* X, int o, int kb, int* bad) {
  const int i = threadIdx.x & 31;
  constexpr unsigned FULL = 0xffffffffu;
  float a[32], y[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    a[c] = (c <= i) ? D[(o + i) * LDD + o + c] : 0.f;
    y[c] = (c == i) ? 1.f : 0.f;
  }
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    float d = __shfl_sync(FULL, a[j], j);
    if (!(d > 0.f) || !isfinite(d)) {
      if (i == 0 && o + j < kb) *bad = 1;
      d = 1.f;
    }
    const float r = rsqrtf(d);
    const float l = (i >= j) ? a[j] * r : 0.f;
    a[j] = l;
#pragma unroll
    for (int c = j + 1; c < 32; ++c) a[c] = fmaf(-l, __shfl_sync(FULL, l, c), a[c]);
#pragma unroll
    for (int c = 0; c <= j; ++c) {
      const float yj = __shfl_sync(FULL, y[c], j) * r;
      y[c] = (i == j) ? yj : fmaf(-l, yj, y[c]);
    }
  }
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    if (c <= i) {
      D[(o + i) * LDD + o + c] = a[c];
      X[(o + i) * LDD + o + c] = y[c];
    }
  }
}

// X = L^-1 for the lower Cholesky factor L of the 128 x 128 block in D
// (fp32; rows / columns kb .. NB-1 padded with the identity by the caller).
// On return D's lower triangle holds L and X (zero above the diagonal)
// holds L^-1.  256 threads.
//
// Right-looking over four 32-wide blocks b (o = 32 b), carrying L^-1 along
// (block forward substitution of L Y = I, accumulators in X below the
// diagonal blocks):
//   1. warp 0: L_bb and Y_bb = L_bb^-1                          (warp_leaf32)
//   2. L_cb = D_cb Y_bb^T (c > b);  Y_bj = Y_bb Acc_bj (j < b)
//   3. D_cd -= L_cb L_db^T (b < d <= c);  Acc_cj -= L_cb Y_bj (c > b, j <= b)
// Steps 2 and 3 are small GEMMs out of shared memory, register-tiled.
__device__ void factor_and_invert(float* D, float* X, int kb, int* bad) {
  const int tid = threadIdx.x;
  for (int e = tid; e < NB * LDD; e += blockDim.x) X[e] = 0.f;
  __syncthreads();
  for (int b = 0; b < NB / 32; ++b) {
    const int o = 32 * b;
    const int o2 = o + 32;
    const int R1 = NB - o2;                 // rows below the diagonal block
    if (tid < 32) warp_leaf32(D, X, o, kb, bad);
    __syncthreads();
    // ---- step 2: thread (tr, tc) = (tid / 8, tid % 8)
    {
      const int tr = tid >> 3, tc = tid & 7;
      float acc1[3][4], acc2[12];
      // L_cb rows o2 + tr + 32 s, columns o + 4 tc .. +3
#pragma unroll
      for (int s = 0; s < 3; ++s)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc1[s][q] = 0.f;
#pragma unroll
      for (int q = 0; q < 12; ++q) acc2[q] = 0.f;
      const int nj = o >> 3;                // Y_bj columns per thread: o / 8
#pragma unroll 4
      for (int t = 0; t < 32; ++t) {
        float bv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) bv[q] = X[(o + 4 * tc + q) * LDD + o + t];   // Y_bb[c][t]
#pragma unroll
        for (int s = 0; s < 3; ++s) {
          if (32 * s < R1) {
            const float av = D[(o2 + tr + 32 * s) * LDD + o + t];
#pragma unroll
            for (int q = 0; q < 4; ++q) acc1[s][q] = fmaf(av, bv[q], acc1[s][q]);
          }
        }
        const float yv = X[(o + tr) * LDD + o + t];                            // Y_bb[r][t]
#pragma unroll
        for (int q = 0; q < 12; ++q)
          if (q < nj) acc2[q] = fmaf(yv, X[(o + t) * LDD + tc * nj + q], acc2[q]);   // Acc[t][c']
      }
      __syncthreads();
#pragma unroll
      for (int s = 0; s < 3; ++s)
        if (32 * s < R1)
#pragma unroll
          for (int q = 0; q < 4; ++q) D[(o2 + tr + 32 * s) * LDD + o + 4 * tc + q] = acc1[s][q];
#pragma unroll
      for (int q = 0; q < 12; ++q)
        if (q < nj) X[(o + tr) * LDD + tc * nj + q] = acc2[q];
      __syncthreads();
    }
    if (R1 == 0) break;
    // ---- step 3: rows o2 + tr + 16 s, columns 8 tc .. 8 tc + 7 (all 128)
    {
      const int tr = tid >> 4, tc = tid & 15;
      const int ns = R1 >> 4;               // 6, 4 or 2 rows per thread
      float acc[6][8];
#pragma unroll
      for (int s = 0; s < 6; ++s)
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[s][q] = 0.f;
      const int c0 = 8 * tc;
      const bool left = c0 < o2;            // Acc / Y columns (j <= b), else trailing D
#pragma unroll 2
      for (int t = 0; t < 32; ++t) {
        float bv[8];
        if (left) {
#pragma unroll
          for (int q = 0; q < 8; ++q) bv[q] = X[(o + t) * LDD + c0 + q];          // Y_b[t][c]
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) bv[q] = D[(c0 + q) * LDD + o + t];          // L[c][o+t]
        }
#pragma unroll
        for (int s = 0; s < 6; ++s) {
          if (s < ns) {
            const float av = D[(o2 + tr + 16 * s) * LDD + o + t];
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[s][q] = fmaf(av, bv[q], acc[s][q]);
          }
        }
      }
#pragma unroll
      for (int s = 0; s < 6; ++s) {
        if (s < ns) {
          const int r = o2 + tr + 16 * s;
          float* dst = left ? &X[r * LDD + c0] : &D[r * LDD + c0];
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (left || c0 + q <= r) dst[q] -= acc[s][q];
        }
      }
      __syncthreads();
    }
  }
}

__global__ void __launch_bounds__(256, 1) panel_kernel(float* R, float* Z, int n, int k, int p,
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
    const int j = blockIdx.x - tiles_L;  // row block of Z's column block p
    if (j < p) {
      // Z_jp = Acc_jp L_pp^-T (in place)
      float* B = Z + (int64_t)(NB * j) * n + k;
      kq::gemm128<true>(gs, B, n, X, LDD, B, n, NB, kb, kb, 1.f, 0.f);
    } else {
      // Z_pp = L_pp^-T (upper; X is zero above its diagonal)
      for (int e = threadIdx.x; e < kb * kb; e += blockDim.x) {
        const int a = e / kb, b = e % kb;
        Z[(int64_t)(k + a) * n + k + b] = X[b * LDD + a];
      }
    }
  }
}

// U[a][b] = Z[n-1-b][n-1-a] for a <= b, 0 below the diagonal (Z has leading
// dimension np): an anti-transpose through 32 x 32 shared-memory tiles,
// coalesced on both sides.
__global__ void __launch_bounds__(256) reverse_out_kernel(const float* __restrict__ Z, int n,
                                                          int np, float* __restrict__ U) {
  __shared__ float tile[32][33];
  const int ta = blockIdx.y * 32, tb = blockIdx.x * 32;     // U tile origin (rows a, cols b)
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 8 rows per pass
  for (int r = ty; r < 32; r += 8) {
    const int b = tb + r, a = ta + 31 - tx;                 // Z row n-1-b, column n-1-a
    float v = 0.f;
    if (b < n && a < n) v = Z[(int64_t)(n - 1 - b) * np + (n - 1 - a)];
    tile[r][31 - tx] = v;                                   // tile[b - tb][a - ta]
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int a = ta + r, b = tb + tx;
    if (a < n && b < n) U[(int64_t)a * n + b] = (a <= b) ? tile[tx][r] : 0.f;
  }
}

size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

constexpr size_t kPanelSmem = (size_t)2 * NB * LDD * sizeof(float) + sizeof(kq::Gemm128Smem);

int64_t padded(int64_t n) { return (n + NB - 1) / NB * NB; }

}  // namespace

size_t kq_cholesky_ws(int64_t n) {
  const int64_t np = padded(n);
  return align256(sizeof(double)) + 2 * align256((size_t)np * np * sizeof(float));
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
  const int np = (int)padded(n64);
  uint8_t* w = static_cast<uint8_t*>(ws);
  double* dsum = reinterpret_cast<double*>(w);
  w += align256(sizeof(double));
  float* R = reinterpret_cast<float*>(w);
  w += align256((size_t)np * np * sizeof(float));
  float* Z = reinterpret_cast<float*>(w);

  const int sms = kqh::num_sms();
  diag_sum_kernel<<<1, 256, 0, st>>>(H, n, dsum);
  KQ_CHECK_LAUNCH();
  reverse_damp_kernel<<<4 * sms, 256, 0, st>>>(H, n, np, R, Z, damp_rel, dsum);
  KQ_CHECK_LAUNCH();
  const int nblk = np / NB;
  for (int p = 0; p < nblk; ++p) {
    const int k = p * NB;
    const int rest = np - k - NB;
    const int tiles_L = rest / NB;
    panel_kernel<<<tiles_L + p + 1, 256, kPanelSmem, st>>>(R, Z, np, k, p, tiles_L, info);
    KQ_CHECK_LAUNCH();
    if (rest > 0) {
      // trailing update on the tensor cores, the panel rows L_ip = L as B:
      //   R[k+128:, k+128:] -= L L^T                 (lower triangle)
      //   Z[:k+128, k+128:] -= Z[:k+128, k:k+128] L^T
      const float* L = R + (int64_t)(k + NB) * np + k;
      kq::GemmNT g[2];
      g[0] = {L, np, L, np, R + (int64_t)(k + NB) * np + (k + NB), np, rest, rest, NB, -1.f, 1};
      g[1] = {Z + k, np, L, np, Z + (k + NB), np, k + NB, rest, NB, -1.f, 0};
      const int s = kq_gemm_nt_tc(g, 2, info, st);
      if (s != KRONQ_OK) return s;
    }
  }
  const dim3 og((n + 31) / 32, (n + 31) / 32);
  reverse_out_kernel<<<og, 256, 0, st>>>(Z, n, np, U);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}
