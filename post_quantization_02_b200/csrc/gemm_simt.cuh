// fp32 CUDA-core GEMM tile: C = alpha * op(A) op(B) + beta * C on 64 x 64
// output tiles, K staged through shared memory in slices of 16.
//   op(A)[i][k] = TA ? A[k * lda + i] : A[i * lda + k]     (M x K)
//   op(B)[k][j] = TB ? B[j * ldb + k] : B[k * ldb + j]     (K x N)
// 256 threads, each owning a 4 x 4 block of the tile.  A CTA reads all of
// its A rows / B columns before it writes C, so C may alias A when the tile
// spans all of N (used for in-place triangular solves).
#pragma once

#include <stdint.h>

namespace kq {

constexpr int GT = 64;   // output tile edge
constexpr int GK = 16;   // K slice

template <bool TA, bool TB>
__device__ __forceinline__ void gemm_tile64(const float* A, int64_t lda,
                                            const float* B, int64_t ldb,
                                            float* C, int64_t ldc, int M, int N, int K,
                                            float alpha, float beta, int tm, int tn) {
  __shared__ float As[GK][GT + 4];
  __shared__ float Bs[GK][GT + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int row0 = tm * GT, col0 = tn * GT;
  float acc[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;

  for (int k0 = 0; k0 < K; k0 += GK) {
    // 64 x 16 slice of op(A) and 16 x 64 slice of op(B): 4 elements per thread each
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int idx = tid + e * 256;
      int i, k;
      if (TA) { i = idx & 63; k = idx >> 6; } else { k = idx & 15; i = idx >> 4; }
      const int gi = row0 + i, gk = k0 + k;
      float v = 0.f;
      if (gi < M && gk < K) v = TA ? A[(int64_t)gk * lda + gi] : A[(int64_t)gi * lda + gk];
      As[k][i] = v;
      int j, kb;
      if (TB) { kb = idx & 15; j = idx >> 4; } else { j = idx & 63; kb = idx >> 6; }
      const int gj = col0 + j, gkb = k0 + kb;
      float u = 0.f;
      if (gj < N && gkb < K) u = TB ? B[(int64_t)gj * ldb + gkb] : B[(int64_t)gkb * ldb + gj];
      Bs[kb][j] = u;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < GK; ++k) {
      const float4 a = *reinterpret_cast<const float4*>(&As[k][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&Bs[k][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int gi = row0 + ty * 4 + r;
    if (gi >= M) continue;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int gj = col0 + tx * 4 + c;
      if (gj >= N) continue;
      float* p = C + (int64_t)gi * ldc + gj;
      *p = (beta == 0.f) ? alpha * acc[r][c] : fmaf(beta, *p, alpha * acc[r][c]);
    }
  }
}

}  // namespace kq
