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

namespace kq {

// 128 x 128 output tile: C = alpha * A op(B) + beta * C, A row-major (M x K).
//   op(B)[k][j] = TB ? B[j * ldb + k] : B[k * ldb + j]
// 256 threads; thread (tx, ty) owns rows {4ty..4ty+3, 64+4ty..} and columns
// {4tx..4tx+3, 64+4tx..}; K in slices of 8 through double-buffered shared
// memory with the next slice prefetched into registers.  All reads of A and
// B happen before C is written, so C may alias A or B when the CTA's tile is
// the only reader of the region it writes.
constexpr int G2 = 128;
constexpr int G2K = 8;

struct Gemm128Smem {
  float a[2][G2K][G2 + 4];
  float b[2][G2K][G2 + 4];
};

template <bool TB>
__device__ __forceinline__ void gemm128_load(const float* A, int64_t lda, const float* B,
                                             int64_t ldb, int M, int N, int K, int k0,
                                             float (&ra)[4], float (&rb)[4]) {
  const int tid = threadIdx.x;
  // A: element (row = tid / 2, k = (tid & 1) * 4 + e)
  {
    const int r = tid >> 1, kk = (tid & 1) * 4;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int k = k0 + kk + e;
      ra[e] = (r < M && k < K) ? A[(int64_t)r * lda + k] : 0.f;
    }
  }
  if (TB) {  // B[k][j] = B_[j][k]: element (j = tid / 2, k = (tid & 1) * 4 + e)
    const int j = tid >> 1, kk = (tid & 1) * 4;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int k = k0 + kk + e;
      rb[e] = (j < N && k < K) ? B[(int64_t)j * ldb + k] : 0.f;
    }
  } else {   // element (k = tid / 32, j = (tid & 31) * 4 + e)
    const int k = k0 + (tid >> 5), j = (tid & 31) * 4;
#pragma unroll
    for (int e = 0; e < 4; ++e) rb[e] = (k < K && j + e < N) ? B[(int64_t)k * ldb + j + e] : 0.f;
  }
}

template <bool TB>
__device__ __forceinline__ void gemm128_stash(Gemm128Smem& s, int buf, const float (&ra)[4],
                                              const float (&rb)[4]) {
  const int tid = threadIdx.x;
  {
    const int r = tid >> 1, kk = (tid & 1) * 4;
#pragma unroll
    for (int e = 0; e < 4; ++e) s.a[buf][kk + e][r] = ra[e];
  }
  if (TB) {
    const int j = tid >> 1, kk = (tid & 1) * 4;
#pragma unroll
    for (int e = 0; e < 4; ++e) s.b[buf][kk + e][j] = rb[e];
  } else {
    const int k = tid >> 5, j = (tid & 31) * 4;
    *reinterpret_cast<float4*>(&s.b[buf][k][j]) = make_float4(rb[0], rb[1], rb[2], rb[3]);
  }
}

template <bool TB>
__device__ __forceinline__ void gemm128(Gemm128Smem& s, const float* A, int64_t lda,
                                        const float* B, int64_t ldb, float* C, int64_t ldc,
                                        int M, int N, int K, float alpha, float beta) {
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  float ra[4], rb[4];
  gemm128_load<TB>(A, lda, B, ldb, M, N, K, 0, ra, rb);
  __syncthreads();  // the previous user of s (if any) is done
  gemm128_stash<TB>(s, 0, ra, rb);
  __syncthreads();
  int buf = 0;
  for (int k0 = 0; k0 < K; k0 += G2K) {
    const bool more = k0 + G2K < K;
    if (more) gemm128_load<TB>(A, lda, B, ldb, M, N, K, k0 + G2K, ra, rb);
#pragma unroll
    for (int kk = 0; kk < G2K; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&s.a[buf][kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&s.a[buf][kk][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&s.b[buf][kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&s.b[buf][kk][64 + tx * 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    if (more) gemm128_stash<TB>(s, buf ^ 1, ra, rb);
    __syncthreads();
    buf ^= 1;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = (i < 4) ? ty * 4 + i : 64 + ty * 4 + (i - 4);
    if (r >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = (j < 4) ? tx * 4 + j : 64 + tx * 4 + (j - 4);
      if (c >= N) continue;
      float* p = C + (int64_t)r * ldc + c;
      *p = (beta == 0.f) ? alpha * acc[i][j] : fmaf(beta, *p, alpha * acc[i][j]);
    }
  }
}

}  // namespace kq
