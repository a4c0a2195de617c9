// Host interface of the tensor-core NT GEMM (gemm_tc.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kq {

// C (M x N, row-major, ldc) += alpha * A B^T with A M x K (lda) and B N x K
// (ldb), both row-major.  lower = 1: M == N and only the lower triangle of C
// (tile by tile, the diagonal tiles on and below the diagonal) is updated.
// Pointers 16-byte aligned, leading dimensions multiples of 4.
struct GemmNT {
  const float* A;
  int64_t lda;
  const float* B;
  int64_t ldb;
  float* C;
  int64_t ldc;
  int M, N, K;
  float alpha;
  int lower;
};

}  // namespace kq

// One launch for up to two independent problems (count 1 or 2); empty
// problems are skipped.  Returns KRONQ_OK, KRONQ_ERR_INVALID_ARG or
// KRONQ_ERR_CUDA.
int kq_gemm_nt_tc(const kq::GemmNT* probs, int count, int32_t* info, cudaStream_t st);
