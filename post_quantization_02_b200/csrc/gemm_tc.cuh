// Host interface of the tensor-core NT GEMM (gemm_tc.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kq {

// C (M x N, row-major, ldc) += alpha * A B^T with A M x K and B N x K, both
// row-major and given pre-split into a hi and a lo plane sharing the leading
// dimension (lda / ldb elements):
//   bf16 = 0: fp32 planes, A_hi exactly a tf32 value (the low 13 mantissa
//             bits clear) and A_lo the fp32 remainder;
//   bf16 = 1: bf16 planes, A_hi = RN_bf16(A) and A_lo = RN_bf16(A - A_hi)
//             (A = A_hi + A_lo to about 2^-17 relative);
//   fp16 = 1: fp16 planes of rows scaled by exact powers of two (row i of A
//             holds A[i][:] * 2^a_i in [2^13, 2^14) at its largest entry,
//             split as fp16 hi / lo: about 2^-22 relative); a_scale[i] =
//             2^-a_i and b_scale[j] = 2^-b_j undo the scaling in the epilogue.
// lower = 1: M == N and only the lower triangle of C (tile by tile, the
// diagonal tiles on and below the diagonal) is updated.  Pointers 16-byte
// aligned, leading dimensions multiples of 16 bytes.
struct GemmNT {
  const void* A_hi;
  const void* A_lo;
  int64_t lda;
  const void* B_hi;
  const void* B_lo;
  int64_t ldb;
  float* C;
  int64_t ldc;
  int M, N, K;
  float alpha;
  int lower;
  // only the problem's output tiles [tile_begin, tile_end) in its own tile
  // order (row-major over 128 x 128 tiles; lower: row by row, columns up to
  // the diagonal); tile_end < 0: to the last tile
  int tile_begin = 0;
  int tile_end = -1;
  int bf16 = 0;
  int fp16 = 0;
  const float* a_scale = nullptr;   // fp16 planes: per A row (M)
  const float* b_scale = nullptr;   // fp16 planes: per B row (N)
};

}  // namespace kq

// One launch for up to two independent problems (count 1 or 2, both with
// the same plane type); empty problems are skipped.  Returns KRONQ_OK, KRONQ_ERR_INVALID_ARG or
// KRONQ_ERR_CUDA.
// max_ctas > 0 caps the persistent grid (to leave SMs to concurrent work).
int kq_gemm_nt_tc(const kq::GemmNT* probs, int count, int32_t* info, cudaStream_t st,
                  int max_ctas = 0);
