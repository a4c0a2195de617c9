// --act_order: the column order of the OBS loop, and the permutations that
// carry W, H_X and the results into and out of it.
//
// KronQ README (GitHub), "Reproduce from scratch": the base recipe passes
// --act_order; the pages do not define it.  Reading: the columns are
// quantized in descending order of the diagonal of the (rotated, undamped)
// H_X handed to the solver, equal diagonals in increasing column order.  The
// solver then runs on W[:, perm] with H[perm][:, perm] (damped and factored
// as usual), and its codes / W_hat go back to the original column order.
#include "common.cuh"

namespace {

constexpr int RANK_THREADS = 256;

// NaN sorts last (as -inf), so that every column gets a distinct rank.
__device__ __forceinline__ float order_key(float v) { return isnan(v) ? -INFINITY : v; }

// rank(i) = #{j : d_j > d_i or (d_j == d_i and j < i)}; perm[rank(i)] = i.
// Each thread ranks one column against all n diagonals, staged through
// shared memory a tile at a time.
__global__ void __launch_bounds__(RANK_THREADS) act_order_kernel(const float* __restrict__ H,
                                                                 int n, int64_t ldh,
                                                                 int32_t* __restrict__ perm) {
  __shared__ float tile[RANK_THREADS];
  const int i = blockIdx.x * RANK_THREADS + threadIdx.x;
  const float di = i < n ? order_key(H[(int64_t)i * ldh + i]) : 0.f;
  int rank = 0;
  for (int t0 = 0; t0 < n; t0 += RANK_THREADS) {
    const int j = t0 + threadIdx.x;
    tile[threadIdx.x] = j < n ? order_key(H[(int64_t)j * ldh + j]) : -INFINITY;
    __syncthreads();
    const int cnt = min(RANK_THREADS, n - t0);
    for (int k = 0; k < cnt; ++k) {
      const float dj = tile[k];
      rank += (dj > di) || (dj == di && t0 + k < i);
    }
    __syncthreads();
  }
  if (i < n) perm[rank] = i;
}

// dst[r][k] = src[r][perm[k]] (gather), dst[r][perm[k]] = src[r][k]
// (scatter), or dst[a][b] = src[perm[a]][perm[b]] (symmetric gather); one
// row per CTA iteration, the columns across its threads.  Entries of perm
// outside [0, n) are skipped and flagged in info.
template <typename T>
__global__ void permute_kernel(const T* __restrict__ src, T* __restrict__ dst, int64_t m, int64_t n,
                               const int32_t* __restrict__ perm, int mode, int32_t* info) {
  for (int64_t r = blockIdx.x; r < m; r += gridDim.x) {
    int64_t pr = r;
    if (mode == KRONQ_PERM_SYM) {
      pr = perm[r];
      if (pr < 0 || pr >= n) {
        if (threadIdx.x == 0) kq::record_error(info, KRONQ_ERR_INVALID_ARG);
        continue;
      }
    }
    const T* s_row = src + r * n;
    const T* s_prow = src + pr * n;
    T* d_row = dst + r * n;
    for (int64_t k = threadIdx.x; k < n; k += blockDim.x) {
      const int64_t pk = perm[k];
      if (pk < 0 || pk >= n) {
        kq::record_error(info, KRONQ_ERR_INVALID_ARG);
        continue;
      }
      if (mode == KRONQ_UNPERM_COLS) d_row[pk] = s_row[k];
      else d_row[k] = s_prow[pk];      // KRONQ_PERM_COLS (pr = r) or KRONQ_PERM_SYM
    }
  }
}

}  // namespace

int kq_act_order(const float* H, int64_t n, int32_t* perm, cudaStream_t st) {
  if (n < 0) return KRONQ_ERR_INVALID_ARG;
  if (n == 0) return KRONQ_OK;
  if (!H || !perm) return KRONQ_ERR_INVALID_ARG;
  if (n > (1 << 24)) return KRONQ_ERR_UNSUPPORTED;
  act_order_kernel<<<(int)((n + RANK_THREADS - 1) / RANK_THREADS), RANK_THREADS, 0, st>>>(H, (int)n, n,
                                                                                         perm);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

int kq_permute(const void* src, void* dst, int64_t m, int64_t n, int elem_bytes,
               const int32_t* perm, int mode, int32_t* info, cudaStream_t st) {
  if (m < 0 || n < 0) return KRONQ_ERR_INVALID_ARG;
  if (m == 0 || n == 0) return KRONQ_OK;
  if (!src || !dst || !perm || src == dst) return KRONQ_ERR_INVALID_ARG;
  if (mode != KRONQ_PERM_COLS && mode != KRONQ_UNPERM_COLS && mode != KRONQ_PERM_SYM)
    return KRONQ_ERR_INVALID_ARG;
  if (mode == KRONQ_PERM_SYM && (m != n || elem_bytes != 4)) return KRONQ_ERR_INVALID_ARG;
  if (elem_bytes != 1 && elem_bytes != 4) return KRONQ_ERR_INVALID_ARG;
  const int grid = (int)(m < 16 * kqh::num_sms() ? m : 16 * kqh::num_sms());
  if (elem_bytes == 4) {
    permute_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(src),
                                                static_cast<float*>(dst), m, n, perm, mode, info);
  } else if (elem_bytes == 1) {
    permute_kernel<uint8_t><<<grid, 256, 0, st>>>(static_cast<const uint8_t*>(src),
                                                  static_cast<uint8_t*>(dst), m, n, perm, mode, info);
  } else {
    return KRONQ_ERR_INVALID_ARG;
  }
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}
