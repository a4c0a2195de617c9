// Lazy block update of the OBS solver on the 5th-generation tensor cores:
//   W[:, i2:] -= E U[i1:i2, i2:]     (E: m x 128 scaled errors, U: inverse Cholesky factor)
//
// KronQ review (pith.science), appendix, Algorithm 2: errors of a block of
// B = 128 columns are buffered in E and applied to the trailing columns at
// once.  The product runs as tcgen05.mma kind::tf32 with a three-term split
// for fp32-level accuracy: x = x_hi + x_lo with x_hi the tf32 truncation the
// tensor core reads and x_lo = x - x_hi (exact in fp32), and
//   E U ~ E_hi U_hi + E_hi U_lo + E_lo U_hi      (relative error ~ 2^-21).
// Both halves are formed in shared memory right after TMA brings a tile in
// (hi: the low 13 mantissa bits cleared, lo = x - hi), so no extra global
// arrays are needed.
//
// Kernel (one CTA per SM, 384 threads): CTA (tn, r) owns column tile tn (128
// columns of W) and the row blocks r, r + R, ...  warp 0 loads the U tile
// (K = 128 rows x 128 columns, MN-major TMA boxes) once; warps 2-3 split it
// into hi / lo and transpose it into resident K-major tiles (the tensor core
// reads both operands K-major).  Then warp 0 streams E (128 rows x 32 K per
// stage, 3 stages) and warps 2-3 split each stage in place; one thread of
// warp 1 issues the MMAs (M = 128, N = 128, K = 8, three per K-step) into one
// of two TMEM accumulators; warps 4-11 read the accumulator back and update
// W in place, with the tile's W loads issued ahead of the MMAs.
#include "tf32x3.cuh"

namespace {

using kq::tf32x3::drain_wait;
using kq::tf32x3::fence_to_tensor_core;
using kq::tf32x3::swz128;
using kq::tf32x3::split_smem;

constexpr int TM = 128, TN = 128, KB = 128;  // tile rows, tile columns, block width (K)
constexpr int KC = 32;                        // K values per 128-byte swizzle row of fp32
constexpr int NKC = KB / KC;                  // 4
constexpr int STAGES = 3;
constexpr int KTILE = 128 * KC * 4;           // 16 KB: 128 rows x 32 fp32, K-major, swizzled
constexpr int B_BYTES = 2 * NKC * KTILE;      // resident U tile, hi + lo: 128 KB
constexpr int STAGE_BYTES = 2 * KTILE;        // E rows x 32 K: landing (becomes hi) + lo
constexpr int U_BOX = KC * 32 * 4;            // 4 KB TMA box of U: 32 K-rows x 32 columns
constexpr int THREADS = 384;
constexpr int SPLITTERS = 64;                 // warps 2 and 3
constexpr int SMEM_BYTES = B_BYTES + STAGES * STAGE_BYTES + 1024 + 256;
constexpr int TMEM_COLS = 2 * TN;

struct Bars {
  uint64_t ufull;            // U tile landed (MN-major, in the stage area)
  uint64_t uready;           // U tile split / transposed into the resident B area
  uint64_t full[STAGES];     // E stage landed
  uint64_t lo[STAGES];       // E stage split
  uint64_t empty[STAGES];    // E stage consumed by the MMAs
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// The U tile (K = 128 rows of U, 128 columns) lands MN-major as 4 K-chunks x
// 4 boxes of 32 K-rows x 32 columns; it is split into hi / lo and transposed
// into K-major tiles (row = column of U, 32 K values per 128-byte row).  Lane
// = K index: a 16-byte read of a landing row (the swizzle spreads the 8 rows
// of a quarter-warp over 8 chunks) and four writes of full 128-byte rows.
__device__ __forceinline__ void split_transpose_u(const uint8_t* land, uint8_t* hi, uint8_t* lo,
                                                  int t, int nthreads) {
  for (int e = t; e < KB * (TN / 4); e += nthreads) {
    const int kk = e & 31, kc = (e >> 5) & (NKC - 1), nq = e >> 7;
    const uint8_t* lt = land + kc * (4 * U_BOX);
    const float4 v = *reinterpret_cast<const float4*>(lt + (nq >> 3) * U_BOX + swz128(kk, (nq & 7) * 16));
    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float h = kq::tf32x3::hi(vv[j]);
      const int d = kc * KTILE + swz128(4 * nq + j, kk * 4);
      *reinterpret_cast<float*>(hi + d) = h;
      *reinterpret_cast<float*>(lo + d) = vv[j] - h;
    }
  }
  fence_to_tensor_core();
}

// CTA (tn, r): column tile tn of W[:, i2:], row blocks r, r + R, ...
__global__ void __launch_bounds__(THREADS, 1)
lazy_tc_kernel(const __grid_constant__ CUtensorMap tm_e, const __grid_constant__ CUtensorMap tm_u,
               float* __restrict__ W, int m, int n, int i1, int mblocks, int32_t* info) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* b_hi = base;
  uint8_t* b_lo = base + B_BYTES / 2;
  uint8_t* stages = base + B_BYTES;
  Bars* bars = reinterpret_cast<Bars*>(stages + STAGES * STAGE_BYTES);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tn = blockIdx.x, r0 = blockIdx.y, R = gridDim.y;
  const int i2 = i1 + KB;
  const int c0 = i2 + tn * TN;

  if (threadIdx.x == 0) {
    kq::mbar_init(&bars->ufull, 1);
    kq::mbar_init(&bars->uready, SPLITTERS);
    for (int s = 0; s < STAGES; ++s) {
      kq::mbar_init(&bars->full[s], 1);
      kq::mbar_init(&bars->lo[s], SPLITTERS);
      kq::mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      kq::mbar_init(&bars->tfull[b], 1);
      kq::mbar_init(&bars->tempty[b], 8);
    }
    kq::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    kq::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    kq::prefetch_tmap(&tm_e);
    kq::prefetch_tmap(&tm_u);
  }
  if (warp == 2) kq::tmem_alloc(&bars->tmem_base, TMEM_COLS);
  kq::tc_fence_before();
  __syncthreads();
  kq::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------- TMA producer
      // the U tile lands in the (still unused) stage area: 64 KB of the 96 KB
      kq::mbar_arrive_expect_tx(&bars->ufull, NKC * 4 * U_BOX);
      for (int kc = 0; kc < NKC; ++kc)
#pragma unroll
        for (int q = 0; q < 4; ++q)
          kq::tma_load_2d(stages + kc * 4 * U_BOX + q * U_BOX, &tm_u, &bars->ufull, c0 + 32 * q,
                          i1 + kc * KC);
      bool ok = kq::mbar_wait(&bars->uready, 0, abort, info);   // stage area free again
      int it = 0;
      for (int mb = r0; mb < mblocks && ok; mb += R) {
        for (int kc = 0; kc < NKC; ++kc, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!kq::mbar_wait(&bars->empty[s], ph ^ 1u, abort, info)) { ok = false; break; }
          kq::mbar_arrive_expect_tx(&bars->full[s], KTILE);
          kq::tma_load_2d(stages + s * STAGE_BYTES, &tm_e, &bars->full[s], kc * KC, mb * TM);
        }
      }
      drain_wait(&bars->ufull, 0, info);
      for (int s = 0; s < STAGES; ++s) {
        const int armed = (it > s) ? (it - s + STAGES - 1) / STAGES : 0;
        if (armed > 0) drain_wait(&bars->full[s], (uint32_t)(armed - 1) & 1u, info);
      }
    }
  } else if (warp == 2 || warp == 3) {
    // ---------------------------------------------- hi / lo splitters (64 threads)
    const int t = (warp - 2) * 32 + lane;
    if (kq::mbar_wait(&bars->ufull, 0, abort, info)) {
      split_transpose_u(stages, b_hi, b_lo, t, SPLITTERS);
      kq::mbar_arrive(&bars->uready);
      int it = 0;
      bool ok = true;
      for (int mb = r0; mb < mblocks && ok; mb += R) {
        for (int kc = 0; kc < NKC; ++kc, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!kq::mbar_wait(&bars->full[s], ph, abort, info)) { ok = false; break; }
          uint8_t* st = stages + s * STAGE_BYTES;
          split_smem(st, st + KTILE, KTILE / 16, t, SPLITTERS);
          kq::mbar_arrive(&bars->lo[s]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------- MMA issuer
      bool ok = kq::mbar_wait(&bars->uready, 0, abort, info);
      kq::tc_fence_after();
      const uint32_t bh = kq::smem_u32(b_hi), bl = kq::smem_u32(b_lo);
      int it = 0, tl = 0;
      for (int mb = r0; mb < mblocks && ok; mb += R, ++tl) {
        const int buf = tl & 1;
        const uint32_t aph = (uint32_t)(tl >> 1) & 1u;
        if (!kq::mbar_wait(&bars->tempty[buf], aph ^ 1u, abort, info)) break;
        kq::tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(buf * TN);
        for (int kc = 0; kc < NKC; ++kc, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!kq::mbar_wait(&bars->full[s], ph, abort, info) ||
              !kq::mbar_wait(&bars->lo[s], ph, abort, info)) { ok = false; break; }
          kq::tc_fence_after();
          const uint32_t ah = kq::smem_u32(stages + s * STAGE_BYTES), al = ah + KTILE;
#pragma unroll
          for (int kk = 0; kk < KC / 8; ++kk)
            kq::tf32x3::mma3(d_tmem, ah, al, bh + kc * KTILE, bl + kc * KTILE, kk,
                             (kc == 0 && kk == 0) ? 0u : 1u);
          kq::mma_commit(&bars->empty[s]);
        }
        if (ok) kq::mma_commit(&bars->tfull[buf]);
      }
      kq::mma_commit(&bars->drain);
      drain_wait(&bars->drain, 0, info);
    }
  } else if (warp >= 4) {
    // ---------------------------------------------- epilogue: W -= acc (8 warps)
    // warp w reads TMEM lane quadrant w % 4 and columns [64 h, 64 h + 64),
    // h = (w - 4) / 4.  The W loads of a tile are issued before its
    // accumulator is waited for, so their latency overlaps the MMAs.
    const int q = warp & 3, h = (warp - 4) >> 2;
    const int cbase = c0 + 64 * h;
    int tl = 0;
    for (int mb = r0; mb < mblocks; mb += R, ++tl) {
      const int buf = tl & 1;
      const uint32_t aph = (uint32_t)(tl >> 1) & 1u;
      const int row = mb * TM + q * 32 + lane;
      float4 w[16];
      const bool full = row < m && cbase + 64 <= n;
      if (full) {
        const float4* src = reinterpret_cast<const float4*>(W + (int64_t)row * n + cbase);
#pragma unroll
        for (int k = 0; k < 16; ++k) w[k] = src[k];
      }
      if (!kq::mbar_wait(&bars->tfull[buf], aph, abort, info)) break;
      kq::tc_fence_after();
      float v[64];
      {
        float v0[32], v1[32];
        __syncwarp();
        kq::tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * TN + 64 * h), v0);
        kq::tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * TN + 64 * h + 32), v1);
        kq::tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) { v[k] = v0[k]; v[32 + k] = v1[k]; }
      }
      kq::tc_fence_before();
      __syncwarp();
      if (lane == 0) kq::mbar_arrive(&bars->tempty[buf]);   // accumulator free again
      if (full) {
        float4* dst = reinterpret_cast<float4*>(W + (int64_t)row * n + cbase);
#pragma unroll
        for (int k = 0; k < 16; ++k)
          dst[k] = make_float4(w[k].x - v[4 * k], w[k].y - v[4 * k + 1], w[k].z - v[4 * k + 2],
                               w[k].w - v[4 * k + 3]);
      } else if (row < m) {
        float* dst = W + (int64_t)row * n + cbase;
#pragma unroll
        for (int k = 0; k < 64; ++k)
          if (cbase + k < n) dst[k] -= v[k];
      }
    }
  }

  kq::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    kq::tc_fence_after();
    kq::tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

// W[:, i1+128:] -= E U[i1:i1+128, i1+128:] with E: m x 128, U: n x n (both fp32, row-major).
int kq_lazy_update_tc(float* W, int64_t m, int64_t n, const float* E, const float* U, int i1,
                      int32_t* info, cudaStream_t st) {
  const int64_t i2 = i1 + KB;
  if (i2 >= n) return KRONQ_OK;
  CUtensorMap me, mu;
  if (!kqh::make_map_f32(&me, E, KB, m, KB, KC, TM) || !kqh::make_map_f32(&mu, U, n, n, n, 32, KC))
    return KRONQ_ERR_CUDA;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(lazy_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES) != cudaSuccess)
      return KRONQ_ERR_CUDA;
    attr = true;
  }
  const int n_tiles = (int)((n - i2 + TN - 1) / TN);
  const int mblocks = (int)((m + TM - 1) / TM);
  int R = kqh::num_sms() / n_tiles;       // one wave: n_tiles x R <= #SMs where possible
  if (R > mblocks) R = mblocks;
  if (R < 1) R = 1;
  lazy_tc_kernel<<<dim3(n_tiles, R), THREADS, SMEM_BYTES, st>>>(me, mu, W, (int)m, (int)n, i1,
                                                                 mblocks, info);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}
