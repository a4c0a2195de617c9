// H = alpha * A^T A + beta * H on the 5th-generation tensor cores.
//
// KronQ summary (hyper.ai), "Method" (Eq. 7): the two Kronecker factors
// H_X = E[x x^T] and H_G = E[g g^T] are covariances over the calibration
// tokens.  A is token-major (N x d, bf16), so a tile of H is a rank-K update
// whose operands are both "MN-major": for a K-slab of tokens the features
// (the M and N indices of the tile) are contiguous in memory.
//
// Kernel structure (one CTA per SM, persistent over work units).  A unit is
// one output tile and one chunk of KC_ITERS K-slabs (4096 tokens); units are
// handed out chunk-major, so all CTAs stream the same token range at about
// the same time (L2 reuse of X) and every CTA gets the same number of units.
//   warp 0      TMA producer: per K-slab of 64 tokens, two 64x64 boxes of the
//               row panel (A, 128 features) and four of the column panel (B,
//               256 features), 128-byte swizzled, into a 4-stage ring.
//   warp 1      one thread issues tcgen05.mma (M=128, N=256, K=16, bf16 in,
//               fp32 accumulate in TMEM) into one of two accumulators (one
//               per unit, alternating) and commits each stage back to the
//               producer and each finished unit to the epilogue.
//   warp 2      allocates / frees the 512 TMEM columns.
//   warps 4-7   epilogue: a unit's partial sum, times alpha, goes to H by TMA
//               reduce-adds of 32 x 32 boxes staged in shared memory (fp32
//               round-to-nearest adds in L2), while the tensor core already
//               fills the other accumulator.
// Folding every 4096-token partial sum with round-to-nearest adds matters:
// the tensor core's own fp32 accumulation rounds towards zero (measured ~
// -6e-8 relative per K=16 step), so it only ever spans one chunk.
// Before the kernel H <- beta H (or 0); only tiles that touch the upper
// triangle are computed, and a last pass copies the upper triangle onto the
// lower one, so the whole symmetric d x d result is written by every call.
// When beta != 0 the old upper triangle is read, so the old H must be
// symmetric.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
// K-slabs per accumulation chunk: the tensor core's fp32 accumulation rounds
// towards zero (measured: ~ -6e-8 relative per K=16 step), so partial sums
// over 4096 tokens are folded into H with round-to-nearest fp32 adds.
constexpr int KC_ITERS = 64;
constexpr int BOX_BYTES = 64 * BK * 2;              // 64 features x 64 tokens of bf16
constexpr int A_BYTES = BM * BK * 2;                // 16 KB
constexpr int B_BYTES = BN * BK * 2;                // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;      // 48 KB
constexpr int TMEM_COLS = 2 * BN;  // two accumulators
constexpr int THREADS = 256;
constexpr int STG_BYTES = 32 * 32 * 4;              // one 32 x 32 fp32 box
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 8 * STG_BYTES + 1024 + 256;
constexpr uint32_t IDESC = kq::idesc_f16(BM, BN, /*bf16*/ 1, /*A MN-major*/ 1, /*B MN-major*/ 1);

struct Bars {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// Tiles are ordered by column block cb; column block cb holds the row blocks
// 0 .. min(nrb, 2 cb + 2) - 1 (those with some element on or above the
// diagonal).  Column blocks before cb hold cb (cb + 1) tiles in all; only the
// last column block can be shorter.
__device__ __forceinline__ void tile_coords(int t, int ncb, int& rb, int& cb) {
  int c = (int)((sqrt(4.0 * (double)t + 1.0) - 1.0) * 0.5);
  while ((long long)(c + 1) * (c + 2) <= t) ++c;
  while ((long long)c * (c + 1) > t) --c;
  if (c > ncb - 1) c = ncb - 1;
  cb = c;
  rb = t - c * (c + 1);
}

// A wait used only while winding down: ignores the abort flag, bounded.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, int32_t* info) {
  if (kq::mbar_try_wait(bar, parity)) return;
  unsigned long long t0 = kq::globaltimer();
  while (!kq::mbar_try_wait(bar, parity)) {
    if (kq::globaltimer() - t0 > kq::kWaitLimitNs) {
      kq::record_error(info, KRONQ_ERR_TIMEOUT);
      return;
    }
  }
}

// C box += the 32 x 32 fp32 box in shared memory (TMA, bulk-group completion).
KQ_DEV void tma_reduce_add_2d(const void* tmap, const void* src, int x, int y) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(tmap)),
      "r"(kq::smem_u32(src)), "r"(x), "r"(y)
      : "memory");
}

__global__ void __launch_bounds__(THREADS, 1)
cov_tc_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap hmap,
              int k_iters, int ncb, int num_tiles, int num_units, float alpha, int32_t* info) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* staging = tiles + STAGES * STAGE_BYTES;      // 1024-byte aligned
  Bars* bars = reinterpret_cast<Bars*>(staging + 8 * STG_BYTES);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      kq::mbar_init(&bars->full[s], 1);
      kq::mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      kq::mbar_init(&bars->tfull[b], 1);
      kq::mbar_init(&bars->tempty[b], 4);
    }
    kq::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    kq::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    kq::prefetch_tmap(&tmap);
    kq::prefetch_tmap(&hmap);
  }
  if (warp == 2) kq::tmem_alloc(&bars->tmem_base, TMEM_COLS);
  kq::tc_fence_before();
  __syncthreads();
  kq::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
        int rb, cb;
        tile_coords(u % num_tiles, ncb, rb, cb);
        const int i0 = rb * BM, j0 = cb * BN;
        const int k0 = (u / num_tiles) * KC_ITERS, k1 = min(k_iters, k0 + KC_ITERS);
        for (int kb = k0; kb < k1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!kq::mbar_wait(&bars->empty[s], ph ^ 1u, abort, info)) { ok = false; break; }
          uint8_t* a = tiles + s * STAGE_BYTES;
          uint8_t* b = a + A_BYTES;
          kq::mbar_arrive_expect_tx(&bars->full[s], STAGE_BYTES);
          const int y = kb * BK;
          kq::tma_load_2d(a, &tmap, &bars->full[s], i0, y);
          kq::tma_load_2d(a + BOX_BYTES, &tmap, &bars->full[s], i0 + 64, y);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            kq::tma_load_2d(b + q * BOX_BYTES, &tmap, &bars->full[s], j0 + 64 * q, y);
        }
      }
      // wind down: every stage's last armed phase must have landed
      for (int s = 0; s < STAGES; ++s) {
        const int armed = (it > s) ? (it - s + STAGES - 1) / STAGES : 0;
        if (armed > 0) drain_wait(&bars->full[s], (uint32_t)(armed - 1) & 1u, info);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      int it = 0, uc = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x, ++uc) {
        const int k0 = (u / num_tiles) * KC_ITERS, k1 = min(k_iters, k0 + KC_ITERS);
        const int buf = uc & 1;
        if (!kq::mbar_wait(&bars->tempty[buf], ((uint32_t)(uc >> 1) & 1u) ^ 1u, abort, info)) break;
        kq::tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(buf * BN);
        for (int kb = k0; kb < k1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!kq::mbar_wait(&bars->full[s], ph, abort, info)) { ok = false; break; }
          kq::tc_fence_after();
          const uint32_t a_addr = kq::smem_u32(tiles + s * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // MN-major, 128B swizzle: 8-row K atoms 1024 B apart (SBO), 64-wide
            // feature atoms one TMA box apart (LBO); K step of 16 rows = 2048 B.
            const uint64_t ad = kq::smem_desc(a_addr + kk * 2048, BOX_BYTES, 1024, kq::kLayoutSwizzle128B);
            const uint64_t bd = kq::smem_desc(b_addr + kk * 2048, BOX_BYTES, 1024, kq::kLayoutSwizzle128B);
            kq::mma_f16(acc, ad, bd, IDESC, (kb != k0) || (kk != 0));
          }
          kq::mma_commit(&bars->empty[s]);
        }
        if (ok) kq::mma_commit(&bars->tfull[buf]);
      }
      // wind down: all MMAs issued by this thread complete before TMEM is freed
      kq::mma_commit(&bars->drain);
      drain_wait(&bars->drain, 0, info);
    }
  } else if (warp >= 4) {
    // -------------------------------------------------- epilogue
    // warp q = warp - 4 reads TMEM lanes 32 q .. 32 q + 31 (tile rows) and
    // adds the unit's partial sum into H box by box (32 columns at a time),
    // alternating between two staging buffers.
    const int q = warp & 3;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    uint8_t* stg = staging + (warp - 4) * 2 * STG_BYTES;
    int uc = 0, nbox = 0;
    for (int u = blockIdx.x; u < num_units; u += gridDim.x, ++uc) {
      int rb, cb;
      tile_coords(u % num_tiles, ncb, rb, cb);
      const int i0 = rb * BM, j0 = cb * BN;
      const int buf = uc & 1;
      if (!kq::mbar_wait(&bars->tfull[buf], (uint32_t)(uc >> 1) & 1u, abort, info)) break;
      kq::tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        if (j0 + c + 31 < i0 + q * 32) continue;     // box strictly below the diagonal: skipped
        float v[32];
        __syncwarp();
        kq::tmem_ld32(tmem + lane_off + (uint32_t)(buf * BN + c), v);
        kq::tmem_wait_ld();
        uint8_t* box = stg + (nbox & 1) * STG_BYTES;
        if (nbox >= 2) {
          if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
          __syncwarp();
        }
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          *reinterpret_cast<float4*>(box + lane * 128 + ((ch ^ (lane & 7)) << 4)) =
              make_float4(alpha * v[4 * ch], alpha * v[4 * ch + 1], alpha * v[4 * ch + 2],
                          alpha * v[4 * ch + 3]);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_2d(&hmap, box, j0 + c, i0 + q * 32);
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
        ++nbox;
      }
      kq::tc_fence_before();
      __syncwarp();
      if (lane == 0) kq::mbar_arrive(&bars->tempty[buf]);   // accumulator free again
    }
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
  }

  kq::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    kq::tc_fence_after();
    kq::tmem_dealloc(tmem, TMEM_COLS);
  }
}

// H[j][i] = H[i][j] for j > i (the computed upper triangle onto the lower
// one), through 32 x 32 shared-memory tiles: coalesced reads and writes.
__global__ void __launch_bounds__(256) mirror_kernel(float* __restrict__ H, int64_t ldh, int d) {
  __shared__ float tile[32][33];
  const int bi = blockIdx.y, bj = blockIdx.x;       // source tile: rows 32 bi, columns 32 bj
  if (bj < bi) return;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int r = ty; r < 32; r += 8) {
    const int i = 32 * bi + r, j = 32 * bj + tx;
    tile[r][tx] = (i < d && j < d) ? H[(int64_t)i * ldh + j] : 0.f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int j = 32 * bj + r, i = 32 * bi + tx;     // destination H[j][i]
    if (i < d && j < d && j > i) H[(int64_t)j * ldh + i] = tile[tx][r];
  }
}

__global__ void scale_kernel(float* __restrict__ H, int64_t ldh, int d, float beta) {
  const int64_t total = (int64_t)d * d;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / d, c = e % d;
    float* p = H + r * ldh + c;
    *p = (beta == 0.f) ? 0.f : beta * *p;
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

int kq_covariance(const uint16_t* A, int64_t N, int64_t d, int64_t lda, float* H, int64_t ldh,
                  float alpha, float beta, int32_t* info, cudaStream_t st) {
  if (d < 0 || N < 0) return KRONQ_ERR_INVALID_ARG;
  if (d == 0) return KRONQ_OK;
  if (!H || ldh < d || (ldh % 4) != 0 || !kqh::aligned(H, 16)) return KRONQ_ERR_INVALID_ARG;
  if (d < 64 || d > (1 << 20) || N > (int64_t)1 << 31) return KRONQ_ERR_UNSUPPORTED;
  if (N == 0) {
    if (beta != 1.f) {
      scale_kernel<<<4 * kqh::num_sms(), 256, 0, st>>>(H, ldh, (int)d, beta);
      KQ_CHECK_LAUNCH();
    }
    return KRONQ_OK;
  }
  if (!A || lda < d || (lda % 8) != 0 || !kqh::aligned(A, 16)) return KRONQ_ERR_INVALID_ARG;

  auto encode = get_encode();
  if (!encode) return KRONQ_ERR_CUDA;
  CUtensorMap tmap, hmap;
  {
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)lda * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)BK};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(A), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return KRONQ_ERR_UNSUPPORTED;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)d};
    cuuint64_t strides[1] = {(cuuint64_t)ldh * 4};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&hmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, H, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return KRONQ_ERR_UNSUPPORTED;
  }

  const int nrb = (int)((d + BM - 1) / BM), ncb = (int)((d + BN - 1) / BN);
  int num_tiles = 0;
  for (int cb = 0; cb < ncb; ++cb) num_tiles += (2 * cb + 2 < nrb) ? 2 * cb + 2 : nrb;
  const int k_iters = (int)((N + BK - 1) / BK);
  const int chunks = (k_iters + KC_ITERS - 1) / KC_ITERS;
  const int64_t units64 = (int64_t)num_tiles * chunks;
  if (units64 > INT32_MAX) return KRONQ_ERR_UNSUPPORTED;
  const int num_units = (int)units64;

  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(cov_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES) != cudaSuccess)
      return KRONQ_ERR_CUDA;
    attr_set = true;
  }
  // H <- beta H, then the units add alpha A^T A into its upper tiles
  if (beta != 1.f) {
    scale_kernel<<<4 * kqh::num_sms(), 256, 0, st>>>(H, ldh, (int)d, beta);
    KQ_CHECK_LAUNCH();
  }
  const int grid = num_units < kqh::num_sms() ? num_units : kqh::num_sms();
  cov_tc_kernel<<<grid, THREADS, SMEM_BYTES, st>>>(tmap, hmap, k_iters, ncb, num_tiles, num_units,
                                                   alpha, info);
  KQ_CHECK_LAUNCH();
  const int nt = (int)((d + 31) / 32);
  mirror_kernel<<<dim3(nt, nt), 256, 0, st>>>(H, ldh, (int)d);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}
