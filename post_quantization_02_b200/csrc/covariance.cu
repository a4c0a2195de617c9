// H = alpha * A^T A + beta * H on the 5th-generation tensor cores.
//
// KronQ summary (hyper.ai), "Method" (Eq. 7): the two Kronecker factors
// H_X = E[x x^T] and H_G = E[g g^T] are covariances over the calibration
// tokens.  A is token-major (N x d, bf16), so a tile of H is a rank-K update
// whose operands are both "MN-major": for a K-slab of tokens the features
// (the M and N indices of the tile) are contiguous in memory.
//
// Kernel structure (one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: per K-slab of 64 tokens, two 64x64 boxes of the
//               row panel (A, 128 features) and four of the column panel (B,
//               256 features), 128-byte swizzled, into a 4-stage ring.
//   warp 1      one thread issues tcgen05.mma (M=128, N=256, K=16, bf16 in,
//               fp32 accumulate in TMEM) and commits each stage back to the
//               producer, and each finished tile to the epilogue.
//   warp 2      allocates / frees the 512 TMEM columns: the accumulator
//               (256) and an fp32 master (256) that the epilogue folds each
//               4096-token partial sum into.
//   warps 4-7   epilogue: folds (tcgen05.ld / add / tcgen05.st), then per tile
//               H = alpha master + beta H for the elements on or above the
//               diagonal, stored twice: in place (row-contiguous vector
//               stores) and mirrored (for a fixed column the 32 lanes of a
//               warp write 32 consecutive floats of the transposed row).
// Only tiles that touch the upper triangle are computed; with the mirrored
// stores every element of the symmetric d x d result is written once per
// call (the diagonal twice, with the same value).  When beta != 0 the old
// upper triangle is read, so the old H must be symmetric.
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
constexpr int TMEM_COLS = 2 * BN;  // accumulator + master
constexpr int THREADS = 256;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
constexpr uint32_t IDESC = kq::idesc_f16(BM, BN, /*bf16*/ 1, /*A MN-major*/ 1, /*B MN-major*/ 1);

struct Bars {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull;
  uint64_t tempty;
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

__global__ void __launch_bounds__(THREADS, 1)
cov_tc_kernel(const __grid_constant__ CUtensorMap tmap, float* __restrict__ H, int64_t ldh, int d,
              int k_iters, int ncb, int num_tiles, float alpha, float beta, int32_t* info) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Bars* bars = reinterpret_cast<Bars*>(tiles + STAGES * STAGE_BYTES);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      kq::mbar_init(&bars->full[s], 1);
      kq::mbar_init(&bars->empty[s], 1);
    }
    kq::mbar_init(&bars->tfull, 1);
    kq::mbar_init(&bars->tempty, 4);
    kq::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    kq::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) kq::prefetch_tmap(&tmap);
  if (warp == 2) kq::tmem_alloc(&bars->tmem_base, TMEM_COLS);
  kq::tc_fence_before();
  __syncthreads();
  kq::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int it = 0;
      for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
        int rb, cb;
        tile_coords(t, ncb, rb, cb);
        const int i0 = rb * BM, j0 = cb * BN;
        bool ok = true;
        for (int kb = 0; kb < k_iters; ++kb, ++it) {
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
        if (!ok) break;
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
      // One accumulator (TMEM columns [0, BN)); it is handed to the epilogue
      // after every chunk of KC_ITERS K-slabs and reused once folded.
      int it = 0, cc = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        for (int k0 = 0; k0 < k_iters && ok; k0 += KC_ITERS, ++cc) {
          const int k1 = min(k_iters, k0 + KC_ITERS);
          if (!kq::mbar_wait(&bars->tempty, ((uint32_t)cc & 1u) ^ 1u, abort, info)) { ok = false; break; }
          kq::tc_fence_after();
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
              kq::mma_f16(tmem, ad, bd, IDESC, (kb != k0) || (kk != 0));
            }
            kq::mma_commit(&bars->empty[s]);
          }
          if (ok) kq::mma_commit(&bars->tfull);
        }
      }
      // wind down: all MMAs issued by this thread complete before TMEM is freed
      kq::mma_commit(&bars->drain);
      drain_wait(&bars->drain, 0, info);
    }
  } else if (warp >= 4) {
    // -------------------------------------------------- epilogue
    // Each chunk's partial sum is folded into the fp32 master (TMEM columns
    // [BN, 2 BN)) with ordinary round-to-nearest adds, so the tensor core's
    // own accumulation only ever spans KC_ITERS * BK tokens.  The accumulator
    // is released as soon as the fold is done; after the last chunk of a tile
    // the master is written out (H = alpha master + beta H_old) together with
    // its mirror image.
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    int cc = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
      int rb, cb;
      tile_coords(t, ncb, rb, cb);
      const int i0 = rb * BM, j0 = cb * BN;
      const int row0 = i0 + q * 32;             // first row of this warp's 32 lanes
      const int row = row0 + lane;
      for (int k0 = 0; k0 < k_iters; k0 += KC_ITERS, ++cc) {
        const bool first = k0 == 0, last = k0 + KC_ITERS >= k_iters;
        if (!kq::mbar_wait(&bars->tfull, (uint32_t)cc & 1u, abort, info)) { ok = false; break; }
        kq::tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          if (j0 + c >= d) break;                   // columns past the matrix (uniform)
          if (j0 + c + 31 < row0) continue;         // strictly below the diagonal: never stored
          float v[32], mst[32];
          __syncwarp();
          kq::tmem_ld32(tmem + lane_off + (uint32_t)c, v);
          if (!first) kq::tmem_ld32(tmem + lane_off + (uint32_t)(BN + c), mst);
          kq::tmem_wait_ld();
          if (!first) {
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] += mst[k];
          }
          kq::tmem_st32(tmem + lane_off + (uint32_t)(BN + c), v);
        }
        kq::tmem_wait_st();
        kq::tc_fence_before();
        __syncwarp();
        if (lane == 0) kq::mbar_arrive(&bars->tempty);   // accumulator free again
        if (!last) continue;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          const int jc = j0 + c;
          if (jc >= d) break;
          if (jc + 31 < row0) continue;
          float v[32];
          __syncwarp();
          kq::tmem_ld32(tmem + lane_off + (uint32_t)(BN + c), v);
          kq::tmem_wait_ld();
          if (row < d) {
            float* dst = H + (int64_t)row * ldh + jc;
            if (jc >= row0 + 31 && jc + 32 <= d) {
              // whole chunk on or above the diagonal for every lane: vector stores
#pragma unroll
              for (int k = 0; k < 32; k += 4) {
                float4 o = make_float4(alpha * v[k], alpha * v[k + 1], alpha * v[k + 2], alpha * v[k + 3]);
                if (beta != 0.f) {
                  const float4 h = *reinterpret_cast<const float4*>(dst + k);
                  o.x = fmaf(beta, h.x, o.x); o.y = fmaf(beta, h.y, o.y);
                  o.z = fmaf(beta, h.z, o.z); o.w = fmaf(beta, h.w, o.w);
                }
                v[k] = o.x; v[k + 1] = o.y; v[k + 2] = o.z; v[k + 3] = o.w;
                *reinterpret_cast<float4*>(dst + k) = o;
              }
            } else {
#pragma unroll
              for (int k = 0; k < 32; ++k) {
                if (jc + k < d && jc + k >= row) {
                  float o = alpha * v[k];
                  if (beta != 0.f) o = fmaf(beta, dst[k], o);
                  v[k] = o;
                  dst[k] = o;
                }
              }
            }
            // mirror: H[j][row] for j > row; for each j the warp writes 32 consecutive floats
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (jc + k < d && jc + k > row) H[(int64_t)(jc + k) * ldh + row] = v[k];
          }
        }
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
  CUtensorMap tmap;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)N};
  cuuint64_t strides[1] = {(cuuint64_t)lda * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)BK};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(A), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return KRONQ_ERR_UNSUPPORTED;

  const int nrb = (int)((d + BM - 1) / BM), ncb = (int)((d + BN - 1) / BN);
  int num_tiles = 0;
  for (int cb = 0; cb < ncb; ++cb) num_tiles += (2 * cb + 2 < nrb) ? 2 * cb + 2 : nrb;
  const int k_iters = (int)((N + BK - 1) / BK);

  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(cov_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES) != cudaSuccess)
      return KRONQ_ERR_CUDA;
    attr_set = true;
  }
  const int grid = num_tiles < kqh::num_sms() ? num_tiles : kqh::num_sms();
  cov_tc_kernel<<<grid, THREADS, SMEM_BYTES, st>>>(tmap, H, ldh, (int)d, k_iters, ncb, num_tiles,
                                                   alpha, beta, info);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}
