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

#include <mutex>

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

// Row `row` of H, columns jc .. jc+31 (v = the fp32 sums): H = alpha v + beta H
// for the elements on or above the diagonal, and their mirror images below
// it.  row0 is the first row of the calling warp (rows row0 .. row0+31).
__device__ __forceinline__ void store_row_chunk(float* __restrict__ H, int64_t ldh, int d, int row,
                                                int row0, int jc, float (&v)[32], float alpha,
                                                float beta) {
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

KQ_DEV void red_add_v4(float* p, float a, float b, float c, float e) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(e)
               : "memory");
}

KQ_DEV void red_add(float* p, float a) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(a) : "memory");
}

// As store_row_chunk, for a tile that several CTA pairs share: adds alpha v
// into H on and above the diagonal with reductions.  The mirror images are
// copied once all parts are in (mirror_tiles_kernel), so that H stays exactly
// symmetric whatever order the parts arrive in.
__device__ __forceinline__ void add_row_chunk(float* __restrict__ H, int64_t ldh, int d, int row,
                                              int row0, int jc, const float (&v)[32], float alpha) {
  float* dst = H + (int64_t)row * ldh + jc;
  if (jc >= row0 + 31 && jc + 32 <= d) {
#pragma unroll
    for (int k = 0; k < 32; k += 4)
      red_add_v4(dst + k, alpha * v[k], alpha * v[k + 1], alpha * v[k + 2], alpha * v[k + 3]);
  } else {
#pragma unroll
    for (int k = 0; k < 32; ++k)
      if (jc + k < d && jc + k >= row) red_add(dst + k, alpha * v[k]);
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
          if (row < d) store_row_chunk(H, ldh, d, row, row0, jc, v, alpha, beta);
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

// ------------------------------------------------------------------------
// The same product on CTA pairs (cta_group::2): a cluster of two CTAs owns a
// 256 x 256 tile of H.  Per K-slab of 64 tokens each CTA loads its 128 rows
// of the tile's row panel and its 128 of the column panel (32 KB, against
// 48 KB per 128 x 256 tile for one CTA alone), and the even CTA issues
// tcgen05.mma.cta_group::2 with M = N = 256: the pair's two tensor cores
// each compute their 128 x 256 half from 128 + 256 features staged across
// both shared memories.  Per unit of tensor-core work the shared-memory
// traffic drops by a third, and the same 192 KB ring covers 50 % more
// K-slabs of load latency.  Each CTA folds and stores its own 128 rows
// exactly as the single-CTA kernel does.
//
// Work is dealt out so that every pair streams the same tokens at the same
// time (one 64-token slab of A then serves all pairs from L2, the reason the
// covariance reads A from DRAM about once): with P pairs and T tiles, the
// first W = T / P waves give each pair whole tiles.  Of the R = T mod P tiles
// left, each goes to one pair for its first k* token chunks (chunks of
// KC_ITERS K-slabs, the fold granularity) while the P - R pairs that would
// otherwise sit idle take the last C - k* chunks of g = ceil(R / (P - R))
// tiles each, k* balancing the two: k* = ceil(g C / (g + 1)).  Only two token
// offsets are then in flight.  A tile split that way is added into H by its
// two pairs with fp32 reductions, onto its region of H zeroed (or scaled by
// beta) by a pass over the split tiles first; with beta = 0 the sum
// 0 + a + b does not depend on the order.
//
// Barriers: full[s] of the even CTA counts the bytes of both CTAs' loads
// (its producer arms it for 2 x 32 KB; the odd CTA's loads complete on it
// through the cta_group::2 form of the TMA load); empty[s] and tfull exist
// in both CTAs and receive one multicast tcgen05.commit each; tempty of the
// even CTA collects the 8 epilogue warps of the pair.
constexpr int P_BM = 128;                            // rows of the tile per CTA
constexpr int P_TILE = 256;                          // the pair's square tile
constexpr int P_STAGES = 7;
constexpr int P_A_BYTES = P_BM * BK * 2;             // 16 KB
constexpr int P_B_BYTES = (P_TILE / 2) * BK * 2;     // 16 KB
constexpr int P_STAGE_BYTES = P_A_BYTES + P_B_BYTES; // 32 KB
constexpr int P_SMEM_BYTES = P_STAGES * P_STAGE_BYTES + 1024 + 256;
// warps 0-3: TMA producer, MMA issuer, TMEM allocator, idle; warps 4-11: the
// epilogue, two per TMEM lane quadrant (128 columns each), so that folding
// the accumulator into the master (which the next chunk's MMAs wait for)
// takes few round trips to TMEM
constexpr int P_THREADS = 384;
constexpr int P_EPI_WARPS = 8;
constexpr uint32_t P_IDESC = kq::idesc_f16(2 * P_BM, P_TILE, /*bf16*/ 1, /*A MN-major*/ 1, /*B MN-major*/ 1);
static_assert(P_SMEM_BYTES <= 227 * 1024, "pair ring exceeds the shared-memory limit");

struct PairBars {
  uint64_t full[P_STAGES];
  uint64_t empty[P_STAGES];
  uint64_t tfull;
  uint64_t tempty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// Tiles per side of a super-block of the tile order below.
constexpr int P_SB = 8;

// Square tiles (rb <= cb) of the upper triangle of an nb x nb tile grid, in
// super-blocks of P_SB x P_SB tiles: super-columns J in order; in each, the
// super-blocks I = 0 .. J -- row-major inside an off-diagonal one, column by
// column inside the diagonal one.  The pairs of one wave take consecutive
// tiles at the same token offset, so with this order a wave's tiles span
// about 2 P_SB row and column panels (instead of a whole column of the
// triangle, i.e. most of the panels): each token slab a wave needs leaves
// DRAM once for a few panels, which L2 then serves to every pair.
__device__ __forceinline__ void pair_tile_coords(int t, int nb, int& rb, int& cb) {
  const int nsb = (nb + P_SB - 1) / P_SB;
  int J = 0, base = 0, w = 0;
  for (;; ++J) {
    w = min(P_SB, nb - J * P_SB);
    const int cnt = J * P_SB * w + w * (w + 1) / 2;
    if (t < base + cnt || J >= nsb - 1) break;
    base += cnt;
  }
  int u = t - base;
  const int off = J * P_SB * w;
  if (u < off) {
    const int I = u / (P_SB * w), v = u - I * (P_SB * w);
    rb = I * P_SB + v / w;
    cb = J * P_SB + v % w;
  } else {
    u -= off;
    int c = (int)((sqrtf(8.f * (float)u + 1.f) - 1.f) * 0.5f);
    while ((c + 1) * (c + 2) / 2 <= u) ++c;
    while (c * (c + 1) / 2 > u) --c;
    rb = J * P_SB + (u - c * (c + 1) / 2);
    cb = J * P_SB + c;
  }
}

struct PairSchedule {
  int nb;              // tiles per side of the tile grid
  int tiles, chunks;   // T, C
  int waves, rest;     // W = T / P, R = T mod P
  int per_helper;      // g
  int kstar;           // k*
};

// The idx-th segment (tile t, chunks [c0, c1)) of pair p; false when p has
// no more.
__device__ __forceinline__ bool pair_segment(const PairSchedule& S, int p, int np, int idx, int& t,
                                             int& c0, int& c1) {
  if (idx < S.waves) {
    t = p + idx * np;
    c0 = 0;
    c1 = S.chunks;
    return true;
  }
  idx -= S.waves;
  if (S.rest == 0) return false;
  const int t0 = S.waves * np;
  if (p < S.rest) {
    if (idx > 0) return false;
    t = t0 + p;
    c0 = 0;
    c1 = S.kstar;
    return true;
  }
  if (S.kstar >= S.chunks || idx >= S.per_helper) return false;
  const int i = (p - S.rest) * S.per_helper + idx;
  if (i >= S.rest) return false;
  t = t0 + i;
  c0 = S.kstar;
  c1 = S.chunks;
  return true;
}

// Keeping the pairs of a launch at the same token offset.  Every pair
// streams all N tokens for each of its tiles, so the pairs of one wave share
// each token slab through L2 only while they stay together; left alone they
// drift apart over many waves (measured: ~1.2 TB of DRAM reads for one
// 28672-wide launch over 262144 tokens, ~80x the input).  Before its next
// wave's tile, a producer waits until every producer of the launch has
// issued the loads of the current wave (the counter reaches target).  The
// wait is a timing hint, not a guard: it gives up after kWaveGateNs without
// recording anything, and nothing depends on it for correctness.
constexpr unsigned long long kWaveGateNs = 2000000ull;  // 2 ms

__device__ __forceinline__ void wave_gate(const unsigned int* ctr, unsigned int target) {
  if (*reinterpret_cast<const volatile unsigned int*>(ctr) >= target) return;
  const unsigned long long t0 = kq::globaltimer();
  while (*reinterpret_cast<const volatile unsigned int*>(ctr) < target) {
    if (kq::globaltimer() - t0 > kWaveGateNs) return;
    __nanosleep(256);
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(P_THREADS, 1)
cov_pair_kernel(const __grid_constant__ CUtensorMap tmap, float* __restrict__ H, int64_t ldh, int d,
                int k_iters, const PairSchedule sched, float alpha, float beta, int32_t* info,
                unsigned int* wave_ctr) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  PairBars* bars = reinterpret_cast<PairBars*>(tiles + P_STAGES * P_STAGE_BYTES);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = kq::cluster_rank();
  const int cid = (int)kq::cluster_id_x(), ncl = (int)kq::num_clusters_x();

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      kq::mbar_init(&bars->full[s], 1);
      kq::mbar_init(&bars->empty[s], 1);
    }
    kq::mbar_init(&bars->tfull, 1);
    kq::mbar_init(&bars->tempty, 2 * P_EPI_WARPS);   // every epilogue warp of both CTAs
    kq::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    kq::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) kq::prefetch_tmap(&tmap);
  if (warp == 2) kq::tmem_alloc_pair(&bars->tmem_base, TMEM_COLS);
  kq::tc_fence_before();
  kq::cluster_sync();          // the peer's barriers are initialised before any remote signal
  kq::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer (both CTAs)
      int it = 0;
      int t, c0, c1;
      for (int sg = 0; pair_segment(sched, cid, ncl, sg, t, c0, c1); ++sg) {
        int rb, cb;
        pair_tile_coords(t, sched.nb, rb, cb);
        const int i0 = rb * P_TILE + P_BM * (int)rank;          // this CTA's rows of the tile
        const int j0 = cb * P_TILE + (P_TILE / 2) * (int)rank;  // this CTA's half of the columns
        if (wave_ctr && sg > 0 && sg < sched.waves) wave_gate(wave_ctr, 2u * (unsigned)ncl * (unsigned)sg);
        bool ok = true;
        const int kb_end = min(k_iters, c1 * KC_ITERS);
        for (int kb = c0 * KC_ITERS; kb < kb_end; ++kb, ++it) {
          const int s = it % P_STAGES;
          const uint32_t ph = (uint32_t)(it / P_STAGES) & 1u;
          if (!kq::mbar_wait(&bars->empty[s], ph ^ 1u, abort, info)) { ok = false; break; }
          uint8_t* a = tiles + s * P_STAGE_BYTES;
          uint8_t* b = a + P_A_BYTES;
          if (rank == 0) kq::mbar_arrive_expect_tx(&bars->full[s], 2 * P_STAGE_BYTES);
          const uint32_t fb = kq::map_to_rank(kq::smem_u32(&bars->full[s]), 0);
          const int y = kb * BK;
          kq::tma_load_2d_pair(a, &tmap, fb, i0, y);
          kq::tma_load_2d_pair(a + BOX_BYTES, &tmap, fb, i0 + 64, y);
          kq::tma_load_2d_pair(b, &tmap, fb, j0, y);
          kq::tma_load_2d_pair(b + BOX_BYTES, &tmap, fb, j0 + 64, y);
        }
        if (!ok) break;
        // this producer has issued its whole tile of the wave
        if (wave_ctr && sg < sched.waves) atomicAdd(wave_ctr, 1u);
      }
      // wind down (even CTA): every armed phase has landed, the odd CTA's
      // bytes included, before the pair may exit
      if (rank == 0) {
        for (int s = 0; s < P_STAGES; ++s) {
          const int armed = (it > s) ? (it - s + P_STAGES - 1) / P_STAGES : 0;
          if (armed > 0) drain_wait(&bars->full[s], (uint32_t)(armed - 1) & 1u, info);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------ MMA issuer (even CTA)
      int it = 0, cc = 0;
      bool ok = true;
      int t, c0, c1;
      for (int sg = 0; ok && pair_segment(sched, cid, ncl, sg, t, c0, c1); ++sg) {
        for (int ch = c0; ch < c1 && ok; ++ch, ++cc) {
          const int k0 = ch * KC_ITERS, k1 = min(k_iters, k0 + KC_ITERS);
          if (!kq::mbar_wait(&bars->tempty, ((uint32_t)cc & 1u) ^ 1u, abort, info)) { ok = false; break; }
          kq::tc_fence_after();
          for (int kb = k0; kb < k1; ++kb, ++it) {
            const int s = it % P_STAGES;
            const uint32_t ph = (uint32_t)(it / P_STAGES) & 1u;
            if (!kq::mbar_wait(&bars->full[s], ph, abort, info)) { ok = false; break; }
            kq::tc_fence_after();
            const uint32_t a_addr = kq::smem_u32(tiles + s * P_STAGE_BYTES);
            const uint32_t b_addr = a_addr + P_A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t ad = kq::smem_desc(a_addr + kk * 2048, BOX_BYTES, 1024, kq::kLayoutSwizzle128B);
              const uint64_t bd = kq::smem_desc(b_addr + kk * 2048, BOX_BYTES, 1024, kq::kLayoutSwizzle128B);
              kq::mma_f16_pair(tmem, ad, bd, P_IDESC, (kb != k0) || (kk != 0));
            }
            kq::mma_commit_pair(&bars->empty[s], 0x3);
          }
          if (ok) kq::mma_commit_pair(&bars->tfull, 0x3);
        }
      }
      kq::mma_commit_pair(&bars->drain, 0x1);
      drain_wait(&bars->drain, 0, info);
    }
  } else if (warp >= 4) {
    // -------------------------------------------------- epilogue (both CTAs)
    // warp 4 + 4 h + q: TMEM lane quadrant q (a warp may only read its own
    // quadrant), tile columns [128 h, 128 h + 128)
    const int q = warp & 3, cbeg = 128 * ((warp - 4) >> 2);
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t tempty_leader = kq::map_to_rank(kq::smem_u32(&bars->tempty), 0);
    int cc = 0;
    bool ok = true;
    int t, c0, c1;
    for (int sg = 0; ok && pair_segment(sched, cid, ncl, sg, t, c0, c1); ++sg) {
      const bool shared_tile = c0 > 0 || c1 < sched.chunks;   // another pair adds the rest
      int rb, cb;
      pair_tile_coords(t, sched.nb, rb, cb);
      const int i0 = rb * P_TILE + P_BM * (int)rank, j0 = cb * P_TILE;
      const int row0 = i0 + q * 32;
      const int row = row0 + lane;
      for (int ch = c0; ch < c1; ++ch, ++cc) {
        const bool first = ch == c0, last = ch == c1 - 1;
        if (!kq::mbar_wait(&bars->tfull, (uint32_t)cc & 1u, abort, info)) { ok = false; break; }
        kq::tc_fence_after();
        // fold: master = acc (first chunk) or master + acc (rounded to nearest)
#pragma unroll 1
        for (int c = cbeg; c < cbeg + 128; c += 32) {
          if (j0 + c >= d) break;
          if (j0 + c + 31 < row0) continue;
          float v[32], mst[32];
          __syncwarp();
          kq::tmem_ld32(tmem + lane_off + (uint32_t)c, v);
          if (!first) kq::tmem_ld32(tmem + lane_off + (uint32_t)(P_TILE + c), mst);
          kq::tmem_wait_ld();
          if (!first) {
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] += mst[k];
          }
          kq::tmem_st32(tmem + lane_off + (uint32_t)(P_TILE + c), v);
        }
        kq::tmem_wait_st();
        kq::tc_fence_before();
        __syncwarp();
        if (lane == 0) kq::mbar_arrive_cluster(tempty_leader);
        if (!last) continue;
#pragma unroll 1
        for (int c = cbeg; c < cbeg + 128; c += 32) {
          const int jc = j0 + c;
          if (jc >= d) break;
          if (jc + 31 < row0) continue;
          float v[32];
          __syncwarp();
          kq::tmem_ld32(tmem + lane_off + (uint32_t)(P_TILE + c), v);
          kq::tmem_wait_ld();
          if (row < d) {
            if (shared_tile) add_row_chunk(H, ldh, d, row, row0, jc, v, alpha);
            else store_row_chunk(H, ldh, d, row, row0, jc, v, alpha, beta);
          }
        }
      }
    }
  }

  kq::tc_fence_before();
  kq::cluster_sync();          // no CTA leaves while the pair's MMAs or loads may touch it
  if (warp == 2) {
    kq::tc_fence_after();
    kq::tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

// The square tiles several pairs shared (at most one per pair boundary).
constexpr int kMaxSharedTiles = 256;
struct SharedTiles {
  int nb;      // tiles per side of the tile grid
  int count;
  int tile[kMaxSharedTiles];
};

// For each listed 256 x 256 tile (rb <= cb): H[j][i] = H[i][j] for the tile's
// elements above the diagonal, through 32 x 32 shared-memory transposes
// (coalesced on both sides).  blockIdx.x = listed tile * 64 + 32 x 32 block.
__global__ void __launch_bounds__(256) mirror_tiles_kernel(float* __restrict__ H, int64_t ldh, int d,
                                                           const __grid_constant__ SharedTiles st) {
  __shared__ float tile[32][33];
  const int li = blockIdx.x >> 6, sb = blockIdx.x & 63;
  int rb, cb;
  pair_tile_coords(st.tile[li], st.nb, rb, cb);
  const int i0 = rb * P_TILE + (sb >> 3) * 32, j0 = cb * P_TILE + (sb & 7) * 32;   // source block
  if (i0 >= d || j0 >= d || j0 + 31 < i0) return;                                  // nothing above the diagonal
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int r = ty; r < 32; r += 8) {
    const int i = i0 + r, j = j0 + tx;
    tile[r][tx] = (i < d && j < d) ? H[(int64_t)i * ldh + j] : 0.f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int j = j0 + r, i = i0 + tx;                 // destination H[j][i] = H[i][j]
    if (i < d && j < d && j > i) H[(int64_t)j * ldh + i] = tile[tx][r];
  }
}

// H = beta H (zeros when beta = 0) on the listed 256 x 256 tiles only: the
// tiles whose parts arrive by reductions.  blockIdx.x = listed tile * 64 +
// 32 x 32 block.
__global__ void __launch_bounds__(256) scale_tiles_kernel(float* __restrict__ H, int64_t ldh, int d,
                                                          float beta,
                                                          const __grid_constant__ SharedTiles st) {
  const int li = blockIdx.x >> 6, sb = blockIdx.x & 63;
  int rb, cb;
  pair_tile_coords(st.tile[li], st.nb, rb, cb);
  const int i0 = rb * P_TILE + (sb >> 3) * 32, j0 = cb * P_TILE + (sb & 7) * 32;
  if (i0 >= d || j0 >= d) return;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int r = ty; r < 32; r += 8) {
    const int i = i0 + r, j = j0 + tx;
    if (i < d && j < d) {
      float* p = H + (int64_t)i * ldh + j;
      *p = (beta == 0.f) ? 0.f : beta * *p;
    }
  }
}

// H = beta H over d x d (ldh), zeros when beta = 0 (no read).
__global__ void scale_kernel(float* __restrict__ H, int64_t ldh, int d, float beta) {
  const bool vec = (d % 4) == 0 && (ldh % 4) == 0;
  for (int r = blockIdx.x; r < d; r += gridDim.x) {
    float* row = H + (int64_t)r * ldh;
    if (vec) {
      float4* row4 = reinterpret_cast<float4*>(row);
      for (int c = threadIdx.x; c < d / 4; c += blockDim.x) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (beta != 0.f) {
          v = row4[c];
          v.x *= beta; v.y *= beta; v.z *= beta; v.w *= beta;
        }
        row4[c] = v;
      }
    } else {
      for (int c = threadIdx.x; c < d; c += blockDim.x) row[c] = (beta == 0.f) ? 0.f : beta * row[c];
    }
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

// The wave counter of cov_pair_kernel: one word per device (a static device
// variable of the library), reset before every launch on the launch's stream.
// Launches that overlap on the GPU share it; then a gate may open early or
// give up after its time limit -- only the timing changes.
static __device__ unsigned int g_cov_wave_ctr;

namespace {
std::mutex g_wave_mutex;
unsigned int* g_wave_ptr[64] = {};

unsigned int* wave_counter() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_wave_mutex);
  if (!g_wave_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_cov_wave_ctr) != cudaSuccess || !p) {
      cudaGetLastError();
      return nullptr;
    }
    g_wave_ptr[dev] = static_cast<unsigned int*>(p);
  }
  return g_wave_ptr[dev];
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

  const int k_iters = (int)((N + BK - 1) / BK);
  if (d > P_TILE) {
    // CTA pairs on 256 x 256 tiles
    const int ncb2 = (int)((d + P_TILE - 1) / P_TILE);
    const int tiles2 = ncb2 * (ncb2 + 1) / 2;
    // the shared-memory attribute and the number of co-resident pairs, once per device
    static kqh::PerDevice pairs_of_device;
    const int P = kqh::per_device(pairs_of_device, [] {
      if (cudaFuncSetAttribute(cov_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               P_SMEM_BYTES) != cudaSuccess)
        return 0;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * (kqh::num_sms() / 2), 1, 1);
      cfg.blockDim = dim3(P_THREADS, 1, 1);
      cfg.dynamicSmemBytes = P_SMEM_BYTES;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, cov_pair_kernel, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = kqh::num_sms() / 2;
      }
      return n < kMaxSharedTiles ? n : kMaxSharedTiles;
    });
    if (P <= 0) return KRONQ_ERR_CUDA;
    PairSchedule sc;
    sc.nb = ncb2;
    sc.tiles = tiles2;
    sc.chunks = (k_iters + KC_ITERS - 1) / KC_ITERS;
    sc.waves = tiles2 / P;
    sc.rest = tiles2 % P;
    sc.per_helper = sc.rest > 0 ? (sc.rest + (P - sc.rest) - 1) / (P - sc.rest) : 0;
    sc.kstar = sc.rest > 0 ? (sc.per_helper * sc.chunks + sc.per_helper) / (sc.per_helper + 1) : sc.chunks;
    if (sc.kstar < 1) sc.kstar = 1;
    if (sc.kstar > sc.chunks) sc.kstar = sc.chunks;
    // the split tiles: the R tiles of the last, partial wave when helpers take their tail
    SharedTiles list;
    list.nb = ncb2;
    list.count = 0;
    if (sc.rest > 0 && sc.kstar < sc.chunks) {
      if (sc.rest > kMaxSharedTiles) return KRONQ_ERR_UNSUPPORTED;
      for (int i = 0; i < sc.rest; ++i) list.tile[list.count++] = sc.waves * P + i;
    }
    const bool shared = list.count > 0;
    const int pairs = (sc.waves == 0 && !shared) ? sc.rest : P;
    if (shared && beta != 1.f) {
      // the split tiles add into H: they start from beta H (zeros when beta = 0);
      // the tiles a single pair owns apply beta themselves
      scale_tiles_kernel<<<list.count * 64, 256, 0, st>>>(H, ldh, (int)d, beta, list);
      KQ_CHECK_LAUNCH();
    }
    const float beta_owned = beta;
    unsigned int* wctr = sc.waves > 1 ? wave_counter() : nullptr;
    if (wctr && cudaMemsetAsync(wctr, 0, sizeof(unsigned int), st) != cudaSuccess) return KRONQ_ERR_CUDA;
    cov_pair_kernel<<<2 * pairs, P_THREADS, P_SMEM_BYTES, st>>>(tmap, H, ldh, (int)d, k_iters, sc,
                                                             alpha, beta_owned, info, wctr);
    KQ_CHECK_LAUNCH();
    if (shared) {
      mirror_tiles_kernel<<<list.count * 64, 256, 0, st>>>(H, ldh, (int)d, list);
      KQ_CHECK_LAUNCH();
    }
    return KRONQ_OK;
  }

  const int nrb = (int)((d + BM - 1) / BM), ncb = (int)((d + BN - 1) / BN);
  int num_tiles = 0;
  for (int cb = 0; cb < ncb; ++cb) num_tiles += (2 * cb + 2 < nrb) ? 2 * cb + 2 : nrb;

  static kqh::PerDevice attr;
  if (kqh::smem_attr_once(attr, cov_tc_kernel, SMEM_BYTES) <= 0) return KRONQ_ERR_CUDA;
  const int grid = num_tiles < kqh::num_sms() ? num_tiles : kqh::num_sms();
  cov_tc_kernel<<<grid, THREADS, SMEM_BYTES, st>>>(tmap, H, ldh, (int)d, k_iters, ncb, num_tiles,
                                                   alpha, beta, info);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}
