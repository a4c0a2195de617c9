// C += alpha * A B^T on the 5th-generation tensor cores from operands split
// into hi / lo planes, three products per K step (hi*hi + hi*lo + lo*hi),
// for up to two problems per launch.  Two plane types (one per launch):
//   tf32: hi tf32-exact, lo the fp32 remainder (fp32-level accuracy; the
//         inverse Cholesky's updates and the GPTAQ correction),
//   bf16: hi = RN_bf16(x), lo = RN_bf16(x - hi) (~2^-17 relative, twice the
//         tf32 rate and half the bytes; the solver's lazy updates).
// All planes row-major, so all four reach the tensor core K-major straight
// from TMA, 128-byte rows (32 tf32 or 64 bf16 K values).  C is M x N
// row-major, updated in place.  A problem may ask for its lower triangle
// only (M = N, tiles with tile column > tile row skipped, diagonal tiles
// written on and below the diagonal): the symmetric rank-K update of a
// Cholesky factorisation.
//
// Persistent kernel, one CTA per SM, 320 threads, 128 x 128 output tiles,
// K streamed in 32-wide chunks through a 3-stage ring:
//   warp 0       TMA loads of A_hi, A_lo, B_hi, B_lo of a stage (16 KB each)
//   warp 1       one thread issues 3 MMAs (M = N = 128, K = 8) per K step
//                into one of two TMEM accumulators
//   warps 2-9    read an accumulator back and add it to C with TMA reduces
//                (32 x 32 boxes staged in shared memory)
// All waits are bounded; a wait that gives up records KRONQ_ERR_TIMEOUT in
// `info` and the CTA winds down.
#include "gemm_tc.cuh"

#include "tf32x3.cuh"

namespace {

constexpr int TM = 128, TN = 128;
constexpr int STAGES = 3;
constexpr int CHUNK = TM * 128;                // 16 KB: 128 rows x 128 bytes (32 fp32 / 64 bf16)
constexpr int STAGE_BYTES = 4 * CHUNK;         // A hi, A lo, B hi, B lo
constexpr int THREADS = 320;
constexpr int EPI_WARP0 = 2;
constexpr int STG_BYTES = 32 * 32 * 4;           // one 32 x 32 fp32 box per epilogue warp
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 8 * STG_BYTES + 1024 + 256;
constexpr int TMEM_COLS = 2 * TN;

struct Bars {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

struct Maps {
  CUtensorMap a_hi[2], a_lo[2];
  CUtensorMap b_hi[2], b_lo[2];
  CUtensorMap c[2];
};

// C box += the 32 x 32 fp32 box in shared memory (TMA, bulk-group completion).
KQ_DEV void tma_reduce_add_2d(const void* tmap, const void* src, int x, int y) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(tmap)),
      "r"(kq::smem_u32(src)), "r"(x), "r"(y)
      : "memory");
}
KQ_DEV void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
KQ_DEV void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
KQ_DEV void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

struct Problem {
  float* C;
  const float* a_scale;   // fp16 planes only: per-row and per-column factors of the product
  const float* b_scale;
  int64_t ldc;
  int M, N, K;
  float alpha;
  int lower;
  int ntn;     // tile columns (rectangular problems)
  int t0;      // first tile of the problem's own tile order
  int tiles;
};

struct Problems {
  Problem p[2];
  int count;
  int total_tiles;
};

struct Tile {
  int prob, tm, tn, kchunks;
};

template <int KC>
__device__ __forceinline__ Tile tile_of(const Problems& P, int t) {
  Tile r;
  r.prob = (P.count > 1 && t >= P.p[0].tiles) ? 1 : 0;
  if (r.prob) t -= P.p[0].tiles;
  const Problem& q = P.p[r.prob];
  t += q.t0;
  if (q.lower) {
    int tm = (int)((sqrtf(8.f * (float)t + 1.f) - 1.f) * 0.5f);
    while ((tm + 1) * (tm + 2) / 2 <= t) ++tm;
    while (tm * (tm + 1) / 2 > t) --tm;
    r.tm = tm;
    r.tn = t - tm * (tm + 1) / 2;
  } else {
    r.tm = t / q.ntn;
    r.tn = t % q.ntn;
  }
  r.kchunks = (q.K + KC - 1) / KC;
  return r;
}

// KIND 0: tf32 planes (32 fp32 K values per 128-byte row); 1: bf16 planes;
// 2: fp16 planes of scaled rows (64 K values per row; the epilogue applies
// the rows' and columns' factors).
template <int KIND>
__global__ void __launch_bounds__(THREADS, 1)
gemm_nt_tc_kernel(const __grid_constant__ Maps maps, const __grid_constant__ Problems P,
                  int32_t* info) {
  constexpr int KC = KIND ? 64 : 32;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stages = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* staging = stages + STAGES * STAGE_BYTES;   // 1024-byte aligned
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
      kq::mbar_init(&bars->tempty[b], 8);
    }
    kq::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    kq::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < P.count; ++i) {
      kq::prefetch_tmap(&maps.a_hi[i]);
      kq::prefetch_tmap(&maps.a_lo[i]);
      kq::prefetch_tmap(&maps.b_hi[i]);
      kq::prefetch_tmap(&maps.b_lo[i]);
      kq::prefetch_tmap(&maps.c[i]);
    }
  }
  if (warp == EPI_WARP0) kq::tmem_alloc(&bars->tmem_base, TMEM_COLS);
  kq::tc_fence_before();
  __syncthreads();
  kq::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < P.total_tiles && ok; t += gridDim.x) {
        const Tile tl = tile_of<KC>(P, t);
        for (int kc = 0; kc < tl.kchunks; ++kc, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!kq::mbar_wait(&bars->empty[s], ph ^ 1u, abort, info)) { ok = false; break; }
          uint8_t* st = stages + s * STAGE_BYTES;
          kq::mbar_arrive_expect_tx(&bars->full[s], 4 * CHUNK);
          const int x = kc * KC, ya = tl.tm * TM, yb = tl.tn * TN;
          kq::tma_load_2d(st, &maps.a_hi[tl.prob], &bars->full[s], x, ya);
          kq::tma_load_2d(st + CHUNK, &maps.a_lo[tl.prob], &bars->full[s], x, ya);
          kq::tma_load_2d(st + 2 * CHUNK, &maps.b_hi[tl.prob], &bars->full[s], x, yb);
          kq::tma_load_2d(st + 3 * CHUNK, &maps.b_lo[tl.prob], &bars->full[s], x, yb);
        }
      }
      // wait for the copies still in flight before the CTA can exit
      for (int s = 0; s < STAGES; ++s) {
        const int armed = (it > s) ? (it - s + STAGES - 1) / STAGES : 0;
        if (armed > 0) kq::tf32x3::drain_wait(&bars->full[s], (uint32_t)(armed - 1) & 1u, info);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      int it = 0, tcount = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < P.total_tiles && ok; t += gridDim.x, ++tcount) {
        const Tile tl = tile_of<KC>(P, t);
        const int buf = tcount & 1;
        const uint32_t aph = (uint32_t)(tcount >> 1) & 1u;
        if (!kq::mbar_wait(&bars->tempty[buf], aph ^ 1u, abort, info)) break;
        kq::tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(buf * TN);
        for (int kc = 0; kc < tl.kchunks; ++kc, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!kq::mbar_wait(&bars->full[s], ph, abort, info)) { ok = false; break; }
          kq::tc_fence_after();
          const uint32_t a = kq::smem_u32(stages + s * STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {     // four 32-byte K steps per 128-byte row
            if (KIND == 1)
              kq::tf32x3::mma3_16(d_tmem, a, a + CHUNK, a + 2 * CHUNK, a + 3 * CHUNK, kk,
                                  (kc == 0 && kk == 0) ? 0u : 1u, kq::tf32x3::kIdescBf16_128);
            else if (KIND == 2)
              kq::tf32x3::mma3_16(d_tmem, a, a + CHUNK, a + 2 * CHUNK, a + 3 * CHUNK, kk,
                                  (kc == 0 && kk == 0) ? 0u : 1u, kq::tf32x3::kIdescFp16_128);
            else
              kq::tf32x3::mma3(d_tmem, a, a + CHUNK, a + 2 * CHUNK, a + 3 * CHUNK, kk,
                               (kc == 0 && kk == 0) ? 0u : 1u);
          }
          kq::mma_commit(&bars->empty[s]);
        }
        if (ok) kq::mma_commit(&bars->tfull[buf]);
      }
      kq::mma_commit(&bars->drain);
      kq::tf32x3::drain_wait(&bars->drain, 0, info);
    }
  } else {
    // ------------------------------------------------------ epilogue: C += alpha acc
    // warp w: TMEM lane quadrant w % 4 (tile rows; a warp may only read its
    // own quadrant), columns [64 h, 64 h + 64) as two 32 x 32 boxes.  Each box
    // is scaled, written to the warp's staging buffer in the 128-byte-swizzled
    // layout and added to C by a TMA reduce (the L2 does the read-modify-write).
    const int q = warp & 3, h = (warp - EPI_WARP0) >> 2;
    uint8_t* stg = staging + (warp - EPI_WARP0) * STG_BYTES;
    int tcount = 0;
    bool pending = false;
    for (int t = blockIdx.x; t < P.total_tiles; t += gridDim.x, ++tcount) {
      const Tile tl = tile_of<KC>(P, t);
      const Problem& pr = P.p[tl.prob];
      const int buf = tcount & 1;
      const uint32_t aph = (uint32_t)(tcount >> 1) & 1u;
      const int rt = q * 32 + lane;                   // row inside the tile
      if (!kq::mbar_wait(&bars->tfull[buf], aph, abort, info)) break;
      kq::tc_fence_after();
      float v[2][32];
      __syncwarp();
      const uint32_t ta = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * TN + 64 * h);
      kq::tmem_ld32(ta, v[0]);
      kq::tmem_ld32(ta + 32, v[1]);
      kq::tmem_wait_ld();
      kq::tc_fence_before();
      __syncwarp();
      if (lane == 0) kq::mbar_arrive(&bars->tempty[buf]);
      // the row's factor (fp16 planes), else alpha alone
      const int grow = tl.tm * TM + rt;
      const float al = (KIND == 2 && grow < pr.M) ? pr.alpha * pr.a_scale[grow] : pr.alpha;
      const bool diag = pr.lower && tl.tm == tl.tn;
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        const int ct = 64 * h + 32 * c2;              // first column inside the tile
        if (pending) {
          if (lane == 0) bulk_wait_read();            // staging free again
          __syncwarp();
        }
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          float4 o;
          o.x = al * v[c2][4 * ch];
          o.y = al * v[c2][4 * ch + 1];
          o.z = al * v[c2][4 * ch + 2];
          o.w = al * v[c2][4 * ch + 3];
          if (KIND == 2) {
            // the columns' factors (B rows); beyond N the box is clipped anyway
            const int gc = tl.tn * TN + ct + 4 * ch;
            o.x *= gc < pr.N ? pr.b_scale[gc] : 0.f;
            o.y *= gc + 1 < pr.N ? pr.b_scale[gc + 1] : 0.f;
            o.z *= gc + 2 < pr.N ? pr.b_scale[gc + 2] : 0.f;
            o.w *= gc + 3 < pr.N ? pr.b_scale[gc + 3] : 0.f;
          }
          if (diag) {                                 // keep the strict upper triangle untouched
            const int c = ct + 4 * ch;
            if (c > rt) o.x = 0.f;
            if (c + 1 > rt) o.y = 0.f;
            if (c + 2 > rt) o.z = 0.f;
            if (c + 3 > rt) o.w = 0.f;
          }
          *reinterpret_cast<float4*>(stg + lane * 128 + ((ch ^ (lane & 7)) << 4)) = o;
        }
        kq::tf32x3::fence_to_tensor_core();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_2d(&maps.c[tl.prob], stg, tl.tn * TN + ct, tl.tm * TM + q * 32);
          bulk_commit();
        }
        pending = true;
      }
    }
    if (lane == 0) bulk_wait_all();                   // the reduces have landed in C
    __syncwarp();
  }

  kq::tc_fence_before();
  __syncthreads();
  if (warp == EPI_WARP0) {
    kq::tc_fence_after();
    kq::tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

int kq_gemm_nt_tc(const kq::GemmNT* probs, int count, int32_t* info, cudaStream_t st,
                  int max_ctas) {
  if (count < 1 || count > 2) return KRONQ_ERR_INVALID_ARG;
  Maps maps;
  Problems P;
  P.count = 0;
  P.total_tiles = 0;
  const int bf16 = probs[0].bf16, fp16 = probs[0].fp16;
  const int kind = fp16 ? 2 : (bf16 ? 1 : 0);
  const int KC = kind ? 64 : 32;
  const int64_t lda_align = kind ? 8 : 4;          // 16-byte rows
  for (int i = 0; i < count; ++i) {
    const kq::GemmNT& g = probs[i];
    if (g.M <= 0 || g.N <= 0 || g.K <= 0) continue;
    if (g.bf16 != bf16 || g.fp16 != fp16 || (bf16 && fp16)) return KRONQ_ERR_INVALID_ARG;
    if (fp16 && (!g.a_scale || !g.b_scale)) return KRONQ_ERR_INVALID_ARG;
    if (!g.A_hi || !g.A_lo || !g.B_hi || !g.B_lo || !g.C || g.lda % lda_align ||
        g.ldb % lda_align || g.ldc % 4 || !kqh::aligned(g.A_hi, 16) ||
        !kqh::aligned(g.A_lo, 16) || !kqh::aligned(g.B_hi, 16) || !kqh::aligned(g.B_lo, 16) ||
        !kqh::aligned(g.C, 16))
      return KRONQ_ERR_INVALID_ARG;
    if (g.lower && g.M != g.N) return KRONQ_ERR_INVALID_ARG;
    const int j = P.count;
    bool ok;
    if (kind)
      ok = kqh::make_map_bf16(&maps.a_hi[j], g.A_hi, g.K, g.M, g.lda, KC, TM, fp16) &&
           kqh::make_map_bf16(&maps.a_lo[j], g.A_lo, g.K, g.M, g.lda, KC, TM, fp16) &&
           kqh::make_map_bf16(&maps.b_hi[j], g.B_hi, g.K, g.N, g.ldb, KC, TN, fp16) &&
           kqh::make_map_bf16(&maps.b_lo[j], g.B_lo, g.K, g.N, g.ldb, KC, TN, fp16);
    else
      ok = kqh::make_map_f32(&maps.a_hi[j], static_cast<const float*>(g.A_hi), g.K, g.M, g.lda, KC, TM) &&
           kqh::make_map_f32(&maps.a_lo[j], static_cast<const float*>(g.A_lo), g.K, g.M, g.lda, KC, TM) &&
           kqh::make_map_f32(&maps.b_hi[j], static_cast<const float*>(g.B_hi), g.K, g.N, g.ldb, KC, TN) &&
           kqh::make_map_f32(&maps.b_lo[j], static_cast<const float*>(g.B_lo), g.K, g.N, g.ldb, KC, TN);
    if (!ok || !kqh::make_map_f32(&maps.c[j], g.C, g.N, g.M, g.ldc, 32, 32)) return KRONQ_ERR_CUDA;
    Problem& q = P.p[j];
    q.C = g.C;
    q.a_scale = g.a_scale;
    q.b_scale = g.b_scale;
    q.ldc = g.ldc;
    q.M = g.M;
    q.N = g.N;
    q.K = g.K;
    q.alpha = g.alpha;
    q.lower = g.lower;
    const int ntm = (g.M + TM - 1) / TM;
    q.ntn = (g.N + TN - 1) / TN;
    const int all = g.lower ? ntm * (ntm + 1) / 2 : ntm * q.ntn;
    const int tb = g.tile_begin < 0 ? 0 : (g.tile_begin > all ? all : g.tile_begin);
    const int te = (g.tile_end < 0 || g.tile_end > all) ? all : g.tile_end;
    if (te <= tb) continue;
    q.t0 = tb;
    q.tiles = te - tb;
    P.total_tiles += q.tiles;
    ++P.count;
  }
  if (P.count == 0) return KRONQ_OK;
  if (P.count == 1) P.p[1] = P.p[0];
  static kqh::PerDevice attr[3];
  const int a_ok = kind == 2   ? kqh::smem_attr_once(attr[2], gemm_nt_tc_kernel<2>, SMEM_BYTES)
                   : kind == 1 ? kqh::smem_attr_once(attr[1], gemm_nt_tc_kernel<1>, SMEM_BYTES)
                               : kqh::smem_attr_once(attr[0], gemm_nt_tc_kernel<0>, SMEM_BYTES);
  if (a_ok <= 0) return KRONQ_ERR_CUDA;
  int grid = P.total_tiles < kqh::num_sms() ? P.total_tiles : kqh::num_sms();
  if (max_ctas > 0 && grid > max_ctas) grid = max_ctas;
  if (kind == 2)
    gemm_nt_tc_kernel<2><<<grid, THREADS, SMEM_BYTES, st>>>(maps, P, info);
  else if (kind == 1)
    gemm_nt_tc_kernel<1><<<grid, THREADS, SMEM_BYTES, st>>>(maps, P, info);
  else
    gemm_nt_tc_kernel<0><<<grid, THREADS, SMEM_BYTES, st>>>(maps, P, info);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}
