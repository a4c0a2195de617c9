// Damping and the inverse Cholesky factor U_c (H_d^-1 = U_c^T U_c, U_c upper).
//
// KronQ review (pith.science), appendix, Algorithm 2, steps 1-2:
// H_X <- H_X + lambda mean(diag H_X) I, then the inverse Cholesky factor.
//
// Route (fp32 throughout): with J the index reversal, R = J H_d J = L L^T
// (lower Cholesky) and U_c = J L^-1 J; then U_c^T U_c = J (L L^T)^-1 J =
// H_d^-1 and U_c is upper triangular.
//
// The matrix is padded with the identity to np = a multiple of 128 (which
// leaves the leading blocks of L and L^-1 unchanged).  One right-looking
// sweep over 128-wide panels computes L and Z = L^-T together (block
// forward substitution of L Y = I carried along with the factorisation,
// stored transposed so that every product has both operands K-major).
// Step p (rows k = 128 p ...):
//   panel kernel   every CTA factors the 128 x 128 diagonal block
//                  R_pp = L_pp L_pp^T and inverts L_pp in shared memory, then
//                  either turns 128 rows of the panel into L_ip = R_ip L_pp^-T,
//                  or finishes 128 rows of block column p of Z:
//                  Z_jp = B_jp L_pp^-T (B_jp = -sum_{q<p} Z_jq L_pq^T), Z_pp = L_pp^-T.
//   update         one tensor-core launch (tf32, three-term split) for
//                  R[k+128:, k+128:] -= L L^T (lower triangle) and
//                  Z[:k+128, k+128:] -= Z[:k+128, k:k+128] L^T, L = the panel rows.
// Then U_c[a][b] = Z[n-1-b][n-1-a] (a <= b).
#include <cuda_fp16.h>

#include "common.cuh"
#include "gemm_tc.cuh"
#include "tf32x3.cuh"

namespace {

constexpr int NB = 128;
constexpr int LDD = NB + 1;   // D: odd row stride, column reads are conflict-free
constexpr int LDX = NB + 4;   // X and the panel tile P: 16-byte rows for float4 reads
constexpr int LDA = 100;      // As: K-major copy of the 32 columns just factored (<= 96 rows)
constexpr int LDY = 36;       // YT: the 32 x 32 inverse block, transposed
// shared memory of the panel kernel, in floats
constexpr int SM_D = 0;
constexpr int SM_X = SM_D + NB * LDD;
constexpr int SM_P = SM_X + NB * LDX;
constexpr int SM_AS = SM_P + 32 * LDX;
constexpr int SM_YT = SM_AS + 32 * LDA;
constexpr int SM_LB = SM_YT + 32 * LDY;       // the leaf's exchange buffers (6 x 32)
constexpr int SM_P2 = SM_LB + 192;            // second slice buffer (double buffering)
constexpr int SM_FLOATS = SM_P2 + 32 * LDX;
static_assert(SM_LB % 4 == 0, "leaf buffers must allow 16-byte loads");

__global__ void __launch_bounds__(1024) diag_sum_kernel(const float* __restrict__ H, int n,
                                                        double* out) {
  __shared__ double red[1024];
  double s = 0.0;
#pragma unroll 4
  for (int i = threadIdx.x; i < n; i += blockDim.x) s += (double)H[(int64_t)i * n + i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = red[0];
}

// R[a][b] = H[n-1-a][n-1-b] + delta [a == b] for a, b < n, the identity on
// the padding up to np (a multiple of 128), delta = damp_rel * mean(diag H);
// Z = 0.  Padding with the identity leaves the leading n x n blocks of the
// factor and of its inverse unchanged.
__global__ void reverse_damp_kernel(const float* __restrict__ H, int n, int np,
                                    float* __restrict__ R, float* __restrict__ Z, float damp_rel,
                                    const double* __restrict__ diag_sum) {
  const float delta = (float)((double)damp_rel * (*diag_sum / (double)n));
  // one row of R (and Z) per CTA iteration, its columns across the threads
  for (int a = blockIdx.x; a < np; a += gridDim.x) {
    float* Ra = R + (int64_t)a * np;
    float* Za = Z + (int64_t)a * np;
    const float* Hr = H + (int64_t)(n - 1 - a) * n + (n - 1);   // H[n-1-a][n-1-b] = Hr[-b]
    for (int b = threadIdx.x; b < np; b += blockDim.x) {
      float v;
      if (a < n && b < n) {
        v = Hr[-b];
        if (a == b) v += delta;
      } else {
        v = (a == b) ? 1.f : 0.f;
      }
      Ra[b] = v;
      Za[b] = 0.f;
    }
  }
}

// Two warps factor the 32 x 32 diagonal block at offset o of D (lower part
// valid, already updated) and invert the factor: on return D holds L_oo,
// X holds Y_oo = L_oo^-1 and YT its transpose.  Pivot step j:
//   L[i][j] = a_i[j] r,  r = 1 / sqrt(a_j[j]),   a_i[c] -= L[i][j] L[c][j]  (c > j)
//   Y[j][:] = y_j[:] r,  y_i[:] -= L[i][j] Y[j][:]                          (i > j)
// Warp 0 does the factorisation: lane i keeps row i of the block in
// registers, shifted so that slot 0 is the current pivot column (slot c =
// column j + c), stores L[i][j] into D and r into lb as it goes, and passes
// the column L[j+1:, j] to its own lanes through lb.  Warp 1 carries the
// inverse one pivot behind: lane i keeps row i of Y; the finished row Y[j][:]
// travels through lb.  Warp 0 arrives on barrier FULL[j&1] after pivot j's
// stores; warp 1 syncs on it, and arrives on EMPTY[j&1] when it is done with
// pivot j, which warp 0 syncs on before pivot j+2 (so lb's double buffers and
// the barriers are never reused early; every arrive has its sync).  The
// pivot loop is not unrolled: the whole leaf is a few hundred instructions,
// so its first pass does not stall on instruction fetch after the update
// kernels ran.  The arithmetic (and its order) is that of the plain update.
// lb: 192 floats, 16-byte aligned (colb 2 x 32 | rowb 2 x 32 | r 32).
// Named barriers 1..4; called by the CTA's warps 0 and 1 together.
KQ_DEV void named_sync64(int id) { asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory"); }
KQ_DEV void named_arrive64(int id) { asm volatile("bar.arrive %0, 64;" ::"r"(id) : "memory"); }

__device__ __forceinline__ void leaf32(float* D, float* X, float* YT, int o, int kb, int* bad,
                                       float* lb) {
  const int i = threadIdx.x & 31, w = threadIdx.x >> 5;
  constexpr unsigned FULL = 0xffffffffu;
  float* rj = lb + 128;
  if (w == 0) {
    float a[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) a[c] = (c <= i) ? D[(o + i) * LDD + o + c] : 0.f;
    *reinterpret_cast<float2*>(lb + 2 * i) = make_float2(0.f, 0.f);
    __syncwarp();
#pragma unroll 1
    for (int j = 0; j < 32; ++j) {
      float* colb = lb + (j & 1) * 32;           // colb[c] = L[j+1+c][j]
      float d = __shfl_sync(FULL, a[0], j);
      if (!(d > 0.f) || !isfinite(d)) {
        if (i == 0 && o + j < kb) *bad = 1;
        d = 1.f;
      }
      const float r = rsqrtf(d);
      const float l = (i >= j) ? a[0] * r : 0.f;
      if (j >= 2) named_sync64(3 + (j & 1));     // warp 1 is done with pivot j - 2
      if (i >= j) D[(o + i) * LDD + o + j] = l;
      if (i > j) colb[i - j - 1] = l;
      if (i == j) rj[j] = r;
      __syncwarp();
      named_arrive64(1 + (j & 1));
      // a_i[j+1+c] -= L[i][j] L[j+1+c][j], shifted down one slot; the slots
      // past the row's last column hold values that are never used
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 v = *reinterpret_cast<const float4*>(colb + 4 * q);
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = 4 * q + u;
          if (c < 31) a[c] = fmaf(-l, vv[u], a[c + 1]);
        }
      }
      a[31] = 0.f;
    }
  } else {
    float y[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) y[c] = (c == i) ? 1.f : 0.f;
#pragma unroll 1
    for (int j = 0; j < 32; ++j) {
      float* rowb = lb + 64 + (j & 1) * 32;      // Y[j][:]
      named_sync64(1 + (j & 1));
      const float r = rj[j];
      const float l = (i >= j) ? D[(o + i) * LDD + o + j] : 0.f;
      if (i == j) {
        // y_j[c] = 0 for c > j, so scaling the whole row changes nothing there
#pragma unroll
        for (int c = 0; c < 32; ++c) y[c] = y[c] * r;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<float4*>(rowb + 4 * q) =
              make_float4(y[4 * q], y[4 * q + 1], y[4 * q + 2], y[4 * q + 3]);
      }
      __syncwarp();
      if (i != j) {
        // rowb[c] = 0 for c > j: those updates leave y (+0) as it is
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 v = *reinterpret_cast<const float4*>(rowb + 4 * q);
          y[4 * q + 0] = fmaf(-l, v.x, y[4 * q + 0]);
          y[4 * q + 1] = fmaf(-l, v.y, y[4 * q + 1]);
          y[4 * q + 2] = fmaf(-l, v.z, y[4 * q + 2]);
          y[4 * q + 3] = fmaf(-l, v.w, y[4 * q + 3]);
        }
      }
      if (j + 2 < 32) named_arrive64(3 + (j & 1));
    }
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      if (c <= i) X[(o + i) * LDX + o + c] = y[c];
      YT[c * LDY + i] = (c <= i) ? y[c] : 0.f;   // YT[c][i] = Y[i][c]
    }
  }
}

// X = L^-1 for the lower Cholesky factor L of the 128 x 128 block in D
// (fp32; rows / columns kb .. NB-1 padded with the identity by the caller).
// On return D's lower triangle holds L and X (zero above the diagonal)
// holds L^-1.  PANEL_THREADS (256) threads.
//
// Right-looking over four 32-wide blocks b (o = 32 b), carrying L^-1 along
// (block forward substitution of L Y = I, accumulators in X below the
// diagonal blocks):
//   1. warps 0-1: L_bb and Y_bb = L_bb^-1                       (leaf32)
//   2. L_cb = D_cb Y_bb^T (c > b), also kept K-major in As;  Y_bj = Y_bb Acc_bj (j < b)
//      (together one 96 x 32 x 32 product whose B operand is Y_bb^T)
//   3a. the next block column: D_{c,b+1} -= L_cb L_{b+1,b}^T
//   3b. the rest: D_cd -= L_cb L_db^T (d > b+1);  Acc_cj -= L_cb Y_bj (j <= b)
// with warps 0-1 factoring block b+1 (step 1 of the next round) while four other
// warps do 3b.  Steps 2 and 3 are small register-tiled GEMMs out of shared
// memory (3 x 4 outputs per thread in steps 2 and 3a) whose wide operands are
// read as contiguous rows (YT, As, rows of X).
constexpr int PANEL_THREADS = 256;

__device__ void factor_and_invert(float* D, float* X, float* As, float* YT, float* LB, int kb,
                                  int* bad) {
  const int tid = threadIdx.x;
  static_assert((NB * LDX) % 4 == 0 && SM_X % 4 == 0, "X is cleared in 16-byte stores");
  for (int e = 4 * tid; e < NB * LDX; e += 4 * blockDim.x)
    *reinterpret_cast<float4*>(X + e) = make_float4(0.f, 0.f, 0.f, 0.f);
  __syncthreads();
  if (tid < 64) leaf32(D, X, YT, 0, kb, bad, LB);
  __syncthreads();
  for (int b = 0; b < NB / 32; ++b) {
    const int o = 32 * b;
    const int o2 = o + 32;
    const int R1 = NB - o2;                 // rows below the diagonal block
    // ---- step 2, one 96 x 32 x 32 product through YT (B[t][q] = Y_bb[q][t]):
    //   rows m < R1:  L_cb[m][q]  = sum_t D[o2+m][o+t] Y_bb[q][t]   -> D, As
    //   rows m >= R1: Y_bj[q][c'] = sum_t Acc[o+t][c'] Y_bb[q][t],  c' = m - R1 -> X
    // thread (g, cg): rows g + 32 k (k < 3), columns 4 cg .. 4 cg + 3; each
    // 32-row block lies on one side of R1 (a multiple of 32)
    {
      const int cg = tid & 7, g = tid >> 3;
      float acc[3][4];
#pragma unroll
      for (int k = 0; k < 3; ++k)
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[k][u] = 0.f;
#pragma unroll 4
      for (int t = 0; t < 32; ++t) {
        const float4 bv = *reinterpret_cast<const float4*>(&YT[t * LDY + 4 * cg]);
#pragma unroll
        for (int k = 0; k < 3; ++k) {
          const int m = g + 32 * k;
          const float av = (32 * k < R1) ? D[(o2 + m) * LDD + o + t] : X[(o + t) * LDX + m - R1];
          acc[k][0] = fmaf(av, bv.x, acc[k][0]);
          acc[k][1] = fmaf(av, bv.y, acc[k][1]);
          acc[k][2] = fmaf(av, bv.z, acc[k][2]);
          acc[k][3] = fmaf(av, bv.w, acc[k][3]);
        }
      }
      __syncthreads();
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        const int m = g + 32 * k;
        if (32 * k < R1) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            D[(o2 + m) * LDD + o + 4 * cg + u] = acc[k][u];
            As[(4 * cg + u) * LDA + m] = acc[k][u];
          }
        } else {
#pragma unroll
          for (int u = 0; u < 4; ++u) X[(o + 4 * cg + u) * LDX + m - R1] = acc[k][u];
        }
      }
      __syncthreads();
    }
    if (R1 == 0) break;
    // ---- step 3a: D[o2+m][o2+n] -= sum_t L[o2+m][o+t] L[o2+n][o+t] (n < 32, m >= n),
    // both operands from the K-major copy As; thread (g, cg) as in step 2
    {
      const int cg = tid & 7, g = tid >> 3;
      float acc[3][4];
#pragma unroll
      for (int k = 0; k < 3; ++k)
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[k][u] = 0.f;
#pragma unroll 4
      for (int t = 0; t < 32; ++t) {
        const float4 bv = *reinterpret_cast<const float4*>(&As[t * LDA + 4 * cg]);
#pragma unroll
        for (int k = 0; k < 3; ++k) {
          if (32 * k < R1) {
            const float av = As[t * LDA + g + 32 * k];
            acc[k][0] = fmaf(av, bv.x, acc[k][0]);
            acc[k][1] = fmaf(av, bv.y, acc[k][1]);
            acc[k][2] = fmaf(av, bv.z, acc[k][2]);
            acc[k][3] = fmaf(av, bv.w, acc[k][3]);
          }
        }
      }
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        const int m = g + 32 * k;
        if (32 * k < R1) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (4 * cg + u <= m) D[(o2 + m) * LDD + o2 + 4 * cg + u] -= acc[k][u];
        }
      }
    }
    __syncthreads();
    // ---- step 3b on warps 2, 3, 6, 7, the next diagonal block on warps 0-1
    if (tid < 64) {
      leaf32(D, X, YT, o2, kb, bad, LB);
    } else if (((tid >> 5) & 3) >= 2) {
      // warps 2, 3, 6, 7: the leaf's warps share no scheduler with them
      // item = 4 rows x 8 columns; 12 column groups: 8 g < o2 (Acc), else past the next block
      const int items = (R1 / 4) * 12;
      for (int it = (tid >> 5) < 4 ? tid - 64 : tid - 128; it < items; it += 128) {
        const int rg = it / 12, g = it % 12;
        const int c0 = (8 * g < o2) ? 8 * g : 8 * g + 32;
        const bool left = c0 < o2;
        const float* Bp = left ? &X[o * LDX + c0] : &As[c0 - o2];
        const int ldb = left ? LDX : LDA;
        float acc[4][8];
#pragma unroll
        for (int s = 0; s < 4; ++s)
#pragma unroll
          for (int q = 0; q < 8; ++q) acc[s][q] = 0.f;
#pragma unroll 2
        for (int t = 0; t < 32; ++t) {
          const float4 b0 = *reinterpret_cast<const float4*>(Bp + t * ldb);
          const float4 b1 = *reinterpret_cast<const float4*>(Bp + t * ldb + 4);
          const float4 a4 = *reinterpret_cast<const float4*>(&As[t * LDA + 4 * rg]);
          const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
          const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
          for (int s = 0; s < 4; ++s)
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[s][q] = fmaf(av[s], bv[q], acc[s][q]);
        }
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const int r = o2 + 4 * rg + s;
          if (left) {
#pragma unroll
            for (int q = 0; q < 8; ++q) X[r * LDX + c0 + q] -= acc[s][q];
          } else {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              if (c0 + q <= r) D[r * LDD + c0 + q] -= acc[s][q];
          }
        }
      }
    }
    __syncthreads();
  }
}

KQ_DEV void bulk_copy_row(float* dst, const float* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          kq::smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(kq::smem_u32(bar))
      : "memory");
}

// Write v to a row of fp32 and to its tf32 hi / lo planes.
KQ_DEV void put_split(float* hi_plane, float* lo_plane, int64_t idx, float v) {
  const float h = kq::tf32x3::hi(v);
  hi_plane[idx] = h;
  lo_plane[idx] = v - h;
}

// Panel step p (rows / columns k = 128 p ...) of the padded np x np matrices,
// in 32-row slices ("tiles", PR rows each):
//   tile t < tiles_L:          L_ip = R_ip L_pp^-T for rows k+128+32t ..
//                              -> the hi / lo planes Lh, Ll
//   tile tiles_L + j, j < 4p:  Z_jp = B_jp L_pp^-T for Z rows 32j .. -> Z and the
//                              planes Zh, Zl
//   tile tiles_L + 4p (last):  Z_pp = L_pp^-T      -> Z and the planes
// The planes are np x ldp, indexed by matrix row; the panel's 128 columns go
// to plane columns pc .. pc + 127 (its place in the current super-block).
// At most one CTA per SM: each factors and inverts the diagonal block once in
// shared memory, then takes tiles t = blockIdx.x, + gridDim.x, ... (the
// first slice is fetched by bulk copies during the factorisation, each
// following one while the previous is multiplied: two slice buffers).
constexpr int PR = 32;

__global__ void __launch_bounds__(PANEL_THREADS, 1) panel_kernel(const float* R, float* Z, float* Lh,
                                                    float* Ll, float* Zh, float* Zl, int np, int k,
                                                    int p, int tiles_L, int tiles_total, int ldp,
                                                    int pc, int32_t* info) {
  extern __shared__ __align__(16) float sm[];
  float* D = sm + SM_D;
  float* X = sm + SM_X;
  float* As = sm + SM_AS;
  float* YT = sm + SM_YT;
  float* LB = sm + SM_LB;
  float* Pbuf[2] = {sm + SM_P, sm + SM_P2};
  __shared__ int bad;
  __shared__ int abort_flag;
  __shared__ __align__(8) uint64_t pbar[2];
  const int tid = threadIdx.x;
  const int z_pp = tiles_L + 4 * p;   // the tile without a slice to fetch (the last one)
  auto slice_src = [&](int t) -> const float* {
    return t < tiles_L ? R + (int64_t)(k + NB + PR * t) * np + k
                       : Z + (int64_t)(PR * (t - tiles_L)) * np + k;
  };
  auto fetch = [&](int t, int b) {
    const float* src = slice_src(t);
    kq::mbar_arrive_expect_tx(&pbar[b], PR * NB * 4);
    for (int r = 0; r < PR; ++r) bulk_copy_row(Pbuf[b] + r * LDX, src + (int64_t)r * np, NB * 4, &pbar[b]);
  };
  if (tid == 0) {
    bad = 0;
    abort_flag = 0;
    kq::mbar_init(&pbar[0], 1);
    kq::mbar_init(&pbar[1], 1);
    kq::fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0 && (int)blockIdx.x < z_pp) fetch(blockIdx.x, 0);
  // the diagonal block, lower triangle: 16-byte loads, all requested before
  // any is stored (one CTA per SM leaves few warps to hide the latency);
  // the chunks wholly above the diagonal are not read
  static_assert(NB * NB / 4 == 16 * PANEL_THREADS, "diagonal block load assumes 256 threads");
  {
    float4 v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int e4 = tid + PANEL_THREADS * u;
      const int i = e4 >> 5, c = (e4 & 31) * 4;
      v[u] = (c <= i) ? *reinterpret_cast<const float4*>(R + (int64_t)(k + i) * np + k + c)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int e4 = tid + PANEL_THREADS * u;
      const int i = e4 >> 5, c = (e4 & 31) * 4;
      float* d = D + i * LDD + c;
      d[0] = (c <= i) ? v[u].x : 0.f;
      d[1] = (c + 1 <= i) ? v[u].y : 0.f;
      d[2] = (c + 2 <= i) ? v[u].z : 0.f;
      d[3] = (c + 3 <= i) ? v[u].w : 0.f;
    }
  }
  __syncthreads();
  factor_and_invert(D, X, As, YT, LB, NB, &bad);
  if (blockIdx.x == 0 && tid == 0 && bad) kq::record_error(info, KRONQ_ERR_NOT_PD);

  const int ty = tid >> 4, tx = tid & 15;
  int n_it = 0;
  for (int t = blockIdx.x; t < tiles_total; t += gridDim.x, ++n_it) {
    const int b = n_it & 1;
    const uint32_t ph = (uint32_t)(n_it >> 1) & 1u;
    const int tn = t + gridDim.x;
    // the next slice into the other buffer (its last reader finished at the
    // barrier that ended the previous iteration)
    if (tid == 0 && tn < z_pp) fetch(tn, b ^ 1);
    if (t == z_pp) {
      // Z_pp = X^T (upper; X is zero above its diagonal)
      for (int e = tid; e < NB * NB; e += blockDim.x) {
        const int a = e / NB, c = e % NB;
        const float v = X[c * LDX + a];
        Z[(int64_t)(k + a) * np + k + c] = v;
        put_split(Zh, Zl, (int64_t)(k + a) * ldp + pc + c, v);
      }
      break;                          // the last tile
    }
    if (!kq::mbar_wait(&pbar[b], ph, &abort_flag, info)) {
      // give the copies in flight a bounded time to land before the CTA exits
      kq::tf32x3::drain_wait(&pbar[b], ph, info);
      if (tn < z_pp) kq::tf32x3::drain_wait(&pbar[b ^ 1], (uint32_t)((n_it + 1) >> 1) & 1u, info);
      return;
    }
    const float* P = Pbuf[b];
    // C = P X^T (32 x 128): thread (ty, tx) owns rows ty, ty + 16 and columns tx + 16 jj
    float acc[2][8];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) acc[i][jj] = 0.f;
#pragma unroll 4
    for (int kk = 0; kk < NB; kk += 4) {
      float4 pa[2], xb[8];
#pragma unroll
      for (int i = 0; i < 2; ++i) pa[i] = *reinterpret_cast<const float4*>(&P[(ty + 16 * i) * LDX + kk]);
#pragma unroll
      for (int jj = 0; jj < 8; ++jj)
        xb[jj] = *reinterpret_cast<const float4*>(&X[(tx + 16 * jj) * LDX + kk]);
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          acc[i][jj] = fmaf(pa[i].x, xb[jj].x, acc[i][jj]);
          acc[i][jj] = fmaf(pa[i].y, xb[jj].y, acc[i][jj]);
          acc[i][jj] = fmaf(pa[i].z, xb[jj].z, acc[i][jj]);
          acc[i][jj] = fmaf(pa[i].w, xb[jj].w, acc[i][jj]);
        }
    }
    if (t < tiles_L) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int64_t r = (int64_t)k + NB + PR * t + ty + 16 * i;   // matrix row
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) put_split(Lh, Ll, r * ldp + pc + tx + 16 * jj, acc[i][jj]);
      }
    } else {
      const int j = t - tiles_L;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int64_t r = (int64_t)PR * j + ty + 16 * i;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int c = tx + 16 * jj;
          Z[r * np + k + c] = acc[i][jj];
          put_split(Zh, Zl, r * ldp + pc + c, acc[i][jj]);
        }
      }
    }
    __syncthreads();                  // P[b] is read; it may be refilled two tiles on
  }
}

// U[a][b] = Z[n-1-b][n-1-a] for a <= b, 0 below the diagonal (Z has leading
// dimension np): an anti-transpose through 32 x 32 shared-memory tiles,
// coalesced on both sides.
__global__ void __launch_bounds__(256) reverse_out_kernel(const float* __restrict__ Z, int n,
                                                          int np, float* __restrict__ U) {
  __shared__ float tile[32][33];
  const int ta = blockIdx.y * 32, tb = blockIdx.x * 32;     // U tile origin (rows a, cols b)
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 8 rows per pass
  for (int r = ty; r < 32; r += 8) {
    const int b = tb + r, a = ta + 31 - tx;                 // Z row n-1-b, column n-1-a
    float v = 0.f;
    if (b < n && a < n) v = Z[(int64_t)(n - 1 - b) * np + (n - 1 - a)];
    tile[r][31 - tx] = v;                                   // tile[b - tb][a - ta]
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int a = ta + r, b = tb + tx;
    if (a < n && b < n) U[(int64_t)a * n + b] = (a <= b) ? tile[tx][r] : 0.f;
  }
}

// Rows of the fp32 values held as tf32 hi / lo planes (x = hi + lo exactly;
// rows * K values from column 0, leading dimension ld) as fp16 hi / lo planes
// of x * 2^e_i with e_i chosen so that the row's largest |x| * 2^e_i lies in
// [2^13, 2^14): fp16 keeps 11 + 11 bits of every entry within 2^-17 of the
// row's largest, smaller ones lose only absolute precision far below that
// entry's contribution.  inv[i] = 2^-e_i (1 for an all-zero row).  One warp
// per row, K a multiple of 128 (up to 1024).
__global__ void __launch_bounds__(256) fp16_rows_kernel(const float* __restrict__ Sh,
                                                        const float* __restrict__ Sl, int rows,
                                                        int K, int ld, __half* __restrict__ Dh,
                                                        __half* __restrict__ Dl,
                                                        float* __restrict__ inv) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float* h = Sh + (int64_t)row * ld;
  const float* l = Sl + (int64_t)row * ld;
  float x[32];
  float mx = 0.f;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int c = 4 * lane + 128 * u;
    if (c < K) {
      const float4 a = *reinterpret_cast<const float4*>(h + c);
      const float4 b = *reinterpret_cast<const float4*>(l + c);
      x[4 * u] = a.x + b.x;
      x[4 * u + 1] = a.y + b.y;
      x[4 * u + 2] = a.z + b.z;
      x[4 * u + 3] = a.w + b.w;
    } else {
      x[4 * u] = x[4 * u + 1] = x[4 * u + 2] = x[4 * u + 3] = 0.f;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) mx = fmaxf(mx, fabsf(x[4 * u + q]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  int e2 = 0;
  if (mx > 0.f) {
    frexpf(mx, &e2);                     // mx = f 2^e2, f in [0.5, 1)
    e2 = 14 - e2;                        // mx 2^e2 in [2^13, 2^14)
  }
  if (lane == 0) inv[row] = ldexpf(1.f, -e2);
  __half* dh = Dh + (int64_t)row * ld;
  __half* dl = Dl + (int64_t)row * ld;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int c = 4 * lane + 128 * u;
    if (c < K) {
      __half hh[4], ll[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float v = ldexpf(x[4 * u + q], e2);
        hh[q] = __float2half_rn(v);
        ll[q] = __float2half_rn(v - __half2float(hh[q]));
      }
      *reinterpret_cast<uint2*>(dh + c) = *reinterpret_cast<const uint2*>(hh);
      *reinterpret_cast<uint2*>(dl + c) = *reinterpret_cast<const uint2*>(ll);
    }
  }
}

size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

constexpr size_t kPanelSmem = (size_t)SM_FLOATS * sizeof(float);

int64_t padded(int64_t n) { return (n + NB - 1) / NB * NB; }

}  // namespace

// Super-block width of the two-level sweep: its panels update only the
// super-block's own columns; the trailing matrix gets one K = SBW update.
constexpr int SBW = 1024;

int64_t plane_ld(int64_t np) { return np < SBW ? np : SBW; }

size_t kq_cholesky_ws(int64_t n) {
  const int64_t np = padded(n);
  return align256(sizeof(double)) + 2 * align256((size_t)np * np * sizeof(float)) +
         4 * align256((size_t)np * plane_ld(np) * sizeof(float)) +
         4 * align256((size_t)np * plane_ld(np) * sizeof(__half)) +
         2 * align256((size_t)np * sizeof(float));
}

int kq_cholesky_inv(const float* H, int64_t n64, float damp_rel, float* U, int32_t* info, void* ws,
                    size_t ws_bytes, cudaStream_t st) {
  if (n64 < 0 || !(damp_rel >= 0.f)) return KRONQ_ERR_INVALID_ARG;
  if (n64 == 0) return KRONQ_OK;
  if (!H || !U || H == U) return KRONQ_ERR_INVALID_ARG;
  if (n64 > 65536) return KRONQ_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < kq_cholesky_ws(n64) || !kqh::aligned(ws, 256)) return KRONQ_ERR_WORKSPACE;
  static kqh::PerDevice attr;
  if (kqh::smem_attr_once(attr, panel_kernel, (int)kPanelSmem) <= 0) return KRONQ_ERR_CUDA;
  const int n = (int)n64;
  const int np = (int)padded(n64);
  uint8_t* w = static_cast<uint8_t*>(ws);
  double* dsum = reinterpret_cast<double*>(w);
  w += align256(sizeof(double));
  float* R = reinterpret_cast<float*>(w);
  w += align256((size_t)np * np * sizeof(float));
  float* Z = reinterpret_cast<float*>(w);
  w += align256((size_t)np * np * sizeof(float));
  float* planes[4];
  const int ldp = (int)plane_ld(np);
  for (int i = 0; i < 4; ++i) {
    planes[i] = reinterpret_cast<float*>(w);
    w += align256((size_t)np * ldp * sizeof(float));
  }
  float *Lh = planes[0], *Ll = planes[1], *Zh = planes[2], *Zl = planes[3];
  // the outer updates' operands: fp16 planes of row-scaled L and Z, and the rows' factors
  __half* p16[4];
  for (int i = 0; i < 4; ++i) {
    p16[i] = reinterpret_cast<__half*>(w);
    w += align256((size_t)np * ldp * sizeof(__half));
  }
  float* sL = reinterpret_cast<float*>(w);
  w += align256((size_t)np * sizeof(float));
  float* sZ = reinterpret_cast<float*>(w);

  const int sms = kqh::num_sms();
  diag_sum_kernel<<<1, 1024, 0, st>>>(H, n, dsum);
  KQ_CHECK_LAUNCH();
  reverse_damp_kernel<<<4 * sms, 256, 0, st>>>(H, n, np, R, Z, damp_rel, dsum);
  KQ_CHECK_LAUNCH();
  for (int kb = 0; kb < np; kb += ldp) {
    const int kb_end = kb + ldp < np ? kb + ldp : np;
    // the Z planes of the super-block's columns are read down to row kb_end
    // by its trailing update: the rows below each panel's block are zero
    const size_t zrows = (size_t)(kb_end - kb) * ldp * sizeof(float);
    if (cudaMemsetAsync(Zh + (size_t)kb * ldp, 0, zrows, st) != cudaSuccess ||
        cudaMemsetAsync(Zl + (size_t)kb * ldp, 0, zrows, st) != cudaSuccess)
      return KRONQ_ERR_CUDA;
    for (int k = kb; k < kb_end; k += NB) {
      const int p = k / NB, pc = k - kb;
      const int below = np - k - NB;
      const int tiles_L = below / PR;
      const int tiles_total = tiles_L + 4 * p + 1;
      const int grid = tiles_total < sms ? tiles_total : sms;
      const int tp = kqh::timer_begin(KRONQ_TIMER_CHOL_PANEL, st);
      panel_kernel<<<grid, PANEL_THREADS, kPanelSmem, st>>>(R, Z, Lh, Ll, Zh, Zl, np, k, p,
                                                            tiles_L, tiles_total, ldp, pc, info);
      kqh::timer_end(tp, st);
      KQ_CHECK_LAUNCH();
      const int inner = kb_end - k - NB;      // the super-block's columns after this panel
      if (inner > 0) {
        // inside the super-block, on the tensor cores (B = the panel rows L_ip):
        //   R[k+128:, k+128:kb_end] -= L L[k+128:kb_end]^T   (every row below; the
        //                                                      part above the diagonal is unused)
        //   Z[:k+128, k+128:kb_end] -= Z[:k+128, k:k+128] L[k+128:kb_end]^T
        const int64_t lr = (int64_t)(k + NB) * ldp + pc;
        kq::GemmNT g[2];
        g[0] = {Lh + lr, Ll + lr, ldp, Lh + lr, Ll + lr, ldp, R + (int64_t)(k + NB) * np + (k + NB),
                np, below, inner, NB, -1.f, 0};
        g[1] = {Zh + pc, Zl + pc, ldp, Lh + lr, Ll + lr, ldp, Z + (k + NB), np, k + NB, inner, NB,
                -1.f, 0};
        const int tu = kqh::timer_begin(KRONQ_TIMER_CHOL_UPDATE, st);
        const int s = kq_gemm_nt_tc(g, 2, info, st);
        kqh::timer_end(tu, st);
        if (s != KRONQ_OK) return s;
      }
    }
    const int rest = np - kb_end;
    if (rest > 0) {
      // the trailing matrix, once per super-block (K = kb_end - kb), on fp16
      // planes of row-scaled operands (twice the tf32 rate, ~2^-22 relative):
      //   R[kb_end:, kb_end:] -= L L^T (lower triangle),  L = L[kb_end:, kb:kb_end]
      //   Z[:kb_end, kb_end:] -= Z[:kb_end, kb:kb_end] L^T
      const int K = kb_end - kb;
      const int64_t lr = (int64_t)kb_end * ldp;
      const int tu = kqh::timer_begin(KRONQ_TIMER_CHOL_UPDATE, st);
      fp16_rows_kernel<<<(rest + 7) / 8, 256, 0, st>>>(Lh + lr, Ll + lr, rest, K, ldp, p16[0] + lr,
                                                       p16[1] + lr, sL + kb_end);
      KQ_CHECK_LAUNCH();
      fp16_rows_kernel<<<(kb_end + 7) / 8, 256, 0, st>>>(Zh, Zl, kb_end, K, ldp, p16[2], p16[3], sZ);
      KQ_CHECK_LAUNCH();
      kq::GemmNT g[2];
      g[0] = {p16[0] + lr, p16[1] + lr, ldp, p16[0] + lr, p16[1] + lr, ldp,
              R + (int64_t)kb_end * np + kb_end, np, rest, rest, K, -1.f, 1};
      g[1] = {p16[2], p16[3], ldp, p16[0] + lr, p16[1] + lr, ldp, Z + kb_end, np, kb_end, rest, K,
              -1.f, 0};
      g[0].fp16 = g[1].fp16 = 1;
      g[0].a_scale = g[0].b_scale = sL + kb_end;
      g[1].a_scale = sZ;
      g[1].b_scale = sL + kb_end;
      const int s = kq_gemm_nt_tc(g, 2, info, st);
      kqh::timer_end(tu, st);
      if (s != KRONQ_OK) return s;
    }
  }
  const dim3 og((n + 31) / 32, (n + 31) / 32);
  reverse_out_kernel<<<og, 256, 0, st>>>(Z, n, np, U);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}
