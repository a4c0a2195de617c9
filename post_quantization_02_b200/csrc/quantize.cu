// Column-wise OBS quantization of the rotated weights (GPTQ-style), packing,
// and the layer-loss helper.
//
// KronQ summary (hyper.ai), "Method", Prop. 1: H_G cancels in the column
// update, so every row of W' is solved with the inverse Cholesky factor U_c
// of H_X alone, and rows never interact.  KronQ review (pith.science),
// appendix, Algorithm 2: columns in blocks of B = 128 with an error buffer E
// and lazy updates of the trailing columns.
//
// Per block of 128 columns:
//   obs_block_kernel  32 rows per CTA, 8 threads per row, 16 columns of the
//                     block held in registers by each thread; the 128 x 128
//                     diagonal block of U_c in shared memory.  For each column
//                     j: the owning thread quantizes, the scaled error
//                     e = (w - w_hat) / U_c[j,j] is broadcast to the row's 8
//                     threads with one shuffle, each thread applies
//                     w_k -= e U_c[j,k] to its columns k > j.  No block-wide
//                     synchronisation inside the column loop.
//                     The kernel also writes E and the slab U_c[i:i+128, i+128:]^T
//                     as tf32 hi / lo planes (tf32x3.cuh) for the lazy update.
//   lazy update       W[:, i+128:] -= E U_c[i:i+128, i+128:] on the tensor cores
//                     (kq_gemm_nt_tc: tf32, three-term split, TMA reduce into W)
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"
#include "tf32x3.cuh"

namespace {

constexpr int QB = 128;          // column block
constexpr int ROWS_PER_CTA = 32;
constexpr int OBS_THREADS = 8 * ROWS_PER_CTA;   // 8 threads per row
constexpr int US_LD = QB + 4;    // padded row of the U_c block in shared memory
constexpr int TT_W = 8;          // columns per transposition slice of the U_c slab
constexpr int TT_LD = TT_W + 1;  // its shared-memory tile (QB x TT_W), padded

struct Grid {
  float scale;
  float zero;
};

// round(x / scale) with x / scale rounded to fp32 first (round half to even),
// i.e. exactly rintf(__fdiv_rn(x, scale)).  Fast path: qa = x * RN(1/scale)
// is within |q| * 1.8e-7 of the correctly rounded quotient q (two roundings
// of 2^-24 each, plus q's own), i.e. within 4.6e-5 for |q| < 256; so both
// round to the same integer unless qa lies within 1e-4 of a half-integer.
// Only then (or for |qa| >= 256) is the division carried out.
__device__ __forceinline__ float round_quotient(float x, float scale, float rscale) {
  const float qa = x * rscale;
  const float fr = qa - floorf(qa);
  if (fabsf(fr - 0.5f) > 1e-4f && fabsf(qa) < 256.f) return rintf(qa);
  return rintf(__fdiv_rn(x, scale));
}

// Asymmetric grid of [lo, hi] in fp32: lo = min(0, min w), hi = max(0, max w).
__device__ __forceinline__ Grid make_grid(float mn, float mx, float maxq) {
  const float lo = fminf(mn, 0.f), hi = fmaxf(mx, 0.f);
  Grid g;
  if (lo == 0.f && hi == 0.f) {
    g.scale = 1.f;
    g.zero = 0.f;
  } else {
    g.scale = __fdiv_rn(hi - lo, maxq);
    g.zero = fminf(fmaxf(rintf(__fdiv_rn(-lo, g.scale)), 0.f), maxq);
  }
  return g;
}

// --w_clip (KronQ README (GitHub), "Reproduce from scratch"; the pages name
// the flag without defining it).  Reading: among the shrunk ranges
// [p lo, p hi], p = 1 - i/100 for i = 0 .. 79, take the first grid with the
// least squared error sum (w - w_hat)^2 over the row or group.  The grid and
// the differences are fp32 operations (no contraction), the squares of the
// fp32 differences are exact in fp64 and summed in fp64, so the choice does
// not depend on the order of the sum.
constexpr int CLIP_STEPS = 80;

__device__ __forceinline__ float clip_ratio(int i) {
  return __double2float_rn(__dadd_rn(1.0, -__dmul_rn((double)i, 0.01)));
}

__device__ __forceinline__ Grid clip_grid(float lo, float hi, float p, float maxq) {
  const float lo1 = __fmul_rn(lo, p), hi1 = __fmul_rn(hi, p);
  Grid g;
  if (lo1 == 0.f && hi1 == 0.f) {
    g.scale = 1.f;
    g.zero = 0.f;
  } else {
    g.scale = __fdiv_rn(__fsub_rn(hi1, lo1), maxq);
    g.zero = fminf(fmaxf(rintf(__fdiv_rn(-lo1, g.scale)), 0.f), maxq);
  }
  return g;
}

// (w - w_hat)^2 for one weight on grid g, exact in fp64.
__device__ __forceinline__ double clip_sq_err(float x, const Grid& g, float rscale, float maxq) {
  const float q = fminf(fmaxf(round_quotient(x, g.scale, rscale) + g.zero, 0.f), maxq);
  const float wh = __fmul_rn(g.scale, q - g.zero);
  const double d = (double)__fsub_rn(x, wh);
  return d * d;
}

// Per-channel grid with the clip search: one CTA of 256 threads per row.
__global__ void __launch_bounds__(256) row_clip_params_kernel(const float* __restrict__ W, int m,
                                                              int n, int bits,
                                                              float* __restrict__ scales,
                                                              uint8_t* __restrict__ zeros) {
  __shared__ float rmn[8], rmx[8];
  __shared__ double part[8][CLIP_STEPS];   // per-warp error sums of every candidate
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* w = W + (int64_t)row * n;
  const float maxq = (float)((1 << bits) - 1);
  float mn = INFINITY, mx = -INFINITY;
  for (int j = tid; j < n; j += blockDim.x) {
    const float v = w[j];
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) { rmn[warp] = mn; rmx[warp] = mx; }
  __syncthreads();
  mn = rmn[0]; mx = rmx[0];
  for (int k = 1; k < 8; ++k) { mn = fminf(mn, rmn[k]); mx = fmaxf(mx, rmx[k]); }
  const float lo = fminf(mn, 0.f), hi = fmaxf(mx, 0.f);
  for (int i = 0; i < CLIP_STEPS; ++i) {
    const Grid g = clip_grid(lo, hi, clip_ratio(i), maxq);
    const float rs = __frcp_rn(g.scale);
    double acc = 0.0;
    for (int j = tid; j < n; j += blockDim.x) acc += clip_sq_err(w[j], g, rs, maxq);
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) part[warp][i] = acc;
  }
  __syncthreads();
  if (tid == 0) {
    double best = INFINITY;
    int best_i = 0;
    for (int i = 0; i < CLIP_STEPS; ++i) {
      double tot = 0.0;
      for (int k = 0; k < 8; ++k) tot += part[k][i];
      if (tot < best) { best = tot; best_i = i; }
    }
    const Grid g = clip_grid(lo, hi, clip_ratio(best_i), maxq);
    scales[row] = g.scale;
    zeros[row] = (uint8_t)g.zero;
  }
}

// Per-channel grid from the whole row, one warp per row.
__global__ void row_params_kernel(const float* __restrict__ W, int m, int n, int bits,
                                  float* __restrict__ scales, uint8_t* __restrict__ zeros) {
  const int row = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= m) return;
  float mn = INFINITY, mx = -INFINITY;
  const float* w = W + (int64_t)row * n;
  for (int j = lane; j < n; j += 32) {
    const float v = w[j];
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    const Grid g = make_grid(mn, mx, (float)((1 << bits) - 1));
    scales[row] = g.scale;
    zeros[row] = (uint8_t)g.zero;
  }
}

// GROUP 0: per-channel grid; else 32, 64 or 128.  CLIP: --w_clip.  ASYM: the
// GPTAQ term (P != null): after column j, later columns k also receive
// v_j P[j][k] (v_j: column j's value the quantizer saw); the kernel then
// also writes -v_j next to e_j (columns QB .. 2 QB - 1 of the block's part of
// the E planes) and P's slab next to U's (columns QB .. 2 QB - 1 of the slab
// planes), so that the lazy update is one product with K = 2 QB per block.
template <int GROUP, bool CLIP, bool ASYM = false>
__global__ void __launch_bounds__(OBS_THREADS)
obs_block_kernel(const float* __restrict__ W, int m, int n, const float* __restrict__ U, int i1,
                 int bits, uint8_t* __restrict__ codes, float* __restrict__ scales,
                 uint8_t* __restrict__ zeros, float* __restrict__ W_hat, uint16_t* __restrict__ Eh,
                 uint16_t* __restrict__ El, int ld_e, uint16_t* __restrict__ Uth,
                 uint16_t* __restrict__ Utl, int slab_end, const float* __restrict__ P = nullptr) {
  // Thread `chunk` (0..7) of a row owns the 16 columns 32 s + 4 chunk + t
  // (s, t in 0..3), held in w[4 s + t]: for a fixed s the 8 threads of a row
  // read 8 consecutive float4 of a U row, so the shared-memory reads are
  // free of bank conflicts.  Column j = 32 s + 4 c + t belongs to thread c.
  extern __shared__ float smem[];
  float* Us = smem;                    // [QB][US_LD]
  float* rdiag = smem + QB * US_LD;    // [QB]
  float* Tt = rdiag + QB;              // [QB][TT_LD]
  float* Ps = Tt + QB * TT_LD;         // [QB][US_LD] (ASYM only)
  const int tid = threadIdx.x, lane = tid & 31;
  constexpr int LDU = ASYM ? 2 * QB : QB;     // slab plane row length

  // The lazy update's B operand: Ut[c - i2][k] = U[i1 + k][c] for
  // i2 <= c < slab_end (the rest of the super-block, or of the matrix with
  // one level), in 8-column slices spread over all the CTAs (so that no CTA
  // starts its column loop much later than the others), as tf32 hi / lo planes.
  {
    const int i2 = i1 + QB;
    const int slices = (slab_end - i2) / TT_W;
#pragma unroll 1
    for (int which = 0; which < (ASYM ? 2 : 1); ++which) {
      const float* S = which ? P : U;
      for (int sl = blockIdx.x; sl < slices; sl += gridDim.x) {
        const int c0 = i2 + TT_W * sl;
        for (int e = tid; e < QB * TT_W; e += blockDim.x) {
          const int k = e / TT_W, cc = e % TT_W;
          Tt[k * TT_LD + cc] = S[(int64_t)(i1 + k) * n + c0 + cc];
        }
        __syncthreads();
        for (int e = tid; e < QB * TT_W; e += blockDim.x) {
          const int cc = e >> 7, k = e & (QB - 1);
          const int64_t o = (int64_t)(c0 - i2 + cc) * LDU + which * QB + k;
          kq::tf32x3::split_bf16(Tt[k * TT_LD + cc], Uth[o], Utl[o]);
        }
        __syncthreads();
      }
    }
  }
  const int chunk = tid & 7;
  const int row = blockIdx.x * ROWS_PER_CTA + (tid >> 3);
  const bool live = row < m;
  const float maxq = (float)((1 << bits) - 1);
  const int G = GROUP ? n / GROUP : 1;

  for (int e = tid; e < QB * QB / 4; e += blockDim.x) {
    const int r = e / (QB / 4), c4 = e % (QB / 4);
    const float4 u = *reinterpret_cast<const float4*>(U + (int64_t)(i1 + r) * n + i1 + c4 * 4);
    *reinterpret_cast<float4*>(Us + r * US_LD + c4 * 4) = u;
  }
  for (int j = tid; j < QB; j += blockDim.x) rdiag[j] = 1.f / U[(int64_t)(i1 + j) * n + i1 + j];
  if (ASYM) {
    for (int e = tid; e < QB * QB / 4; e += blockDim.x) {
      const int r = e / (QB / 4), c4 = e % (QB / 4);
      const float4 u = *reinterpret_cast<const float4*>(P + (int64_t)(i1 + r) * n + i1 + c4 * 4);
      *reinterpret_cast<float4*>(Ps + r * US_LD + c4 * 4) = u;
    }
  }

  float w[16];
  {
    const float* src = W + (int64_t)(live ? row : 0) * n + i1 + 4 * chunk;
#pragma unroll
    for (int sg = 0; sg < 4; ++sg) {
      const float4 v = live ? *reinterpret_cast<const float4*>(src + 32 * sg) : make_float4(0.f, 0.f, 0.f, 0.f);
      w[4 * sg] = v.x; w[4 * sg + 1] = v.y; w[4 * sg + 2] = v.z; w[4 * sg + 3] = v.w;
    }
  }
  float scale = 1.f, zero = 0.f;
  if (GROUP == 0 && live) {
    scale = scales[row];
    zero = (float)zeros[row];
  }
  float rscale = __frcp_rn(scale);
  __syncthreads();

  float qv[16], ev[16], hv[16];
  float vv[ASYM ? 16 : 1];
#pragma unroll
  for (int sg = 0; sg < 4; ++sg) {
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      const bool own = chunk == c;
      const int src = (lane & ~7) | c;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int j = 32 * sg + 4 * c + t;
        if (GROUP > 0 && t == 0 && (j % (GROUP > 0 ? GROUP : 1)) == 0) {
          // grid of columns j .. j+GROUP-1 (groups sg .. sg + GROUP/32 - 1 of every thread)
          float mn = INFINITY, mx = -INFINITY;
#pragma unroll
          for (int k = 4 * sg; k < 4 * sg + (GROUP >= 32 ? GROUP / 8 : 4) && k < 16; ++k) {
            mn = fminf(mn, w[k]);
            mx = fmaxf(mx, w[k]);
          }
#pragma unroll
          for (int o = 1; o < 8; o <<= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          }
          Grid g = make_grid(mn, mx, maxq);
          if (CLIP) {
            // the clip search over this group: every candidate's error summed
            // over the row's 8 threads, the total taken from the row's first
            // thread so that all 8 make the same choice
            const float lo = fminf(mn, 0.f), hi = fmaxf(mx, 0.f);
            double best = INFINITY;
            int best_i = 0;
#pragma unroll 1
            for (int ci = 0; ci < CLIP_STEPS; ++ci) {
              const Grid gc = clip_grid(lo, hi, clip_ratio(ci), maxq);
              const float rs = __frcp_rn(gc.scale);
              double acc = 0.0;
#pragma unroll
              for (int k = 4 * sg; k < 4 * sg + (GROUP >= 32 ? GROUP / 8 : 4) && k < 16; ++k)
                acc += clip_sq_err(w[k], gc, rs, maxq);
#pragma unroll
              for (int o = 1; o < 8; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
              acc = __shfl_sync(0xffffffffu, acc, lane & ~7);
              if (acc < best) { best = acc; best_i = ci; }
            }
            g = clip_grid(lo, hi, clip_ratio(best_i), maxq);
          }
          scale = g.scale;
          zero = g.zero;
          rscale = __frcp_rn(scale);
          if (live && own) {
            const int gi = (i1 + j) / (GROUP > 0 ? GROUP : 1);
            scales[(int64_t)row * G + gi] = scale;
            zeros[(int64_t)row * G + gi] = (uint8_t)zero;
          }
        }
        // quantize this thread's copy of column j (meaningful on the owner only)
        const float x = w[4 * sg + t];
        const float q = fminf(fmaxf(round_quotient(x, scale, rscale) + zero, 0.f), maxq);
        const float wh = scale * (q - zero);
        const float e_own = (x - wh) * rdiag[j];
        const float e_bc = __shfl_sync(0xffffffffu, e_own, src);
        const float e = own ? e_own : e_bc;          // the owner skips the shuffle latency
        qv[4 * sg + t] = own ? q : qv[4 * sg + t];
        hv[4 * sg + t] = own ? wh : hv[4 * sg + t];
        ev[4 * sg + t] = own ? e_own : ev[4 * sg + t];
        float v = 0.f;
        if (ASYM) {
          const float v_bc = __shfl_sync(0xffffffffu, x, src);
          v = own ? x : v_bc;
          vv[(4 * sg + t) % (ASYM ? 16 : 1)] = own ? x : vv[(4 * sg + t) % (ASYM ? 16 : 1)];
        }
        // w_k -= e U[j][k] (and, ASYM, += v P[j][k]) for this thread's
        // columns k > j (groups left of sg are done)
        const float* ur = Us + j * US_LD + 4 * chunk;
        const float* pr = Ps + j * US_LD + 4 * chunk;
#pragma unroll
        for (int s2 = sg; s2 < 4; ++s2) {
          const float4 u = *reinterpret_cast<const float4*>(ur + 32 * s2);
          const float uu[4] = {u.x, u.y, u.z, u.w};
          float pp[4] = {0.f, 0.f, 0.f, 0.f};
          if (ASYM) {
            const float4 p4 = *reinterpret_cast<const float4*>(pr + 32 * s2);
            pp[0] = p4.x; pp[1] = p4.y; pp[2] = p4.z; pp[3] = p4.w;
          }
#pragma unroll
          for (int t2 = 0; t2 < 4; ++t2) {
            const bool later = s2 > sg || 4 * chunk + t2 > 4 * c + t;
            const float coef = later ? uu[t2] : 0.f;
            w[4 * s2 + t2] = fmaf(-e, coef, w[4 * s2 + t2]);
            if (ASYM) w[4 * s2 + t2] = fmaf(v, later ? pp[t2] : 0.f, w[4 * s2 + t2]);
          }
        }
      }
    }
  }
  if (!live) return;
#pragma unroll
  for (int sg = 0; sg < 4; ++sg) {
    const int64_t off = (int64_t)row * n + i1 + 32 * sg + 4 * chunk;
    const uint32_t pk = (uint32_t)qv[4 * sg] | ((uint32_t)qv[4 * sg + 1] << 8) |
                        ((uint32_t)qv[4 * sg + 2] << 16) | ((uint32_t)qv[4 * sg + 3] << 24);
    *reinterpret_cast<uint32_t*>(codes + off) = pk;
    {
      // E as bf16 hi / lo planes (four values: one 8-byte store per plane)
      uint16_t h[4], l[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) kq::tf32x3::split_bf16(ev[4 * sg + u], h[u], l[u]);
      const int64_t eo = (int64_t)row * ld_e + 32 * sg + 4 * chunk;
      *reinterpret_cast<uint2*>(Eh + eo) = make_uint2(h[0] | ((uint32_t)h[1] << 16), h[2] | ((uint32_t)h[3] << 16));
      *reinterpret_cast<uint2*>(El + eo) = make_uint2(l[0] | ((uint32_t)l[1] << 16), l[2] | ((uint32_t)l[3] << 16));
      if (ASYM) {
        // -v next to e: the lazy update subtracts [E | -V] [U ; P]
        const int b = (4 * sg) % (ASYM ? 16 : 1);
#pragma unroll
        for (int u = 0; u < 4; ++u) kq::tf32x3::split_bf16(-vv[b + u], h[u], l[u]);
        *reinterpret_cast<uint2*>(Eh + eo + QB) = make_uint2(h[0] | ((uint32_t)h[1] << 16), h[2] | ((uint32_t)h[3] << 16));
        *reinterpret_cast<uint2*>(El + eo + QB) = make_uint2(l[0] | ((uint32_t)l[1] << 16), l[2] | ((uint32_t)l[3] << 16));
      }
    }
    if (W_hat)
      *reinterpret_cast<float4*>(W_hat + off) =
          make_float4(hv[4 * sg], hv[4 * sg + 1], hv[4 * sg + 2], hv[4 * sg + 3]);
  }
}

template <bool TA, bool TB>
__global__ void __launch_bounds__(256) gemm_kernel(const float* A, int64_t lda, const float* B,
                                                   int64_t ldb, float* C, int64_t ldc, int M, int N,
                                                   int K, float alpha, float beta) {
  kq::gemm_tile64<TA, TB>(A, lda, B, ldb, C, ldc, M, N, K, alpha, beta, blockIdx.y, blockIdx.x);
}

__global__ void sub_kernel(const float* __restrict__ a, const float* __restrict__ b,
                           float* __restrict__ c, int64_t total) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x)
    c[e] = a[e] - b[e];
}

__global__ void dot_kernel(const float* __restrict__ a, const float* __restrict__ b, int64_t total,
                           double* out) {
  __shared__ double red[256];
  double s = 0.0;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x)
    s += (double)a[e] * (double)b[e];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) atomicAdd(out, red[0]);
}

// ------------------------------------------------------------------ packing
__global__ void pack_kernel(const uint8_t* __restrict__ codes, int64_t m, int64_t n, int bits,
                            int64_t wpr, uint32_t* __restrict__ packed, int32_t* bad) {
  const int per = 32 / bits;
  const uint32_t mask = (1u << bits) - 1u;
  const int64_t total = m * wpr;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / wpr, wi = e % wpr;
    const int64_t j0 = wi * per;
    uint32_t word = 0;
    for (int t = 0; t < per; ++t) {
      const int64_t j = j0 + t;
      if (j >= n) break;
      const uint32_t c = codes[r * n + j];
      if (c > mask && bad) atomicCAS(bad, 0, KRONQ_ERR_INVALID_ARG);
      word |= (c & mask) << (t * bits);
    }
    packed[e] = word;
  }
}

// Fast path for n % 16 == 0: 16 codes (one 16-byte load) per item give two
// 32-bit words (4-bit) or one (2-bit); the flattened code index maps to the
// flattened word index because rows hold whole items.
template <int BITS>
__global__ void pack16_kernel(const uint4* __restrict__ codes, int64_t items,
                              uint32_t* __restrict__ packed) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < items;
       e += (int64_t)gridDim.x * blockDim.x) {
    const uint4 v = codes[e];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    if (BITS == 4) {
      uint32_t o[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t a = w[2 * h], b = w[2 * h + 1];   // bytes c0..c3, c4..c7
        o[h] = (a & 0xFu) | ((a >> 4) & 0xF0u) | ((a >> 8) & 0xF00u) | ((a >> 12) & 0xF000u) |
               ((b & 0xFu) << 16) | ((b << 12) & 0xF00000u) | ((b << 8) & 0xF000000u) |
               ((b << 4) & 0xF0000000u);
      }
      reinterpret_cast<uint2*>(packed)[e] = make_uint2(o[0], o[1]);
    } else {
      uint32_t o = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t a = w[q];
        const uint32_t c = (a & 0x3u) | ((a >> 6) & 0xCu) | ((a >> 12) & 0x30u) | ((a >> 18) & 0xC0u);
        o |= c << (8 * q);
      }
      packed[e] = o;
    }
  }
}

__global__ void unpack_kernel(const uint32_t* __restrict__ packed, int64_t m, int64_t n, int bits,
                              int64_t wpr, uint8_t* __restrict__ codes) {
  const int per = 32 / bits;
  const uint32_t mask = (1u << bits) - 1u;
  const int64_t total = m * n;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / n, j = e % n;
    codes[e] = (uint8_t)((packed[r * wpr + j / per] >> ((j % per) * bits)) & mask);
  }
}

size_t a256(size_t b) { return (b + 255) & ~(size_t)255; }

// The lazy update's operands are bf16 hi / lo planes (x = hi + lo to about
// 2^-17 relative; three bf16 tensor-core products per fp32 product).
struct SolverScratch {
  int B2;                  // outer (super-)block width: 128 (one level) or 1024
  uint16_t *Eh, *El;       // E of the super-block, m x B2 each
  uint16_t *Uth, *Utl;     // inner slab U[i1:i1+128, i1+128:sb_end]^T, n x 128 each
  uint16_t *Voh, *Vol;     // outer slab U[sb:sb_end, sb_end:]^T, n x B2 each (two levels only)
};

// Ut[c - col0][k] = U[row0 + k][c] for k < rows, col0 <= c < n, as tf32
// hi / lo planes with leading dimension ld: one 32 x 32 tile per CTA.
__global__ void __launch_bounds__(256) slab_transpose_kernel(const float* __restrict__ U, int n,
                                                             int row0, int rows, int col0,
                                                             uint16_t* __restrict__ Th,
                                                             uint16_t* __restrict__ Tl, int ld) {
  __shared__ float t[32][33];
  const int kb = blockIdx.y * 32, cb = col0 + blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int r = ty; r < 32; r += 8) {
    const int k = kb + r, c = cb + tx;
    t[r][tx] = (k < rows && c < n) ? U[(int64_t)(row0 + k) * n + c] : 0.f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int c = cb + r, k = kb + tx;
    if (c < n && k < rows) {
      const int64_t o = (int64_t)(c - col0) * ld + k;
      kq::tf32x3::split_bf16(t[tx][r], Th[o], Tl[o]);
    }
  }
}

template <int GROUP, bool CLIP, bool ASYM = false>
int launch_block(const float* W, int m, int n, const float* U, int i1, int bits, uint8_t* codes,
                 float* scales, uint8_t* zeros, float* W_hat, const SolverScratch& sc, int sb,
                 int slab_end, cudaStream_t st, const float* P = nullptr) {
  static kqh::PerDevice attr;
  const size_t smem = (size_t)(QB * US_LD + QB + QB * TT_LD + (ASYM ? QB * US_LD : 0)) * sizeof(float);
  if (kqh::smem_attr_once(attr, obs_block_kernel<GROUP, CLIP, ASYM>, (int)smem) <= 0)
    return KRONQ_ERR_CUDA;
  const int grid = (m + ROWS_PER_CTA - 1) / ROWS_PER_CTA;
  constexpr int KM = ASYM ? 2 : 1;               // E planes: [E | -V] per block with ASYM
  const int ts = kqh::timer_begin(KRONQ_TIMER_OBS_BLOCK, st);
  obs_block_kernel<GROUP, CLIP, ASYM><<<grid, OBS_THREADS, smem, st>>>(
      W, m, n, U, i1, bits, codes, scales, zeros, W_hat, sc.Eh + KM * (i1 - sb),
      sc.El + KM * (i1 - sb), KM * sc.B2, sc.Uth, sc.Utl, slab_end, P);
  kqh::timer_end(ts, st);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

// The GPTAQ variant of slab_transpose_kernel: rows row0 .. row0 + rows - 1 of
// U and of P, transposed, interleaved per 128-row block b as the K layout of
// the asymmetric lazy update: T[c - col0][2 QB b + k] = U[row0 + QB b + k][c]
// and T[c - col0][2 QB b + QB + k] = P[row0 + QB b + k][c].
__global__ void __launch_bounds__(256) slab_transpose2_kernel(const float* __restrict__ U,
                                                              const float* __restrict__ P, int n,
                                                              int row0, int rows, int col0,
                                                              uint16_t* __restrict__ Th,
                                                              uint16_t* __restrict__ Tl, int ld) {
  __shared__ float t[32][33];
  const float* S = blockIdx.z ? P : U;
  const int kb = blockIdx.y * 32, cb = col0 + blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int r = ty; r < 32; r += 8) {
    const int k = kb + r, c = cb + tx;
    t[r][tx] = (k < rows && c < n) ? S[(int64_t)(row0 + k) * n + c] : 0.f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int c = cb + r, k = kb + tx;
    if (c < n && k < rows) {
      const int kk = 2 * QB * (k / QB) + (int)blockIdx.z * QB + k % QB;
      const int64_t o = (int64_t)(c - col0) * ld + kk;
      kq::tf32x3::split_bf16(t[tx][r], Th[o], Tl[o]);
    }
  }
}

constexpr int QB2 = 1024;        // outer super-block of the two-level lazy update

// Scratch of the solver with outer block B2: E of a super-block as hi / lo
// planes (m x B2 each), the inner U_c slab transposed (n x 128 each) and,
// with two levels, the outer slab transposed (n x B2 each).
size_t solver_ws(int64_t m, int64_t n, int B2) {
  size_t b = 2 * a256((size_t)m * B2 * sizeof(uint16_t)) + 2 * a256((size_t)n * QB * sizeof(uint16_t));
  if (B2 > QB) b += 2 * a256((size_t)n * B2 * sizeof(uint16_t));
  return b;
}

}  // namespace

// The size that enables the two-level lazy update; a workspace of at least
// solver_ws(m, n, 128) runs the one-level update.
size_t kq_quantize_ws(int64_t m, int64_t n) { return solver_ws(m, n, QB2); }

size_t kq_loss_ws(int64_t m, int64_t n) { return 3 * a256((size_t)m * n * sizeof(float)); }

int kq_quantize_layer(float* W, int64_t m64, int64_t n64, const float* U, int bits, int group,
                      int block, int options, uint8_t* codes, float* scales, uint8_t* zeros,
                      float* W_hat, int32_t* info, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!W || !U || !codes || !scales || !zeros || m64 <= 0 || n64 <= 0) return KRONQ_ERR_INVALID_ARG;
  if (options & ~KRONQ_QUANT_CLIP) return KRONQ_ERR_INVALID_ARG;
  const bool clip = (options & KRONQ_QUANT_CLIP) != 0;
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return KRONQ_ERR_INVALID_ARG;
  if (group != -1 && (group <= 0 || n64 % group)) return KRONQ_ERR_INVALID_ARG;
  if (block != QB) return KRONQ_ERR_UNSUPPORTED;
  if (group != -1 && group != 32 && group != 64 && group != 128) return KRONQ_ERR_UNSUPPORTED;
  if (n64 % QB) return KRONQ_ERR_UNSUPPORTED;
  if (m64 > INT32_MAX || n64 > 65536) return KRONQ_ERR_UNSUPPORTED;
  if (!kqh::aligned(W, 16) || !kqh::aligned(U, 16) || !kqh::aligned(codes, 16) ||
      (W_hat && !kqh::aligned(W_hat, 16)))
    return KRONQ_ERR_INVALID_ARG;
  if (!ws || !kqh::aligned(ws, 256)) return KRONQ_ERR_WORKSPACE;
  // two levels (B2 = 1024: the outer update is a K = 1024 tensor-core GEMM)
  // when the workspace allows, else one level
  const int B2 = (n64 > QB && ws_bytes >= solver_ws(m64, n64, QB2)) ? QB2 : QB;
  if (ws_bytes < solver_ws(m64, n64, B2)) return KRONQ_ERR_WORKSPACE;
  const int m = (int)m64, n = (int)n64;
  SolverScratch sc;
  {
    uint8_t* w = static_cast<uint8_t*>(ws);
    sc.B2 = B2;
    sc.Eh = reinterpret_cast<uint16_t*>(w);
    w += a256((size_t)m * B2 * sizeof(uint16_t));
    sc.El = reinterpret_cast<uint16_t*>(w);
    w += a256((size_t)m * B2 * sizeof(uint16_t));
    sc.Uth = reinterpret_cast<uint16_t*>(w);
    w += a256((size_t)n * QB * sizeof(uint16_t));
    sc.Utl = reinterpret_cast<uint16_t*>(w);
    w += a256((size_t)n * QB * sizeof(uint16_t));
    sc.Voh = sc.Vol = nullptr;
    if (B2 > QB) {
      sc.Voh = reinterpret_cast<uint16_t*>(w);
      w += a256((size_t)n * B2 * sizeof(uint16_t));
      sc.Vol = reinterpret_cast<uint16_t*>(w);
    }
  }

  if (group == -1 && clip) {
    row_clip_params_kernel<<<m, 256, 0, st>>>(W, m, n, bits, scales, zeros);
    KQ_CHECK_LAUNCH();
  } else if (group == -1) {
    row_params_kernel<<<(m + 7) / 8, 256, 0, st>>>(W, m, n, bits, scales, zeros);
    KQ_CHECK_LAUNCH();
  }
  for (int sb = 0; sb < n; sb += B2) {
    const int sb_end = sb + B2 < n ? sb + B2 : n;
    const int slab_end = B2 > QB ? sb_end : n;
    for (int i1 = sb; i1 < sb_end; i1 += QB) {
      int s;
#define KQ_BLOCK(G, C) launch_block<G, C>(W, m, n, U, i1, bits, codes, scales, zeros, W_hat, sc, sb, slab_end, st)
      switch (group) {
        case -1: s = KQ_BLOCK(0, false); break;   // per-channel: the clip search ran before the loop
        case 32: s = clip ? KQ_BLOCK(32, true) : KQ_BLOCK(32, false); break;
        case 64: s = clip ? KQ_BLOCK(64, true) : KQ_BLOCK(64, false); break;
        default: s = clip ? KQ_BLOCK(128, true) : KQ_BLOCK(128, false); break;
      }
#undef KQ_BLOCK
      if (s != KRONQ_OK) return s;
      const int i2 = i1 + QB;
      if (i2 < sb_end) {
        // inner: W[:, i2:sb_end] -= E_blk U[i1:i2, i2:sb_end]
        kq::GemmNT g = {sc.Eh + (i1 - sb), sc.El + (i1 - sb), B2, sc.Uth, sc.Utl, QB,
                        W + i2, n, m, sb_end - i2, QB, -1.f, 0};
        g.bf16 = 1;
        const int ts = kqh::timer_begin(KRONQ_TIMER_LAZY_UPDATE, st);
        s = kq_gemm_nt_tc(&g, 1, info, st);
        kqh::timer_end(ts, st);
        if (s != KRONQ_OK) return s;
      }
    }
    if (sb_end < n) {
      // outer: W[:, sb_end:] -= E_sb U[sb:sb_end, sb_end:]   (K = sb_end - sb)
      const int K = sb_end - sb;
      const uint16_t* Bh = sc.Uth;
      const uint16_t* Bl = sc.Utl;
      int ldb = QB;
      if (B2 > QB) {
        const dim3 g((n - sb_end + 31) / 32, (K + 31) / 32);
        slab_transpose_kernel<<<g, 256, 0, st>>>(U, n, sb, K, sb_end, sc.Voh, sc.Vol, B2);
        KQ_CHECK_LAUNCH();
        Bh = sc.Voh;
        Bl = sc.Vol;
        ldb = B2;
      }
      // (one level: the block kernel already wrote U[sb:sb_end, sb_end:]^T into Ut)
      kq::GemmNT g = {sc.Eh, sc.El, B2, Bh, Bl, ldb, W + sb_end, n, m, n - sb_end, K, -1.f, 0};
      g.bf16 = 1;
      const int ts = kqh::timer_begin(KRONQ_TIMER_LAZY_UPDATE, st);
      const int s = kq_gemm_nt_tc(&g, 1, info, st);
      kqh::timer_end(ts, st);
      if (s != KRONQ_OK) return s;
    }
  }
  return KRONQ_OK;
}

// ---------------------------------------------------------------------------
// The solver with the GPTAQ term (asymmetric calibration): the block kernel
// adds v_j P[j][k] next to -e_j U[j][k], and every lazy update subtracts
// [E | -V] [U ; P] with K = 2 QB per block (E and -V interleaved per block,
// U's and P's slabs likewise), as one tensor-core product.
namespace {
size_t solver_ws_asym(int64_t m, int64_t n, int B2) {
  size_t b = 2 * a256((size_t)m * 2 * B2 * sizeof(uint16_t)) +
             2 * a256((size_t)n * 2 * QB * sizeof(uint16_t));
  if (B2 > QB) b += 2 * a256((size_t)n * 2 * B2 * sizeof(uint16_t));
  return b;
}
}  // namespace

size_t kq_quantize_asym_ws(int64_t m, int64_t n) { return solver_ws_asym(m, n, QB2); }

int kq_quantize_layer_asym(float* W, int64_t m64, int64_t n64, const float* U, const float* P,
                           int bits, int group, int block, uint8_t* codes, float* scales,
                           uint8_t* zeros, float* W_hat, int32_t* info, void* ws, size_t ws_bytes,
                           cudaStream_t st) {
  if (!W || !U || !P || !codes || !scales || !zeros || m64 <= 0 || n64 <= 0)
    return KRONQ_ERR_INVALID_ARG;
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return KRONQ_ERR_INVALID_ARG;
  if (group != -1 && (group <= 0 || n64 % group)) return KRONQ_ERR_INVALID_ARG;
  if (block != QB) return KRONQ_ERR_UNSUPPORTED;
  if (group != -1 && group != 128) return KRONQ_ERR_UNSUPPORTED;
  if (n64 % QB) return KRONQ_ERR_UNSUPPORTED;
  if (m64 > INT32_MAX || n64 > 32768) return KRONQ_ERR_UNSUPPORTED;
  if (!kqh::aligned(W, 16) || !kqh::aligned(U, 16) || !kqh::aligned(P, 16) ||
      !kqh::aligned(codes, 16) || (W_hat && !kqh::aligned(W_hat, 16)))
    return KRONQ_ERR_INVALID_ARG;
  if (!ws || !kqh::aligned(ws, 256)) return KRONQ_ERR_WORKSPACE;
  const int B2 = (n64 > QB && ws_bytes >= solver_ws_asym(m64, n64, QB2)) ? QB2 : QB;
  if (ws_bytes < solver_ws_asym(m64, n64, B2)) return KRONQ_ERR_WORKSPACE;
  const int m = (int)m64, n = (int)n64;
  SolverScratch sc;
  {
    uint8_t* w = static_cast<uint8_t*>(ws);
    sc.B2 = B2;
    sc.Eh = reinterpret_cast<uint16_t*>(w);
    w += a256((size_t)m * 2 * B2 * sizeof(uint16_t));
    sc.El = reinterpret_cast<uint16_t*>(w);
    w += a256((size_t)m * 2 * B2 * sizeof(uint16_t));
    sc.Uth = reinterpret_cast<uint16_t*>(w);
    w += a256((size_t)n * 2 * QB * sizeof(uint16_t));
    sc.Utl = reinterpret_cast<uint16_t*>(w);
    w += a256((size_t)n * 2 * QB * sizeof(uint16_t));
    sc.Voh = sc.Vol = nullptr;
    if (B2 > QB) {
      sc.Voh = reinterpret_cast<uint16_t*>(w);
      w += a256((size_t)n * 2 * B2 * sizeof(uint16_t));
      sc.Vol = reinterpret_cast<uint16_t*>(w);
    }
  }
  if (group == -1) {
    row_params_kernel<<<(m + 7) / 8, 256, 0, st>>>(W, m, n, bits, scales, zeros);
    KQ_CHECK_LAUNCH();
  }
  for (int sb = 0; sb < n; sb += B2) {
    const int sb_end = sb + B2 < n ? sb + B2 : n;
    const int slab_end = B2 > QB ? sb_end : n;
    for (int i1 = sb; i1 < sb_end; i1 += QB) {
      const int s = group == -1
          ? launch_block<0, false, true>(W, m, n, U, i1, bits, codes, scales, zeros, W_hat, sc, sb,
                                         slab_end, st, P)
          : launch_block<128, false, true>(W, m, n, U, i1, bits, codes, scales, zeros, W_hat, sc,
                                           sb, slab_end, st, P);
      if (s != KRONQ_OK) return s;
      const int i2 = i1 + QB;
      if (i2 < sb_end) {
        // inner: W[:, i2:sb_end] -= [E_blk | -V_blk] [U ; P][i1:i2, i2:sb_end]
        kq::GemmNT g = {sc.Eh + 2 * (i1 - sb), sc.El + 2 * (i1 - sb), 2 * B2, sc.Uth, sc.Utl,
                        2 * QB, W + i2, n, m, sb_end - i2, 2 * QB, -1.f, 0};
        g.bf16 = 1;
        const int ts = kqh::timer_begin(KRONQ_TIMER_LAZY_UPDATE, st);
        const int s2 = kq_gemm_nt_tc(&g, 1, info, st);
        kqh::timer_end(ts, st);
        if (s2 != KRONQ_OK) return s2;
      }
    }
    if (sb_end < n) {
      // outer: W[:, sb_end:] -= [E | -V]_sb [U ; P][sb:sb_end, sb_end:]
      const int K = sb_end - sb;
      const uint16_t* Bh = sc.Uth;
      const uint16_t* Bl = sc.Utl;
      int ldb = 2 * QB;
      if (B2 > QB) {
        const dim3 g((n - sb_end + 31) / 32, (K + 31) / 32, 2);
        slab_transpose2_kernel<<<g, 256, 0, st>>>(U, P, n, sb, K, sb_end, sc.Voh, sc.Vol, 2 * B2);
        KQ_CHECK_LAUNCH();
        Bh = sc.Voh;
        Bl = sc.Vol;
        ldb = 2 * B2;
      }
      kq::GemmNT g = {sc.Eh, sc.El, 2 * B2, Bh, Bl, ldb, W + sb_end, n, m, n - sb_end, 2 * K,
                      -1.f, 0};
      g.bf16 = 1;
      const int ts = kqh::timer_begin(KRONQ_TIMER_LAZY_UPDATE, st);
      const int s = kq_gemm_nt_tc(&g, 1, info, st);
      kqh::timer_end(ts, st);
      if (s != KRONQ_OK) return s;
    }
  }
  return KRONQ_OK;
}

int kq_pack(const uint8_t* codes, int64_t m, int64_t n, int bits, uint32_t* packed,
            cudaStream_t st) {
  if (bits == 3) return KRONQ_ERR_UNSUPPORTED;
  if (bits != 2 && bits != 4) return KRONQ_ERR_INVALID_ARG;
  if (m < 0 || n < 0) return KRONQ_ERR_INVALID_ARG;
  if (m == 0 || n == 0) return KRONQ_OK;
  if (!codes || !packed || !kqh::aligned(packed, 4)) return KRONQ_ERR_INVALID_ARG;
  const int64_t wpr = (n * bits + 31) / 32;
  if (n % 16 == 0 && kqh::aligned(codes, 16) && kqh::aligned(packed, bits == 4 ? 8 : 4)) {
    const int64_t items = m * n / 16;
    const int grid = (int)std::min<int64_t>((items + 255) / 256, 8 * (int64_t)kqh::num_sms());
    if (bits == 4)
      pack16_kernel<4><<<grid, 256, 0, st>>>(reinterpret_cast<const uint4*>(codes), items, packed);
    else
      pack16_kernel<2><<<grid, 256, 0, st>>>(reinterpret_cast<const uint4*>(codes), items, packed);
    KQ_CHECK_LAUNCH();
    return KRONQ_OK;
  }
  pack_kernel<<<4 * kqh::num_sms(), 256, 0, st>>>(codes, m, n, bits, wpr, packed, nullptr);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

int kq_unpack(const uint32_t* packed, int64_t m, int64_t n, int bits, uint8_t* codes,
              cudaStream_t st) {
  if (bits == 3) return KRONQ_ERR_UNSUPPORTED;
  if (bits != 2 && bits != 4) return KRONQ_ERR_INVALID_ARG;
  if (m < 0 || n < 0) return KRONQ_ERR_INVALID_ARG;
  if (m == 0 || n == 0) return KRONQ_OK;
  if (!codes || !packed || !kqh::aligned(packed, 4)) return KRONQ_ERR_INVALID_ARG;
  const int64_t wpr = (n * bits + 31) / 32;
  unpack_kernel<<<4 * kqh::num_sms(), 256, 0, st>>>(packed, m, n, bits, wpr, codes);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

int kq_layer_loss(const float* Wr, const float* Wh, int64_t m64, int64_t n64, const float* HX,
                  const float* HG, double* out, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!Wr || !Wh || !HX || !HG || !out || m64 <= 0 || n64 <= 0) return KRONQ_ERR_INVALID_ARG;
  if (m64 > INT32_MAX || n64 > INT32_MAX) return KRONQ_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < kq_loss_ws(m64, n64) || !kqh::aligned(ws, 256)) return KRONQ_ERR_WORKSPACE;
  const int m = (int)m64, n = (int)n64;
  const size_t slab = a256((size_t)m * n * sizeof(float));
  float* dW = static_cast<float*>(ws);
  float* T1 = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + slab);
  float* T2 = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + 2 * slab);
  const int sms = kqh::num_sms();
  sub_kernel<<<4 * sms, 256, 0, st>>>(Wr, Wh, dW, (int64_t)m * n);
  KQ_CHECK_LAUNCH();
  const dim3 g((n + 63) / 64, (m + 63) / 64);
  gemm_kernel<false, false><<<g, 256, 0, st>>>(dW, n, HX, n, T1, n, m, n, n, 1.f, 0.f);
  KQ_CHECK_LAUNCH();
  gemm_kernel<false, false><<<g, 256, 0, st>>>(HG, m, dW, n, T2, n, m, n, m, 1.f, 0.f);
  KQ_CHECK_LAUNCH();
  if (cudaMemsetAsync(out, 0, sizeof(double), st) != cudaSuccess) return KRONQ_ERR_CUDA;
  dot_kernel<<<2 * sms, 256, 0, st>>>(T1, T2, (int64_t)m * n, out);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

// ---------------------------------------------------------------------------
// Allocation-free variant of kronq_quantize_layer.
//
// Some callers cannot allocate device memory while they run: a host framework
// that owns the device allocator and forbids plugins from calling cudaMalloc,
// a process that plans all of its memory at start-up and must not grow it
// later, or a latency-sensitive loop in which cudaMalloc / cudaFree would
// synchronise the device and stall other streams.  For them the solver's
// scratch (the error block and the transposed U_c slab, each as bf16 hi / lo
// planes) lives in the static device array below instead of a caller
// workspace.
//
// The array is part of the library image: every GPU that loads libkronq holds
// its 64 MiB until the process exits; it holds the one-level scratch of up
// to m = 32768 rows and n = 32768 columns (half of it), and the two-level
// scratch whenever that fits too.  Host code cannot use the symbol as a device address,
// so its address is looked up with cudaGetSymbolAddress once per device (with
// that device current), on the first call made on that device.  All calls
// share the one array and it keeps the previous call's contents: nothing in
// it has to start at zero (every element the lazy update reads was written
// by the block solve of the same call), but two calls whose work overlaps on
// the GPU race on it.
constexpr int64_t kNoAllocMaxRows = 32768;
constexpr int64_t kNoAllocMaxCols = 32768;
constexpr size_t kNoAllocBytes = (size_t)2 * (kNoAllocMaxRows + kNoAllocMaxCols) * QB * sizeof(float);
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocBytes / sizeof(float)];

namespace {

std::mutex g_noalloc_mutex;
float* g_noalloc_ptr[64] = {};

// Device address of g_noalloc_scratch on the current device (nullptr on failure).
float* noalloc_scratch() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  }
  return g_noalloc_ptr[dev];
}

}  // namespace

int kq_quantize_layer_noalloc(float* W, int64_t m, int64_t n, const float* U, int bits, int group,
                              int block, uint8_t* codes, float* scales, uint8_t* zeros,
                              float* W_hat, int32_t* info, cudaStream_t st) {
  // the static scratch holds 32768 rows and 32768 columns
  if (m > kNoAllocMaxRows || n > kNoAllocMaxCols) return KRONQ_ERR_UNSUPPORTED;
  float* scratch = noalloc_scratch();
  if (!scratch) return KRONQ_ERR_CUDA;
  return kq_quantize_layer(W, m, n, U, bits, group, block, 0, codes, scales, zeros, W_hat, info,
                           scratch, sizeof(g_noalloc_scratch), st);
}
