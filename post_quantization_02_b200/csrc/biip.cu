// Bidirectional incoherence processing and the sensitivity score.
//
// KronQ summary (hyper.ai), "Method", Eqs. 11-12: diagonal rescale of both
// dimensions of W (S_X on columns, S_G on rows; S_G is KronQ's addition),
// then W' = U W V^T, H_X' = V H_X V^T, H_G' = U H_G U^T with randomized
// Hadamard transforms; Eq. 14: s = tr(H_G') tr(H_X').
//
// Transform of a length-d vector, d = Q * L2 with L2 = 2^k2 <= 4096:
//   x -> (M_Q (x) H_L2 / sqrt(L2)) D x,   M_Q = C_q (x) H_{2^k1} / sqrt(2^k1)
// (C_q the orthonormal DCT-II, q the odd part of d).  This is the same matrix
// as C_q (x) H_{2^k} / sqrt(2^k): a Sylvester Hadamard of size 2^k1 L2 splits
// into H_{2^k1} on the high index bits and H_L2 on the low ones.  Within a
// segment of L2 consecutive entries: Walsh-Hadamard butterflies; across the
// Q segments: a dense Q x Q mix.
//
// Passes over HBM: a row pass (per row segment: butterflies in registers,
// scaling and signs fused into the load; rows with an odd factor: the row
// staged in shared memory with the Q-mix) and a column pass (each thread
// one column of a group of rows in registers, two launches for segments
// longer than 64 rows, then the Q-mix).
#include "common.cuh"

namespace {

constexpr int RT_THREADS = 256;

struct Split {
  int L2, Q, q, k1;
};

bool split_width(int64_t d, Split& s) {
  if (d < 16 || d % 16) return false;
  int64_t q = d;
  int k = 0;
  while (q % 2 == 0) { q /= 2; ++k; }
  if (q > 63) return false;
  const int k2 = k < 12 ? k : 12;
  s.L2 = 1 << k2;
  s.k1 = k - k2;
  s.q = (int)q;
  s.Q = (int)q << s.k1;
  return s.Q <= 64;
}

// M = C_q (x) H_{2^k1} / sqrt(2^k1), Q x Q, row-major.
__global__ void make_mix_kernel(float* __restrict__ M, int q, int k1) {
  const int Q = q << k1;
  const double PI = 3.14159265358979323846;
  for (int e = threadIdx.x; e < Q * Q; e += blockDim.x) {
    const int s = e / Q, t = e % Q;
    const int p = s >> k1, a = s & ((1 << k1) - 1);
    const int p2 = t >> k1, a2 = t & ((1 << k1) - 1);
    double c = sqrt(2.0 / q) * cos(PI * (2 * p2 + 1) * p / (2.0 * q));
    if (p == 0) c *= sqrt(0.5);
    const double h = (__popc(a & a2) & 1) ? -1.0 : 1.0;
    M[e] = (float)(c * h / sqrt((double)(1 << k1)));
  }
}

__global__ void colnorm_kernel(const float* __restrict__ W, int m, int n, double* __restrict__ cn) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const int rows_per = (m + gridDim.y - 1) / gridDim.y;
  const int r0 = blockIdx.y * rows_per, r1 = min(m, r0 + rows_per);
  double s = 0.0;
#pragma unroll 8
  for (int i = r0; i < r1; ++i) {
    const double v = W[(int64_t)i * n + j];
    s += v * v;
  }
  atomicAdd(&cn[j], s);
}

// S = (H_jj / norm2_j)^alpha (1 when either is not positive); also 1/S.
__global__ void scale_from_diag_kernel(const float* __restrict__ H, int d,
                                       const double* __restrict__ norm2, float alpha,
                                       float* __restrict__ S, float* __restrict__ rS, int active) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= d) return;
  float s = 1.f;
  if (active) {
    const double h = H[(int64_t)j * d + j], nn = norm2[j];
    if (h > 0.0 && nn > 0.0) s = (float)pow(h / nn, (double)alpha);
  }
  S[j] = s;
  rS[j] = 1.f / s;
}

// ||(W S_X)_i,:||^2, one warp per row.
__global__ void rownorm_kernel(const float* __restrict__ W, int m, int n,
                               const float* __restrict__ SX, double* __restrict__ rn) {
  const int row = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= m) return;
  double s = 0.0;
  for (int j = lane; j < n; j += 32) {
    const double v = (double)(W[(int64_t)row * n + j] * SX[j]);
    s += v * v;
  }
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) rn[row] = s;
}

__global__ void recip_kernel(const float* __restrict__ S, float* __restrict__ rS, int d) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j < d) rS[j] = 1.f / S[j];
}

// X[r][c] *= rs[r] cs[c]
__global__ void scale_only_kernel(float* __restrict__ X, int R, int C, const float* __restrict__ rs,
                                  const float* __restrict__ cs) {
  const int64_t total = (int64_t)R * C;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int r = (int)(e / C), c = (int)(e % C);
    X[e] *= rs[r] * cs[c];
  }
}

// In-shared-memory Walsh-Hadamard butterflies on Q segments of L2 = 2^lg2
// entries (pair p of stage h = 2^lh: i = (p >> lh) << (lh+1) | (p & (h-1))).
__device__ void fwht_segments(float* x, int lg2, int Q) {
  const int half = 1 << (lg2 - 1);
  const int pairs = half * Q;
  for (int lh = 0; lh < lg2; ++lh) {
    const int h = 1 << lh;
    for (int p = threadIdx.x; p < pairs; p += blockDim.x) {
      const int i = ((p >> lh) << (lh + 1)) | (p & (h - 1));
      const float a = x[i], b = x[i + h];
      x[i] = a + b;
      x[i + h] = a - b;
    }
    __syncthreads();
  }
}

// y[s L2 + r] = sum_t M[s][t] x[t L2 + r]  (M^T when transpose), in place.
__device__ void mix_segments(float* x, int L2, int Q, const float* __restrict__ M, bool transpose) {
  float v[64];
  for (int r = threadIdx.x; r < L2; r += blockDim.x) {
    for (int t = 0; t < Q; ++t) v[t] = x[t * L2 + r];
    for (int s = 0; s < Q; ++s) {
      float acc = 0.f;
      for (int t = 0; t < Q; ++t) acc = fmaf(transpose ? M[t * Q + s] : M[s * Q + t], v[t], acc);
      x[s * L2 + r] = acc;
    }
  }
  __syncthreads();
}

// One row per CTA.  forward: x <- T D (rs[r] cs[c] x);  inverse: x <- rs[r] cs[c] D T^T x.
__global__ void __launch_bounds__(RT_THREADS)
row_transform_kernel(float* __restrict__ X, int R, int C, const float* __restrict__ rs,
                     const float* __restrict__ cs, const int8_t* __restrict__ sign, int L2, int Q,
                     const float* __restrict__ M, int inverse) {
  extern __shared__ float x[];
  const int r = blockIdx.x;
  if (r >= R) return;
  float* row = X + (int64_t)r * C;
  const float rsc = rs ? rs[r] : 1.f;
  const float norm = rsqrtf((float)L2);
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    float v = row[c];
    if (!inverse) v = v * (rsc * (cs ? cs[c] : 1.f)) * (float)sign[c];
    x[c] = v;
  }
  __syncthreads();
  if (inverse && Q > 1) mix_segments(x, L2, Q, M, true);
  fwht_segments(x, 31 - __clz(L2), Q);
  if (!inverse && Q > 1) mix_segments(x, L2, Q, M, false);
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    float v = x[c] * norm;
    if (inverse) v = v * (float)sign[c] * (rsc * (cs ? cs[c] : 1.f));
    row[c] = v;
  }
}

// Column pass, step 2: rows {s L2 + r : s < Q} mixed by M (or M^T), 64 columns per CTA.
__global__ void __launch_bounds__(64)
col_mix_kernel(float* __restrict__ X, int C, int L2, int Q, const float* __restrict__ M,
               int transpose) {
  __shared__ float v[64][65];
  __shared__ float Ms[64 * 64];
  const int r = blockIdx.y, c = blockIdx.x * 64 + threadIdx.x;
  for (int e = threadIdx.x; e < Q * Q; e += blockDim.x) Ms[e] = M[e];
  for (int t = 0; t < Q; ++t) v[t][threadIdx.x] = (c < C) ? X[(int64_t)(t * L2 + r) * C + c] : 0.f;
  __syncthreads();
  if (c >= C) return;
  for (int s = 0; s < Q; ++s) {
    float acc = 0.f;
    for (int t = 0; t < Q; ++t) acc = fmaf(transpose ? Ms[t * Q + s] : Ms[s * Q + t], v[t][threadIdx.x], acc);
    X[(int64_t)(s * L2 + r) * C + c] = acc;
  }
}

// Row pass, fast path (no odd factor): one segment of L2 = 128 E entries of
// two rows per CTA, Walsh-Hadamard butterflies in registers.  Thread t first
// holds entries t + 128 k (coalesced loads; the row scale and the column
// factor cf = column scale x sign fused, cf loaded once for both rows), which
// makes the stages with h >= 128 thread-local; one padded shared-memory
// transpose gives it entries E t .. E t + E - 1 for the stages h < E; the
// stages E <= h < 128 pair thread t with t ^ (h / E) by shuffles.
template <int E>
__global__ void __launch_bounds__(128)
row_fht_kernel(float* __restrict__ X, int R, int C, const float* __restrict__ rs,
               const float* __restrict__ cf, int inverse) {
  constexpr int L2 = 128 * E;
  constexpr int RPC = 2;                      // rows per CTA
  __shared__ float sm[RPC][L2 + L2 / 32];
  const int t = threadIdx.x;
  const int c0 = blockIdx.y * L2;
  const int64_t r0 = (int64_t)blockIdx.x * RPC;
  const int nr = (R - r0) < RPC ? (int)(R - r0) : RPC;
  float v[RPC][E];
  float f[E];
#pragma unroll
  for (int k = 0; k < E; ++k) f[k] = cf[c0 + t + 128 * k];
#pragma unroll
  for (int q = 0; q < RPC; ++q) {
    if (q < nr) {
      const float* base = X + (r0 + q) * C + c0;
      const float rsc = rs ? rs[r0 + q] : 1.f;
#pragma unroll
      for (int k = 0; k < E; ++k) {
        const float x = base[t + 128 * k];
        v[q][k] = inverse ? x : x * (rsc * f[k]);
      }
    } else {
#pragma unroll
      for (int k = 0; k < E; ++k) v[q][k] = 0.f;
    }
  }
#pragma unroll
  for (int q = 0; q < RPC; ++q) {
#pragma unroll
    for (int h = 1; h < E; h <<= 1)
#pragma unroll
      for (int k = 0; k < E; ++k)
        if (!(k & h)) {
          const float a = v[q][k], b = v[q][k + h];
          v[q][k] = a + b;
          v[q][k + h] = a - b;
        }
#pragma unroll
    for (int k = 0; k < E; ++k) {
      const int i = t + 128 * k;
      sm[q][i + (i >> 5)] = v[q][k];
    }
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < RPC; ++q) {
#pragma unroll
    for (int k = 0; k < E; ++k) {
      const int i = E * t + k;
      v[q][k] = sm[q][i + (i >> 5)];
    }
#pragma unroll
    for (int h = 1; h < E; h <<= 1)
#pragma unroll
      for (int k = 0; k < E; ++k)
        if (!(k & h)) {
          const float a = v[q][k], b = v[q][k + h];
          v[q][k] = a + b;
          v[q][k + h] = a - b;
        }
#pragma unroll
    for (int m = 1; m < 128 / E; m <<= 1) {
      const bool upper = (t & m) != 0;
#pragma unroll
      for (int k = 0; k < E; ++k) {
        const float o = __shfl_xor_sync(0xffffffffu, v[q][k], m);
        v[q][k] = upper ? (o - v[q][k]) : (v[q][k] + o);
      }
    }
  }
  // back to entries t + 128 k through shared memory, so that every store
  // instruction writes 128 contiguous bytes per warp
  __syncthreads();
#pragma unroll
  for (int q = 0; q < RPC; ++q)
#pragma unroll
    for (int k = 0; k < E; ++k) {
      const int i = E * t + k;
      sm[q][i + (i >> 5)] = v[q][k];
    }
  __syncthreads();
  const float norm = rsqrtf((float)L2);
#pragma unroll
  for (int q = 0; q < RPC; ++q) {
    if (q >= nr) break;
    float* base = X + (r0 + q) * C + c0;
    const float rsc = rs ? rs[r0 + q] : 1.f;
#pragma unroll
    for (int k = 0; k < E; ++k) {
      const int i = t + 128 * k;
      float o = sm[q][i + (i >> 5)] * norm;
      if (inverse) o *= rsc * f[k];
      base[i] = o;
    }
  }
}

// Row pass for widths with an odd factor (forward only), one row per CTA:
// segment g of the row (L2 = 128 E entries) belongs to threads
// [128 g, 128 g + 128), which transform it in registers exactly as
// row_fht_kernel does (scaling and signs fused into the load), then leave it
// in shared memory; after one barrier every thread mixes the Q segments at
// its positions r (y[s L2 + r] = sum_t M[s][t] x[t L2 + r]) straight into
// global memory.  One read and one write of the row, like the power-of-two
// rows.
template <int Q, int E>
__global__ void __launch_bounds__(128 * Q, 1)
row_fht_mix_kernel(float* __restrict__ X, int C, const float* __restrict__ rs,
                   const float* __restrict__ cf, const float* __restrict__ M) {
  constexpr int L2 = 128 * E;
  constexpr int LD = L2 + L2 / 32;            // padded segment in shared memory
  extern __shared__ float sm[];               // [Q][LD], then M (Q x Q)
  float* Ms = sm + Q * LD;
  const int tid = threadIdx.x, g = tid >> 7, t = tid & 127;
  const int64_t row = blockIdx.x;
  float* base = X + row * C;
  if (tid < Q * Q) Ms[tid] = M[tid];
  {
    const int c0 = g * L2;
    const float rsc = rs ? rs[row] : 1.f;
    float v[E];
#pragma unroll
    for (int k = 0; k < E; ++k) {
      const int c = c0 + t + 128 * k;
      v[k] = base[c] * (rsc * cf[c]);
    }
#pragma unroll
    for (int h = 1; h < E; h <<= 1)
#pragma unroll
      for (int k = 0; k < E; ++k)
        if (!(k & h)) {
          const float a = v[k], b = v[k + h];
          v[k] = a + b;
          v[k + h] = a - b;
        }
    float* seg = sm + g * LD;
#pragma unroll
    for (int k = 0; k < E; ++k) {
      const int i = t + 128 * k;
      seg[i + (i >> 5)] = v[k];
    }
    // the stages E <= h < L2 among the segment's 128 threads: a transpose
    // within the segment (named barrier per segment: 4 warps)
    asm volatile("bar.sync %0, 128;" ::"r"(g + 1) : "memory");
#pragma unroll
    for (int k = 0; k < E; ++k) {
      const int i = E * t + k;
      v[k] = seg[i + (i >> 5)];
    }
#pragma unroll
    for (int h = 1; h < E; h <<= 1)
#pragma unroll
      for (int k = 0; k < E; ++k)
        if (!(k & h)) {
          const float a = v[k], b = v[k + h];
          v[k] = a + b;
          v[k + h] = a - b;
        }
#pragma unroll
    for (int m = 1; m < 128 / E; m <<= 1) {
      const bool upper = (t & m) != 0;
#pragma unroll
      for (int k = 0; k < E; ++k) {
        const float o = __shfl_xor_sync(0xffffffffu, v[k], m);
        v[k] = upper ? (o - v[k]) : (v[k] + o);
      }
    }
    asm volatile("bar.sync %0, 128;" ::"r"(g + 1) : "memory");
#pragma unroll
    for (int k = 0; k < E; ++k) {
      const int i = E * t + k;
      seg[i + (i >> 5)] = v[k];
    }
  }
  __syncthreads();
  const float norm = rsqrtf((float)L2);
  for (int r = tid; r < L2; r += 128 * Q) {
    const int ri = r + (r >> 5);
    float x[Q];
#pragma unroll
    for (int u = 0; u < Q; ++u) x[u] = sm[u * LD + ri];
#pragma unroll
    for (int s2 = 0; s2 < Q; ++s2) {
      float acc = 0.f;
#pragma unroll
      for (int u = 0; u < Q; ++u) acc = fmaf(Ms[s2 * Q + u], x[u], acc);
      base[s2 * L2 + r] = acc * norm;
    }
  }
}

// Column pass, last launch for heights with an odd factor (forward only): the
// Walsh-Hadamard factor H_{NR} on the rows with stride st (as
// col_fht_reg_kernel) for each of the Q segments, then the Q-mix across the
// segments, in one read and one write.  Warp s of the CTA owns segment s
// (32 columns, coalesced 128-byte row pieces); the transformed values meet in
// shared memory for the mix.  first: the row signs before (when this launch
// is the whole Walsh-Hadamard part); the 1/sqrt(L2) normalisation is applied.
template <int Q, int LG>
__global__ void __launch_bounds__(32 * Q)
col_fht_mix_kernel(float* __restrict__ X, int C, int L2, int st, const int8_t* __restrict__ sign,
                   const float* __restrict__ M, int first) {
  constexpr int NR = 1 << LG;
  extern __shared__ float dyn[];
  float(*buf)[NR][33] = reinterpret_cast<float(*)[NR][33]>(dyn);   // [Q][NR][33]
  float* Ms = dyn + Q * NR * 33;
  const int lane = threadIdx.x & 31, s = threadIdx.x >> 5;
  if (threadIdx.x < Q * Q) Ms[threadIdx.x] = M[threadIdx.x];
  const int c = blockIdx.x * 32 + lane;
  const bool live = c < C;
  const int g = blockIdx.y;
  const int hi = g / st, lo = g % st;
  const int64_t r0 = (int64_t)hi * st * NR + lo;      // row within the segment
  const int64_t step = (int64_t)st * C;
  float v[NR];
  {
    const float* p = X + ((int64_t)s * L2 + r0) * C + (live ? c : 0);
#pragma unroll
    for (int j = 0; j < NR; ++j) {
      v[j] = live ? *p : 0.f;
      p += step;
    }
  }
  if (first) {
    const int8_t* sg = sign + (int64_t)s * L2 + r0;
#pragma unroll
    for (int j = 0; j < NR; ++j) v[j] = (sg[(int64_t)j * st] < 0) ? -v[j] : v[j];
  }
#pragma unroll
  for (int h = 1; h < NR; h <<= 1)
#pragma unroll
    for (int j = 0; j < NR; ++j)
      if (!(j & h)) {
        const float a = v[j], b = v[j + h];
        v[j] = a + b;
        v[j + h] = a - b;
      }
#pragma unroll
  for (int j = 0; j < NR; ++j) buf[s][j][lane] = v[j];
  __syncthreads();
  if (!live) return;
  const float norm = rsqrtf((float)L2);
  float* p = X + ((int64_t)s * L2 + r0) * C + c;
#pragma unroll 4
  for (int j = 0; j < NR; ++j) {
    float acc = 0.f;
#pragma unroll
    for (int u = 0; u < Q; ++u) acc = fmaf(Ms[s * Q + u], buf[u][j][lane], acc);
    *p = acc * norm;
    p += step;
  }
}

// cf[c] = cs[c] sign[c] (cs may be null: 1).
__global__ void col_factor_kernel(const float* __restrict__ cs, const int8_t* __restrict__ sign,
                                  int C, float* __restrict__ cf) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c < C) cf[c] = (cs ? cs[c] : 1.f) * (float)sign[c];
}

// Column pass, one factor H_{NR} (NR = 2^LG <= 64) of the Walsh-Hadamard
// transform along rows, in registers: each thread owns one column and the
// NR rows row(s) = seg L2 + hi (st NR) + lo + s st, s < NR, of one group
// (coalesced row segments, no shared memory).  With st = 1 the groups are
// NR consecutive rows; with st = 2^a and NR = L2 / st the rows with stride
// st, so the two launches (I (x) H_{2^a}) then (H_{L2/2^a} (x) I) make the
// whole H_{L2}.  first: signs of the rows before (forward); last: the
// 1/sqrt(L2) normalisation and, when inverse, the signs after.
template <int LG>
__global__ void __launch_bounds__(128)
col_fht_reg_kernel(float* __restrict__ X, int C, int L2, int st, const int8_t* __restrict__ sign,
                   int first, int last, int inverse) {
  constexpr int NR = 1 << LG;
  const int c = blockIdx.x * 128 + threadIdx.x;
  if (c >= C) return;
  const int groups_per_seg = L2 / NR;
  const int seg = blockIdx.y / groups_per_seg, g = blockIdx.y % groups_per_seg;
  const int hi = g / st, lo = g % st;
  const int64_t r0 = (int64_t)seg * L2 + (int64_t)hi * st * NR + lo;
  const int64_t step = (int64_t)st * C;
  float v[NR];
  {
    const float* p = X + r0 * C + c;
#pragma unroll
    for (int s = 0; s < NR; ++s) {
      v[s] = *p;
      p += step;
    }
  }
  if (first && !inverse) {
    const int8_t* sg = sign + r0;
#pragma unroll
    for (int s = 0; s < NR; ++s) v[s] = (sg[(int64_t)s * st] < 0) ? -v[s] : v[s];
  }
#pragma unroll
  for (int h = 1; h < NR; h <<= 1)
#pragma unroll
    for (int s = 0; s < NR; ++s)
      if (!(s & h)) {
        const float a = v[s], b = v[s + h];
        v[s] = a + b;
        v[s + h] = a - b;
      }
  const float norm = last ? rsqrtf((float)L2) : 1.f;
  if (last && inverse) {
    const int8_t* sg = sign + r0;
#pragma unroll
    for (int s = 0; s < NR; ++s) v[s] = (sg[(int64_t)s * st] < 0) ? -v[s] : v[s];
  }
  float* p = X + r0 * C + c;
#pragma unroll
  for (int s = 0; s < NR; ++s) {
    *p = v[s] * norm;
    p += step;
  }
}

__global__ void __launch_bounds__(1024) sensitivity_kernel(const float* __restrict__ HX, int n,
                                                           const float* __restrict__ HG, int m,
                                                           double* __restrict__ out) {
  // one CTA of 1024 threads: every diagonal entry is a separate cache line,
  // so the loads are spread over as many threads as possible
  __shared__ double sx[1024], sg[1024];
  double a = 0.0, b = 0.0;
#pragma unroll 4
  for (int i = threadIdx.x; i < n; i += blockDim.x) a += (double)HX[(int64_t)i * n + i];
#pragma unroll 4
  for (int i = threadIdx.x; i < m; i += blockDim.x) b += (double)HG[(int64_t)i * m + i];
  sx[threadIdx.x] = a;
  sg[threadIdx.x] = b;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) {
      sx[threadIdx.x] += sx[threadIdx.x + w];
      sg[threadIdx.x] += sg[threadIdx.x + w];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    out[0] = sx[0] * sg[0];
    out[1] = sx[0];
    out[2] = sg[0];
  }
}

size_t a256(size_t b) { return (b + 255) & ~(size_t)255; }

kqh::PerDevice g_row_attr;

int set_attrs() {
  return kqh::smem_attr_once(g_row_attr, row_transform_kernel, 200 * 1024) > 0 ? KRONQ_OK
                                                                                : KRONQ_ERR_CUDA;
}

template <int Q, int E>
int launch_row_fht_mix(float* X, int R, int C, const float* rs, const float* cf, const float* M,
                       cudaStream_t st) {
  constexpr int LD = 128 * E + 4 * E;
  const int smem = (Q * LD + Q * Q) * (int)sizeof(float);
  static kqh::PerDevice attr;
  if (kqh::smem_attr_once(attr, row_fht_mix_kernel<Q, E>, smem) <= 0) return KRONQ_ERR_CUDA;
  row_fht_mix_kernel<Q, E><<<R, 128 * Q, smem, st>>>(X, C, rs, cf, M);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

// Apply T D along rows (row pass, with scaling) of an R x C matrix.
int row_pass(float* X, int R, int C, const float* rs, const float* cs, const int8_t* sign,
             const Split& sp, const float* M, int inverse, float* cf, cudaStream_t st,
             bool cf_ready = false) {
  if (sp.Q == 1 && sp.L2 >= 512) {
    if (!cf_ready) {
      col_factor_kernel<<<(C + 255) / 256, 256, 0, st>>>(cs, sign, C, cf);
      KQ_CHECK_LAUNCH();
    }
    const dim3 g((R + 1) / 2, C / sp.L2);
    switch (sp.L2) {
      case 512: row_fht_kernel<4><<<g, 128, 0, st>>>(X, R, C, rs, cf, inverse); break;
      case 1024: row_fht_kernel<8><<<g, 128, 0, st>>>(X, R, C, rs, cf, inverse); break;
      case 2048: row_fht_kernel<16><<<g, 128, 0, st>>>(X, R, C, rs, cf, inverse); break;
      default: row_fht_kernel<32><<<g, 128, 0, st>>>(X, R, C, rs, cf, inverse); break;
    }
    KQ_CHECK_LAUNCH();
    return KRONQ_OK;
  }
  if (!inverse && (sp.Q == 7 || sp.Q == 2) && (sp.L2 == 2048 || sp.L2 == 4096)) {
    // a factor 7 (widths 14336, 28672) or a second 4096 segment (8192): one
    // fused pass (for Q = 2 the "mix" is the last Walsh-Hadamard stage)
    if (!cf_ready) {
      col_factor_kernel<<<(C + 255) / 256, 256, 0, st>>>(cs, sign, C, cf);
      KQ_CHECK_LAUNCH();
    }
    if (sp.Q == 7)
      return sp.L2 == 4096 ? launch_row_fht_mix<7, 32>(X, R, C, rs, cf, M, st)
                           : launch_row_fht_mix<7, 16>(X, R, C, rs, cf, M, st);
    return sp.L2 == 4096 ? launch_row_fht_mix<2, 32>(X, R, C, rs, cf, M, st)
                         : launch_row_fht_mix<2, 16>(X, R, C, rs, cf, M, st);
  }
  const size_t smem = (size_t)C * sizeof(float);
  if (smem > 200 * 1024) return KRONQ_ERR_UNSUPPORTED;
  row_transform_kernel<<<R, RT_THREADS, smem, st>>>(X, R, C, rs, cs, sign, sp.L2, sp.Q, M, inverse);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

// One launch of col_fht_reg_kernel<lg> over every segment of an R x C matrix.
int col_fht_launch(float* X, int R, int C, int L2, int lg, int stride, const int8_t* sign,
                   int first, int last, int inverse, cudaStream_t st) {
  const dim3 g((C + 127) / 128, R >> lg);
  switch (lg) {
    case 1: col_fht_reg_kernel<1><<<g, 128, 0, st>>>(X, C, L2, stride, sign, first, last, inverse); break;
    case 2: col_fht_reg_kernel<2><<<g, 128, 0, st>>>(X, C, L2, stride, sign, first, last, inverse); break;
    case 3: col_fht_reg_kernel<3><<<g, 128, 0, st>>>(X, C, L2, stride, sign, first, last, inverse); break;
    case 4: col_fht_reg_kernel<4><<<g, 128, 0, st>>>(X, C, L2, stride, sign, first, last, inverse); break;
    case 5: col_fht_reg_kernel<5><<<g, 128, 0, st>>>(X, C, L2, stride, sign, first, last, inverse); break;
    case 6: col_fht_reg_kernel<6><<<g, 128, 0, st>>>(X, C, L2, stride, sign, first, last, inverse); break;
    default: return KRONQ_ERR_UNSUPPORTED;
  }
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

// Apply T D along columns of an R x C matrix (R = Q * L2): the Hadamard part
// as H_{2^a} within groups of 2^a consecutive rows, then (when L2 > 64)
// H_{L2 / 2^a} across them; the odd factor as a Q x Q mix of the segments.
template <int Q, int LG>
int col_fht_mix_launch_lg(float* X, int C, int L2, int stride, const int8_t* sign, const float* M,
                          int first, cudaStream_t st) {
  const int smem = (Q * (1 << LG) * 33 + Q * Q) * (int)sizeof(float);
  static kqh::PerDevice attr;
  if (kqh::smem_attr_once(attr, col_fht_mix_kernel<Q, LG>, smem) <= 0) return KRONQ_ERR_CUDA;
  const dim3 g((C + 31) / 32, L2 >> LG);
  col_fht_mix_kernel<Q, LG><<<g, 32 * Q, smem, st>>>(X, C, L2, stride, sign, M, first);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

template <int Q>
int col_fht_mix_launch(float* X, int C, int L2, int lg, int stride, const int8_t* sign,
                       const float* M, int first, cudaStream_t st) {
  switch (lg) {
    case 5: return col_fht_mix_launch_lg<Q, 5>(X, C, L2, stride, sign, M, first, st);
    case 6: return col_fht_mix_launch_lg<Q, 6>(X, C, L2, stride, sign, M, first, st);
    default: return KRONQ_ERR_UNSUPPORTED;
  }
}

int col_pass(float* X, int R, int C, const int8_t* sign, const Split& sp, const float* M,
             int inverse, cudaStream_t st) {
  if (!inverse && (sp.Q == 7 || sp.Q == 2) && (sp.L2 == 2048 || sp.L2 == 4096)) {
    // heights 14336, 28672 (factor 7) and 8192 (two 4096 segments): H_64 on
    // consecutive rows, then H_{L2/64} with stride 64 fused with the mix of
    // the segments
    const int k2 = 31 - __builtin_clz((unsigned)sp.L2);
    int s = col_fht_launch(X, R, C, sp.L2, 6, 1, sign, 1, 0, 0, st);
    if (s != KRONQ_OK) return s;
    return sp.Q == 7 ? col_fht_mix_launch<7>(X, C, sp.L2, k2 - 6, 64, sign, M, 0, st)
                     : col_fht_mix_launch<2>(X, C, sp.L2, k2 - 6, 64, sign, M, 0, st);
  }
  if (inverse && sp.Q > 1) {
    col_mix_kernel<<<dim3((C + 63) / 64, sp.L2), 64, 0, st>>>(X, C, sp.L2, sp.Q, M, 1);
    KQ_CHECK_LAUNCH();
  }
  const int k2 = 31 - __builtin_clz((unsigned)sp.L2);
  const int a = k2 < 6 ? k2 : 6, b = k2 - a;
  int s = col_fht_launch(X, R, C, sp.L2, a, 1, sign, 1, b == 0, inverse, st);
  if (s != KRONQ_OK) return s;
  if (b > 0) {
    s = col_fht_launch(X, R, C, sp.L2, b, 1 << a, sign, 0, 1, inverse, st);
    if (s != KRONQ_OK) return s;
  }
  if (!inverse && sp.Q > 1) {
    col_mix_kernel<<<dim3((C + 63) / 64, sp.L2), 64, 0, st>>>(X, C, sp.L2, sp.Q, M, 0);
    KQ_CHECK_LAUNCH();
  }
  return KRONQ_OK;
}

}  // namespace

size_t kq_biip_ws(int64_t m, int64_t n) {
  return a256((size_t)(m + n) * sizeof(double)) + 2 * a256((size_t)(m + n) * sizeof(float)) +
         2 * a256(64 * 64 * sizeof(float));
}

int kq_sensitivity(const float* HX, int64_t n, const float* HG, int64_t m, double* out,
                   cudaStream_t st) {
  if (!HX || !HG || !out || n <= 0 || m <= 0 || n > INT32_MAX || m > INT32_MAX)
    return KRONQ_ERR_INVALID_ARG;
  sensitivity_kernel<<<1, 1024, 0, st>>>(HX, (int)n, HG, (int)m, out);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

int kq_biip_rotate(float* W, int64_t m64, int64_t n64, float* HX, float* HG, const int8_t* su,
                   const int8_t* sv, float alpha, int mode, int inverse, float* SX, float* SG,
                   void* ws, size_t ws_bytes, cudaStream_t st) {
  if (mode < 0 || mode > 3 || (inverse != 0 && inverse != 1)) return KRONQ_ERR_INVALID_ARG;
  if (!W || !su || !sv || !SX || !SG || m64 <= 0 || n64 <= 0) return KRONQ_ERR_INVALID_ARG;
  if (!inverse && (!HX || !HG)) return KRONQ_ERR_INVALID_ARG;
  if (!(alpha >= 0.f)) return KRONQ_ERR_INVALID_ARG;
  if (m64 % 16 || n64 % 16) return KRONQ_ERR_INVALID_ARG;
  if (m64 > 65536 || n64 > 65536) return KRONQ_ERR_UNSUPPORTED;
  Split spm, spn;
  if (!split_width(m64, spm) || !split_width(n64, spn)) return KRONQ_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < kq_biip_ws(m64, n64) || !kqh::aligned(ws, 256)) return KRONQ_ERR_WORKSPACE;
  int st0 = set_attrs();
  if (st0 != KRONQ_OK) return st0;
  const int m = (int)m64, n = (int)n64;
  const bool in_s = mode == 0 || mode == 3, out_s = mode == 0 || mode == 2;
  const bool in_r = mode != 2, out_r = mode != 3;

  uint8_t* w = static_cast<uint8_t*>(ws);
  double* cn = reinterpret_cast<double*>(w);
  double* rn = cn + n;
  w += a256((size_t)(m + n) * sizeof(double));
  float* rSX = reinterpret_cast<float*>(w);
  float* rSG = rSX + n;
  w += a256((size_t)(m + n) * sizeof(float));
  float* cf = reinterpret_cast<float*>(w);      // column factors of a row pass
  w += a256((size_t)(m + n) * sizeof(float));
  float* Mn = reinterpret_cast<float*>(w);
  w += a256(64 * 64 * sizeof(float));
  float* Mm = reinterpret_cast<float*>(w);

  if (spn.Q > 1) { make_mix_kernel<<<1, 256, 0, st>>>(Mn, spn.q, spn.k1); KQ_CHECK_LAUNCH(); }
  if (spm.Q > 1) { make_mix_kernel<<<1, 256, 0, st>>>(Mm, spm.q, spm.k1); KQ_CHECK_LAUNCH(); }
  const int sms = kqh::num_sms();

  if (inverse) {
    recip_kernel<<<(n + 255) / 256, 256, 0, st>>>(SX, rSX, n);
    KQ_CHECK_LAUNCH();
    recip_kernel<<<(m + 255) / 256, 256, 0, st>>>(SG, rSG, m);
    KQ_CHECK_LAUNCH();
    if (out_r) {
      int s = col_pass(W, m, n, su, spm, Mm, 1, st);
      if (s) return s;
    }
    if (in_r) {
      int s = row_pass(W, m, n, rSG, rSX, sv, spn, Mn, 1, cf, st);
      if (s) return s;
    } else {
      scale_only_kernel<<<4 * sms, 256, 0, st>>>(W, m, n, rSG, rSX);
      KQ_CHECK_LAUNCH();
    }
    return KRONQ_OK;
  }

  // ---- rescale factors
  if (cudaMemsetAsync(cn, 0, (size_t)n * sizeof(double), st) != cudaSuccess) return KRONQ_ERR_CUDA;
  if (in_s) {
    colnorm_kernel<<<dim3((n + 255) / 256, (m + 31) / 32), 256, 0, st>>>(W, m, n, cn);
    KQ_CHECK_LAUNCH();
  }
  scale_from_diag_kernel<<<(n + 255) / 256, 256, 0, st>>>(HX, n, cn, alpha, SX, rSX, in_s);
  KQ_CHECK_LAUNCH();
  if (out_s) {
    rownorm_kernel<<<(m + 7) / 8, 256, 0, st>>>(W, m, n, SX, rn);
    KQ_CHECK_LAUNCH();
  }
  scale_from_diag_kernel<<<(m + 255) / 256, 256, 0, st>>>(HG, m, rn, alpha, SG, rSG, out_s);
  KQ_CHECK_LAUNCH();

  // ---- W' = U (S_G W S_X) V^T
  if (in_r) {
    int s = row_pass(W, m, n, SG, SX, sv, spn, Mn, 0, cf, st);
    if (s) return s;
  } else {
    scale_only_kernel<<<4 * sms, 256, 0, st>>>(W, m, n, SG, SX);
    KQ_CHECK_LAUNCH();
  }
  if (out_r) {
    int s = col_pass(W, m, n, su, spm, Mm, 0, st);
    if (s) return s;
  }
  // ---- H_X' = V S_X^-1 H_X S_X^-1 V^T
  if (in_r) {
    int s = row_pass(HX, n, n, rSX, rSX, sv, spn, Mn, 0, cf, st);
    if (s) return s;
    s = col_pass(HX, n, n, sv, spn, Mn, 0, st);
    if (s) return s;
  } else if (in_s) {
    scale_only_kernel<<<4 * sms, 256, 0, st>>>(HX, n, n, rSX, rSX);
    KQ_CHECK_LAUNCH();
  }
  // ---- H_G' = U S_G^-1 H_G S_G^-1 U^T
  if (out_r) {
    int s = row_pass(HG, m, m, rSG, rSG, su, spm, Mm, 0, cf, st);
    if (s) return s;
    s = col_pass(HG, m, m, su, spm, Mm, 0, st);
    if (s) return s;
  } else if (out_s) {
    scale_only_kernel<<<4 * sms, 256, 0, st>>>(HG, m, m, rSG, rSG);
    KQ_CHECK_LAUNCH();
  }
  return KRONQ_OK;
}

// ---------------------------------------------------------------------------
// Vectors through one side of BiIP (the deployment path): each row x of the
// R x C matrix X becomes V diag(1/S) x (forward) or diag(1/S) V^T x
// (inverse), V = T_C D (rotate = 1), or only the scaling (rotate = 0).
// Scratch: kq_vec_transform_ws(C) bytes.
size_t kq_vec_transform_ws(int64_t C) {
  return 2 * a256((size_t)C * sizeof(float)) + a256(64 * 64 * sizeof(float));
}

namespace {
// rS[c] = 1 / S[c] and cf[c] = sign[c] / S[c] (the row pass's column factor).
__global__ void recip_factor_kernel(const float* __restrict__ S, const int8_t* __restrict__ sign,
                                    int C, float* __restrict__ rS, float* __restrict__ cf) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c < C) {
    const float r = 1.f / S[c];
    rS[c] = r;
    if (sign) cf[c] = r * (float)sign[c];
  }
}

__global__ void vec_scale_kernel(float* __restrict__ X, int64_t R, int C, const float* __restrict__ rS) {
  const int64_t total = R * C;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x)
    X[e] *= rS[e % C];
}
}  // namespace

int kq_vec_transform(float* X, int64_t R, int64_t C, const float* S, const int8_t* sign, int rotate,
                     int inverse, void* ws, cudaStream_t st) {
  if (!X || !S || (rotate && !sign) || R <= 0 || C <= 0) return KRONQ_ERR_INVALID_ARG;
  Split sp;
  if (!split_width(C, sp) || C > 65536 || R > (1 << 30)) return KRONQ_ERR_UNSUPPORTED;
  int s0 = set_attrs();
  if (s0 != KRONQ_OK) return s0;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* rS = reinterpret_cast<float*>(w);
  w += a256((size_t)C * sizeof(float));
  float* cf = reinterpret_cast<float*>(w);
  w += a256((size_t)C * sizeof(float));
  float* M = reinterpret_cast<float*>(w);
  recip_factor_kernel<<<(int)((C + 255) / 256), 256, 0, st>>>(S, rotate ? sign : nullptr, (int)C,
                                                               rS, cf);
  KQ_CHECK_LAUNCH();
  if (!rotate) {
    vec_scale_kernel<<<2 * kqh::num_sms(), 256, 0, st>>>(X, R, (int)C, rS);
    KQ_CHECK_LAUNCH();
    return KRONQ_OK;
  }
  if (sp.Q > 1) {
    make_mix_kernel<<<1, 256, 0, st>>>(M, sp.q, sp.k1);
    KQ_CHECK_LAUNCH();
  }
  return row_pass(X, (int)R, (int)C, nullptr, rS, sign, sp, M, inverse, cf, st, /*cf_ready=*/true);
}


// ---------------------------------------------------------------------------
// The input side of BiIP applied to another n x n matrix built from input
// vectors (the drift covariance of the asymmetric calibration):
// A <- V S_X^-1 A S_X^-1 V^T with the S_X and V of H_X; mode as in
// kq_biip_rotate (the output side is not touched).
int kq_biip_rotate_input(float* A, int64_t n64, const float* SX, const int8_t* sv, int mode,
                         void* ws, size_t ws_bytes, cudaStream_t st) {
  if (mode < 0 || mode > 3 || !A || !SX || !sv || n64 <= 0) return KRONQ_ERR_INVALID_ARG;
  if (n64 % 16) return KRONQ_ERR_INVALID_ARG;
  if (n64 > 65536) return KRONQ_ERR_UNSUPPORTED;
  Split spn;
  if (!split_width(n64, spn)) return KRONQ_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < kq_biip_ws(n64, n64) || !kqh::aligned(ws, 256)) return KRONQ_ERR_WORKSPACE;
  int s0 = set_attrs();
  if (s0 != KRONQ_OK) return s0;
  const int n = (int)n64;
  const bool in_s = mode == 0 || mode == 3, in_r = mode != 2;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* rSX = reinterpret_cast<float*>(w);
  w += a256((size_t)n * sizeof(float));
  float* cf = reinterpret_cast<float*>(w);
  w += a256((size_t)n * sizeof(float));
  float* Mn = reinterpret_cast<float*>(w);
  recip_kernel<<<(n + 255) / 256, 256, 0, st>>>(SX, rSX, n);
  KQ_CHECK_LAUNCH();
  if (in_r) {
    if (spn.Q > 1) {
      make_mix_kernel<<<1, 256, 0, st>>>(Mn, spn.q, spn.k1);
      KQ_CHECK_LAUNCH();
    }
    int s = row_pass(A, n, n, in_s ? rSX : nullptr, in_s ? rSX : nullptr, sv, spn, Mn, 0, cf, st);
    if (s) return s;
    return col_pass(A, n, n, sv, spn, Mn, 0, st);
  }
  if (in_s) {
    scale_only_kernel<<<4 * kqh::num_sms(), 256, 0, st>>>(A, n, n, rSX, rSX);
    KQ_CHECK_LAUNCH();
  }
  return KRONQ_OK;
}
