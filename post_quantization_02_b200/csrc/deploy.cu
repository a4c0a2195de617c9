// Deployment matvec of a quantized layer: y = W_hat x from the packed codes,
// with the BiIP transforms applied to the vectors online.
//
// KronQ README (GitHub), deploy path: a fused dequant + BiIP matvec serves
// the packed int4 / int2 layer at batch-1 decode.  KronQ summary (hyper.ai),
// "Method", Eqs. 11-12: W' = U S_G W S_X V^T, so the layer the codes stand
// for is W_hat = S_G^-1 U^T W_hat' V S_X^-1 and
//   y = S_G^-1 U^T ( W_hat' ( V S_X^-1 x ) ).
// Three steps on the stream: x2 = V S_X^-1 x (row transform of the batch),
// y1 = W_hat' x2 (dequant_matvec_kernel, the HBM-bound step: every packed
// byte is read once), y = S_G^-1 U^T y1 (inverse row transform in place).
// (One fused launch -- x transformed per CTA in shared memory, y by the last
// CTA to finish -- measured slower: 22.5 against 19.8 us per 4096 x 4096
// layer, its shared-memory transforms being latency-bound.)
//
// dequant_matvec_kernel: x2 staged in shared memory (float4 blocks with one
// pad block per lane-run, so that the 8 lanes of each LDS.128 phase hit
// distinct banks); one warp per row at a time; each lane streams one uint4
// of packed codes per step (32 lanes x 16 B = 512 B per load instruction,
// read-only and not kept in L1); a code c becomes the float c - zero
// exactly as float(0x4B000000 | c) - (2^23 + zero).
#include "common.cuh"

size_t kq_vec_transform_ws(int64_t C);
int kq_vec_transform(float* X, int64_t R, int64_t C, const float* S, const int8_t* sign, int rotate,
                     int inverse, void* ws, cudaStream_t st);

namespace {

constexpr int MV_THREADS = 512;

KQ_DEV uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// One lane's share of a 128-uint4 chunk of row i: q[u] holds uint4 v0 + lane + 32 u.
template <int BITS, int BATCH>
__device__ __forceinline__ void chunk_dot(const uint4 (&q)[4], int v0, int lane, int vpr, int64_t i,
                                          int G, int lg_group, const float* __restrict__ scales,
                                          const uint8_t* __restrict__ zeros, const float4* xs4,
                                          int ld4, float s_row, float kz_row, float (&acc)[BATCH]) {
  constexpr int CPW = 32 / BITS, CPL = 4 * CPW, F4L = CPL / 4;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int v = v0 + lane + 32 * u;
    if (v >= vpr) break;
    const uint32_t wv[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
    const float4* xb = xs4 + v * (F4L + 1);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float s = s_row, kz = kz_row;
      if (G > 1) {
        const int g = (v * CPL + k * CPW) >> lg_group;
        s = scales[i * G + g];
        kz = -(8388608.f + (float)zeros[i * G + g]);
      }
      float p[BATCH];
#pragma unroll
      for (int b = 0; b < BATCH; ++b) p[b] = 0.f;
#pragma unroll
      for (int c4 = 0; c4 < CPW / 4; ++c4) {
        float cz[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const uint32_t code = (wv[k] >> ((4 * c4 + t) * BITS)) & MASK;
          cz[t] = __fadd_rn(__uint_as_float(0x4B000000u | code), kz);   // code - zero, exact
        }
#pragma unroll
        for (int b = 0; b < BATCH; ++b) {
          const float4 xv = xb[b * ld4 + k * (CPW / 4) + c4];
          p[b] = fmaf(cz[0], xv.x, p[b]);
          p[b] = fmaf(cz[1], xv.y, p[b]);
          p[b] = fmaf(cz[2], xv.z, p[b]);
          p[b] = fmaf(cz[3], xv.w, p[b]);
        }
      }
#pragma unroll
      for (int b = 0; b < BATCH; ++b) acc[b] = fmaf(s, p[b], acc[b]);
    }
  }
}

// The warp's first chunk is requested before x2 is staged (the two latencies
// overlap); afterwards the next chunk (of this row or the warp's next row)
// is always in flight while the current one is consumed.
template <int BITS, int BATCH>
__global__ void __launch_bounds__(MV_THREADS)
dequant_matvec_kernel(const uint4* __restrict__ packed, int m, int n, int lg_group, int G,
                      const float* __restrict__ scales, const uint8_t* __restrict__ zeros,
                      const float* __restrict__ x2, float* __restrict__ y) {
  constexpr int CPL = 4 * (32 / BITS);   // codes per lane per uint4
  constexpr int F4L = CPL / 4;           // float4 blocks per lane run (8 or 16)
  extern __shared__ float4 xs4[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  const int vpr = n / CPL;               // uint4 per row
  const int stride = gridDim.x * nw;
  int i = blockIdx.x * nw + warp;
  uint4 q[4];
  if (i < m) {
    const uint4* pr = packed + (int64_t)i * vpr;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int v = lane + 32 * u;
      q[u] = v < vpr ? ld_stream(pr + v) : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  const int nb4 = n / 4;
  const int ld4 = nb4 + nb4 / F4L;       // one pad block after every lane run
  {
    const float4* src = reinterpret_cast<const float4*>(x2);
    for (int e = threadIdx.x; e < BATCH * nb4; e += blockDim.x) {
      const int b = e / nb4, qq = e - b * nb4;
      xs4[b * ld4 + qq + qq / F4L] = src[e];
    }
  }
  __syncthreads();
  for (; i < m; i += stride) {
    float acc[BATCH];
#pragma unroll
    for (int b = 0; b < BATCH; ++b) acc[b] = 0.f;
    const float s_row = scales[(int64_t)i * G];
    const float kz_row = -(8388608.f + (float)zeros[(int64_t)i * G]);
    for (int v0 = 0; v0 < vpr; v0 += 128) {
      uint4 nq[4];
      const bool more = v0 + 128 < vpr;
      const int ni = more ? i : i + stride, nv0 = more ? v0 + 128 : 0;
#pragma unroll
      for (int u = 0; u < 4; ++u) nq[u] = make_uint4(0u, 0u, 0u, 0u);
      if (ni < m) {
        const uint4* pn = packed + (int64_t)ni * vpr;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int v = nv0 + lane + 32 * u;
          if (v < vpr) nq[u] = ld_stream(pn + v);
        }
      }
      chunk_dot<BITS, BATCH>(q, v0, lane, vpr, i, G, lg_group, scales, zeros, xs4, ld4, s_row,
                             kz_row, acc);
#pragma unroll
      for (int u = 0; u < 4; ++u) q[u] = nq[u];
    }
#pragma unroll
    for (int b = 0; b < BATCH; ++b) {
      float a = acc[b];
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0) y[(int64_t)b * m + i] = a;
    }
  }
}

size_t a256(size_t b) { return (b + 255) & ~(size_t)255; }

template <int BITS, int BATCH>
int launch_mv(const uint32_t* packed, int m, int n, int lg_group, int G, const float* scales,
              const uint8_t* zeros, const float* x2, float* y, cudaStream_t st) {
  constexpr int F4L = (32 / BITS);
  const int nb4 = n / 4;
  const size_t smem = (size_t)BATCH * (nb4 + nb4 / F4L) * sizeof(float4);
  if (smem > 200 * 1024) return KRONQ_ERR_UNSUPPORTED;
  static kqh::PerDevice attr;
  if (kqh::smem_attr_once(attr, dequant_matvec_kernel<BITS, BATCH>, 200 * 1024) <= 0)
    return KRONQ_ERR_CUDA;
  const int warps = MV_THREADS / 32;
  const int grid = (m + warps - 1) / warps;
  dequant_matvec_kernel<BITS, BATCH><<<grid, MV_THREADS, smem, st>>>(
      reinterpret_cast<const uint4*>(packed), m, n, lg_group, G, scales, zeros, x2, y);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

template <int BITS>
int launch_mv_batch(int batch, const uint32_t* packed, int m, int n, int lg_group, int G,
                    const float* scales, const uint8_t* zeros, const float* x2, float* y,
                    cudaStream_t st) {
  switch (batch) {
    case 1: return launch_mv<BITS, 1>(packed, m, n, lg_group, G, scales, zeros, x2, y, st);
    case 2: return launch_mv<BITS, 2>(packed, m, n, lg_group, G, scales, zeros, x2, y, st);
    case 4: return launch_mv<BITS, 4>(packed, m, n, lg_group, G, scales, zeros, x2, y, st);
    case 8: return launch_mv<BITS, 8>(packed, m, n, lg_group, G, scales, zeros, x2, y, st);
    default: return KRONQ_ERR_UNSUPPORTED;
  }
}

}  // namespace

// Workspace: x2 (batch x n) and the scratch of the vector transforms.
size_t kq_deploy_ws(int64_t m, int64_t n, int64_t batch) {
  if (m <= 0 || n <= 0 || batch <= 0) return 0;
  const int64_t c = m > n ? m : n;
  return a256((size_t)batch * n * sizeof(float)) + kq_vec_transform_ws(c);
}

int kq_deploy_matvec(const uint32_t* packed, int64_t m64, int64_t n64, int bits, int group,
                     const float* scales, const uint8_t* zeros, const float* SX, const float* SG,
                     const int8_t* su, const int8_t* sv, int mode, const float* x, int64_t batch,
                     float* y, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!packed || !scales || !zeros || !SX || !SG || !su || !sv || !x || !y) return KRONQ_ERR_INVALID_ARG;
  if (m64 <= 0 || n64 <= 0 || batch <= 0) return KRONQ_ERR_INVALID_ARG;
  if (bits != 2 && bits != 4) return KRONQ_ERR_UNSUPPORTED;
  if (mode < 0 || mode > 3) return KRONQ_ERR_INVALID_ARG;
  if (group != -1 && group != 32 && group != 64 && group != 128) return KRONQ_ERR_UNSUPPORTED;
  if (n64 % 64 || m64 % 16) return KRONQ_ERR_INVALID_ARG;
  if (batch != 1 && batch != 2 && batch != 4 && batch != 8) return KRONQ_ERR_UNSUPPORTED;
  if (m64 > 65536 || n64 > 65536) return KRONQ_ERR_UNSUPPORTED;
  if (!kqh::aligned(packed, 16) || !kqh::aligned(x, 16) || !kqh::aligned(y, 16) ||
      !kqh::aligned(SX, 16) || !kqh::aligned(SG, 16) || !kqh::aligned(su, 4) || !kqh::aligned(sv, 4))
    return KRONQ_ERR_INVALID_ARG;
  if (!ws || ws_bytes < kq_deploy_ws(m64, n64, batch) || !kqh::aligned(ws, 256))
    return KRONQ_ERR_WORKSPACE;
  const int m = (int)m64, n = (int)n64, B = (int)batch;
  const bool in_r = mode != 2, out_r = mode != 3;   // incoh modes: full, no_rescale, su_only, sv_only
  float* x2 = static_cast<float*>(ws);
  void* tws = static_cast<uint8_t*>(ws) + a256((size_t)batch * n * sizeof(float));
  const int G = group == -1 ? 1 : n / group;
  const int lg = group == -1 ? 30 : 31 - __builtin_clz((unsigned)group);
  if (cudaMemcpyAsync(x2, x, (size_t)batch * n * sizeof(float), cudaMemcpyDeviceToDevice, st) !=
      cudaSuccess)
    return KRONQ_ERR_CUDA;
  int s = kq_vec_transform(x2, batch, n, SX, sv, in_r, 0, tws, st);   // x2 = V S_X^-1 x
  if (s != KRONQ_OK) return s;
  // the dot products stage x2 in shared memory: one batch row at a time when
  // the whole batch does not fit
  const size_t row_smem = (size_t)(n / 4 + n / 4 / (32 / bits)) * 16;
  const int per = (size_t)B * row_smem <= 200 * 1024 ? B : 1;
  for (int b0 = 0; b0 < B; b0 += per) {
    s = bits == 4 ? launch_mv_batch<4>(per, packed, m, n, lg, G, scales, zeros, x2 + (int64_t)b0 * n,
                                       y + (int64_t)b0 * m, st)
                  : launch_mv_batch<2>(per, packed, m, n, lg, G, scales, zeros, x2 + (int64_t)b0 * n,
                                       y + (int64_t)b0 * m, st);
    if (s != KRONQ_OK) return s;
  }
  return kq_vec_transform(y, batch, m, SG, su, out_r, 1, tws, st);   // y = S_G^-1 U^T y1
}
