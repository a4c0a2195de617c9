// fp32-accurate products on the 5th-generation tensor cores (tcgen05.mma
// kind::tf32) by a three-term split, shared by the lazy block update and
// the inverse-Cholesky updates.
//
// A tf32 operand keeps 10 explicit mantissa bits.  Each fp32 x is written as
// x = hi + lo with hi = x with its low 13 mantissa bits cleared (exactly a
// tf32 value, so the tensor core reads it unchanged whatever its own
// conversion does) and lo = x - hi (exact in fp32).  Then
//   A B ~ A_hi B_hi + A_hi B_lo + A_lo B_hi
// with the dropped A_lo B_lo term ~2^-22 relative, and fp32 accumulation.
//
// Operand tiles are K-major with the 128-byte swizzle: rows of 32 fp32 K
// values, 8-row atoms 1024 bytes apart (the layout a TMA box of 32 x rows
// fp32 with CU_TENSOR_MAP_SWIZZLE_128B writes).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace kq {
namespace tf32x3 {

constexpr int KC = 32;  // fp32 K values per 128-byte swizzle row

// kind::tf32, fp32 accumulate, A and B K-major, M = 128, N = 128
constexpr uint32_t kIdesc128 = (1u << 4) | (2u << 7) | (2u << 10) | (0u << 15) | (0u << 16) |
                               ((uint32_t)(128 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);

KQ_DEV void mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kIdesc128), "r"(accumulate)
      : "memory");
}

// Byte address inside a tile of 128-byte rows written with the 128-byte
// swizzle (16-byte chunk index XOR row mod 8); tiles are 1024-byte aligned.
KQ_DEV int swz128(int row, int byte) {
  return row * 128 + ((((byte >> 4) ^ (row & 7)) << 4) | (byte & 15));
}

KQ_DEV float hi(float v) { return __uint_as_float(__float_as_uint(v) & 0xFFFFE000u); }

// Generic-proxy writes to shared memory become visible to the tensor core.
KQ_DEV void fence_to_tensor_core() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// In place: src <- hi(src), dst <- src - hi(src); n4 float4, `nthreads`
// threads with index t.  The swizzle is a permutation of 16-byte chunks
// within a row, so the split can ignore it.
KQ_DEV void split_smem(uint8_t* src, uint8_t* dst, int n4, int t, int nthreads) {
  float4* s4 = reinterpret_cast<float4*>(src);
  float4* d4 = reinterpret_cast<float4*>(dst);
  for (int e = t; e < n4; e += nthreads) {
    const float4 v = s4[e];
    float4 h, o;
    h.x = hi(v.x); h.y = hi(v.y); h.z = hi(v.z); h.w = hi(v.w);
    o.x = v.x - h.x; o.y = v.y - h.y; o.z = v.z - h.z; o.w = v.w - h.w;
    s4[e] = h;
    d4[e] = o;
  }
  fence_to_tensor_core();
}

// The three products of one K = 8 step into d_tmem (accumulate = 0 starts
// the accumulator).  a_h / a_l / b_h / b_l: shared addresses of the hi and
// lo K-major tiles, kk: the K = 8 step inside the 32-wide row.
KQ_DEV void mma3(uint32_t d_tmem, uint32_t a_h, uint32_t a_l, uint32_t b_h, uint32_t b_l, int kk,
                 uint32_t accumulate) {
  const uint64_t ah = smem_desc(a_h + kk * 32, 16, 1024, kLayoutSwizzle128B);
  const uint64_t al = smem_desc(a_l + kk * 32, 16, 1024, kLayoutSwizzle128B);
  const uint64_t bh = smem_desc(b_h + kk * 32, 16, 1024, kLayoutSwizzle128B);
  const uint64_t bl = smem_desc(b_l + kk * 32, 16, 1024, kLayoutSwizzle128B);
  mma(d_tmem, al, bh, accumulate);
  mma(d_tmem, ah, bl, 1u);
  mma(d_tmem, ah, bh, 1u);
}

// The same three products from bf16 planes (kind::f16 with bf16 operands,
// K = 16 per instruction: a K step is again 32 bytes of the 128-byte row).
constexpr uint32_t kIdescBf16_128 = idesc_f16(128, 128, /*bf16*/ 1, /*A K-major*/ 0, /*B K-major*/ 0);

constexpr uint32_t kIdescFp16_128 = idesc_f16(128, 128, /*fp16*/ 0, /*A K-major*/ 0, /*B K-major*/ 0);

// idesc: kIdescBf16_128 (bf16 planes) or kIdescFp16_128 (fp16 planes)
KQ_DEV void mma3_16(uint32_t d_tmem, uint32_t a_h, uint32_t a_l, uint32_t b_h, uint32_t b_l, int kk,
                    uint32_t accumulate, uint32_t idesc) {
  const uint64_t ah = smem_desc(a_h + kk * 32, 16, 1024, kLayoutSwizzle128B);
  const uint64_t al = smem_desc(a_l + kk * 32, 16, 1024, kLayoutSwizzle128B);
  const uint64_t bh = smem_desc(b_h + kk * 32, 16, 1024, kLayoutSwizzle128B);
  const uint64_t bl = smem_desc(b_l + kk * 32, 16, 1024, kLayoutSwizzle128B);
  mma_f16(d_tmem, al, bh, idesc, accumulate);
  mma_f16(d_tmem, ah, bl, idesc, 1u);
  mma_f16(d_tmem, ah, bh, idesc, 1u);
}

// Split x into bf16 hi = RN(x) and lo = RN(x - hi), as raw bits.
KQ_DEV void split_bf16(float x, uint16_t& h, uint16_t& l) {
  const __nv_bfloat16 hb = __float2bfloat16_rn(x);
  const __nv_bfloat16 lb = __float2bfloat16_rn(x - __bfloat162float(hb));
  h = __bfloat16_as_ushort(hb);
  l = __bfloat16_as_ushort(lb);
}

// Bounded wait used while winding down (records a timeout, never aborts).
KQ_DEV void drain_wait(uint64_t* bar, uint32_t parity, int32_t* info) {
  if (mbar_try_wait(bar, parity)) return;
  unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > kWaitLimitNs) {
      record_error(info, KRONQ_ERR_TIMEOUT);
      return;
    }
  }
}

}  // namespace tf32x3
}  // namespace kq

namespace kqh {

// 2-D fp32 tensor map over a row-major matrix (rows x cols, leading
// dimension ld elements), boxes of box_cols x box_rows, 128-byte swizzle,
// out-of-range elements read as zero.  False if the driver entry point is
// missing or the map is rejected (alignment of ptr / ld).
inline bool make_map_f32(CUtensorMap* map, const float* ptr, int64_t cols, int64_t rows, int64_t ld,
                         uint32_t box_cols, uint32_t box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same for a 2-byte matrix (bf16, or fp16 with fp16 = true; ld in elements).
inline bool make_map_bf16(CUtensorMap* map, const void* ptr, int64_t cols, int64_t rows, int64_t ld,
                          uint32_t box_cols, uint32_t box_rows, bool fp16 = false) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
            const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace kqh
