// Small tcgen05 / bf16 helpers shared by the sequential-phase tensor-core
// kernels (the backward and the split-operand forward).
#pragma once

#include "gdr_sm100.cuh"

namespace gdr {
namespace tcu {

using namespace sm100;

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&t);
}

__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u));
}

// x = hi + lo + O(2^-18 |x|) with hi, lo bf16: the two-term split that lets
// three bf16 products (hi hi, hi lo, lo hi) stand in for one fp32 product.
__device__ __forceinline__ void split_bf16(float x, float &hi, float &lo) {
  hi = __bfloat162float(__float2bfloat16_rn(x));
  lo = x - hi;
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16 (bf16 in, fp32 acc).
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 16 consecutive 32-bit TMEM columns of this thread's lane (raw words).
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t *v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  float a[16], b[16];
  tmem_ld16(taddr, a);
  tmem_ld16(taddr + 16, b);
  tmem_wait_ld();
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    v[e] = a[e];
    v[16 + e] = b[e];
  }
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  tmem_st16(taddr, *reinterpret_cast<const float(*)[16]>(v));
  tmem_st16(taddr + 16, *reinterpret_cast<const float(*)[16]>(v + 16));
}

// 32 bf16 of x into columns [32 q, 32 q + 32) of row `row` of a 128B-swizzled
// tile whose rows are 64 bf16.
__device__ __forceinline__ void st_row32(uint8_t *tile, int row, int q, const float *x) {
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    uint4 u;
    u.x = pack_bf16(x[8 * ch + 0], x[8 * ch + 1]);
    u.y = pack_bf16(x[8 * ch + 2], x[8 * ch + 3]);
    u.z = pack_bf16(x[8 * ch + 4], x[8 * ch + 5]);
    u.w = pack_bf16(x[8 * ch + 6], x[8 * ch + 7]);
    *reinterpret_cast<uint4 *>(tile + sw128_off(row, 32 * q + 8 * ch)) = u;
  }
}

}  // namespace tcu
}  // namespace gdr
