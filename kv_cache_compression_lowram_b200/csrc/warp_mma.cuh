// Warp-level bf16 matrix products (mma.sync m16n8k16, fp32 accumulation) and their shared-
// memory fragment loads, for the small per-unit products of the selection and combine kernels
// (projections, score and logit GEMVs, the second predictor layer): a few dozen instructions
// where CUDA-core loops would issue thousands.  The chunk-attention kernel's large tiles use
// tcgen05 instead.
//
// Fragment layout of m16n8k16 (lane l, g = l / 4, c = (l % 4) * 2):
//   A (16 x 16, row-major): a0 = (row g, k c..c+1), a1 = (g + 8, c..c+1), a2 = (g, c+8..c+9),
//                           a3 = (g + 8, c+8..c+9)
//   B (16 x 8, k x n):      b0 = (k c..c+1, col g), b1 = (k c+8..c+9, col g)
//   C (16 x 8, fp32):       c0, c1 = (row g, cols c, c+1), c2, c3 = (row g + 8, cols c, c+1)
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace lowram {
namespace wm {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Four 8x8 bf16 matrices; lane l supplies the row address of row l % 8 of matrix l / 8.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr(row_addr)));
}
// Two 8x8 matrices (lanes 0-15 supply the row addresses).
__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(smem_addr(row_addr)));
}
// The same, transposed (for a B operand stored k-major, i.e. [k][n] rows).
__device__ __forceinline__ void ldsm_x2_t(uint32_t (&r)[2], const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(smem_addr(row_addr)));
}

// D = A B + D, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// An fp32 value as the sum of two bf16 values (hi = x rounded, lo = the rest rounded): used
// where an fp32 operand meets bf16 data in an MMA, so the product keeps ~16 significant bits.
__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

}  // namespace wm
}  // namespace lowram
