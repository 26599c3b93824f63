// Warp-level tensor-core helpers: bf16 mma.sync m16n8k16 with fp32 accumulate,
// ldmatrix fragment loads, and the hi/lo bf16 split used for fp32-accurate
// products (x = hi + lo, hi = bf16(x), lo = bf16(x - hi); a product is taken
// as hi*hi + hi*lo + lo*hi, which leaves a relative error near 2^-16).
//
// Fragment layout of m16n8k16 (g = lane/4, c = lane%4):
//   A (16x16): a0 = (g, 2c..2c+1), a1 = (g+8, 2c..), a2 = (g, 8+2c..), a3 = (g+8, 8+2c..)
//   B (16x8):  b0 = (k 2c..2c+1, n g), b1 = (k 8+2c.., n g)
//   C (16x8):  c0 = (g, 2c), c1 = (g, 2c+1), c2 = (g+8, 2c), c3 = (g+8, 2c+1)
// so the accumulators of two adjacent n-tiles are exactly an A fragment.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace wkv7 {

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* row_ptr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(row_ptr)));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo_elem, float hi_elem) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo_elem, hi_elem);
  return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace wkv7

namespace wkv7 {

// ------------------------------------------------------------------ tf32 (m16n8k8, fp32 accumulate)
// Fragment layout (g = lane/4, c = lane%4):
//   A (16x8): a0 = (g, c), a1 = (g+8, c), a2 = (g, c+4), a3 = (g+8, c+4)
//   B (8x8):  b0 = (k c, n g), b1 = (k c+4, n g)
//   C (16x8): c0 = (g, 2c), c1 = (g, 2c+1), c2 = (g+8, 2c), c3 = (g+8, 2c+1)
// ldmatrix on fp32 data treats each fp32 as two b16 halves: thread l receives element
// (row l/4, column l%4) of an 8-row x 4-fp32 tile, which is exactly the A/B pattern above
// when the tile is stored with k contiguous.  An accumulator tile used as an A operand is
// read with a permuted k order (column 2c -> k c, column 2c+1 -> k c+4); the matching B
// fragment is then the adjacent pair (k 2c, 2c+1) of a [n][k] tile, one 8-byte load.

__device__ __forceinline__ void mma1688(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Round an fp32 value to tf32 (nearest, ties away), returned as its 32-bit pattern.
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;\n" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float tf32f(float x) { return __uint_as_float(to_tf32(x)); }

// ldmatrix address of an A fragment (16 m x 8 k) from fp32 [m][k] storage at (m0, k0).
__device__ __forceinline__ const float* a32_addr(const float* base, int stride, int m0, int k0, int lane) {
  const int mat = lane >> 3, r = lane & 7;
  return base + (m0 + (mat & 1) * 8 + r) * stride + k0 + (mat >> 1) * 4;
}
// ldmatrix address of B fragments for two n-tiles (n0.., n0+8..) x one k-step (k0..k0+7) from fp32 [n][k].
__device__ __forceinline__ const float* b32_2n_addr(const float* base, int stride, int n0, int k0, int lane) {
  const int mat = lane >> 3, r = lane & 7;
  return base + (n0 + (mat >> 1) * 8 + r) * stride + k0 + (mat & 1) * 4;
}
// ldmatrix address of B fragments for one n-tile (n0..n0+7) x two k-steps (k0.., k0+8..) from fp32 [n][k].
__device__ __forceinline__ const float* b32_2k_addr(const float* base, int stride, int n0, int k0, int lane) {
  const int mat = lane >> 3, r = lane & 7;
  return base + (n0 + r) * stride + k0 + mat * 4;
}

}  // namespace wkv7
