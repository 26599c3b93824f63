// sm_100a fifth-generation tensor-core helpers (tcgen05): tensor-memory (TMEM) allocation, loads
// and stores between registers and TMEM, single-thread MMA issue and its completion on an mbarrier.
//
// Layouts used here (cta_group::1, M = 64):
//   * an M=64 accumulator or A operand in TMEM keeps row m in lane (m % 16) + 32 (m / 16) and
//     column n in TMEM column base + n: warp w of a warpgroup reaches rows 16w..16w+15;
//   * tcgen05.{ld,st}.16x256b moves, per thread (g = lane/4, c = lane%4), registers
//     {(g, 2c), (g, 2c+1), (g+8, 2c), (g+8, 2c+1)} of an 8-column block -- the m16n8 accumulator
//     fragment of mma.sync -- and .xR repeats it over R consecutive 8-column blocks;
//   * shared-memory operands are K-major without swizzle: element (r, k) of a 32-bit operand
//     sits at byte (r / 8) * SBO + (k / 4) * 128 + (r % 8) * 16 + (k % 4) * 4, i.e. 8x16-byte
//     core matrices, K-adjacent ones 128 bytes apart (LBO = 128); one kind::tf32 MMA consumes
//     K = 8, so its descriptor starts 256 bytes further per K step.
#pragma once

#include <stdint.h>

namespace wkv7 {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- TMEM allocation (one full warp; the address is written to shared memory)
__device__ __forceinline__ void alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32addr(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// ---- ordering
__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// Generic-proxy shared-memory writes become visible to the tensor core (async proxy).
__device__ __forceinline__ void fence_smem_to_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---- registers <-> TMEM in the m16n8 fragment layout: x8 = 64 columns, x2 = 16 columns
__device__ __forceinline__ void st_16x256b_x8(uint32_t taddr, const float (&v)[8][4]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "f"(v[0][0]), "f"(v[0][1]), "f"(v[0][2]), "f"(v[0][3]), "f"(v[1][0]), "f"(v[1][1]), "f"(v[1][2]), "f"(v[1][3]),
      "f"(v[2][0]), "f"(v[2][1]), "f"(v[2][2]), "f"(v[2][3]), "f"(v[3][0]), "f"(v[3][1]), "f"(v[3][2]), "f"(v[3][3]),
      "f"(v[4][0]), "f"(v[4][1]), "f"(v[4][2]), "f"(v[4][3]), "f"(v[5][0]), "f"(v[5][1]), "f"(v[5][2]), "f"(v[5][3]),
      "f"(v[6][0]), "f"(v[6][1]), "f"(v[6][2]), "f"(v[6][3]), "f"(v[7][0]), "f"(v[7][1]), "f"(v[7][2]), "f"(v[7][3])
      : "memory");
}
__device__ __forceinline__ void ld_16x256b_x8(uint32_t taddr, float (&v)[8][4]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=f"(v[0][0]), "=f"(v[0][1]), "=f"(v[0][2]), "=f"(v[0][3]), "=f"(v[1][0]), "=f"(v[1][1]), "=f"(v[1][2]),
        "=f"(v[1][3]), "=f"(v[2][0]), "=f"(v[2][1]), "=f"(v[2][2]), "=f"(v[2][3]), "=f"(v[3][0]), "=f"(v[3][1]),
        "=f"(v[3][2]), "=f"(v[3][3]), "=f"(v[4][0]), "=f"(v[4][1]), "=f"(v[4][2]), "=f"(v[4][3]), "=f"(v[5][0]),
        "=f"(v[5][1]), "=f"(v[5][2]), "=f"(v[5][3]), "=f"(v[6][0]), "=f"(v[6][1]), "=f"(v[6][2]), "=f"(v[6][3]),
        "=f"(v[7][0]), "=f"(v[7][1]), "=f"(v[7][2]), "=f"(v[7][3])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void ld_16x256b_x2(uint32_t taddr, float (&v)[2][4]) {
  asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=f"(v[0][0]), "=f"(v[0][1]), "=f"(v[0][2]), "=f"(v[0][3]), "=f"(v[1][0]), "=f"(v[1][1]),
                 "=f"(v[1][2]), "=f"(v[1][3])
               : "r"(taddr)
               : "memory");
}

// ---- descriptors
// Shared-memory matrix descriptor: K-major, no swizzle, LBO = 128 bytes (see the header comment).
__device__ __forceinline__ uint64_t smem_desc(const void* start, uint32_t sbo_bytes) {
  const uint64_t addr = smem_u32addr(start);
  return ((addr >> 4) & 0x3FFFull)                        // start address, 16-byte units
         | ((uint64_t(128) >> 4) << 16)                   // leading byte offset
         | ((uint64_t(sbo_bytes) >> 4) << 32)             // stride byte offset
         | (uint64_t(1) << 46);                           // descriptor version (sm_100)
  // base offset 0, LBO mode 0, layout type 0 (no swizzle)
}
// Instruction descriptor of kind::tf32: fp32 accumulate, tf32 A and B, both K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N) {
  return (1u << 4)                      // D format: f32
         | (2u << 7)                    // A format: tf32
         | (2u << 10)                   // B format: tf32
         | (uint32_t(N >> 3) << 17)     // N / 8
         | (uint32_t(M >> 4) << 24);    // M / 16
}

// Shared-memory matrix descriptors without swizzle (the backward builds its own at compile time with
// these rules): for a K-major operand the leading byte offset (LBO) is the distance between
// K-adjacent core matrices and the stride byte offset (SBO) the distance between M/N-adjacent 8-row
// groups; for an MN-major one (16-bit types only: tf32 operands must be K-major) SBO is the distance
// between M/N-adjacent core matrices and LBO the distance between K-adjacent 8-row groups.

// Instruction descriptor of kind::f16 with bf16 A and B, fp32 accumulate, and the major-ness of A
// and B (0 = K-major, 1 = MN-major).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                      // D format: f32
         | (1u << 7)                    // A format: bf16
         | (1u << 10)                   // B format: bf16
         | (uint32_t(a_mn) << 15) | (uint32_t(b_mn) << 16)
         | (uint32_t(N >> 3) << 17)     // N / 8
         | (uint32_t(M >> 4) << 24);    // M / 16
}
// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16 (K = 16 per MMA)
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         bool accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u), "r"(0u)
      : "memory");
}

// ---- 32x32b register <-> TMEM moves: thread l of warp w reaches lane 32 (w % 4) + l; register r is
// column base + r.
__device__ __forceinline__ void ld_32x32b_x16(uint32_t taddr, float (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]), "=f"(v[8]),
        "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]), "=f"(v[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void st_32x32b_x16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]), "f"(v[9]),
      "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15])
      : "memory");
}

// ---- 16x32bx2 register <-> TMEM moves for M = 64 accumulators (rows in lanes 0-15 of the warp's
// quadrant): thread l < 16 reaches row l, columns base .. base+15; thread l >= 16 reaches row l - 16,
// columns base+16 .. base+31, so that all 32 threads of the warp share the 16 rows.
__device__ __forceinline__ void ld_16x32bx2_x16(uint32_t taddr, float (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16], 16;"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]), "=f"(v[8]),
        "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]), "=f"(v[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void st_16x32bx2_x16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], 16, {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]), "f"(v[9]),
      "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15])
      : "memory");
}
// Same with 8 columns per half: thread l < 16 reaches columns base .. base+7 of row l, thread l >= 16
// columns base+8 .. base+15 of row l - 16.
__device__ __forceinline__ void ld_16x32bx2_x8(uint32_t taddr, float (&v)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8], 8;"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
      : "r"(taddr)
      : "memory");
}

// ---- MMA issue (one thread) and completion
// D[tmem] (+)= A[smem desc] * B[smem desc]; no output lane is disabled
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       bool accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u), "r"(0u)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       bool accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u), "r"(0u)
      : "memory");
}
// Arrive on `bar` once every MMA this thread issued before has completed.
__device__ __forceinline__ void commit(unsigned long long* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32addr(bar))
               : "memory");
}

}  // namespace tc
}  // namespace wkv7
