// Shared device helpers for the WKV-7 kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace wkv7 {

constexpr int kN = 64;       // head size
constexpr int kChunk = 16;   // checkpoint interval / chunk length

// ------------------------------------------------------------------ element I/O
template <typename T> struct Elt;

template <> struct Elt<float> {
  static __device__ __forceinline__ float to_f32(float x) { return x; }
  static __device__ __forceinline__ float from_f32(float x) { return x; }
};
template <> struct Elt<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f32(float x) { return __float2bfloat16_rn(x); }
};
template <> struct Elt<__half> {
  static __device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }
  static __device__ __forceinline__ __half from_f32(float x) { return __float2half_rn(x); }
};

// Two adjacent elements of T (4- or 8-byte aligned) as fp32.
__device__ __forceinline__ float2 load2(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ float2 load2(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}
__device__ __forceinline__ float2 load2(const __half* p) { return __half22float2(*reinterpret_cast<const __half2*>(p)); }

// Store two fp32 values as adjacent elements of T (round to nearest).
__device__ __forceinline__ void store2(float* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }
__device__ __forceinline__ void store2(__nv_bfloat16* p, float2 v) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v.x, v.y);
}
__device__ __forceinline__ void store2(__half* p, float2 v) { *reinterpret_cast<__half2*>(p) = __floats2half2_rn(v.x, v.y); }

// Number of elements of T in one 16-byte vector.
template <typename T> struct Vec16 { static constexpr int n = 16 / sizeof(T); };

// Unpack one 16-byte vector of T into fp32 values.
template <typename T>
__device__ __forceinline__ void unpack16(const uint4& raw, float* out) {
  const T* p = reinterpret_cast<const T*>(&raw);
#pragma unroll
  for (int e = 0; e < Vec16<T>::n; ++e) out[e] = Elt<T>::to_f32(p[e]);
}

// ------------------------------------------------------------------ cp.async (16 B)
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

// Offset of element (i, j) inside one checkpointed 64x64 fp32 state.  The order is the one
// in which the chunked kernels hold the state as m16n8 accumulator fragments (warp i/16,
// lane 4(i%8) + (j%8)/2, register 4(j/8) + 2((i/8)%2) + j%2), so that each warp stores and
// loads 512 contiguous bytes per instruction.
__host__ __device__ __forceinline__ int ckpt_off(int i, int j) {
  return (i >> 4) * 1024 + (j >> 3) * 128 + ((i & 7) * 4 + ((j & 7) >> 1)) * 4 + ((i >> 3) & 1) * 2 + (j & 1);
}

// Offset (in elements) of x[b][t][h][0] in a [B,T,H,64] tensor.
__device__ __forceinline__ int64_t tok_off(int64_t b, int64_t t, int64_t h, int64_t T, int64_t H) {
  return ((b * T + t) * H + h) * kN;
}
// The same in a [B,T,H,N] tensor.
template <int N>
__device__ __forceinline__ int64_t tok_offn(int64_t b, int64_t t, int64_t h, int64_t T, int64_t H) {
  return ((b * T + t) * H + h) * N;
}

}  // namespace wkv7

namespace wkv7 {

// ------------------------------------------------------------------ packed fp32 pairs (sm_100 f32x2)
// One instruction operates on two adjacent fp32 values; on sm_100a this issues half the
// instructions of the scalar form at the same arithmetic throughput.
__device__ __forceinline__ unsigned long long f2_pack(float2 v) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(v.x), "f"(v.y));
  return r;
}
__device__ __forceinline__ float2 f2_unpack(unsigned long long r) {
  float2 v;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
  return v;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(f2_pack(a)), "l"(f2_pack(b)), "l"(f2_pack(c)));
  return f2_unpack(d);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_pack(a)), "l"(f2_pack(b)));
  return f2_unpack(d);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_pack(a)), "l"(f2_pack(b)));
  return f2_unpack(d);
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  unsigned long long d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_pack(a)), "l"(f2_pack(b)));
  return f2_unpack(d);
}

// The decay from its stored input: w itself, or, under the log-space convention, x with
// w = exp(-exp(x)) (log w = -exp(x)).  The fast exponential (a few ulp) keeps the chunked kernels'
// decay scan, which the context warps sit on, short; it is far inside every tolerance.
__device__ __forceinline__ float decay_of(float x, bool log_decay) { return log_decay ? __expf(-__expf(x)) : x; }
// dL/dx from dL/d(log w) under the log-space convention: d(log w)/dx = -exp(x).
__device__ __forceinline__ float dx_of_dlogw(float dlogw, float x) { return -dlogw * expf(x); }

// Segment index of token t inside a chunk: number of resets among tokens 1..t.
__device__ __forceinline__ int seg_of(unsigned mask, int t) { return __popc(mask & ((2u << t) - 2u)); }

// Bits of the tokens that belong to the chunk's last segment.
__device__ __forceinline__ unsigned last_segment_bits(unsigned mask) {
  if (!(mask & 0xfffeu)) return 0xffffu;
  const int last = 31 - __clz(mask & 0xfffeu);   // start of the last segment
  return 0xffffu & ~((1u << last) - 1u);
}

// ------------------------------------------------------------------ bulk copies and mbarriers
// One-dimensional bulk copies (TMA engine, no tensor map) from global to shared memory complete
// on an mbarrier's transaction count; threads wait on the barrier phase with a wall-clock bound.
__device__ __forceinline__ unsigned smem_addr(const void* p) {
  return static_cast<unsigned>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(unsigned long long* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(unsigned long long* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(unsigned long long* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait for completion of the barrier phase with the given parity; false if limit_ns passed first.
__device__ __forceinline__ bool mbar_wait_bounded(unsigned long long* bar, unsigned parity, unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity))
    if (global_ns() - t0 > limit_ns) return false;
  return true;
}
// Copy `bytes` (a multiple of 16; both addresses 16-byte aligned) and count them on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, unsigned long long* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}

// Tiled 4-D tensor load (TMA) of one box into shared memory, counted on `bar`.  `map` is the
// address of a CUtensorMap in kernel parameter space; coordinates are innermost first.
__device__ __forceinline__ void tma_load_4d(void* dst, const void* map, int c0, int c1, int c2, int c3,
                                            unsigned long long* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];"
      ::"r"(smem_addr(dst)), "l"(reinterpret_cast<unsigned long long>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
        "r"(smem_addr(bar))
      : "memory");
}

}  // namespace wkv7
