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

// Offset (in elements) of x[b][t][h][0] in a [B,T,H,64] tensor.
__device__ __forceinline__ int64_t tok_off(int64_t b, int64_t t, int64_t h, int64_t T, int64_t H) {
  return ((b * T + t) * H + h) * kN;
}

}  // namespace wkv7
