// WKV-7 single-token decode step on B*H resident fp32 states, in place.
//
// The rwkv-metal page runs one token as plain array ops ("wkv7_step(...,
// h_in)") and keeps "exact right-padding for ragged batches".  Here one
// launch steps every (b,h) state: it is a pure stream over the 16 KiB state
// (read once, written once) and therefore HBM-bound.  One CTA per (b,h), 256
// threads; thread t owns row t/4 and the 16 columns 16*(t%4)..+15, held as
// four float4 -- each warp reads and writes 2 KiB of contiguous state with
// 16-byte accesses.  The two row dot products (sa and y) reduce over the 4
// lanes of a row with two xor-shuffles.  Rows of the batch with active[b]==0
// exit before touching the state, which therefore stays bitwise unchanged,
// and write y = 0.
#include "common.cuh"
#include "kernels.h"

namespace wkv7 {
namespace {

constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ void load16(const T* g, float* out) {
  constexpr int n = Vec16<T>::n;
#pragma unroll
  for (int u = 0; u < 16 / n; ++u) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(g + u * n));
    unpack16<T>(raw, out + u * n);
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) step_kernel(StepArgs p) {
  const int64_t unit = blockIdx.x;
  const int64_t b = unit / p.H;
  const int t = threadIdx.x;
  const int i = t >> 2, q = t & 3;
  T* y = static_cast<T*>(p.y) + unit * kN;
  if (p.active && !p.active[b]) {
    if (q == 0) y[i] = Elt<T>::from_f32(0.f);
    return;
  }
  float4* row = reinterpret_cast<float4*>(p.state + (unit * kN + i) * kN + q * 16);
  float S[16];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float4 s4 = row[u];
    S[4 * u] = s4.x; S[4 * u + 1] = s4.y; S[4 * u + 2] = s4.z; S[4 * u + 3] = s4.w;
  }
  const int64_t o = unit * kN + q * 16;
  float wv[16], kv[16], av[16], bv[16], rv[16];
  load16<T>(static_cast<const T*>(p.a) + o, av);
  load16<T>(static_cast<const T*>(p.w) + o, wv);
  load16<T>(static_cast<const T*>(p.b) + o, bv);
  load16<T>(static_cast<const T*>(p.k) + o, kv);
  load16<T>(static_cast<const T*>(p.r) + o, rv);
  const float vi = Elt<T>::to_f32(static_cast<const T*>(p.v)[unit * kN + i]);

  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int j = 0; j < 16; j += 2) {
    s0 = fmaf(S[j], av[j], s0);
    s1 = fmaf(S[j + 1], av[j + 1], s1);
  }
  float sa = s0 + s1;
  sa += __shfl_xor_sync(0xffffffffu, sa, 1);
  sa += __shfl_xor_sync(0xffffffffu, sa, 2);

  float y0 = 0.f, y1 = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    S[j] = fmaf(S[j], wv[j], fmaf(sa, bv[j], vi * kv[j]));
    if (j & 1) y1 = fmaf(S[j], rv[j], y1); else y0 = fmaf(S[j], rv[j], y0);
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) row[u] = make_float4(S[4 * u], S[4 * u + 1], S[4 * u + 2], S[4 * u + 3]);
  float yy = y0 + y1;
  yy += __shfl_xor_sync(0xffffffffu, yy, 1);
  yy += __shfl_xor_sync(0xffffffffu, yy, 2);
  if (q == 0) y[i] = Elt<T>::from_f32(yy);
}

template <typename T>
cudaError_t launch(const StepArgs& p, cudaStream_t stream) {
  step_kernel<T><<<dim3(unsigned(p.B * p.H)), dim3(kThreads), 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_step(const StepArgs& p, int dtype, cudaStream_t stream) {
  switch (dtype) {
    case 0: return launch<float>(p, stream);
    case 1: return launch<__nv_bfloat16>(p, stream);
    case 2: return launch<__half>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wkv7
