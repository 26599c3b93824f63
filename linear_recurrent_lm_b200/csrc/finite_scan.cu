// Optional check of a call's floating outputs for NaN and infinities (desc->flags bit
// WKV7_FLAG_CHECK_FINITE): one pass over the output, 16 bytes per load, that sets the
// non-finite bit of the device status word if any element is NaN or +-Inf.  It reads the
// output once more (a plain HBM stream), so it is off by default.
#include "common.cuh"
#include "kernels.h"

namespace wkv7 {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxBlocks = 1184;   // enough 16-byte loads in flight to stream at HBM rate

template <typename T>
__global__ void __launch_bounds__(kThreads) finite_scan_kernel(const T* x, int64_t n, int* status) {
  constexpr int kPer = Vec16<T>::n;
  const int64_t nv = n / kPer;
  bool bad = false;
  for (int64_t i = int64_t(blockIdx.x) * kThreads + threadIdx.x; i < nv; i += int64_t(gridDim.x) * kThreads) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(x) + i);
    float f[kPer];
    unpack16<T>(raw, f);
#pragma unroll
    for (int e = 0; e < kPer; ++e) bad |= !isfinite(f[e]);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0)   // elements past the last whole 16-byte vector
    for (int64_t i = nv * kPer; i < n; ++i) bad |= !isfinite(Elt<T>::to_f32(x[i]));
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, kStatusNonFinite);
}

template <typename T>
cudaError_t launch(const void* x, int64_t n, int* status, cudaStream_t stream) {
  const int64_t nv = n / Vec16<T>::n;
  int64_t blocks = (nv + kThreads - 1) / kThreads;
  if (blocks < 1) blocks = 1;
  if (blocks > kMaxBlocks) blocks = kMaxBlocks;
  finite_scan_kernel<T><<<dim3(unsigned(blocks)), dim3(kThreads), 0, stream>>>(static_cast<const T*>(x), n, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_finite_scan(const void* x, int64_t n, int dtype, int* status, cudaStream_t stream) {
  if (!x || n <= 0) return cudaSuccess;
  switch (dtype) {
    case 0: return launch<float>(x, n, status, stream);
    case 1: return launch<__nv_bfloat16>(x, n, status, stream);
    case 2: return launch<__half>(x, n, status, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wkv7
