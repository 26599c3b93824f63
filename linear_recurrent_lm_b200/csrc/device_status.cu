// Device status word: kernels record device-side errors in it (a bounded wait on staged inputs
// that ran out); wkv7_get_device_status() reads it after synchronising.  One word per device.
#include <cuda_runtime.h>

#include <mutex>

#include "kernels.h"
#include "wkv7.h"

namespace {

static __device__ int g_device_status;

constexpr int kMaxDevices = 256;
std::mutex g_lock;
int* g_status_ptr[kMaxDevices] = {};

}  // namespace

namespace wkv7 {

cudaError_t device_status_ptr(int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> guard(g_lock);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_device_status);
    if (e != cudaSuccess) return e;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  *out = g_status_ptr[dev];
  return cudaSuccess;
}

}  // namespace wkv7

extern "C" wkv7_status_t wkv7_get_device_status(int clear) {
  if (cudaDeviceSynchronize() != cudaSuccess) return WKV7_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return WKV7_ERR_CUDA;
  if (clear && v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return WKV7_ERR_CUDA;
  }
  if (v & wkv7::kStatusWaitTimeout) return WKV7_ERR_TIMEOUT;
  return (v & wkv7::kStatusNonFinite) ? WKV7_ERR_NONFINITE : WKV7_OK;
}
