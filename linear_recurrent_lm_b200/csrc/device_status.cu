// Device status word: kernels record device-side errors in it (a bounded wait on staged inputs
// that ran out, a non-finite checked output, a failed debug-build bounds check);
// wkv7_get_device_status() reads it after synchronising.  One word per device.
#include <cuda_runtime.h>

#include "kernels.h"
#include "wkv7.h"

namespace {

static __device__ int g_device_status;

}  // namespace

namespace wkv7 {

// Looked up on every call, never cached: after a cudaDeviceReset the module is loaded again and the
// word may sit at another address.  (Host code sees g_device_status only as a host-side stand-in.)
cudaError_t device_status_ptr(int** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_device_status);
  *out = static_cast<int*>(p);
  return e;
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
  if (v & wkv7::kStatusBounds) return WKV7_ERR_BOUNDS;
  return (v & wkv7::kStatusNonFinite) ? WKV7_ERR_NONFINITE : WKV7_OK;
}

extern "C" int wkv7_debug_checks(void) { return wkv7::kDebugChecks ? 1 : 0; }
