// wkv7_train_step_noalloc: a forward + backward pass that allocates nothing.
//
// Some callers cannot call cudaMalloc: hosts whose device memory is owned by
// another allocator (a framework's caching allocator, or a serving engine
// that reserves all free memory up front) and code paths where allocating
// is not allowed.  The regular entry points need a caller-provided
// checkpoint workspace; this one keeps that scratch (the 16-token state
// checkpoints and the backward's per-head marks) in a fixed array of this
// library instead.  Inputs and outputs are still the caller's buffers.
//
// The array is a file-scope __device__ object: every GPU that loads the
// library holds its WKV7_NOALLOC_SCRATCH_BYTES until the process exits.  Its
// device address is looked up on every call (cudaGetSymbolAddress, with the
// calling device current), never cached: after a cudaDeviceReset the module
// is loaded again and the array may sit elsewhere.  Only the first call on a
// device loads the module, so that first call should come before any stream
// capture.  Every call shares the one array and it keeps the previous call's
// contents; nothing in it needs to start at zero (the forward writes every
// checkpoint and the backward writes every mark before reading them), but
// two calls that overlap on the GPU race on it.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "wkv7.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[WKV7_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array on the current device.  Host code sees g_noalloc_scratch only
// as a host-side stand-in, so the address comes from the runtime, looked up afresh on every call.
cudaError_t scratch_for_current_device(void** out) {
  *out = nullptr;
  return cudaGetSymbolAddress(out, g_noalloc_scratch);
}

}  // namespace

extern "C" wkv7_status_t wkv7_train_step_noalloc(const wkv7_desc_t* d, const void* r, const void* w, const void* k,
                                                 const void* v, const void* a, const void* b, const float* s0,
                                                 const uint8_t* reset, void* y, float* s_out, const void* dy,
                                                 const float* dsT, void* dr, void* dw, void* dk, void* dv, void* da,
                                                 void* db, float* ds0, void* stream) {
  const wkv7_status_t valid = wkv7::validate_desc(d);
  if (valid != WKV7_OK) return valid;
  if (d->N != 64) return WKV7_ERR_UNSUPPORTED;   // the backward is written for heads of 64
  const size_t need = wkv7_workspace_bytes(d);
  if (need == 0 && d->T != 0) return WKV7_ERR_SHAPE;   // (an accepted descriptor always has a size)
  if (need > size_t(WKV7_NOALLOC_SCRATCH_BYTES)) return WKV7_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  if (d->T > 0) {
    if (scratch_for_current_device(&scratch) != cudaSuccess) return WKV7_ERR_CUDA;
  }
  wkv7_status_t st = wkv7_forward(d, r, w, k, v, a, b, s0, reset, y, s_out, scratch, stream);
  if (st != WKV7_OK) return st;
  return wkv7_backward(d, r, w, k, v, a, b, s0, reset, dy, dsT, scratch, dr, dw, dk, dv, da, db, ds0, stream);
}
