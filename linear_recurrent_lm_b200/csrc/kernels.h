// Internal launch interface between the C-ABI layer (wkv7_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace wkv7 {

struct FwdArgs {
  int64_t B, T, H;
  const void *r, *w, *k, *v, *a, *b;
  const float* s0;        // [B,H,64,64] or null
  const uint8_t* reset;   // [B,T] or null
  void* y;                // [B,T,H,64]
  float* s_out;           // [B,H,64,64] or null
  float* ckpt;            // [B,H,ceil(T/16),64,64] or null
};

struct BwdArgs {
  int64_t B, T, H;
  const void *r, *w, *k, *v, *a, *b;
  const float* s0;
  const uint8_t* reset;
  const void* dy;
  const float* dsT;
  const float* ckpt;
  void *dr, *dw, *dk, *dv, *da, *db;
  float* ds0;
  int* unit_flags;   // [B*H] in the workspace tail: the chunked backward marks units it could not handle
};

struct StepArgs {
  int64_t B, H;
  const void *r, *w, *k, *v, *a, *b;
  float* state;
  const uint8_t* active;
  void* y;
};

// dtype: 0 = f32, 1 = bf16, 2 = f16.  Each returns the launch status.
cudaError_t launch_scan_fwd(const FwdArgs& p, int dtype, cudaStream_t stream);
// only_flagged: run only the (b,h) units whose unit_flags entry is non-zero (others exit at once).
cudaError_t launch_scan_bwd(const BwdArgs& p, int dtype, bool only_flagged, cudaStream_t stream);
cudaError_t launch_step(const StepArgs& p, int dtype, cudaStream_t stream);
cudaError_t launch_chunk_fwd(const FwdArgs& p, int dtype, cudaStream_t stream);
cudaError_t launch_chunk_bwd(const BwdArgs& p, int dtype, cudaStream_t stream);

}  // namespace wkv7
